// The probability weights P enter the bf16 tensor-core products as two
// terms, its bf16 value and the bf16 value of the residual, so that P keeps
// about 17 significant bits (one bf16 term alone, relative error ~2^-9 per
// weight, gives an expected relative-L2 error near 1.1e-3 on unit-variance
// values: above the 1e-3 bound of the attention output).
#pragma once

#include <cstdint>

#include "pa_common.cuh"

namespace pa {

// Two-term bf16 split of the pair (a, b): hi = (bf16(a), bf16(b)) and
// lo = (bf16(a - bf16(a)), bf16(b - bf16(b))), both rounded to nearest, a in
// the low half of each word.  hi + lo carries a to within 2^-18 relative
// (the residual is exact in fp32); the error has no sign bias.
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi,
                                             uint32_t& lo) {
    hi = pack_bf16x2(a, b);
    const float ah = __uint_as_float(hi << 16);
    const float bh = __uint_as_float(hi & 0xFFFF0000u);
    lo = pack_bf16x2(a - ah, b - bh);
}

}  // namespace pa
