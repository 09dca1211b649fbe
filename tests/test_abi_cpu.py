"""C-ABI checks that need no GPU: the library loads, exports every entry point
include/pa.h declares, and rejects bad arguments on the host with the
documented status before any CUDA call."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

from paged_kv_cache_435_b200 import _native as nat
from paged_kv_cache_435_b200 import build as pa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")


@pytest.fixture(scope="module")
def lib():
    pa_build.build()
    return nat.raw()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w \*]*?\b(pa_\w+)\s*\(", text,
                                 flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("pa_reshape_and_cache", "pa_decode_attention", "pa_copy_blocks",
              "pa_decode_workspace_size", "pa_decode_partition_size",
              "pa_status_string", "pa_launch_count", "pa_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings(lib):
    assert nat.status_string(0) == "PA_OK"
    assert nat.status_string(-1) == "PA_ERR_INVALID_ARG"
    assert nat.status_string(-2) == "PA_ERR_UNSUPPORTED"
    assert nat.status_string(-3) == "PA_ERR_WORKSPACE"
    assert nat.status_string(-4) == "PA_ERR_CUDA"
    assert nat.status_string(7) == "PA_UNKNOWN_STATUS"
    assert lib.pa_version() >> 16 == 1


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def decode_args(**kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, mb=8, cl=FAKE,
             maxlen=100, B=4, Hq=8, Hkv=2, D=128, bs=16, NB=64, scale=0.1,
             part=0, ws=None, wsb=0, err=None, stream=None)
    a.update(kw)
    return [a[k] for k in ("out", "q", "k", "v", "bt", "mb", "cl", "maxlen",
                           "B", "Hq", "Hkv", "D", "bs", "NB", "scale", "part",
                           "ws", "wsb", "err", "stream")]


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=6, Hkv=4), nat.PA_ERR_INVALID_ARG),          # Hq % Hkv != 0
    (dict(B=-1), nat.PA_ERR_INVALID_ARG),
    (dict(Hkv=0), nat.PA_ERR_INVALID_ARG),
    (dict(maxlen=129), nat.PA_ERR_INVALID_ARG),           # > mb*bs
    (dict(part=24), nat.PA_ERR_INVALID_ARG),              # not multiple of bs
    (dict(part=-16), nat.PA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), nat.PA_ERR_INVALID_ARG),
    (dict(out=None), nat.PA_ERR_INVALID_ARG),
    (dict(q=FAKE + 2), nat.PA_ERR_INVALID_ARG),           # misaligned
    (dict(D=96), nat.PA_ERR_UNSUPPORTED),
    (dict(bs=8, mb=16), nat.PA_ERR_UNSUPPORTED),
    (dict(Hq=32, Hkv=2), nat.PA_ERR_UNSUPPORTED),         # group 16
    (dict(part=16, ws=None, wsb=0), nat.PA_ERR_WORKSPACE),  # split, no ws
    (dict(part=16, ws=FAKE, wsb=16), nat.PA_ERR_WORKSPACE),
    (dict(part=16, ws=FAKE + 16, wsb=1 << 30), nat.PA_ERR_INVALID_ARG),
])
def test_decode_host_validation(lib, kw, status):
    assert lib.pa_decode_attention(*decode_args(**kw)) == status


def test_decode_zero_sequences_is_a_no_op(lib):
    assert lib.pa_decode_attention(*decode_args(B=0, out=None, q=None)) == nat.PA_OK


def test_partition_plan_and_workspace(lib):
    # Big batch: no split (one partition covering the longest context).
    p = nat.pa_decode_partition_size(256, 64, 8, 128, 16, 4096, 0)
    assert p >= 4096 and p % 16 == 0
    assert nat.pa_decode_workspace_size(256, 64, 8, 128, 16, 4096, 0) == 0
    # Few (seq, kv head) units with a long context: 512-token partitions.
    p = nat.pa_decode_partition_size(32, 32, 8, 128, 32, 131072, 0)
    assert p == 512
    ws = nat.pa_decode_workspace_size(32, 32, 8, 128, 32, 131072, 0)
    rows = 32 * 32 * 256
    assert ws >= rows * 128 * 4 + 2 * rows * 4
    # Explicit partition wins.
    assert nat.pa_decode_partition_size(4, 4, 4, 64, 16, 100, 32) == 32
    assert nat.pa_decode_workspace_size(4, 4, 4, 64, 16, 100, 32) > 0
    with pytest.raises(nat.PAError):
        nat.pa_decode_partition_size(4, 4, 4, 64, 16, 100, 24)


def reshape_args(**kw):
    a = dict(key=FAKE, value=FAKE, ks=512, vs=512, kc=FAKE, vc=FAKE, sm=FAKE,
             T=4, NB=8, bs=16, Hkv=4, D=128, err=None, stream=None)
    a.update(kw)
    return [a[k] for k in ("key", "value", "ks", "vs", "kc", "vc", "sm", "T",
                           "NB", "bs", "Hkv", "D", "err", "stream")]


@pytest.mark.parametrize("kw,status", [
    (dict(T=-1), nat.PA_ERR_INVALID_ARG),
    (dict(ks=100), nat.PA_ERR_INVALID_ARG),               # stride < Hkv*D
    (dict(kc=None), nat.PA_ERR_INVALID_ARG),
    (dict(sm=None), nat.PA_ERR_INVALID_ARG),
    (dict(sm=FAKE + 4), nat.PA_ERR_INVALID_ARG),          # int64 misaligned
    (dict(key=FAKE + 1), nat.PA_ERR_INVALID_ARG),
    (dict(bs=0), nat.PA_ERR_INVALID_ARG),
    (dict(T=0, key=None, value=None, sm=None), nat.PA_OK),
])
def test_reshape_host_validation(lib, kw, status):
    assert lib.pa_reshape_and_cache(*reshape_args(**kw)) == status


def test_copy_blocks_host_validation(lib):
    arr = (ctypes.c_void_p * 2)(FAKE, FAKE)
    bad = (ctypes.c_void_p * 2)(FAKE, None)
    mis = (ctypes.c_void_p * 2)(FAKE, FAKE + 8)
    f = lib.pa_copy_blocks
    a = ctypes.cast(arr, ctypes.c_void_p)
    assert f(a, a, 2, FAKE, -1, 8, 16, 4, 128, None, None) == nat.PA_ERR_INVALID_ARG
    assert f(a, a, 0, FAKE, 1, 8, 16, 4, 128, None, None) == nat.PA_ERR_INVALID_ARG
    assert f(ctypes.cast(bad, ctypes.c_void_p), a, 2, FAKE, 1, 8, 16, 4, 128,
             None, None) == nat.PA_ERR_INVALID_ARG
    assert f(ctypes.cast(mis, ctypes.c_void_p), a, 2, FAKE, 1, 8, 16, 4, 128,
             None, None) == nat.PA_ERR_INVALID_ARG
    assert f(a, a, 2, None, 1, 8, 16, 4, 128, None, None) == nat.PA_ERR_INVALID_ARG
    assert f(a, a, 2, None, 0, 8, 16, 4, 128, None, None) == nat.PA_OK
    assert f(None, a, 2, FAKE, 1, 8, 16, 4, 128, None, None) == nat.PA_ERR_INVALID_ARG


def test_launch_counter_is_monotonic(lib):
    a = nat.pa_launch_count()
    # host-rejected calls launch nothing
    lib.pa_decode_attention(*decode_args(Hkv=0))
    assert nat.pa_launch_count() == a


def test_product_package_does_not_reach_the_oracle():
    pkg = os.path.join(ROOT, "paged_kv_cache_435_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text
                assert "pa_oracle" not in text, f


def test_swap_blocks_host_validation(lib):
    arr = (ctypes.c_void_p * 1)(FAKE)
    a = ctypes.cast(arr, ctypes.c_void_p)
    f = lib.pa_swap_blocks
    assert f(a, a, 0, FAKE, 1, 4096, 4, 4, None, None) == nat.PA_ERR_INVALID_ARG
    assert f(a, a, 1, FAKE, 1, 4100, 4, 4, None, None) == nat.PA_ERR_INVALID_ARG
    assert f(a, a, 1, FAKE, -1, 4096, 4, 4, None, None) == nat.PA_ERR_INVALID_ARG
    assert f(a, a, 1, FAKE, 1, 4096, 0, 4, None, None) == nat.PA_ERR_INVALID_ARG
    assert f(a, a, 1, None, 0, 4096, 4, 4, None, None) == nat.PA_OK
    assert f(None, a, 1, FAKE, 1, 4096, 4, 4, None, None) == nat.PA_ERR_INVALID_ARG


def test_multi_query_host_validation(lib):
    f = lib.pa_multi_query_attention
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, 8, FAKE, 100, FAKE, 4, 2, 8, 2, 128,
            16, 64, 0.1, None, None]
    def call(**kw):
        a = list(args)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return f(*a)
    assert call(a12=4, a11=6) == nat.PA_ERR_INVALID_ARG        # Hq % Hkv
    assert call(a9=101) == nat.PA_ERR_INVALID_ARG              # mq > max len
    assert call(a7=129) == nat.PA_ERR_INVALID_ARG              # > MB*bs
    assert call(a13=96) == nat.PA_ERR_UNSUPPORTED
    assert call(a8=None) == nat.PA_ERR_INVALID_ARG
    assert call(a9=0) == nat.PA_OK


def test_shared_prefix_host_validation(lib):
    f = lib.pa_decode_attention_shared_prefix
    #       out   q     k     v     bt   mb cl   maxlen gs    pl   G mgs B   Hq Hkv D   bs  NB  scale part ws    wsb       err   stream
    base = [FAKE, FAKE, FAKE, FAKE, FAKE, 8, FAKE, 100, FAKE, FAKE, 2, 4, 8, 32, 8, 128, 16, 64, 0.1, 0, FAKE, 1 << 30, None, None]

    def call(**kw):
        a = list(base)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return f(*a)
    assert call(a10=-1) == nat.PA_ERR_INVALID_ARG          # negative group count
    assert call(a11=0) == nat.PA_ERR_INVALID_ARG           # max_group_size 0
    assert call(a8=None) == nat.PA_ERR_INVALID_ARG         # group_start missing
    assert call(a9=FAKE + 2) == nat.PA_ERR_INVALID_ARG     # prefix_lens misaligned
    assert call(a15=64) == nat.PA_ERR_UNSUPPORTED          # head size 64
    assert call(a13=128) == nat.PA_ERR_UNSUPPORTED         # 128 q / 8 kv: group 16
    # 64-token partitions split the 100-token contexts: scratch is needed
    assert call(a19=64, a20=None) == nat.PA_ERR_WORKSPACE          # no workspace
    assert call(a19=64, a21=16) == nat.PA_ERR_WORKSPACE            # too small
    assert call(a19=64, a20=FAKE + 16) == nat.PA_ERR_INVALID_ARG   # not 256-aligned
    assert call(a12=0, a0=None, a1=None) == nat.PA_OK      # empty batch


def test_shared_prefix_workspace_grows_with_rows(lib):
    # The per-sequence pass's split scratch, then the group pass's pieces:
    # (B + 148 / Hkv) slots x Hkv x 32 rows of D + 2 floats, and B x Hkv
    # counters, each region 256-byte aligned (no device here: 148 SMs).
    def a256(x):
        return (x + 255) // 256 * 256
    for B in (8, 16):
        for part in (0, 64):
            split = nat.pa_decode_workspace_size(B, 32, 8, 128, 16, 1000, part)
            rows = (B + 148 // 8) * 8 * 32
            want = a256(a256(a256(a256(split) + rows * 128 * 4) + rows * 2 * 4) + B * 8 * 4)
            assert nat.pa_shared_prefix_workspace_size(B, 32, 8, 128, 16, 1000, part) == want
    a = nat.pa_shared_prefix_workspace_size(8, 32, 8, 128, 16, 1000)
    b = nat.pa_shared_prefix_workspace_size(16, 32, 8, 128, 16, 1000)
    assert b > a > 0


def test_missing_library_raises_instead_of_falling_back():
    """No CPU path exists: without the shared library the first call fails."""
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "from paged_kv_cache_435_b200 import _native\n"
        "_native.LIB_PATH = '/nonexistent/libpagedattn.so'\n"
        "try:\n"
        "    _native.raw()\n"
        "except ImportError as e:\n"
        "    print('raised', e)\n"
        "else:\n"
        "    print('loaded')\n" % ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True,
                         text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.startswith("raised"), out.stdout


def test_cpu_tensors_are_rejected_not_computed():
    import torch
    import paged_kv_cache_435_b200 as pa
    q = torch.zeros(1, 4, 64, dtype=torch.bfloat16)
    pool = torch.zeros(4, 16, 4, 64, dtype=torch.bfloat16)
    out = torch.zeros(1, 4, 64, dtype=torch.float32)
    with pytest.raises(TypeError, match="CUDA"):
        pa.pa_decode_attention(out, q, pool, pool, torch.zeros(1, 1, dtype=torch.int32),
                               torch.ones(1, dtype=torch.int32), 1, 0.125)
