"""Paged decode attention for NVIDIA B200 (sm_100a).

The product is ``libpagedattn.so`` (C ABI in ``include/pa.h``); its entry
points are bound here under the same names:

* ``pa_reshape_and_cache``: write each new token's K/V into its paged-cache
  slot;
* ``pa_decode_attention``: one-query-token-per-sequence attention over the
  paged K/V pool through per-sequence block tables (GQA folded, split-KV for
  long contexts);
* ``pa_copy_blocks``: copy-on-write block copies;
* ``pa_multi_query_attention``: k causal query tokens per sequence (chunked
  prefill chunks, speculative-decoding verification);
* ``pa_swap_blocks``: whole-block moves between GPU and pinned CPU pools
  (preemption by swapping);
* ``pa_decode_attention_shared_prefix``: decode attention that reads the
  prompt blocks shared by a group of sequences (parallel samples, beams)
  once for the whole group;
* ``pa_decode_attention_static_ws``: ``pa_decode_attention`` with scratch
  built into the library, for callers that cannot allocate device memory.

``inputs`` builds seeded synthetic workloads.  The library is loaded lazily on
first use and its absence raises; nothing here computes on the CPU.
"""
from ._native import (  # noqa: F401
    PA_DEVERR_BLOCK_ID, PA_DEVERR_CONTEXT_LEN, PA_DEVERR_COPY_PAIR,
    PA_DEVERR_SLOT, PA_DEVERR_TIMEOUT, PA_ERR_CUDA, PA_ERR_INVALID_ARG,
    PA_DEVERR_PREFIX, PA_DEVERR_QUERY_LEN, PA_ERR_UNSUPPORTED,
    PA_ERR_WORKSPACE, PA_OK, PAError, library_path,
    pa_copy_blocks, pa_decode_attention, pa_decode_attention_shared_prefix,
    pa_decode_attention_static_ws,
    pa_decode_partition_size, pa_shared_prefix_workspace_size,
    pa_decode_workspace_size, pa_launch_count, pa_multi_query_attention,
    pa_reshape_and_cache, pa_swap_blocks, raw, status_string)
