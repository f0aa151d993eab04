"""B200-native causal GQA + RoPE (+ QK-RMSNorm): prefill and KV-cache decode.

The compute lives in libgqa.so (hand-written sm_100a CUDA behind the C ABI of
include/gqa.h); this package is its thin Python binding plus the seeded
workload generator used by the tests and the benchmark.
"""
from . import inputs  # noqa: F401
from .decode_graph import DecodeGraph  # noqa: F401
from ._lib import (GQA_DEV_BAD_LEN, GQA_DEV_CAPACITY, GQA_DEV_TIMEOUT,  # noqa: F401
                   LIB_PATH, SIGNATURES, GqaError, RopeScaling, decode_workspace,
                   gqa_attention_backward, gqa_backward_workspace_bytes, gqa_decode,
                   gqa_decode_noalloc, gqa_decode_workspace_bytes, gqa_doc_start, gqa_prefill,
                   gqa_prefill_chunk, gqa_prefill_docs, gqa_prefill_lse, gqa_rope_append,
                   gqa_rope_apply, kv_cache_append, load, status_string)
