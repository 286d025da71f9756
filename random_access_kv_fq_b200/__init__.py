"""FibQuant KV-cache codec for NVIDIA B200 (sm_100a).

The compute path is libfq.so (hand-written CUDA behind the C ABI of include/fq.h); this package
holds its thin ctypes binding (``_lib``), the table loader (``tables``), the seeded synthetic
workloads (``workloads``) and the in-tree build step (``build``).  Importing the package does
not load the library; the first compute call does, and raises if it is missing.
"""
from ._lib import (FQ_ATTN_NOALLOC_SCRATCH_BYTES, FQ_F16, FQ_F32, FQ_INDEX_EXACT,  # noqa: F401
                   FQ_INDEX_TENSOR, FQ_INDEX_TOPC, FQ_RESCALE_MSE, FQ_RESCALE_PLAIN,
                   FQ_RESCALE_UNBIASED, FQError,
                   fq_attn_decode, fq_attn_decode_append, fq_attn_decode_lengths,
                   fq_attn_decode_noalloc, fq_decode_gather, fq_decode_prod, fq_decode_rescaled,
                   fq_encode_prod, fq_encode_rho, fq_attn_workspace_bytes, fq_build_search_index, fq_decode,
                   fq_encode, fq_padded_dim, fq_payload_bytes, fq_wait_status, lib,
                   status_string)
