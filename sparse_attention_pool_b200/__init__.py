"""B200-native CSA + HCA hybrid attention (libsparse_attn.so + a thin binding).

The compute path is the CUDA library; ``api`` only marshals torch tensors
into its C ABI and ``synth`` only generates seeded inputs.
"""
from .api import (Cache, CapturedDecode, DecodeGraph, alloc_cache, alloc_workspace, attn_lse_merge,  # noqa: F401
                  csa_append, csa_compress, decode_io_layout,
                  csa_index_topk, csa_index_topk_noalloc, hca_append, swa_attn,
                  csa_index_quantize_mxfp4, csa_index_topk_mxfp4, hybrid_attn_decode_mxfp4, hybrid_attn_decode_swa,
                  hybrid_attn_prefill_mxfp4,
                  cp_decode_candidates, cp_decode_merge_select, cp_decode_merge_select_packed, attn_lse_merge_n,
                  attn_lse_merge_n_packed,
                  csa_sparse_attn,
                  hca_compress, hca_dense_attn, hybrid_attn_decode, hybrid_attn_prefill, read_device_status,
                  selftest_wait_timeout, set_option, get_option,
                  workspace_size)
from ._lib import (SA_OP_DENSE_ATTN, SA_OP_HYBRID_DECODE, SA_OP_HYBRID_PREFILL, SA_OP_INDEX_TOPK,  # noqa: F401
                   SA_OP_SPARSE_ATTN, SA_OP_WINDOW_ATTN, SA_OP_CP_CANDIDATES,
                   SA_OP_HYBRID_DECODE_SWA, SA_OPT_DECODE_FAST, SA_OPT_HCA_PREFILL, SA_OPT_PREFILL_SELECT,
                   SparseAttnError)
