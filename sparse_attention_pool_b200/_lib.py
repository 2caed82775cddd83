"""ctypes view of libsparse_attn.so: the C structs and function signatures of
include/sparse_attn.h, nothing else.  Loading fails loudly if the library has
not been built; there is no fallback implementation."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsparse_attn.so")
TRACE_LIB_PATH = os.path.join(HERE, "libsparse_attn_trace.so")  # loaded instead when SA_TRACE_LIB=1

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_WORKSPACE, SA_ERR_CUDA, SA_ERR_TIMEOUT, SA_ERR_DEVICE = range(7)
SA_BF16, SA_FP8_E4M3, SA_KV_MIXED = 0, 1, 2
SA_OP_INDEX_TOPK, SA_OP_SPARSE_ATTN, SA_OP_DENSE_ATTN, SA_OP_HYBRID_DECODE, SA_OP_HYBRID_PREFILL = 1, 2, 3, 4, 5
SA_OP_WINDOW_ATTN = 6
SA_OP_CP_CANDIDATES = 7
SA_OP_HYBRID_DECODE_SWA = 8

STATUS_NAMES = {0: "SA_OK", 1: "SA_ERR_INVALID_ARG", 2: "SA_ERR_UNSUPPORTED", 3: "SA_ERR_WORKSPACE",
                4: "SA_ERR_CUDA", 5: "SA_ERR_TIMEOUT", 6: "SA_ERR_DEVICE"}

# every symbol the header declares
EXPORTS = ["csa_compress", "hca_compress", "csa_index_topk", "csa_sparse_attn", "hca_dense_attn",
           "hybrid_attn_decode", "hybrid_attn_prefill", "sa_workspace_size", "sa_read_device_status",
           "sa_last_error", "sa_abi_version", "sa_set_stage_events", "sa_launch_count",
           "csa_index_topk_noalloc", "csa_append", "hca_append", "swa_attn", "attn_lse_merge",
           "csa_index_quantize_mxfp4", "csa_index_topk_mxfp4", "hybrid_attn_decode_mxfp4",
           "cp_decode_candidates", "cp_decode_merge_select", "attn_lse_merge_n", "hybrid_attn_decode_swa",
           "sa_selftest_wait_timeout", "sa_trace_install", "sa_trace_count", "hybrid_attn_prefill_mxfp4",
           "sa_set_option", "sa_get_option", "sa_decode_io_layout", "sa_decode_graph_create",
           "sa_decode_graph_step", "sa_decode_graph_destroy"]
SA_NOALLOC_SCRATCH_BYTES = 32 << 20
SA_STAGE_INDEX_SCORE, SA_STAGE_TOPK_SELECT, SA_STAGE_CSA_ATTN, SA_STAGE_HCA_ATTN = 0, 1, 2, 3
SA_OPT_PREFILL_SELECT = 1
SA_OPT_DECODE_FAST = 2
SA_OPT_HCA_PREFILL = 3
SA_DG_KERNEL_IN, SA_DG_DIRECT_OUT = 1, 2

P = ctypes.c_void_p
I32 = ctypes.c_int32
F32 = ctypes.c_float
SZ = ctypes.c_size_t


class SaRaw(ctypes.Structure):
    _fields_ = [("k", P), ("v", P), ("kidx", P), ("len", P),
                ("B", I32), ("Lcap", I32), ("d", I32), ("d_idx", I32)]


class SaCache(ctypes.Structure):
    _fields_ = [("k", P), ("v", P), ("k_scale", P), ("v_scale", P), ("kidx", P), ("n", P),
                ("B", I32), ("Ncap", I32), ("d", I32), ("d_idx", I32), ("m", I32), ("dtype", I32)]


class SaDecodeIO(ctypes.Structure):
    _fields_ = [(n, SZ) for n in ("in_bytes", "q_idx_off", "q_off", "out_bytes", "out_hca_off", "lse_hca_off",
                                  "out_csa_off", "lse_csa_off")]


class SparseAttnError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn} -> {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None


def lib():
    """The loaded library (raises if it is missing)."""
    global _lib
    if _lib is None:
        path = TRACE_LIB_PATH if os.environ.get("SA_TRACE_LIB") == "1" else LIB_PATH
        if not os.path.exists(path):
            raise ImportError(f"{os.path.basename(path)} is not built ({path}); run "
                              f"`python -m sparse_attention_pool_b200.build`")
        L = ctypes.CDLL(path)
        RP, CP = ctypes.POINTER(SaRaw), ctypes.POINTER(SaCache)
        L.csa_compress.argtypes = [RP, CP, P]
        L.hca_compress.argtypes = [RP, CP, P]
        L.csa_append.argtypes = [RP, CP, I32, P]
        L.swa_attn.argtypes = [P, I32, I32, P, RP, I32, F32, P, P, P, SZ, P]
        L.attn_lse_merge.argtypes = [P, P, P, P, ctypes.c_int64, P, P, P]
        L.hca_append.argtypes = [RP, CP, I32, P]
        L.csa_index_topk.argtypes = [P, I32, P, CP, I32, P, P, P, SZ, P]
        L.csa_index_topk_noalloc.argtypes = [P, CP, I32, P, P, P]
        L.csa_index_quantize_mxfp4.argtypes = [CP, I32, P, P, P]
        L.csa_index_topk_mxfp4.argtypes = [P, I32, P, CP, P, P, I32, P, P, P, SZ, P]
        L.csa_sparse_attn.argtypes = [P, I32, I32, CP, P, P, I32, F32, P, P, P, SZ, P]
        L.hca_dense_attn.argtypes = [P, I32, I32, P, CP, F32, P, P, P, SZ, P]
        L.hybrid_attn_decode.argtypes = [P, P, I32, CP, CP, I32, F32, P, P, P, P, P, P, P, SZ, P]
        L.cp_decode_candidates.argtypes = [P, CP, I32, P, P, P, P, P, SZ, P]
        I64 = ctypes.c_int64
        L.cp_decode_merge_select.argtypes = [P, P, P, I64, I64, I32, I32, I32, I32, P, P, P, P, P, P]
        L.attn_lse_merge_n.argtypes = [P, P, I32, I64, I64, I64, P, P, P]
        L.hybrid_attn_decode_swa.argtypes = [P, P, I32, CP, CP, RP, I32, I32, F32, P, P, P, P, P, P, P, SZ, P]
        L.hybrid_attn_prefill_mxfp4.argtypes = [P, P, I32, I32, CP, CP, P, P, I32, F32, P, P, P, P, P, P, P, SZ, P]
        L.hybrid_attn_decode_mxfp4.argtypes = [P, P, I32, CP, CP, P, P, I32, F32, P, P, P, P, P, P, P, SZ, P]
        L.hybrid_attn_prefill.argtypes = [P, P, I32, I32, CP, CP, I32, F32, P, P, P, P, P, P, P, SZ, P]
        L.sa_workspace_size.argtypes = [I32, I32, I32, I32, I32, I32, I32]
        L.sa_workspace_size.restype = SZ
        L.sa_read_device_status.argtypes = [P]
        L.sa_last_error.argtypes = []
        L.sa_last_error.restype = ctypes.c_char_p
        L.sa_abi_version.argtypes = []
        L.sa_abi_version.restype = I32
        L.sa_set_stage_events.argtypes = [I32, P, P]
        L.sa_selftest_wait_timeout.argtypes = [ctypes.c_uint32, P]
        L.sa_trace_install.argtypes = [P, ctypes.c_uint32, P]
        L.sa_trace_count.argtypes = [ctypes.POINTER(ctypes.c_uint32), P]
        L.sa_set_option.argtypes = [I32, ctypes.c_int64]
        L.sa_get_option.argtypes = [I32, ctypes.POINTER(ctypes.c_int64)]
        L.sa_launch_count.argtypes = []
        L.sa_decode_io_layout.argtypes = [I32, I32, ctypes.POINTER(SaDecodeIO)]
        L.sa_decode_graph_create.argtypes = [CP, CP, I32, I32, F32, P, P, P, P, P, P, P, P, P, SZ,
                                             ctypes.c_uint32, ctypes.POINTER(P)]
        L.sa_decode_graph_step.argtypes = [P, P]
        L.sa_decode_graph_destroy.argtypes = [P]
        L.sa_launch_count.restype = ctypes.c_uint64
        for name in EXPORTS:
            if name not in ("sa_workspace_size", "sa_last_error", "sa_abi_version", "sa_launch_count"):
                getattr(L, name).restype = I32
        _lib = L
    return _lib


def check(fn: str, status: int):
    if status != SA_OK:
        raise SparseAttnError(fn, status, lib().sa_last_error().decode(errors="replace"))
