"""Thin Python binding of libsparse_attn.so.

Every function here only marshals torch tensors (device memory owned by the
caller) into the C ABI of include/sparse_attn.h and raises on a non-OK
status; every step of the computation runs in the library's CUDA kernels.
Function names follow the C entry points.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import SaCache, SaRaw, check, lib

D, D_IDX = 128, 64
MIXED_K_ROW = 192  # bytes of a mixed-storage K row


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, dtype, name):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise TypeError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    return t


@dataclass
class Cache:
    """A compressed KV cache (caller-owned device tensors) and its descriptor."""
    k: torch.Tensor
    v: torch.Tensor
    n: torch.Tensor
    m: int
    kidx: torch.Tensor | None = None
    k_scale: torch.Tensor | None = None
    v_scale: torch.Tensor | None = None

    @property
    def B(self):
        return self.k.shape[0]

    @property
    def Ncap(self):
        return self.k.shape[1]

    @property
    def fp8(self):
        """e4m3 storage (with per-64-entry scales), plain or mixed."""
        return self.k.dtype == torch.uint8

    @property
    def mixed(self):
        """Mixed storage: K rows of 192 bytes (64 e4m3 codes, then the 64 rotary
        dims in bf16), V in e4m3."""
        return self.k.dtype == torch.uint8 and self.k.shape[2] == MIXED_K_ROW

    def struct(self) -> SaCache:
        dtype = _lib.SA_KV_MIXED if self.mixed else _lib.SA_FP8_E4M3 if self.fp8 else _lib.SA_BF16
        return SaCache(_ptr(self.k), _ptr(self.v), _ptr(self.k_scale), _ptr(self.v_scale), _ptr(self.kidx),
                       _ptr(self.n), self.B, self.Ncap, D, D_IDX, self.m, dtype)


def alloc_cache(B: int, Ncap: int, m: int, *, fp8: bool = False, with_kidx: bool = False, mixed: bool = False,
                device="cuda") -> Cache:
    """A zeroed cache: bf16, e4m3 (fp8=True) or mixed storage (mixed=True)."""
    fp8 = fp8 or mixed
    kv_dtype = torch.uint8 if fp8 else torch.bfloat16
    nG = (Ncap + 63) // 64
    return Cache(
        k=torch.zeros(B, Ncap, MIXED_K_ROW if mixed else D, dtype=kv_dtype, device=device),
        v=torch.zeros(B, Ncap, D, dtype=kv_dtype, device=device),
        n=torch.zeros(B, dtype=torch.int32, device=device),
        m=m,
        kidx=torch.zeros(B, Ncap, D_IDX, dtype=torch.bfloat16, device=device) if with_kidx else None,
        k_scale=torch.zeros(B, max(nG, 1), dtype=torch.float32, device=device) if fp8 else None,
        v_scale=torch.zeros(B, max(nG, 1), dtype=torch.float32, device=device) if fp8 else None,
    )


def _raw(k, v, kidx, lengths):
    _need(k, torch.bfloat16, "k")
    _need(v, torch.bfloat16, "v")
    _need(lengths, torch.int32, "lengths")
    if kidx is not None:
        _need(kidx, torch.bfloat16, "kidx")
    B, Lcap = k.shape[0], k.shape[1]
    return SaRaw(_ptr(k), _ptr(v), _ptr(kidx), _ptr(lengths), B, Lcap, D, D_IDX)


def csa_compress(k, v, kidx, lengths, cache: Cache, stream=None):
    raw = _raw(k, v, kidx, lengths)
    cs = cache.struct()
    check("csa_compress", lib().csa_compress(ctypes.byref(raw), ctypes.byref(cs), _stream(stream)))


def hca_compress(k, v, lengths, cache: Cache, stream=None):
    raw = _raw(k, v, None, lengths)
    cs = cache.struct()
    check("hca_compress", lib().hca_compress(ctypes.byref(raw), ctypes.byref(cs), _stream(stream)))


def csa_append(k, v, kidx, lengths, cache: Cache, max_new_tokens: int, stream=None):
    """Brings a CSA cache up to date with raw sequences that have grown by at most
    max_new_tokens tokens each since cache.n was set (bit-identical to a full
    csa_compress of the new lengths)."""
    raw = _raw(k, v, kidx, lengths)
    cs = cache.struct()
    check("csa_append", lib().csa_append(ctypes.byref(raw), ctypes.byref(cs), int(max_new_tokens), _stream(stream)))


def hca_append(k, v, lengths, cache: Cache, max_new_tokens: int, stream=None):
    """As csa_append, for an HCA cache (k and v only)."""
    raw = _raw(k, v, None, lengths)
    cs = cache.struct()
    check("hca_append", lib().hca_append(ctypes.byref(raw), ctypes.byref(cs), int(max_new_tokens), _stream(stream)))


def swa_attn(q, k_raw, v_raw, lengths, window: int, ws, *, q_pos=None, scale=0.0, out=None, lse=None, stream=None):
    """Sliding-window branch: attention over the last `window` raw tokens visible
    to each query (q [B][H][128] for decode, or [B][Tq][H][128] with q_pos)."""
    _need(q, torch.bfloat16, "q")
    Tq, H = (q.shape[1] if q.dim() == 4 else 1), q.shape[-2]
    if out is None:
        out = torch.empty_like(q)
    raw = _raw(k_raw, v_raw, None, lengths)
    check("swa_attn", lib().swa_attn(_ptr(q), Tq, H, _ptr(q_pos), ctypes.byref(raw), int(window), float(scale),
                                     _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def attn_lse_merge(out_a, lse_a, out_b, lse_b, *, out=None, lse=None, stream=None):
    """Attention over the union of two disjoint key sets from the two partial
    attentions (outputs [..., 128] bf16 and their natural-log lse [...])."""
    _need(out_a, torch.bfloat16, "out_a")
    _need(out_b, torch.bfloat16, "out_b")
    _need(lse_a, torch.float32, "lse_a")
    _need(lse_b, torch.float32, "lse_b")
    if out is None:
        out = torch.empty_like(out_a)
    check("attn_lse_merge", lib().attn_lse_merge(_ptr(out_a), _ptr(lse_a), _ptr(out_b), _ptr(lse_b),
                                                 lse_a.numel(), _ptr(out), _ptr(lse), _stream(stream)))
    return out


def workspace_size(op: int, B: int, Tq: int, H: int, Ncap_csa: int, Ncap_hca: int, k: int) -> int:
    return int(lib().sa_workspace_size(op, B, Tq, H, Ncap_csa, Ncap_hca, k))


def alloc_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Zeroed scratch; torch's allocator returns 512-byte aligned blocks."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def csa_index_topk(q_idx, csa: Cache, k: int, ws, *, q_pos=None, idx=None, cnt=None, stream=None):
    _need(q_idx, torch.bfloat16, "q_idx")
    B = csa.B
    Tq = 1 if q_pos is None else q_idx.shape[1]
    if idx is None:
        idx = torch.empty(B, Tq, k, dtype=torch.int32, device=q_idx.device)
    if cnt is None:
        cnt = torch.empty(B, Tq, dtype=torch.int32, device=q_idx.device)
    cs = csa.struct()
    check("csa_index_topk", lib().csa_index_topk(_ptr(q_idx), Tq, _ptr(q_pos), ctypes.byref(cs), k, _ptr(idx),
                                                 _ptr(cnt), _ptr(ws), ws.numel(), _stream(stream)))
    return idx, cnt


def csa_index_topk_noalloc(q_idx, csa: Cache, k: int, *, idx=None, cnt=None, stream=None):
    """Decode top-k without a workspace: the library's static device scratch is
    used instead (for callers that cannot allocate; see the C header)."""
    _need(q_idx, torch.bfloat16, "q_idx")
    B = csa.B
    if idx is None:
        idx = torch.empty(B, 1, k, dtype=torch.int32, device=q_idx.device)
    if cnt is None:
        cnt = torch.empty(B, 1, dtype=torch.int32, device=q_idx.device)
    cs = csa.struct()
    check("csa_index_topk_noalloc", lib().csa_index_topk_noalloc(_ptr(q_idx), ctypes.byref(cs), k, _ptr(idx),
                                                                 _ptr(cnt), _stream(stream)))
    return idx, cnt


def csa_index_quantize_mxfp4(csa: Cache, *, codes=None, scales=None, row_from: int = 0, stream=None):
    """MXFP4 copy of the cache's bf16 indexer keys (entries row_from .. n-1):
    codes [B][Ncap][32] uint8 (two e2m1 per byte, even element low), scales
    [B][Ncap][2] uint8 (E8M0).  Returns (codes, scales)."""
    dev = csa.k.device
    if codes is None:
        codes = torch.zeros(csa.B, csa.Ncap, 32, dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.zeros(csa.B, csa.Ncap, 2, dtype=torch.uint8, device=dev)
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.uint8, "scales")
    cs = csa.struct()
    check("csa_index_quantize_mxfp4", lib().csa_index_quantize_mxfp4(ctypes.byref(cs), int(row_from), _ptr(codes),
                                                                     _ptr(scales), _stream(stream)))
    return codes, scales


def csa_index_topk_mxfp4(q_idx, csa: Cache, codes, scales, k: int, ws, *, q_pos=None, idx=None, cnt=None,
                         stream=None):
    """Top-k on FP4 (MXFP4) indexer scores, decode (q_pos None: q_idx [B][64])
    or causal prefill (q_idx [B][T][64], q_pos [B][T]); idx [B][Tq][k], cnt
    [B][Tq]."""
    _need(q_idx, torch.bfloat16, "q_idx")
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.uint8, "scales")
    B = csa.B
    Tq = 1 if q_pos is None else q_idx.shape[1]
    if idx is None:
        idx = torch.empty(B, Tq, k, dtype=torch.int32, device=q_idx.device)
    if cnt is None:
        cnt = torch.empty(B, Tq, dtype=torch.int32, device=q_idx.device)
    cs = csa.struct()
    check("csa_index_topk_mxfp4", lib().csa_index_topk_mxfp4(_ptr(q_idx), Tq, _ptr(q_pos), ctypes.byref(cs),
                                                             _ptr(codes), _ptr(scales), k, _ptr(idx), _ptr(cnt),
                                                             _ptr(ws), ws.numel(), _stream(stream)))
    return idx, cnt


def cp_decode_candidates(q_idx, csa: Cache, k: int, base, ws, *, keys=None, gidx=None, gcnt=None, stream=None):
    """This rank's exact local top-k with the order keys and global indices of
    its winners: (keys [B][k] int32 holding the uint32 order keys, gidx [B][k],
    gcnt [B])."""
    _need(q_idx, torch.bfloat16, "q_idx")
    _need(base, torch.int32, "base")
    B, dev = csa.B, q_idx.device
    keys = torch.empty(B, k, dtype=torch.int32, device=dev) if keys is None else keys
    gidx = torch.empty(B, k, dtype=torch.int32, device=dev) if gidx is None else gidx
    gcnt = torch.empty(B, dtype=torch.int32, device=dev) if gcnt is None else gcnt
    cs = csa.struct()
    check("cp_decode_candidates", lib().cp_decode_candidates(_ptr(q_idx), ctypes.byref(cs), k, _ptr(base), _ptr(keys),
                                                             _ptr(gidx), _ptr(gcnt), _ptr(ws), ws.numel(),
                                                             _stream(stream)))
    return keys, gidx, gcnt


def cp_decode_merge_select(keys, gidx, gcnt, rank: int, base, *, local_idx=None, local_cnt=None, sel_idx=None,
                           sel_cnt=None, stream=None):
    """From the candidates of all ranks stacked in rank order (keys, gidx
    [W][B][k], gcnt [W][B]): (local_idx [B][k], local_cnt [B], sel_idx [B][k],
    sel_cnt [B]), this rank's share of the global top-k and the selection."""
    for t, name in ((keys, "keys"), (gidx, "gidx"), (gcnt, "gcnt"), (base, "base")):
        _need(t, torch.int32, name)
    W, B, k = gidx.shape
    return _merge_select(keys.data_ptr(), gidx.data_ptr(), gcnt.data_ptr(), B * k, B, W, B, k, rank, base,
                         gidx.device, local_idx, local_cnt, sel_idx, sel_cnt, stream)


def cp_decode_merge_select_packed(gathered, B: int, k: int, rank: int, base, *, stream=None):
    """The same from one gathered int32 buffer [W][L], rank w's row holding its
    packed [keys B*k | gidx B*k | gcnt B] (L >= 2*B*k + B)."""
    _need(gathered, torch.int32, "gathered")
    _need(base, torch.int32, "base")
    W, L = gathered.shape
    p = gathered.data_ptr()
    return _merge_select(p, p + 4 * B * k, p + 8 * B * k, L, L, W, B, k, rank, base, gathered.device,
                         None, None, None, None, stream)


def _merge_select(pk, pg, pc, stride_list, stride_cnt, W, B, k, rank, base, dev, local_idx, local_cnt, sel_idx,
                  sel_cnt, stream):
    local_idx = torch.empty(B, k, dtype=torch.int32, device=dev) if local_idx is None else local_idx
    local_cnt = torch.empty(B, dtype=torch.int32, device=dev) if local_cnt is None else local_cnt
    sel_idx = torch.empty(B, k, dtype=torch.int32, device=dev) if sel_idx is None else sel_idx
    sel_cnt = torch.empty(B, dtype=torch.int32, device=dev) if sel_cnt is None else sel_cnt
    P = ctypes.c_void_p
    check("cp_decode_merge_select",
          lib().cp_decode_merge_select(P(pk), P(pg), P(pc), stride_list, stride_cnt, W, B, k, rank, _ptr(base),
                                       _ptr(local_idx), _ptr(local_cnt), _ptr(sel_idx), _ptr(sel_cnt),
                                       _stream(stream)))
    return local_idx, local_cnt, sel_idx, sel_cnt


def attn_lse_merge_n(outs, lses, *, out=None, lse=None, stream=None):
    """W-way log-sum-exp merge: outs [W][..][128] bf16, lses [W][..] fp32 ->
    (out [..][128], lse [..])."""
    _need(outs, torch.bfloat16, "outs")
    _need(lses, torch.float32, "lses")
    W = outs.shape[0]
    rows = lses[0].numel()
    out = torch.empty(outs.shape[1:], dtype=torch.bfloat16, device=outs.device) if out is None else out
    lse = torch.empty(lses.shape[1:], dtype=torch.float32, device=outs.device) if lse is None else lse
    check("attn_lse_merge_n", lib().attn_lse_merge_n(_ptr(outs), _ptr(lses), W, rows, rows * 128, rows, _ptr(out),
                                                     _ptr(lse), _stream(stream)))
    return out, lse


def attn_lse_merge_n_packed(gathered, rows: int, lse_offset: int, *, out=None, lse=None, stream=None):
    """The same from one gathered byte buffer [W][L]: part w's [rows][128]
    bf16 outputs at byte 0 of its row and its [rows] fp32 lse at byte
    lse_offset (L a multiple of 16)."""
    _need(gathered, torch.uint8, "gathered")
    W, L = gathered.shape
    if L % 16 or lse_offset % 4:
        raise ValueError("packed partials: row bytes must be a multiple of 16, the lse offset of 4")
    dev = gathered.device
    out = torch.empty(rows, 128, dtype=torch.bfloat16, device=dev) if out is None else out
    lse = torch.empty(rows, dtype=torch.float32, device=dev) if lse is None else lse
    p = gathered.data_ptr()
    check("attn_lse_merge_n", lib().attn_lse_merge_n(ctypes.c_void_p(p), ctypes.c_void_p(p + lse_offset), W, rows,
                                                     L // 2, L // 4, _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def csa_sparse_attn(q, csa: Cache, idx, cnt, k: int, ws, *, scale=0.0, out=None, lse=None, stream=None):
    _need(q, torch.bfloat16, "q")
    B, Tq, H = q.shape[0], (q.shape[1] if q.dim() == 4 else 1), q.shape[-2]
    if out is None:
        out = torch.empty_like(q)
    cs = csa.struct()
    check("csa_sparse_attn", lib().csa_sparse_attn(_ptr(q), Tq, H, ctypes.byref(cs), _ptr(idx), _ptr(cnt), k,
                                                   float(scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                                   _stream(stream)))
    return out


def hca_dense_attn(q, hca: Cache, ws, *, q_pos=None, scale=0.0, out=None, lse=None, stream=None):
    _need(q, torch.bfloat16, "q")
    Tq, H = (q.shape[1] if q.dim() == 4 else 1), q.shape[-2]
    if out is None:
        out = torch.empty_like(q)
    cs = hca.struct()
    check("hca_dense_attn", lib().hca_dense_attn(_ptr(q), Tq, H, _ptr(q_pos), ctypes.byref(cs), float(scale),
                                                 _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def hybrid_attn_decode(q, q_idx, csa: Cache, hca: Cache, k: int, ws, *, scale=0.0, out_csa=None, out_hca=None,
                       lse_csa=None, lse_hca=None, idx_out=None, cnt_out=None, stream=None):
    """q [B][H][128] bf16, q_idx [B][64] bf16 -> (out_csa, out_hca) [B][H][128] bf16."""
    _need(q, torch.bfloat16, "q")
    _need(q_idx, torch.bfloat16, "q_idx")
    H = q.shape[1]
    out_csa = torch.empty_like(q) if out_csa is None else out_csa
    out_hca = torch.empty_like(q) if out_hca is None else out_hca
    c, h = csa.struct(), hca.struct()
    check("hybrid_attn_decode",
          lib().hybrid_attn_decode(_ptr(q), _ptr(q_idx), H, ctypes.byref(c), ctypes.byref(h), k, float(scale),
                                   _ptr(out_csa), _ptr(out_hca), _ptr(lse_csa), _ptr(lse_hca), _ptr(idx_out),
                                   _ptr(cnt_out), _ptr(ws), ws.numel(), _stream(stream)))
    return out_csa, out_hca


def hybrid_attn_decode_swa(q, q_idx, csa: Cache, hca: Cache, k_raw, v_raw, lengths, window: int, k: int, ws, *,
                           scale=0.0, out_csa=None, out_hca=None, lse_csa=None, lse_hca=None, idx_out=None,
                           cnt_out=None, stream=None):
    """hybrid_attn_decode with the sliding-window branch of both layers: each
    output is the attention over its branch joined with the last `window` raw
    tokens (k_raw, v_raw [B][Lcap][128] bf16, lengths [B] int32)."""
    _need(q, torch.bfloat16, "q")
    _need(q_idx, torch.bfloat16, "q_idx")
    H = q.shape[1]
    out_csa = torch.empty_like(q) if out_csa is None else out_csa
    out_hca = torch.empty_like(q) if out_hca is None else out_hca
    raw = _raw(k_raw, v_raw, None, lengths)
    c, h = csa.struct(), hca.struct()
    check("hybrid_attn_decode_swa",
          lib().hybrid_attn_decode_swa(_ptr(q), _ptr(q_idx), H, ctypes.byref(c), ctypes.byref(h), ctypes.byref(raw),
                                       int(window), k, float(scale), _ptr(out_csa), _ptr(out_hca), _ptr(lse_csa),
                                       _ptr(lse_hca), _ptr(idx_out), _ptr(cnt_out), _ptr(ws), ws.numel(),
                                       _stream(stream)))
    return out_csa, out_hca


def hybrid_attn_decode_mxfp4(q, q_idx, csa: Cache, hca: Cache, codes, scales, k: int, ws, *, scale=0.0,
                             out_csa=None, out_hca=None, lse_csa=None, lse_hca=None, idx_out=None, cnt_out=None,
                             stream=None):
    """hybrid_attn_decode with the CSA selection on FP4 (MXFP4) indexer scores;
    codes / scales from csa_index_quantize_mxfp4."""
    _need(q, torch.bfloat16, "q")
    _need(q_idx, torch.bfloat16, "q_idx")
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.uint8, "scales")
    H = q.shape[1]
    out_csa = torch.empty_like(q) if out_csa is None else out_csa
    out_hca = torch.empty_like(q) if out_hca is None else out_hca
    c, h = csa.struct(), hca.struct()
    check("hybrid_attn_decode_mxfp4",
          lib().hybrid_attn_decode_mxfp4(_ptr(q), _ptr(q_idx), H, ctypes.byref(c), ctypes.byref(h), _ptr(codes),
                                         _ptr(scales), k, float(scale), _ptr(out_csa), _ptr(out_hca), _ptr(lse_csa),
                                         _ptr(lse_hca), _ptr(idx_out), _ptr(cnt_out), _ptr(ws), ws.numel(),
                                         _stream(stream)))
    return out_csa, out_hca


def hybrid_attn_prefill_mxfp4(q, q_idx, csa: Cache, hca: Cache, codes, scales, k: int, ws, idx_out, cnt_out, *,
                              scale=0.0, out_csa=None, out_hca=None, lse_csa=None, lse_hca=None, stream=None):
    """hybrid_attn_prefill with the CSA selection on FP4 (MXFP4) indexer scores."""
    _need(q, torch.bfloat16, "q")
    _need(q_idx, torch.bfloat16, "q_idx")
    _need(codes, torch.uint8, "codes")
    _need(scales, torch.uint8, "scales")
    T, H = q.shape[1], q.shape[2]
    out_csa = torch.empty_like(q) if out_csa is None else out_csa
    out_hca = torch.empty_like(q) if out_hca is None else out_hca
    c, h = csa.struct(), hca.struct()
    check("hybrid_attn_prefill_mxfp4",
          lib().hybrid_attn_prefill_mxfp4(_ptr(q), _ptr(q_idx), T, H, ctypes.byref(c), ctypes.byref(h), _ptr(codes),
                                          _ptr(scales), k, float(scale), _ptr(out_csa), _ptr(out_hca),
                                          _ptr(lse_csa), _ptr(lse_hca), _ptr(idx_out), _ptr(cnt_out), _ptr(ws),
                                          ws.numel(), _stream(stream)))
    return out_csa, out_hca


def hybrid_attn_prefill(q, q_idx, csa: Cache, hca: Cache, k: int, ws, idx_out, cnt_out, *, scale=0.0,
                        out_csa=None, out_hca=None, lse_csa=None, lse_hca=None, stream=None):
    """q [B][T][H][128] bf16, q_idx [B][T][64] bf16; idx_out [B][T][k], cnt_out [B][T] int32."""
    _need(q, torch.bfloat16, "q")
    _need(q_idx, torch.bfloat16, "q_idx")
    T, H = q.shape[1], q.shape[2]
    out_csa = torch.empty_like(q) if out_csa is None else out_csa
    out_hca = torch.empty_like(q) if out_hca is None else out_hca
    c, h = csa.struct(), hca.struct()
    check("hybrid_attn_prefill",
          lib().hybrid_attn_prefill(_ptr(q), _ptr(q_idx), T, H, ctypes.byref(c), ctypes.byref(h), k, float(scale),
                                    _ptr(out_csa), _ptr(out_hca), _ptr(lse_csa), _ptr(lse_hca), _ptr(idx_out),
                                    _ptr(cnt_out), _ptr(ws), ws.numel(), _stream(stream)))
    return out_csa, out_hca


def set_option(option: int, value: int):
    """A process-wide library option (host-only; applies to calls made
    afterwards).  SA_OPT_PREFILL_SELECT: 1 to 4 (default 4), the prefill top-k's
    selection kernel (the same indices in every form)."""
    check("sa_set_option", lib().sa_set_option(int(option), int(value)))


def get_option(option: int) -> int:
    v = ctypes.c_int64(0)
    check("sa_get_option", lib().sa_get_option(int(option), ctypes.byref(v)))
    return int(v.value)


def read_device_status(stream=None):
    """Synchronises the stream and raises if a kernel recorded a device-side anomaly."""
    check("sa_read_device_status", lib().sa_read_device_status(_stream(stream)))


def selftest_wait_timeout(wait_tries: int = 65536, stream=None):
    """Launch the failure-detection self-test (a bounded wait that cannot
    complete); the next read_device_status raises SA_ERR_TIMEOUT."""
    check("sa_selftest_wait_timeout", lib().sa_selftest_wait_timeout(int(wait_tries), _stream(stream)))


class CapturedDecode:
    """A hybrid decode step captured once into a CUDA graph, for serving loops
    that decode the same batch step after step.

    The graph reads the caches in place (appends between steps are seen) and
    its own static buffers: ``q`` [B][H][128] and ``q_idx`` [B][64] bf16 in,
    ``out_csa`` / ``out_hca`` [B][H][128] bf16, ``lse_csa`` / ``lse_hca`` [B][H]
    fp32, ``idx`` [B][k] / ``cnt`` [B] int32 out.  ``step`` copies new queries
    in (from host or device tensors, asynchronously on the current stream),
    replays the graph and, if given host tensors, copies the outputs out.
    With MXFP4 ``codes`` / ``scales`` the CSA selection runs on FP4 scores.
    """

    def __init__(self, csa: Cache, hca: Cache, k: int, H: int, *, scale: float = 0.0, codes=None, scales=None):
        dev = csa.k.device
        B = csa.B
        self.csa, self.hca, self.k, self.scale = csa, hca, k, scale
        self.codes, self.scales = codes, scales
        self.q = torch.zeros(B, H, D, dtype=torch.bfloat16, device=dev)
        self.q_idx = torch.zeros(B, D_IDX, dtype=torch.bfloat16, device=dev)
        self.out_csa = torch.empty(B, H, D, dtype=torch.bfloat16, device=dev)
        self.out_hca = torch.empty_like(self.out_csa)
        self.lse_csa = torch.empty(B, H, dtype=torch.float32, device=dev)
        self.lse_hca = torch.empty_like(self.lse_csa)
        self.idx = torch.empty(B, k, dtype=torch.int32, device=dev)
        self.cnt = torch.empty(B, dtype=torch.int32, device=dev)
        self.ws = alloc_workspace(workspace_size(_lib.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k), device=dev)
        self._call()  # first call outside the capture: one-time kernel attributes and the side stream
        torch.cuda.synchronize(dev)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self._call()
        torch.cuda.synchronize(dev)

    def _call(self):
        kw = dict(scale=self.scale, out_csa=self.out_csa, out_hca=self.out_hca, lse_csa=self.lse_csa,
                  lse_hca=self.lse_hca, idx_out=self.idx, cnt_out=self.cnt)
        if self.codes is not None:
            hybrid_attn_decode_mxfp4(self.q, self.q_idx, self.csa, self.hca, self.codes, self.scales, self.k, self.ws,
                                     **kw)
        else:
            hybrid_attn_decode(self.q, self.q_idx, self.csa, self.hca, self.k, self.ws, **kw)

    def step(self, q=None, q_idx=None, out_csa=None, out_hca=None, lse_csa=None, lse_hca=None):
        """Copy q / q_idx in (when given), replay, copy outputs to the given
        tensors (when given).  Asynchronous on the current stream."""
        if q is not None:
            self.q.copy_(q.view(torch.bfloat16) if q.dtype == torch.int16 else q, non_blocking=True)
        if q_idx is not None:
            self.q_idx.copy_(q_idx.view(torch.bfloat16) if q_idx.dtype == torch.int16 else q_idx, non_blocking=True)
        self.graph.replay()
        for dst, src in ((out_csa, self.out_csa), (out_hca, self.out_hca), (lse_csa, self.lse_csa),
                         (lse_hca, self.lse_hca)):
            if dst is not None:
                dst.copy_(src.view(dst.dtype) if dst.dtype != src.dtype else src, non_blocking=True)


def decode_io_layout(B: int, H: int) -> _lib.SaDecodeIO:
    """Byte offsets of the packed decode I/O (sa_decode_io_layout)."""
    io = _lib.SaDecodeIO()
    check("sa_decode_io_layout", lib().sa_decode_io_layout(B, H, ctypes.byref(io)))
    return io


class DecodeGraph:
    """sa_decode_graph_*: a hybrid decode step captured by the library into a
    CUDA graph together with its host copies (one H2D copy of the packed
    queries, the HCA outputs copied back from the HCA branch, the CSA outputs
    at the end), launched by one call per step.

    The pinned host buffers are exposed as views: write ``q`` [B][H][128] and
    ``q_idx`` [B][64] (bf16) before ``step``; read ``out_csa`` / ``out_hca``
    [B][H][128] (bf16) and ``lse_csa`` / ``lse_hca`` [B][H] (fp32) once the
    stream has finished the step.  ``idx`` [B][k] / ``cnt`` [B] stay on the
    device.  All buffers are allocated here (torch) and owned by this object.
    ``flags`` (SA_DG_KERNEL_IN, SA_DG_DIRECT_OUT) choose how the I/O moves:
    copy-engine copies (0), a kernel reading the mapped host queries, the
    kernels writing the outputs straight into the mapped host buffer.
    """

    DEFAULT_FLAGS = _lib.SA_DG_KERNEL_IN  # measured fastest on a B200 at 1M context

    def __init__(self, csa: Cache, hca: Cache, k: int, H: int, *, scale: float = 0.0, codes=None, scales=None,
                 flags: int | None = None):
        dev = csa.k.device
        B = csa.B
        self.io = io = decode_io_layout(B, H)
        self.csa, self.hca, self.k, self.H = csa, hca, k, H
        self.codes, self.scales = codes, scales
        self.host_in = torch.zeros(io.in_bytes, dtype=torch.uint8).pin_memory()
        self.host_out = torch.zeros(io.out_bytes, dtype=torch.uint8).pin_memory()
        self.dev_in = torch.zeros(io.in_bytes, dtype=torch.uint8, device=dev)
        self.dev_out = torch.zeros(io.out_bytes, dtype=torch.uint8, device=dev)
        self.idx = torch.empty(B, k, dtype=torch.int32, device=dev)
        self.cnt = torch.empty(B, dtype=torch.int32, device=dev)
        self.ws = alloc_workspace(workspace_size(_lib.SA_OP_HYBRID_DECODE, B, 1, H, csa.Ncap, hca.Ncap, k), device=dev)

        def view(buf, off, shape, dtype):
            n = 1
            for x in shape:
                n *= x
            nb = n * torch.tensor([], dtype=dtype).element_size()
            return buf[off:off + nb].view(dtype).view(*shape)

        self.q_idx = view(self.host_in, io.q_idx_off, (B, D_IDX), torch.bfloat16)
        self.q = view(self.host_in, io.q_off, (B, H, D), torch.bfloat16)
        self.out_hca = view(self.host_out, io.out_hca_off, (B, H, D), torch.bfloat16)
        self.lse_hca = view(self.host_out, io.lse_hca_off, (B, H), torch.float32)
        self.out_csa = view(self.host_out, io.out_csa_off, (B, H, D), torch.bfloat16)
        self.lse_csa = view(self.host_out, io.lse_csa_off, (B, H), torch.float32)
        self.h2d_bytes, self.d2h_bytes = io.in_bytes, io.out_bytes
        self.flags = self.DEFAULT_FLAGS if flags is None else flags
        self._cs, self._hs = csa.struct(), hca.struct()
        handle = ctypes.c_void_p()
        torch.cuda.synchronize(dev)
        check("sa_decode_graph_create",
              lib().sa_decode_graph_create(ctypes.byref(self._cs), ctypes.byref(self._hs), H, k, scale, _ptr(codes),
                                           _ptr(scales), _ptr(self.host_in), _ptr(self.host_out), _ptr(self.dev_in),
                                           _ptr(self.dev_out), _ptr(self.idx), _ptr(self.cnt), _ptr(self.ws),
                                           self.ws.numel(), self.flags, ctypes.byref(handle)))
        self._handle = handle

    def step(self, stream=None):
        """Launch one captured step on the stream (asynchronous)."""
        check("sa_decode_graph_step", lib().sa_decode_graph_step(self._handle, _stream(stream)))

    def close(self):
        if getattr(self, "_handle", None) is not None and self._handle.value:
            check("sa_decode_graph_destroy", lib().sa_decode_graph_destroy(self._handle))
            self._handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001 -- interpreter shutdown
            pass
