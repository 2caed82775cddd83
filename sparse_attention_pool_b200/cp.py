"""Context-parallel decode over torch.distributed.

One long sequence's compressed entries are split over the W ranks of a
process group in contiguous shards, one per rank; each rank compresses and
holds only its shard (the review's section 3-2 (4) lists contextual
parallelism among the inference infrastructure; this exchange is the
library's own).  Every entry of the global top-k is in the top-k of its own
shard, so one decode step is exact:

  1. ``cp_decode_candidates``: this rank's exact local top-k, with the order
     key and global index of each winner;
  2. one all-gather of the candidates (k per rank and sequence, packed with
     their global indices and counts in one int32 buffer);
  3. ``cp_decode_merge_select``: the global top-k, and this rank's share;
  4. CSA attention over the share and HCA attention over the HCA shard, each
     with its log-sum-exp;
  5. one all-gather of the partials (outputs and lse of both branches packed
     in one byte buffer) and one W-way log-sum-exp merge (``attn_lse_merge_n``).

Two collectives per step: at decode sizes their latency, not their bytes,
is what they cost.

Every rank ends with the same outputs and the same selection.  The compute
runs in the library's kernels; this module holds the host logic: the shard
boundaries and the collectives (NCCL over NVLink on B200s; any backend whose
``all_gather`` takes tensors on the data's device).
"""
from __future__ import annotations

import contextlib

import torch
import torch.distributed as dist

from . import api as S
from ._lib import SA_OP_CP_CANDIDATES, SA_OP_DENSE_ATTN, SA_OP_SPARSE_ATTN

HCA_BLOCK = 128  # shard boundaries fall on whole HCA blocks (hence whole CSA blocks)


def shard_bounds(length: int, world: int, align: int = HCA_BLOCK) -> list[tuple[int, int]]:
    """Token ranges [t0, t1) of the W shards of a sequence of `length` tokens:
    contiguous, in rank order, covering [0, length), every inner boundary a
    multiple of `align`, with the aligned blocks spread as evenly as that
    allows (the tail of an incomplete block goes to the shard holding the
    last block).  A shard may be empty."""
    if length < 0 or world < 1 or align < 1:
        raise ValueError(f"length={length}, world={world}, align={align}")
    blocks = -(-length // align)
    per, extra = divmod(blocks, world)
    out, b0 = [], 0
    for w in range(world):
        b1 = b0 + per + (1 if w < extra else 0)
        out.append((min(length, b0 * align), min(length, b1 * align)))
        b0 = b1
    return out


def entry_base(bounds: list[tuple[int, int]], rank: int, m: int) -> int:
    """Global index of the first compressed entry of `rank`'s shard (an empty
    shard, which holds no entry, may start anywhere)."""
    t0, t1 = bounds[rank]
    if t0 % m and t1 > t0:
        raise ValueError(f"shard start {t0} is not a multiple of m={m}")
    return t0 // m


def workspace_size(B: int, H: int, Ncap_csa: int, Ncap_hca: int, k: int) -> int:
    """Scratch bytes of one cp_decode_step (its calls run in order on one stream)."""
    return max(S.workspace_size(SA_OP_CP_CANDIDATES, B, 1, H, Ncap_csa, 0, k),
               S.workspace_size(SA_OP_SPARSE_ATTN, B, 1, H, Ncap_csa, 0, k),
               S.workspace_size(SA_OP_DENSE_ATTN, B, 1, H, 0, Ncap_hca, 0))


def candidate_layout(B: int, k: int) -> tuple[int, int, int, int]:
    """One rank's packed candidates, in int32 elements: (offset of the keys,
    of the global indices, of the counts, row length) = [keys B*k | gidx B*k
    | counts B]."""
    return 0, B * k, 2 * B * k, 2 * B * k + B


def partial_layout(B: int, H: int) -> tuple[int, int, int, int]:
    """One rank's packed partials, in bytes: (rows, bytes of the outputs,
    offset of the lse, row length).  rows = 2*B*H (CSA then HCA); the
    [rows][128] bf16 outputs come first, the [rows] fp32 lse at a 16-byte
    boundary after them, the row padded to a multiple of 16 bytes."""
    rows = 2 * B * H
    o_bytes = rows * 128 * 2
    l_off = -(-o_bytes // 16) * 16
    return rows, o_bytes, l_off, -(-(l_off + rows * 4) // 16) * 16


def gather_ranks(t: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather `t` from every rank of the group into one [W, *t.shape]
    tensor, in rank order (each rank's slice written in place)."""
    W = dist.get_world_size(group)
    buf = torch.empty((W,) + tuple(t.shape), dtype=t.dtype, device=t.device)
    dist.all_gather(list(buf.unbind(0)), t.contiguous(), group=group)
    return buf


def cp_decode_step(q, q_idx, csa: S.Cache, hca: S.Cache, base_csa, k: int, ws, *, group=None, scale=0.0,
                   stream=None):
    """One decode step of both branches for B sequences sharded over the group.

    q [B][H][128] and q_idx [B][64] bf16 (the same on every rank); csa / hca:
    this rank's shards (m = 4 / 128); base_csa [B] int32: the global index of
    the CSA shard's entry 0 (entry_base).  Returns (out_csa, out_hca, lse_csa,
    lse_hca, sel_idx, sel_cnt): the outputs of the whole sequence and the
    global selection (ascending global indices, -1 padded), equal on every
    rank.  Kernels and collectives are ordered on one stream: `stream`, made
    current for the step, or the current one."""
    with (torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()):
        return _step(q, q_idx, csa, hca, base_csa, k, ws, group, scale)


def _step(q, q_idx, csa, hca, base_csa, k, ws, group, scale):
    rank = dist.get_rank(group)
    B, H = q.shape[0], q.shape[1]
    dev = q.device
    # candidates: [keys | global indices | counts], one int32 row per rank
    ok, og, oc, ln = candidate_layout(B, k)
    cand = torch.empty(ln, dtype=torch.int32, device=dev)
    S.cp_decode_candidates(q_idx, csa, k, base_csa, ws, keys=cand[ok:og].view(B, k), gidx=cand[og:oc].view(B, k),
                           gcnt=cand[oc:ln])
    local_idx, local_cnt, sel_idx, sel_cnt = S.cp_decode_merge_select_packed(gather_ranks(cand, group), B, k, rank,
                                                                             base_csa)
    # partials: both branches' [2][B][H][128] bf16 outputs, then their [2][B][H] fp32 lse
    rows, o_bytes, l_off, row_bytes = partial_layout(B, H)
    part = torch.empty(row_bytes, dtype=torch.uint8, device=dev)
    part_o = part[:o_bytes].view(torch.bfloat16).view(2, B, H, 128)
    part_l = part[l_off:l_off + rows * 4].view(torch.float32).view(2, B, H)
    S.csa_sparse_attn(q, csa, local_idx, local_cnt, k, ws, scale=scale, out=part_o[0], lse=part_l[0])
    S.hca_dense_attn(q, hca, ws, scale=scale, out=part_o[1], lse=part_l[1])
    # both branches merge row by row in one launch
    out, lse = S.attn_lse_merge_n_packed(gather_ranks(part, group), rows, l_off)
    out, lse = out.view(2, B, H, 128), lse.view(2, B, H)
    return out[0], out[1], lse[0], lse[1], sel_idx, sel_cnt
