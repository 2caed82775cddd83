"""Context-parallel decode on the host: the shard boundaries, the rank-ordered
all-gather of sparse_attention_pool_b200.cp (gloo ranks on CPU), and the
exchange protocol itself -- every rank computing its shard with the oracle,
exchanging packed rows through cp.gather_ranks (cp.candidate_layout,
cp.partial_layout), selecting from the union of the local top-k lists and
merging the partial attentions by log-sum-exp -- against the oracle's
single-rank answer (indices exact; outputs within the bf16 rounding of the
exchanged partials).
"""
from __future__ import annotations

import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_attention_pool_b200 import cp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("length", [0, 1, 127, 128, 129, 1000, 4096, 12345, 1 << 20])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_bounds_cover_contiguously_on_block_boundaries(length, world):
    b = cp.shard_bounds(length, world)
    assert len(b) == world
    assert b[0][0] == 0 and b[-1][1] == length
    for (t0, t1), (u0, _) in zip(b, b[1:]):
        assert t1 == u0 and t0 <= t1
    for t0, t1 in b[:-1]:
        assert t1 % cp.HCA_BLOCK == 0 or t1 == length
    sizes = [-(-(t1 - t0) // cp.HCA_BLOCK) for t0, t1 in b]  # blocks per shard
    assert max(sizes) - min(sizes) <= 1
    for r in range(world):
        if b[r][1] > b[r][0]:
            assert cp.entry_base(b, r, 4) * 4 == b[r][0]
            assert cp.entry_base(b, r, 128) * 128 == b[r][0]


def test_shard_bounds_rejects_bad_arguments():
    with pytest.raises(ValueError):
        cp.shard_bounds(-1, 2)
    with pytest.raises(ValueError):
        cp.shard_bounds(10, 0)
    with pytest.raises(ValueError):
        cp.entry_base([(0, 6), (6, 10)], 1, 4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _order_key(s: np.ndarray) -> np.ndarray:
    """uint32 order key of fp32 scores: sign bit set for s >= 0, all bits
    flipped for s < 0 (scores arrive with -0 already mapped to +0)."""
    u = np.asarray(s, dtype=np.float32).view(np.uint32)
    return np.where(u >> 31, ~u, u | np.uint32(0x80000000)).astype(np.uint32)


def _rank_main(rank, world, port, L, k, out):
    sys.path.insert(0, ROOT)
    from oracle import oracle as O
    from sparse_attention_pool_b200 import cp as CP
    from sparse_attention_pool_b200 import synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        H, sc = 4, 128 ** -0.5
        K = synth.normal_bf16(77, "k", (1, L, 128))[0]
        V = synth.normal_bf16(77, "v", (1, L, 128))[0]
        KI = synth.normal_bf16(77, "kidx", (1, L, 64))[0]
        q = synth.normal_bf16(77, "q", (1, H, 128))[0]
        qI = synth.normal_bf16(77, "qidx", (1, 64))[0]
        bounds = CP.shard_bounds(L, world)
        t0, t1 = bounds[rank]
        base = CP.entry_base(bounds, rank, 4)
        # this rank's shard, compressed on its own
        ck, cv, ci = O.compress(K[t0:t1], 4), O.compress(V[t0:t1], 4), O.compress(KI[t0:t1], 4)
        hk, hv = O.compress(K[t0:t1], 128), O.compress(V[t0:t1], 128)
        # 1. local top-k with order keys and global indices
        s = O.index_scores(qI, ci)
        idx, cnt = O.topk(s, k)
        keys = np.zeros(k, np.uint32)
        gidx = np.full(k, -1, np.int32)
        keys[:cnt] = _order_key(s[idx[:cnt]])
        gidx[:cnt] = base + idx[:cnt]
        # 2. one exchange of the packed candidates (rank order)
        ok_, og, oc_, ln = CP.candidate_layout(1, k)
        row = np.zeros(ln, np.int32)
        row[ok_:og], row[og:oc_], row[oc_] = keys.view(np.int32), gidx, cnt
        allc = CP.gather_ranks(torch.from_numpy(row)).numpy()
        all_keys, all_gidx, all_cnt = allc[:, ok_:og].view(np.uint32), allc[:, og:oc_], allc[:, oc_:oc_ + 1]
        # 3. the global top-k of the union, by plain sorting
        cand = [(int(all_keys[w, i]), int(all_gidx[w, i]))
                for w in range(world) for i in range(int(all_cnt[w, 0]))]
        gl = sorted(cand, key=lambda c: (-c[0], c[1]))[:k]
        sel = sorted(g for _, g in gl)
        mine = [g - base for g in sel if base <= g < base + ck.shape[0]]
        # 4. partial attentions over this rank's share and HCA shard
        oc, lc = O.attention(q, ck, cv, np.asarray(mine, np.int32), sc)
        oh, lh = O.attention(q, hk, hv, np.arange(hk.shape[0], dtype=np.int32), sc)
        # 5. one exchange of the packed partials, then the log-sum-exp merge
        #    (the oracle's fp64 outputs travel as bf16 here, as on the GPU)
        rows, o_bytes, l_off, row_bytes = CP.partial_layout(1, H)
        buf = np.zeros(row_bytes, np.uint8)
        o16 = np.stack([oc, oh]).astype(np.float32).view(np.uint32)
        o16 = ((o16 + 0x7FFF + ((o16 >> 16) & 1)) >> 16).astype(np.uint16)  # RNE to bf16
        buf[:o_bytes] = o16.reshape(-1).view(np.uint8)
        buf[l_off:l_off + rows * 4] = np.stack([lc, lh]).astype(np.float32).reshape(-1).view(np.uint8)
        allp = CP.gather_ranks(torch.from_numpy(buf)).numpy()
        po = (allp[:, :o_bytes].copy().view(np.uint16).astype(np.uint32) << 16).view(np.float32)
        po = po.astype(np.float64).reshape(world, 2, H, 128)
        pl = allp[:, l_off:l_off + rows * 4].copy().view(np.float32).astype(np.float64).reshape(world, 2, H)
        M = pl.max(axis=0)
        wts = np.where(np.isneginf(pl), 0.0, np.exp(pl - np.where(np.isneginf(M), 0.0, M)))
        merged = (wts[..., None] * po).sum(axis=0) / wts.sum(axis=0)[..., None]
        mlse = M + np.log(wts.sum(axis=0))
        out.put((rank, sel, merged, mlse, [int(all_cnt[w, 0]) for w in range(world)]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,L,k", [(2, 6000, 128), (3, 5000, 300), (3, 300, 64)])
def test_exchange_protocol_matches_the_single_rank_oracle(world, L, k):
    from oracle import oracle as O
    from sparse_attention_pool_b200 import synth
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, L, k, q_)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q_.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    H, sc = 4, 128 ** -0.5
    K = synth.normal_bf16(77, "k", (1, L, 128))[0]
    V = synth.normal_bf16(77, "v", (1, L, 128))[0]
    KI = synth.normal_bf16(77, "kidx", (1, L, 64))[0]
    q = synth.normal_bf16(77, "q", (1, H, 128))[0]
    qI = synth.normal_bf16(77, "qidx", (1, 64))[0]
    ref = O.hybrid_query(O.CompressedSeq(K, V, KI), q, qI, t=L, k=k, scale=sc)
    want = ref["idx"][:ref["cnt"]].tolist()
    for rank, sel, merged, mlse, counts in res:
        assert sel == want, rank                      # the same exact selection on every rank
        # partials travelled as bf16 outputs and fp32 lse: the merge is within their rounding
        assert np.abs(merged[0] - ref["out_csa"]).max() < 4e-3, rank
        assert np.abs(merged[1] - ref["out_hca"]).max() < 4e-3, rank
        assert np.abs(mlse[0] - ref["lse_csa"]).max() < 1e-5, rank
        if L >= 128:
            assert np.abs(mlse[1] - ref["lse_hca"]).max() < 1e-5, rank
        assert sum(counts) >= min(k, L // 4)          # the union holds at least the global top-k


@pytest.mark.parametrize("B,k,H", [(1, 1, 1), (3, 300, 64), (4, 2048, 64), (2, 7, 3)])
def test_packed_layouts(B, k, H):
    ok, og, oc, ln = cp.candidate_layout(B, k)
    assert (ok, og, oc, ln) == (0, B * k, 2 * B * k, 2 * B * k + B)
    rows, o_bytes, l_off, row_bytes = cp.partial_layout(B, H)
    assert rows == 2 * B * H and o_bytes == rows * 256
    assert l_off % 16 == 0 and l_off >= o_bytes and row_bytes % 16 == 0 and row_bytes >= l_off + rows * 4
    assert (row_bytes // 2) % 8 == 0  # the bf16 stride between ranks suits 8-byte loads
