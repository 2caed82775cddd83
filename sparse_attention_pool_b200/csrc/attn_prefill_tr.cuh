// attn_prefill_tr.cuh -- the softmax attention of a causal prefill on the
// 5th-generation tensor cores (tcgen05 + tensor memory) with transposed
// tiles, for both branches of "DeepSeek-V4 ... Review", section 3-2 (2)
// component table: CSA attends over each query's sparse top-k of the
// compressed entries (GATHER), HCA over all of its visible entries (dense).
//
// Every query position has its own entry list (CSA: up to kmax listed
// entries; HCA: entries 0 .. n_t - 1), shared by its 64 heads (one KV head).
// A query's 64 heads fill only half of a 128-row MMA, so the tiles are
// transposed: the MMA's 128 rows are list entries,
//     S^T = K_sel Q^T    (M = 128 entries, N = 64 heads, K = 128 dims)
//     O^T = V_sel^T P^T  (M = 128 dims,    N = 64 heads, K = 128 entries)
// with every row of both MMAs used.  Per tile of 128 list entries: the K and
// V rows are copied by cp.async into the 128-byte-swizzled canonical layout
// (one row of 512 contiguous bytes per warp instruction), S^T lands in
// tensor memory, the softmax runs per head over the tile's entries (thread =
// entry, a butterfly exchange per warp gives each lane one head's maximum),
// P^T goes to shared memory in bf16, and O^T accumulates in tensor memory; a
// head's maximum is raised (and the sums and O^T rescaled) only when a score
// passes it by 2^8.  The next tile's rows are copied while the softmax runs
// (two buffers).  A persistent grid, one CTA per SM, walks the queries.
// Completion of each MMA group goes through tcgen05.commit on an mbarrier;
// every wait is bounded.
#pragma once
#include "attn_prefill_tc.cuh"

namespace sa {

constexpr int kCtThreads = 512;       // 16 warps: 4 TMEM lane quarters x 4 groups of 16 heads
constexpr int kCtRows = 128;          // list entries per tile
constexpr int kCtQ = 0;               // Q: 64 heads x 128 dims, K-major SW128, halves 8 KB apart
constexpr int kCtK = 16384;           // [2] K tiles: 128 x 128, K-major SW128, halves 16 KB apart
constexpr int kCtV = kCtK + 2 * 32768;  // [3] V tiles (the MN-major A operand of O^T)
constexpr int kCtP = kCtV + 3 * 32768;  // [2] P^T tiles: 128 entries x 64 heads bf16 (the MN-major B operand)
constexpr int kCtSmem = kCtP + 2 * 16384 + 1024;  // + alignment slack
constexpr uint32_t kCtCols = 256;      // tensor memory: [2] S^T tiles of 64 columns, then O^T (64 columns)
// A head's running maximum is raised only when a score passes it by more
// than 2^8 (the softmax is shift-invariant: the weights stay below 2^8, far
// inside bf16 and fp32, and the rescale of the sums and of O^T is rare).
constexpr float kCtLazy = 8.f;

struct CtArgs {
    const uint16_t* q;   // [BQ][H][128], BQ = B * T
    const uint16_t* K;   // [B][Ncap][128] bf16
    const uint16_t* V;
    const int32_t* n;    // [B]
    const int32_t* idx;  // [BQ][kmax] (GATHER)
    const int32_t* cnt;  // [BQ] (GATHER)
    const int32_t* pos;  // [BQ] token position of each query (dense: entries c with (c + 1) * m <= pos)
    int m;               // tokens per entry (dense)
    long long BQ;
    int T, H, Ncap, kmax;
    float scale_log2;    // softmax scale * log2(e)
    uint16_t* out;       // [BQ][H][128]
    float* lse;          // [BQ][H] or NULL
};

// 2^x on the special-function unit (subnormal results flush to zero: a
// weight below 2^-126 of the row's largest does not change the sum)
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Transposed reduction of 16 values per lane over the warp's 32 lanes (max
// or sum per value index): at each of four butterfly steps a lane keeps one
// half of its values and sends the other half to its partner; a last
// exchange joins the two half-warps, so that lanes l and l + 16 end with the
// reduction of value index l & 15.
template <bool MAX>
__device__ __forceinline__ float warp_transpose_reduce16(float (&v)[16], int lane) {
#pragma unroll
    for (int step = 0; step < 4; ++step) {
        const int half = 8 >> step;
        const bool upper = (lane & half) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float keep = upper ? v[half + i] : v[i];
            const float send = upper ? v[i] : v[half + i];
            const float got = __shfl_xor_sync(0xFFFFFFFFu, send, half);
            v[i] = MAX ? fmaxf(keep, got) : keep + got;
        }
    }
    const float got = __shfl_xor_sync(0xFFFFFFFFu, v[0], 16);
    return MAX ? fmaxf(v[0], got) : v[0] + got;
}

// Byte offset of (row r, 16-byte chunk c) in a K-major SW128 operand whose
// two 64-element halves lie `half` bytes apart.
__device__ __forceinline__ uint32_t sw128_off(int r, int c, uint32_t half) {
    return (uint32_t)(c >> 3) * half + (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Instruction descriptor, kind::f16 with fp32 D and bf16 A / B: M = 128,
// N = 64; a_mn / b_mn select MN-major operands.
__device__ __forceinline__ uint32_t ct_idesc(uint32_t a_mn, uint32_t b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn << 15) | (b_mn << 16) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
}

struct CtStatic {
    float red[16][16];  // per warp: one value per head of its group
    float m[64];       // running max of scale*log2e*s per head (raised lazily)
    float alpha[64];   // the rescale of the earlier sums when it is raised
    float l[64];       // the query's sums, at its end
    uint32_t tmem;
    uint64_t bar_s[2], bar_o[2];  // S^T(t) and O^T(t) complete on barrier t & 1
#ifdef SA_TRACE
    unsigned long long tt[kCtRows / 8][6];  // profiling build: thread 0's step times of one query's tiles
#endif
};

// 16 consecutive fp32 columns of this thread's TMEM lane: loaded without
// the wait (tc_wait_ld completes them), and stored
__device__ __forceinline__ void tc_ld16_nw(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Persistent grid; CTA c takes queries c, c + gridDim.x, ...  The pipeline
// of a query's tiles (K in two buffers, V in three, S^T and P^T in two):
//   1.  wait for S^T(i); copy the K rows of tile i + 2 (into the buffer
//       S^T(i) has read);
//   2.  softmax of tile i (thread = entry, 16 of its heads) into P^T(i);
//   3.  wait for this thread's copies of V(i) and K(i + 1), barrier;
//   4.  issue S^T(i + 1) = K(i + 1) Q^T and, behind it, O^T += V(i)^T P^T(i);
//   5.  wait for O^T(i - 1), then copy the V rows of tile i + 2 (into the
//       buffer O^T(i - 1) has read).
// So the copies of a tile go out about two tiles before its MMAs, and the
// next tile's scores come first in the tensor pipe.  O^T accumulates in
// tensor memory and is read once, at the query's end.  Each thread keeps,
// for its entry slot, the sums of its 16 heads' weights over the tiles; they
// are reduced once per query.
template <bool GATHER>
__global__ void __launch_bounds__(kCtThreads, 1) attn_prefill_tr_kernel(CtArgs a) {
    extern __shared__ uint8_t ct_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ct_raw) + 1023) & ~uintptr_t(1023));
    __shared__ CtStatic S;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3, hg = warp >> 2;  // TMEM lane quarter; group of 16 heads
    const uint32_t sQ = smem_u32(sm + kCtQ), sK = smem_u32(sm + kCtK), sV = smem_u32(sm + kCtV),
                   sP = smem_u32(sm + kCtP);
    pdl_wait();
    pdl_release();
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S.tmem)),
                     "r"(kCtCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.bar_s[i], 1);
            mbar_init(&S.bar_o[i], 1);
        }
        fence_barrier_init();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem;
    const uint32_t t_o = tmem + 128;
    const uint32_t lane_q = (uint32_t)(quarter * 32) << 16;
    const uint32_t id_s = ct_idesc(0, 0), id_o = ct_idesc(1, 1);
    // completions waited for on each barrier (every thread waits for every
    // one, so the counts are uniform), and commits issued (thread 0)
    uint32_t ws0 = 0, ws1 = 0, wo0 = 0, wo1 = 0, is0 = 0, is1 = 0, io0 = 0, io1 = 0;
    bool bad = false;  // a wait ran out (recorded in the status word); the CTA stops
    auto wait_s = [&](int t) {
        uint32_t& w = (t & 1) ? ws1 : ws0;
        bad |= !mbar_wait(&S.bar_s[t & 1], w & 1);
        ++w;
    };
    int o_done = -1;  // the query's O^T groups are complete up to this tile
    auto wait_o_until = [&](int t) {
        for (; o_done < t; ++o_done) {
            const int u = o_done + 1;
            uint32_t& w = (u & 1) ? wo1 : wo0;
            bad |= !mbar_wait(&S.bar_o[u & 1], w & 1);
            ++w;
        }
    };
    // Row copies: warp w copies tile rows 8w .. 8w + 7, two rows per
    // instruction (16 lanes a row: 512 contiguous bytes for consecutive
    // rows); lane l holds the entry of row 8w + (l & 7), -1 for none.
    const int grow = warp * 8 + (lane & 7);
    const int gchunk = lane & 15;
    auto copy_rows = [&](const uint16_t* base, uint8_t* dst, int jo) {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const int j = __shfl_sync(0xFFFFFFFFu, jo, 2 * p + (lane >> 4));
            cp_async16_zfill(dst + sw128_off(warp * 8 + 2 * p + (lane >> 4), gchunk, 16384),
                             base + (size_t)(j >= 0 ? j : 0) * 128 + gchunk * 8, j >= 0);
        }
    };

    for (long long bq = blockIdx.x; bq < a.BQ && !bad; bq += gridDim.x) {
        const int b = (int)(bq / a.T);
        int nb = a.n[b];
        if (nb < 0 || nb > a.Ncap) {
            if (tid == 0) flag(DEV_LEN);
            nb = nb < 0 ? 0 : a.Ncap;
        }
        int R;  // the query's list length
        if (GATHER) {
            R = a.cnt[bq];
            if (R < 0 || R > a.kmax) {
                if (tid == 0) flag(DEV_LEN);
                R = R < 0 ? 0 : a.kmax;
            }
        } else {
            const int tp = a.pos[bq];
            R = tp < 0 ? 0 : min(nb, tp / a.m);
        }
        const int ntiles = (R + kCtRows - 1) / kCtRows;
        const int32_t* lidx = GATHER ? a.idx + (size_t)bq * a.kmax : nullptr;
        const uint16_t* Kb = a.K + (size_t)b * a.Ncap * 128;
        const uint16_t* Vb = a.V + (size_t)b * a.Ncap * 128;
        // this lane's row of tile t: its list entry as loaded (gathered lists) ...
        auto load_idx = [&](int t) -> int {
            const int p = t * kCtRows + grow;
            return GATHER && t < ntiles && p < R ? (int)ld_cg_u32(lidx + p) : 0;
        };
        // ... and checked: the entry to copy, or -1 (past the list; out of range, flagged)
        auto entry = [&](int t, int jl) -> int {
            const int p = t * kCtRows + grow;
            if (t >= ntiles || p >= R) return -1;
            if (!GATHER) return p;
            if (jl >= 0 && jl < nb) return jl;
            if (lane < 16) flag(DEV_INDEX);
            return -1;
        };
        if (tid < 64) S.m[tid] = -INFINITY;
        float lsum[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) lsum[j] = 0.f;
        o_done = -1;
        if (ntiles > 0) {
            // Q (64 rows of 16 chunks, rows at or past H zero), K(0), V(0), K(1), V(1)
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int h = u * 32 + (tid >> 4), c = tid & 15;
                const bool ok = h < a.H;
                const uint16_t* src = a.q + ((size_t)bq * a.H + (ok ? h : 0)) * 128 + c * 8;
                cp_async16_zfill(sm + kCtQ + sw128_off(h, c, 8192), src, ok);
            }
            const int j0 = entry(0, load_idx(0)), j1 = entry(1, load_idx(1));
            copy_rows(Kb, sm + kCtK, j0);
            cp_async_commit();
            if (ntiles > 1) copy_rows(Kb, sm + kCtK + 32768, j1);
            cp_async_commit();
            copy_rows(Vb, sm + kCtV, j0);
            cp_async_commit();
            if (ntiles > 1) copy_rows(Vb, sm + kCtV + 32768, j1);
            cp_async_commit();
            cp_async_wait<3>();  // Q and K(0)
            fence_async_smem();
            __syncthreads();
            if (tid == 0) {  // S^T(0) = K(0) Q^T over 8 k-steps of 16 dims
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc_mma(tmem, tc_desc(sK + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                           tc_desc(sQ + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), id_s, ks > 0);
                tc_commit(&S.bar_s[0]);
                ++is0;
            }
        }
        int jn = load_idx(2);  // the entries of tile i + 2, loaded a tile ahead

        // profiling build: thread 0's step times for the gathered lists of
        // CTA 0's last two queries (full lists), written after each query
        const bool traced = GATHER && blockIdx.x == 0 && bq / gridDim.x + 2 >= a.BQ / gridDim.x;
        auto tnow = [&](int i, int step) {
#ifdef SA_TRACE
            if (traced && tid == 0 && i < kCtRows / 8) S.tt[i][step] = SA_TRACE_NOW();
#else
            (void)traced, (void)i, (void)step;
#endif
        };
        for (int i = 0; i < ntiles; ++i) {
            const int bi = i & 1;
            tnow(i, 0);
            // 1. S^T(i) complete; K(i + 2) into the buffer it has read
            wait_s(i);
            tnow(i, 1);
            tc_fence_after();
            const int j2 = entry(i + 2, jn);
            if (i + 2 < ntiles) copy_rows(Kb, sm + kCtK + bi * 32768, j2);
            cp_async_commit();
            jn = load_idx(i + 3);
            // 2. softmax of tile i: thread = entry e, heads 16 hg .. 16 hg + 15;
            //    d = scale * log2(e) * s - m, the weight's exponent (-inf off the list)
            const int e = quarter * 32 + lane;
            const bool valid = i * kCtRows + e < R;
            uint32_t raw[16];
            tc_ld16_nw(tmem + 64 * bi + lane_q + 16 * hg, raw);
            tc_wait_ld();
            float d[16];
            bool over = false;
            {
                const float4* m4 = reinterpret_cast<const float4*>(S.m + 16 * hg);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float4 mm = m4[c];
                    const float ms[4] = {mm.x, mm.y, mm.z, mm.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int h = 4 * c + u;
                        d[h] = valid ? fmaf(__uint_as_float(raw[h]), a.scale_log2, -ms[u]) : -INFINITY;
                        over |= d[h] > kCtLazy;
                    }
                }
            }
            if (__syncthreads_or(over)) {
                // raise the maxima to the exact ones of this tile, rescale the
                // sums and O^T (once its last group, i - 1, is complete)
                float vm[16];
#pragma unroll
                for (int h = 0; h < 16; ++h) vm[h] = valid ? __uint_as_float(raw[h]) * a.scale_log2 : -INFINITY;
                const float r = warp_transpose_reduce16<true>(vm, lane);  // head 16 hg + (lane & 15)
                if (lane < 16) S.red[warp][lane] = r;
                __syncthreads();
                if (tid < 64) {  // head tid: the warps of its group, one per lane quarter
                    const int g = tid >> 4, j = tid & 15;
                    float mt = S.red[4 * g][j];
#pragma unroll
                    for (int q = 1; q < 4; ++q) mt = fmaxf(mt, S.red[4 * g + q][j]);
                    const float mo = S.m[tid], mn = fmaxf(mo, mt);
                    S.alpha[tid] = mo == -INFINITY ? 0.f : ex2_ftz(mo - mn);  // earlier sums are 0 while m is -inf
                    S.m[tid] = mn;
                }
                __syncthreads();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float mn = S.m[16 * hg + j];
                    lsum[j] *= S.alpha[16 * hg + j];
                    d[j] = valid ? fmaf(__uint_as_float(raw[j]), a.scale_log2, -mn) : -INFINITY;
                }
                if (i > 0) {  // thread = dim here: its row of O^T for its 16 heads
                    wait_o_until(i - 1);
                    tc_fence_after();
                    uint32_t rr[16];
                    tc_ld16_nw(t_o + lane_q + 16 * hg, rr);
                    tc_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) rr[j] = __float_as_uint(__uint_as_float(rr[j]) * S.alpha[16 * hg + j]);
                    tc_st16(t_o + lane_q + 16 * hg, rr);
                    tc_wait_st();
                }
            }
            // P^T(i) (bf16, heads contiguous): p = 2^d < 2^8, 0 off the list
            // (2^-inf).  Its buffer was last read by O^T(i - 2), complete
            // since tile i - 1.
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t pk[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const int h = c * 8 + w * 2;
                    const float p0 = ex2_ftz(d[h]), p1 = ex2_ftz(d[h + 1]);
                    lsum[h] += p0;
                    lsum[h + 1] += p1;
                    pk[w] = pack_bf16x2(p0, p1);
                }
                const int cc = 2 * hg + c;  // 16-byte chunk of the entry's 128-byte P^T row
                *reinterpret_cast<uint4*>(sm + kCtP + bi * 16384 + (e >> 3) * 1024 + (e & 7) * 128 +
                                          ((cc ^ (e & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            tnow(i, 2);
            // 3. V(i) and K(i + 1) landed (the two newest groups, K(i + 2) and
            // V(i + 1), may still be in flight)
            cp_async_wait<2>();
            fence_async_smem();
            tc_fence_before();
            if (__syncthreads_or(bad)) {
                bad = true;
                break;
            }
            tnow(i, 3);
            // 4. S^T(i + 1) (the next softmax waits for it), then O^T += V(i)^T P^T(i)
            if (tid == 0) {
                tc_fence_after();
                if (i + 1 < ntiles) {
                    const uint32_t kb = sK + (bi ^ 1) * 32768;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        tc_mma(tmem + 64 * (bi ^ 1), tc_desc(kb + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                               tc_desc(sQ + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024), id_s, ks > 0);
                    tc_commit(&S.bar_s[bi ^ 1]);
                    ++(bi ? is0 : is1);
                }
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc_mma(t_o, tc_desc(sV + (i % 3) * 32768 + ks * 2048, 16384, 1024),
                           tc_desc(sP + bi * 16384 + ks * 2048, 16384, 1024), id_o, (i > 0 || ks > 0) ? 1u : 0u);
                tc_commit(&S.bar_o[bi]);
                ++(bi ? io1 : io0);
            }
            tnow(i, 4);
            // 5. O^T(i - 1) complete: V(i + 2) into the buffer it has read
            if (i > 0) wait_o_until(i - 1);
            if (i + 2 < ntiles) copy_rows(Vb, sm + kCtV + ((i + 2) % 3) * 32768, j2);
            cp_async_commit();
            tnow(i, 5);
        }
#ifdef SA_TRACE
        if (traced && tid == 0)
            for (int i = 0; i < min(ntiles, kCtRows / 8); ++i)
                for (int step = 0; step < 6; ++step)
                    SA_TRACE_PUT(S.tt[i][step], TR_PATTN, step, (uint32_t)((bq / gridDim.x) % 2) * 16 + i);
#endif
        if (ntiles > 0 && !bad) wait_o_until(ntiles - 1);  // the query's last O^T group
        cp_async_wait<0>();
        tc_fence_after();
        if (__syncthreads_or(bad)) {
            bad = true;
            break;
        }
        // the sums per head over the entry slots
        {
            const float r = warp_transpose_reduce16<false>(lsum, lane);  // head 16 hg + (lane & 15)
            if (lane < 16) S.red[warp][lane] = r;
        }
        __syncthreads();
        if (tid < 64) {
            const int g = tid >> 4, j = tid & 15;
            float sum = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) sum += S.red[4 * g + q][j];
            S.l[tid] = sum;
        }
        __syncthreads();
        // this query's output: dim d of each of the thread's 16 heads, and the lse
        {
            const int dd = quarter * 32 + lane;
            uint32_t rr[16];
            if (ntiles > 0) {
                tc_ld16_nw(t_o + lane_q + 16 * hg, rr);
                tc_wait_ld();
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int h = 16 * hg + j;
                if (h < a.H) {
                    const float L = S.l[h];
                    const float ov = ntiles > 0 ? __uint_as_float(rr[j]) : 0.f;
                    const __nv_bfloat16 y = __float2bfloat16_rn(L > 0.f ? ov / L : 0.f);
                    a.out[((size_t)bq * a.H + h) * 128 + dd] = *reinterpret_cast<const uint16_t*>(&y);
                }
            }
            if (a.lse && tid < a.H && tid < 64) {
                const float L = S.l[tid];
                a.lse[(size_t)bq * a.H + tid] = L > 0.f ? (S.m[tid] + __log2f(L)) * 0.6931471805599453f : -INFINITY;
            }
        }
        tc_fence_before();
        __syncthreads();  // tensor memory, shared buffers, S.m and S.l are reused by the next query
    }
    // after a timeout: the MMA groups still in flight are waited for
    // (bounded) before their tensor memory is released
    if (tid == 0) {
        for (; ws0 < is0; ++ws0) mbar_wait(&S.bar_s[0], ws0 & 1);
        for (; ws1 < is1; ++ws1) mbar_wait(&S.bar_s[1], ws1 & 1);
        for (; wo0 < io0; ++wo0) mbar_wait(&S.bar_o[0], wo0 & 1);
        for (; wo1 < io1; ++wo1) mbar_wait(&S.bar_o[1], wo1 & 1);
    }
    cp_async_wait<0>();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCtCols));
    }
}

// --------------------------------------------------- dense, query pairs --
// The dense (HCA) causal prefill with 64 heads, two query positions per
// tile: with m even, positions 2p and 2p + 1 see the same entries (entry c
// needs (c + 1) m <= t, and 2p + 1 is never a multiple of m), so one tile of
// K and V rows serves both.  The MMAs take both queries' 128 heads as N:
//     S^T = K Q^T    (M = 128 entries, N = 128 = 2 queries x 64 heads)
//     O^T = V^T P^T  (M = 128 dims,    N = 128)
// which halves the row copies per query and doubles the work per MMA.  The
// pipeline is the single-query kernel's with V in two buffers and P^T in one
// (shared memory holds Q 32 KB, K 2 x 32, V 2 x 32, P^T 32 KB): a tile's
// P^T is written once the previous tile's products are complete.  Positions that are not
// consecutive (q_pos is the caller's) are handled too: each query's heads
// mask the entries past its own count.
constexpr int kPrThreads = 512;         // 16 warps: 4 TMEM lane quarters x 4 groups of 32 heads
constexpr int kPrQ = 0;                 // Q: 128 rows (2 queries x 64 heads) x 128 dims, K-major SW128
constexpr int kPrK = 32768;             // [2] K tiles
constexpr int kPrV = kPrK + 2 * 32768;  // [2] V tiles
constexpr int kPrP = kPrV + 2 * 32768;  // P^T: 128 entries x 128 heads, two 64-head halves
constexpr int kPrSmem = kPrP + 32768 + 1024;
constexpr uint32_t kPrCols = 512;       // tensor memory: [2] S^T tiles of 128 columns, then O^T (128)

struct PrStatic {
    float red[16][32];  // per warp: one value per head of its group
    float m[128];       // running max of scale*log2e*s per (query, head), raised lazily
    float alpha[128];
    float l[128];
    uint32_t tmem;
    uint64_t bar_s[2], bar_o[2];
};

__device__ __forceinline__ uint32_t pr_idesc(uint32_t a_mn, uint32_t b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn << 15) | (b_mn << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
}

// Transposed reduction of 32 values per lane over the warp's 32 lanes (max
// or sum per value index): at each of five butterfly steps a lane keeps one
// half of its values and sends the other half to its partner, so that lane
// l ends with the reduction of value index l.
template <bool MAX>
__device__ __forceinline__ float warp_transpose_reduce32(float (&v)[32], int lane) {
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int half = 16 >> step;
        const bool upper = (lane & half) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float keep = upper ? v[half + i] : v[i];
            const float send = upper ? v[i] : v[half + i];
            const float got = __shfl_xor_sync(0xFFFFFFFFu, send, half);
            v[i] = MAX ? fmaxf(keep, got) : keep + got;
        }
    }
    return v[0];
}

// Persistent grid over query pairs (b, positions 2p and 2p + 1 of sequence
// b; the second is absent at an odd end).  Per tile i:
//   1. wait for S^T(i); copy K(i + 2) into the buffer S^T(i) has read;
//   2. softmax (thread = entry, 32 heads of one query); wait for O^T(i - 1),
//      then write P^T(i);
//   3. wait for this thread's copies of V(i) and K(i + 1), barrier;
//   4. issue S^T(i + 1), then O^T += V(i)^T P^T(i);
//   5. copy V(i + 1) into the buffer O^T(i - 1) has read.
__global__ void __launch_bounds__(kPrThreads, 1) attn_prefill_pair_kernel(CtArgs a) {
    extern __shared__ uint8_t pr_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pr_raw) + 1023) & ~uintptr_t(1023));
    __shared__ PrStatic S;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3, hg = warp >> 2;  // TMEM lane quarter; group of 32 heads (query hg >> 1)
    const int qi = hg >> 1;                        // this thread's query of the pair (softmax)
    const uint32_t sQ = smem_u32(sm + kPrQ), sK = smem_u32(sm + kPrK), sV = smem_u32(sm + kPrV),
                   sP = smem_u32(sm + kPrP);
    pdl_wait();
    pdl_release();
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S.tmem)),
                     "r"(kPrCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.bar_s[i], 1);
            mbar_init(&S.bar_o[i], 1);
        }
        fence_barrier_init();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem;
    const uint32_t t_o = tmem + 256;
    const uint32_t lane_q = (uint32_t)(quarter * 32) << 16;
    const uint32_t id_s = pr_idesc(0, 0), id_o = pr_idesc(1, 1);
    uint32_t ws0 = 0, ws1 = 0, wo0 = 0, wo1 = 0, is0 = 0, is1 = 0, io0 = 0, io1 = 0;
    bool bad = false;
    auto wait_s = [&](int t) {
        uint32_t& w = (t & 1) ? ws1 : ws0;
        bad |= !mbar_wait(&S.bar_s[t & 1], w & 1);
        ++w;
    };
    int o_done = -1;
    auto wait_o_until = [&](int t) {
        for (; o_done < t; ++o_done) {
            const int u = o_done + 1;
            uint32_t& w = (u & 1) ? wo1 : wo0;
            bad |= !mbar_wait(&S.bar_o[u & 1], w & 1);
            ++w;
        }
    };
    // row copies: warp w copies tile rows 8w .. 8w + 7 (entries e0 + row), two rows an instruction
    const int gchunk = lane & 15;
    auto copy_rows = [&](const uint16_t* base, uint8_t* dst, int first, int R) {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const int row = warp * 8 + 2 * p + (lane >> 4);
            const bool ok = first + row < R;
            cp_async16_zfill(dst + sw128_off(row, gchunk, 16384), base + (size_t)(ok ? first + row : 0) * 128 + gchunk * 8,
                             ok);
        }
    };
    const long long npair = (a.T + 1) / 2;
    const long long total = npair * (a.BQ / a.T);

    for (long long pp = blockIdx.x; pp < total && !bad; pp += gridDim.x) {
        const int b = (int)(pp / npair);
        const int t0 = 2 * (int)(pp % npair);
        const bool has1 = t0 + 1 < a.T;
        const long long bq0 = (long long)b * a.T + t0;
        int nb = a.n[b];
        if (nb < 0 || nb > a.Ncap) {
            if (tid == 0) flag(DEV_LEN);
            nb = nb < 0 ? 0 : a.Ncap;
        }
        int Rq[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int tp = (u == 0 || has1) ? a.pos[bq0 + u] : -1;
            Rq[u] = tp < 0 ? 0 : min(nb, tp / a.m);
        }
        const int R = max(Rq[0], Rq[1]);
        const int Rmine = Rq[qi];
        const int ntiles = (R + kCtRows - 1) / kCtRows;
        const uint16_t* Kb = a.K + (size_t)b * a.Ncap * 128;
        const uint16_t* Vb = a.V + (size_t)b * a.Ncap * 128;
        if (tid < 128) S.m[tid] = -INFINITY;
        float lsum[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) lsum[j] = 0.f;
        o_done = -1;
        if (ntiles > 0) {
            // Q: row u * 64 + h of query u (zero when the query is absent), 16 chunks
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int r = v * 32 + (tid >> 4), c = tid & 15;
                const int u = r >> 6, h = r & 63;
                const bool ok = u == 0 || has1;
                const uint16_t* src = a.q + ((size_t)(bq0 + (ok ? u : 0)) * 64 + h) * 128 + c * 8;
                cp_async16_zfill(sm + kPrQ + sw128_off(r, c, 16384), src, ok);
            }
            copy_rows(Kb, sm + kPrK, 0, R);
            cp_async_commit();
            if (ntiles > 1) copy_rows(Kb, sm + kPrK + 32768, kCtRows, R);
            cp_async_commit();
            copy_rows(Vb, sm + kPrV, 0, R);
            cp_async_commit();
            cp_async_wait<2>();  // Q and K(0)
            fence_async_smem();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc_mma(tmem, tc_desc(sK + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                           tc_desc(sQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024), id_s, ks > 0);
                tc_commit(&S.bar_s[0]);
                ++is0;
            }
        }

        for (int i = 0; i < ntiles; ++i) {
            const int bi = i & 1;
            // 1. S^T(i) complete; K(i + 2) into the buffer it has read
            wait_s(i);
            tc_fence_after();
            if (i + 2 < ntiles) copy_rows(Kb, sm + kPrK + bi * 32768, (i + 2) * kCtRows, R);
            cp_async_commit();
            // 2. softmax: thread = entry e, heads 32 hg .. 32 hg + 31 (query qi), in
            //    two halves of 16 read from tensor memory (once to test the
            //    maxima, once more for the weights: fewer live registers)
            const int e = quarter * 32 + lane;
            const bool valid = i * kCtRows + e < Rmine;
            const uint32_t t_s = tmem + 128 * bi + lane_q + 32 * hg;
            bool over = false;
            // (the tensor-memory loads are warp-collective: every lane takes them)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t raw[16];
                tc_ld16_nw(t_s + 16 * hf, raw);
                tc_wait_ld();
                const float4* m4 = reinterpret_cast<const float4*>(S.m + 32 * hg + 16 * hf);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float4 mm = m4[c];
                    const float ms[4] = {mm.x, mm.y, mm.z, mm.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        over |= valid && fmaf(__uint_as_float(raw[4 * c + u]), a.scale_log2, -ms[u]) > kCtLazy;
                }
            }
            if (__syncthreads_or(over)) {
                // raise the maxima to the exact ones of this tile, rescale the
                // sums and O^T
                {
                    float vm[32];
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        uint32_t raw[16];
                        tc_ld16_nw(t_s + 16 * hf, raw);
                        tc_wait_ld();
#pragma unroll
                        for (int h = 0; h < 16; ++h)
                            vm[16 * hf + h] = valid ? __uint_as_float(raw[h]) * a.scale_log2 : -INFINITY;
                    }
                    S.red[warp][lane] = warp_transpose_reduce32<true>(vm, lane);  // head 32 hg + lane
                }
                __syncthreads();
                if (tid < 128) {  // (query, head) tid: the warps of its group, one per lane quarter
                    const int g = tid >> 5, j = tid & 31;
                    float mt = S.red[4 * g][j];
#pragma unroll
                    for (int q = 1; q < 4; ++q) mt = fmaxf(mt, S.red[4 * g + q][j]);
                    const float mo = S.m[tid], mn = fmaxf(mo, mt);
                    S.alpha[tid] = mo == -INFINITY ? 0.f : ex2_ftz(mo - mn);
                    S.m[tid] = mn;
                }
                __syncthreads();
#pragma unroll
                for (int j = 0; j < 32; ++j) lsum[j] *= S.alpha[32 * hg + j];
                if (i > 0) {  // thread = dim here: its row of O^T for its 32 heads
                    wait_o_until(i - 1);
                    tc_fence_after();
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        uint32_t rr[16];
                        tc_ld16_nw(t_o + lane_q + 32 * hg + 16 * hf, rr);
                        tc_wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            rr[j] = __float_as_uint(__uint_as_float(rr[j]) * S.alpha[32 * hg + 16 * hf + j]);
                        tc_st16(t_o + lane_q + 32 * hg + 16 * hf, rr);
                    }
                    tc_wait_st();
                }
            }
            // P^T(i): p = 2^(scale log2(e) s - m) < 2^8, 0 off the list.  Heads
            // 32 hg .. + 31 are 16-byte chunks 4 (hg & 1) .. + 3 of half hg >> 1
            // of the entry's row; the buffer's last reader is O^T(i - 1).
            if (i > 0) wait_o_until(i - 1);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t raw[16];
                tc_ld16_nw(t_s + 16 * hf, raw);
                tc_wait_ld();
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    uint32_t pk[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const int h = 16 * hf + 8 * c2 + 2 * w;  // head within the thread's 32
                        const float m0 = S.m[32 * hg + h], m1 = S.m[32 * hg + h + 1];
                        const float p0 = valid ? ex2_ftz(fmaf(__uint_as_float(raw[8 * c2 + 2 * w]), a.scale_log2, -m0)) : 0.f;
                        const float p1 =
                            valid ? ex2_ftz(fmaf(__uint_as_float(raw[8 * c2 + 2 * w + 1]), a.scale_log2, -m1)) : 0.f;
                        lsum[h] += p0;
                        lsum[h + 1] += p1;
                        pk[w] = pack_bf16x2(p0, p1);
                    }
                    const int cc = 4 * (hg & 1) + 2 * hf + c2;
                    *reinterpret_cast<uint4*>(sm + kPrP + (hg >> 1) * 16384 + (e >> 3) * 1024 +
                                              (e & 7) * 128 + ((cc ^ (e & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            // 3. V(i) and K(i + 1) landed (the newest group, K(i + 2), may be in flight)
            cp_async_wait<1>();
            fence_async_smem();
            tc_fence_before();
            if (__syncthreads_or(bad)) {
                bad = true;
                break;
            }
            // 4. S^T(i + 1), then O^T += V(i)^T P^T(i)
            if (tid == 0) {
                tc_fence_after();
                if (i + 1 < ntiles) {
                    const uint32_t kb = sK + (bi ^ 1) * 32768;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        tc_mma(tmem + 128 * (bi ^ 1), tc_desc(kb + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                               tc_desc(sQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024), id_s, ks > 0);
                    tc_commit(&S.bar_s[bi ^ 1]);
                    ++(bi ? is0 : is1);
                }
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc_mma(t_o, tc_desc(sV + bi * 32768 + ks * 2048, 16384, 1024),
                           tc_desc(sP + ks * 2048, 16384, 1024), id_o, (i > 0 || ks > 0) ? 1u : 0u);
                tc_commit(&S.bar_o[bi]);
                ++(bi ? io1 : io0);
            }
            // 5. V(i + 1) into the buffer O^T(i - 1) has read (complete since step 2)
            if (i + 1 < ntiles) copy_rows(Vb, sm + kPrV + (bi ^ 1) * 32768, (i + 1) * kCtRows, R);
            cp_async_commit();
        }
        if (ntiles > 0 && !bad) wait_o_until(ntiles - 1);
        cp_async_wait<0>();
        tc_fence_after();
        if (__syncthreads_or(bad)) {
            bad = true;
            break;
        }
        // the sums per (query, head) over the entry slots
        S.red[warp][lane] = warp_transpose_reduce32<false>(lsum, lane);
        __syncthreads();
        if (tid < 128) {
            const int g = tid >> 5, j = tid & 31;
            float sum = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) sum += S.red[4 * g + q][j];
            S.l[tid] = sum;
        }
        __syncthreads();
        // the outputs: dim dd of each of the thread's 32 heads (query qi), and the lse
        {
            const int dd = quarter * 32 + lane;
            uint32_t rr[32];
            if (ntiles > 0) {
                tc_ld32_nw(t_o + lane_q + 32 * hg, rr);
                tc_wait_ld();
            }
            if (qi == 0 || has1) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int h = 32 * (hg & 1) + j;
                    const float L = S.l[32 * hg + j];
                    const float ov = ntiles > 0 ? __uint_as_float(rr[j]) : 0.f;
                    const __nv_bfloat16 y = __float2bfloat16_rn(L > 0.f ? ov / L : 0.f);
                    a.out[((size_t)(bq0 + qi) * 64 + h) * 128 + dd] = *reinterpret_cast<const uint16_t*>(&y);
                }
            }
            if (a.lse && tid < 128 && ((tid >> 6) == 0 || has1)) {
                const float L = S.l[tid];
                a.lse[(size_t)(bq0 + (tid >> 6)) * 64 + (tid & 63)] =
                    L > 0.f ? (S.m[tid] + __log2f(L)) * 0.6931471805599453f : -INFINITY;
            }
        }
        tc_fence_before();
        __syncthreads();
    }
    if (tid == 0) {
        for (; ws0 < is0; ++ws0) mbar_wait(&S.bar_s[0], ws0 & 1);
        for (; ws1 < is1; ++ws1) mbar_wait(&S.bar_s[1], ws1 & 1);
        for (; wo0 < io0; ++wo0) mbar_wait(&S.bar_o[0], wo0 & 1);
        for (; wo1 < io1; ++wo1) mbar_wait(&S.bar_o[1], wo1 & 1);
    }
    cp_async_wait<0>();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kPrCols));
    }
}

}  // namespace sa
