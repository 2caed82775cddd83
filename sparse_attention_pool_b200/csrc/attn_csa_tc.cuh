// attn_csa_tc.cuh -- the gathered (CSA) softmax attention of a causal
// prefill on the 5th-generation tensor cores (tcgen05 + tensor memory),
// "DeepSeek-V4 ... Review", section 3-2 (2) component table (CSA attends over
// its sparse top-k of the compressed entries).
//
// Every query position has its own list of up to kmax entries, shared by its
// 64 heads (one KV head).  A query's 64 heads fill only half of a 128-row
// MMA, so the tiles are transposed: the MMA's 128 rows are list entries,
//     S^T = K_sel Q^T    (M = 128 entries, N = 64 heads, K = 128 dims)
//     O^T = V_sel^T P^T  (M = 128 dims,    N = 64 heads, K = 128 entries)
// with every row of both MMAs used.  Per tile of 128 list entries: the K and
// V rows are gathered by cp.async into the 128-byte-swizzled canonical
// layout, S^T lands in tensor memory, the softmax runs per head over the
// tile's entries (thread = entry, a butterfly exchange per warp gives each
// lane one head's maximum), P^T goes to shared memory in bf16, and O^T
// accumulates in tensor memory; a head's maximum is raised (and the sums and
// O^T rescaled) only when a score passes it by 2^8.  The next tile's rows
// are gathered while the softmax runs (two buffers).  A persistent grid, one
// CTA per SM, walks the queries.  Completion of each MMA group goes through
// tcgen05.commit on an mbarrier; every wait is bounded.
#pragma once
#include "attn_prefill_tc.cuh"

namespace sa {

constexpr int kCtThreads = 256;       // 8 warps
constexpr int kCtRows = 128;          // list entries per tile
constexpr int kCtQ = 0;               // Q: 64 heads x 128 dims, K-major SW128, halves 8 KB apart
constexpr int kCtK = 16384;           // [2] K tiles: 128 x 128, K-major SW128, halves 16 KB apart
constexpr int kCtV = kCtK + 2 * 32768;  // [2] V tiles (the MN-major A operand of O^T)
constexpr int kCtP = kCtV + 2 * 32768;  // [2] P^T tiles: 128 entries x 64 heads bf16 (the MN-major B operand)
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
    const int32_t* idx;  // [BQ][kmax]
    const int32_t* cnt;  // [BQ]
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

// Transposed reduction of 32 values per lane over the warp's 32 lanes (max
// or sum per value index): at each of the five butterfly steps a lane keeps
// one half of its values and sends the other half to its partner, so that
// lane l ends with the reduction of value index l.
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
    float red[8][32];  // per warp: one value per head of its half
    float m[64];       // running max of scale*log2e*s per head (raised lazily)
    float alpha[64];   // the rescale of the earlier sums when it is raised
    float l[64];       // the query's sums, at its end
    uint32_t tmem;
    int bad;
    uint64_t bar_s, bar_o;
};

// 32 consecutive fp32 columns of this thread's TMEM lane, stored
__device__ __forceinline__ void tc_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Persistent grid; CTA c takes queries c, c + gridDim.x, ...  Per tile i of
// a query's list: the tile's K and V rows were gathered during tile i - 1;
// S^T(i) is issued, the gather of tile i + 1 goes out once O^T(i - 1) has
// released its buffers, the softmax of tile i writes P^T(i), and O^T(i)
// accumulates in tensor memory (read once, at the query's end).  Each
// thread keeps, for its entry slot, the sums of its 32 heads' weights over
// the tiles; they are reduced once per query.
__global__ void __launch_bounds__(kCtThreads, 1) attn_csa_prefill_tc_kernel(CtArgs a) {
    extern __shared__ uint8_t ct_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ct_raw) + 1023) & ~uintptr_t(1023));
    __shared__ CtStatic S;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int quarter = warp & 3, hh = warp >> 2;  // TMEM lane quarter; half of the heads
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
        mbar_init(&S.bar_s, 1);
        mbar_init(&S.bar_o, 1);
        fence_barrier_init();
        S.bad = 0;
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem;
    const uint32_t t_o = tmem + 128;
    const uint32_t lane_q = (uint32_t)(quarter * 32) << 16;
    const uint32_t id_s = ct_idesc(0, 0), id_o = ct_idesc(1, 1);
    uint32_t ph_s = 0, ph_o = 0;
    int pend_s = 0, pend_o = 0;  // (thread 0) commits not yet seen complete
    // The gather: warp w copies tile rows 16w .. 16w + 15, one row per
    // instruction, lanes 0-15 the row's 16 K chunks and lanes 16-31 its V
    // chunks (512 contiguous bytes per instruction); lane l holds the entry
    // of row 16w + (l & 15).
    const int grow = warp * 16 + (lane & 15);
    const int gchunk = lane & 15;
    const bool isv = lane >= 16;

    for (long long bq = blockIdx.x; bq < a.BQ; bq += gridDim.x) {
        const int b = (int)(bq / a.T);
        int nb = a.n[b];
        if (nb < 0 || nb > a.Ncap) {
            if (tid == 0) flag(DEV_LEN);
            nb = nb < 0 ? 0 : a.Ncap;
        }
        int R = a.cnt[bq];
        if (R < 0 || R > a.kmax) {
            if (tid == 0) flag(DEV_LEN);
            R = R < 0 ? 0 : a.kmax;
        }
        const int ntiles = (R + kCtRows - 1) / kCtRows;
        const int32_t* lidx = a.idx + (size_t)bq * a.kmax;
        // Q: 64 rows of 16 chunks, rows at or past H zero; 16 threads a row,
        // two consecutive (contiguous) rows per instruction
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int h = u * 16 + (tid >> 4), c = tid & 15;
            const bool ok = h < a.H;
            const uint16_t* src = a.q + ((size_t)bq * a.H + (ok ? h : 0)) * 128 + c * 8;
            cp_async16_zfill(sm + kCtQ + sw128_off(h, c, 8192), src, ok);
        }
        // the gather of tile t's rows into buffer t & 1 (zero past the list);
        // jn holds the entry of this lane's row of that tile, loaded a tile ahead
        int jn = ntiles > 0 && grow < R ? (int)ld_cg_u32(lidx + grow) : 0;
        auto gather = [&](int t) {
            int jo = -1;  // this lane's row: its entry, or -1 past the list or when out of range (flagged)
            if (t * kCtRows + grow < R) {
                if (jn >= 0 && jn < nb)
                    jo = jn;
                else if (!isv)
                    flag(DEV_INDEX);
            }
            const uint16_t* src = (isv ? a.V : a.K) + (size_t)b * a.Ncap * 128 + gchunk * 8;
            uint8_t* dst = sm + (isv ? kCtV : kCtK) + (t & 1) * 32768;
#pragma unroll
            for (int p = 0; p < 16; ++p) {
                const int j = __shfl_sync(0xFFFFFFFFu, jo, p);  // lane p holds row 16w + p
                cp_async16_zfill(dst + sw128_off(warp * 16 + p, gchunk, 16384), src + (size_t)(j >= 0 ? j : 0) * 128,
                                 j >= 0);
            }
            const int pn = (t + 1) * kCtRows + grow;
            jn = t + 1 < ntiles && pn < R ? (int)ld_cg_u32(lidx + pn) : 0;
        };
        if (ntiles > 0) gather(0);
        cp_async_commit();
        if (tid < 64) S.m[tid] = -INFINITY;
        float lsum[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) lsum[j] = 0.f;

        for (int i = 0; i < ntiles; ++i) {
            const int bi = i & 1;
            cp_async_wait<0>();  // tile i (and the query's Q) landed
            fence_async_smem();
            __syncthreads();
            // S^T(i) = K Q^T over 8 k-steps of 16 dims
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t ka = sK + bi * 32768 + (ks >> 2) * 16384 + (ks & 3) * 32;
                    const uint32_t qb = sQ + (ks >> 2) * 8192 + (ks & 3) * 32;
                    tc_mma(tmem + 64 * bi, tc_desc(ka, 16, 1024), tc_desc(qb, 16, 1024), id_s, ks > 0);
                }
                tc_commit(&S.bar_s);
                ++pend_s;
            }
            // O^T(i - 1) done: V, P^T of buffer 1 - bi are free for tile i + 1
            if (i >= 1) {
                if (mbar_wait(&S.bar_o, ph_o)) {
                    if (tid == 0) --pend_o;
                } else {
                    S.bad = 1;  // recorded in the status word; this CTA stops below
                }
                ph_o ^= 1;
            }
            if (i + 1 < ntiles) gather(i + 1);
            cp_async_commit();
            if (mbar_wait(&S.bar_s, ph_s)) {
                if (tid == 0) --pend_s;
            } else {
                S.bad = 1;
            }
            ph_s ^= 1;
            tc_fence_after();
            // softmax of tile i: thread = entry, its 32 heads
            const int e = quarter * 32 + lane;
            const bool valid = i * kCtRows + e < R;
            float v[32];
            {
                uint32_t rr[32];
                tc_ld32_nw(tmem + 64 * bi + lane_q + 32 * hh, rr);
                tc_wait_ld();
#pragma unroll
                for (int h = 0; h < 32; ++h) v[h] = valid ? __uint_as_float(rr[h]) * a.scale_log2 : -INFINITY;
            }
            bool over = false;
#pragma unroll
            for (int h = 0; h < 32; ++h) over |= v[h] > S.m[32 * hh + h] + kCtLazy;
            if (__syncthreads_or(over)) {
                // raise the maxima to the exact ones of this tile, rescale the
                // sums and O^T (whose last tile, i - 1, is complete)
                float vm[32];
#pragma unroll
                for (int h = 0; h < 32; ++h) vm[h] = v[h];
                S.red[warp][lane] = warp_transpose_reduce32<true>(vm, lane);  // head 32 * hh + lane
                __syncthreads();
                if (tid < 64) {
                    const int w0 = (tid >> 5) * 4;
                    float mt = S.red[w0][tid & 31];
#pragma unroll
                    for (int q = 1; q < 4; ++q) mt = fmaxf(mt, S.red[w0 + q][tid & 31]);
                    const float mo = S.m[tid], mn = fmaxf(mo, mt);
                    S.alpha[tid] = mo == -INFINITY ? 0.f : ex2_ftz(mo - mn);  // earlier sums are 0 while m is -inf
                    S.m[tid] = mn;
                }
                __syncthreads();
#pragma unroll
                for (int j = 0; j < 32; ++j) lsum[j] *= S.alpha[32 * hh + j];
                if (i > 0) {  // thread = dim here: its row of O^T for its 32 heads
                    uint32_t rr[32];
                    tc_ld32_nw(t_o + lane_q + 32 * hh, rr);
                    tc_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) rr[j] = __float_as_uint(__uint_as_float(rr[j]) * S.alpha[32 * hh + j]);
                    tc_st32(t_o + lane_q + 32 * hh, rr);
                    tc_wait_st();
                }
            }
            // P^T(i) (bf16, heads contiguous): p = 2^(s - m) < 2^8; 0 off the list
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pk[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const int h = c * 8 + w * 2;
                    const float p0 = valid ? ex2_ftz(v[h] - S.m[32 * hh + h]) : 0.f;  // valid: m is finite
                    const float p1 = valid ? ex2_ftz(v[h + 1] - S.m[32 * hh + h + 1]) : 0.f;
                    lsum[h] += p0;
                    lsum[h + 1] += p1;
                    pk[w] = pack_bf16x2(p0, p1);
                }
                const int cc = 4 * hh + c;  // 16-byte chunk of the entry's 128-byte P^T row
                *reinterpret_cast<uint4*>(sm + kCtP + bi * 16384 + (e >> 3) * 1024 + (e & 7) * 128 +
                                          ((cc ^ (e & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            // O^T += V^T P^T over 8 k-steps of 16 entries
            if (tid == 0 && !S.bad) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    tc_mma(t_o, tc_desc(sV + bi * 32768 + ks * 2048, 16384, 1024),
                           tc_desc(sP + bi * 16384 + ks * 2048, 16384, 1024), id_o, (i > 0 || ks > 0) ? 1u : 0u);
                tc_commit(&S.bar_o);
                ++pend_o;
            }
            if (S.bad) break;
        }
        // the query's last O^T group (or, with no tiles, its Q copies)
        if (ntiles > 0 && !S.bad) {
            if (mbar_wait(&S.bar_o, ph_o)) {
                if (tid == 0) --pend_o;
            } else {
                S.bad = 1;
            }
            ph_o ^= 1;
        }
        cp_async_wait<0>();
        tc_fence_after();
        // the sums per head over the entry slots
        S.red[warp][lane] = warp_transpose_reduce32<false>(lsum, lane);
        __syncthreads();
        if (tid < 64) {
            const int w0 = (tid >> 5) * 4;
            float sum = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) sum += S.red[w0 + q][tid & 31];
            S.l[tid] = sum;
        }
        __syncthreads();
        // this query's output: dim d of each of the thread's 32 heads, and the lse
        {
            const int d = quarter * 32 + lane;
            uint32_t rr[32];
            if (ntiles > 0) {
                tc_ld32_nw(t_o + lane_q + 32 * hh, rr);
                tc_wait_ld();
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int h = 32 * hh + j;
                if (h < a.H) {
                    const float L = S.l[h];
                    const float ov = ntiles > 0 ? __uint_as_float(rr[j]) : 0.f;
                    const __nv_bfloat16 y = __float2bfloat16_rn(L > 0.f ? ov / L : 0.f);
                    a.out[((size_t)bq * a.H + h) * 128 + d] = *reinterpret_cast<const uint16_t*>(&y);
                }
            }
            if (a.lse && tid < a.H && tid < 64) {
                const float L = S.l[tid];
                a.lse[(size_t)bq * a.H + tid] = L > 0.f ? (S.m[tid] + __log2f(L)) * 0.6931471805599453f : -INFINITY;
            }
        }
        tc_fence_before();
        __syncthreads();  // tensor memory, S.m and S.l are reused by the next query
        if (S.bad) break;
    }
    // an MMA still in flight after a timeout is waited for (bounded) before
    // its tensor memory is released
    if (tid == 0) {
        for (; pend_s > 0; --pend_s, ph_s ^= 1) mbar_wait(&S.bar_s, ph_s);
        for (; pend_o > 0; --pend_o, ph_o ^= 1) mbar_wait(&S.bar_o, ph_o);
    }
    cp_async_wait<0>();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCtCols));
    }
}

}  // namespace sa
