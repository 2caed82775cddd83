// topk_decode.cuh -- CSA indexer scores and exact top-k for decode (one query
// per sequence), "DeepSeek-V4 ... Review", section 3-2 (2) (CSA keeps a sparse
// top-k of the compressed entries) and 3-2 (4) (the CSA indexer QK path).
//
// The selection is defined on s_j = fp32( fp64 sum_{i=0..63, ascending}
// qI[i] * Ic[j][i] ): keep the k entries with the largest (s_j, -j), report
// them in ascending j.  The kernels reach exactly that set without computing
// every s_j in fp64:
//
//   screen   s~_j = fp32 FMA chain over the same products (each bf16 x bf16
//            product is exact in fp32), a~_j = fp32 FMA chain of |q||k|.
//            Recursive summation bounds |s~_j - s_j| <= e_j with
//              e_j = 2^-16 a~_j + 2^-22 |s~_j| + 2^-140
//            (2^-18 would already cover the 64-term fp32 chain, the fp64
//            chain and the final fp32 rounding; the absolute term covers
//            products that underflow fp32).  E = max_j e_j per sequence.
//   order    if t~ is the k-th largest s~, the k-th largest s lies within E
//            of it, so entries with s~ > t~ + 2E are surely selected, entries
//            with s~ < t~ - 2E surely not, and only the band |s~ - t~| <= 2E
//            is rescored exactly (the fp64 definition) and ranked exactly.
//
// Four kernels, ordered on one stream (every hand-off is a kernel boundary,
// chained by programmatic dependent launch; no CTA waits on another):
//   1. score_decode_kernel -- streams Ic through a 4-stage TMA pipeline
//      (128-byte rows, 128B swizzle, one row per thread) and writes an order
//      key of s~ per entry, a histogram of the top 11 key bits (per CTA in
//      shared memory, then added to the sequence's) and each CTA's max e_j;
//      the sequence's last CTA to finish then finds the bin d1 of t~, the
//      keys above it and E, once.
//   2. topk_filter_kernel  -- one CTA per 2048 rows: entries above bin d1
//      widened by 2E become bitmap bits (surely selected, counted per chunk),
//      entries in the widened bin become candidates (compact slots of the
//      chunk), and those inside bin d1 feed a histogram of key bits 20..10.
//   3. topk_resolve_kernel -- one 1024-thread CTA per sequence: the second
//      histogram gives the fine bin of t~, whose few keys are ranked; the band
//      is rescored exactly and ranked by (s, -j); the winners join the bitmap
//      and every chunk gets the output position of its first selected entry.
//   4. topk_emit_kernel    -- one CTA per chunk writes its selected indices,
//      ascending, from that position on.
#pragma once
#include "sa_common.cuh"

namespace sa {

constexpr int kScRows = 128;      // rows per TMA tile (box height)
constexpr int kScStages = 4;      // TMA pipeline depth
constexpr int kScThreads = 128;   // one row per thread per tile
constexpr int kScTileBytes = kScRows * 128;
constexpr int kBins = 2048;       // 11-bit digits
constexpr int kBinsLow = 1024;    // last 10-bit digit

// totals[B][kTotals] (zeroed per call): the score CTAs' finish ticket, and
// from the last of them the bin d1 of t~, the bound E and the count of keys
// above bin d1
constexpr int kTotals = 4;
constexpr int kTotTicket = 0, kTotBin = 1, kTotE = 2, kTotAbove = 3;
constexpr int kFiltRows = 2048;  // rows per filter / emit CTA (one pass of 256 threads x 8 keys)
constexpr int kSlots = 64;       // compact candidate slots per filter chunk

struct TopkDecodeArgs {
    const uint16_t* q_idx;  // [B][64]
    const uint16_t* kidx;   // [B][Ncap][64] (exact rescoring)
    const int32_t* n;       // [B]
    uint32_t* keys;         // [B][Ncap]     order keys of the screened scores
    uint32_t* hist1;        // [B][2048]     histogram of key bits 31..21 (zeroed per call)
    uint32_t* hist2;        // [B][2048]     bits 20..10 of the keys in bin d1 (zeroed per call)
    float* emax_part;       // [B][nchunks]  per score CTA: max e_j
    uint32_t* chunk_in;     // [B][nfch]     per filter chunk: surely selected entries
    uint32_t* chunk_cnt;    // [B][nfch]     per filter chunk: candidates
    uint32_t* chunk_pos;    // [B][nfch]     output position of each filter chunk's first selected entry
    uint2* cslot;           // [B][nfch][kSlots] the first kSlots candidates of each filter chunk (key, index)
    uint32_t* cand_key;     // [B][Ncap]     further candidates of a chunk, in the chunk's own rows
    int32_t* cand_idx;      // [B][Ncap]
    uint32_t* cmp_key;      // [B][Ncap]     all candidates in one list, when they overflow shared memory
    int32_t* cmp_idx;       // [B][Ncap]
    uint32_t* totals;       // [B][kTotals]
    uint32_t* bitmap;       // [B][Wcap]     selection bitmap
    uint32_t* amb_key;      // [B][Ncap]     exact keys of the band, when it is large
    int32_t* amb_idx;       // [B][Ncap]
    int32_t* idx;           // [B][k]
    int32_t* cnt;           // [B]
    int Ncap, Wcap, chunk, nchunks, fchunk, nfch, k;
};

__device__ __forceinline__ int clamp_n(const int32_t* n, int b, int Ncap) {
    int v = n[b];
    if (v < 0 || v > Ncap) {
        flag(DEV_LEN);
        v = v < 0 ? 0 : Ncap;
    }
    return v;
}

__device__ __forceinline__ float key_to_float(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// The exact score of one indexer row (the definition): fp64 FMA chain in
// ascending i over exact products, rounded once to fp32, -0 -> +0, as a key.
// q2 holds qI[i] * 2^768 in fp64 (see below); the row's bf16 values enter as
// x * 2^-896 through bit placement, so each product is qI*k * 2^-128 exactly
// and no conversion instruction is needed per element.
// SMEM: the row is staged in shared memory (read with ordinary loads);
// otherwise it is read from global memory through the read-only path.
template <bool SMEM = false>
__device__ __noinline__ uint32_t exact_key(const double* q2, const uint16_t* row) {
    const uint4* r4 = reinterpret_cast<const uint4*>(row);
    double acc = 0.0;
#pragma unroll 2
    for (int c = 0; c < 8; ++c) {
        const uint4 w = SMEM ? r4[c] : __ldg(r4 + c);
        acc = fma(q2[8 * c + 0], bf16lo_scaled(w.x), acc);
        acc = fma(q2[8 * c + 1], bf16hi_scaled(w.x), acc);
        acc = fma(q2[8 * c + 2], bf16lo_scaled(w.y), acc);
        acc = fma(q2[8 * c + 3], bf16hi_scaled(w.y), acc);
        acc = fma(q2[8 * c + 4], bf16lo_scaled(w.z), acc);
        acc = fma(q2[8 * c + 5], bf16hi_scaled(w.z), acc);
        acc = fma(q2[8 * c + 6], bf16lo_scaled(w.w), acc);
        acc = fma(q2[8 * c + 7], bf16hi_scaled(w.w), acc);
    }
    return score_key(__double2float_rn(acc * 0x1p128));
}

// --------------------------------------------------- digit search helpers --
// Descending: the digit d with  above(d) < K <= above(d) + h[d], where
// above(d) = sum of h[e] for e > d.  Every thread gets (d, above(d)).
template <int NB>
__device__ __forceinline__ void find_digit_desc(const uint32_t* h, uint32_t K, uint32_t* sh32, int* out_d, uint32_t* out_above,
                                int* res) {
    const int T = blockDim.x;
    const int per = (NB + T - 1) / T;
    const int u = T - 1 - threadIdx.x;  // thread t handles the bins of thread u, so the scan runs high -> low
    const int lo = u * per, hi = min(NB, lo + per);
    uint32_t local = 0;
#pragma unroll 1
    for (int e = lo; e < hi; ++e) local += h[e];
    uint32_t above = block_exclusive_scan(local, sh32, nullptr);
    if (threadIdx.x == 0) {
        res[0] = -1;
        res[1] = 0;
    }
    __syncthreads();
#pragma unroll 1
    for (int e = hi - 1; e >= lo; --e) {
        const uint32_t c = h[e];
        if (above < K && K <= above + c) {
            res[0] = e;
            res[1] = (int)above;
        }
        above += c;
    }
    __syncthreads();
    *out_d = res[0];
    *out_above = (uint32_t)res[1];
    __syncthreads();
}

// Ascending: the digit d with  below(d) < R <= below(d) + h[d].
template <int NB>
__device__ __forceinline__ void find_digit_asc(const uint32_t* h, uint32_t R, uint32_t* sh32, int* out_d, uint32_t* out_below,
                               int* res) {
    const int T = blockDim.x;
    const int per = (NB + T - 1) / T;
    const int lo = threadIdx.x * per, hi = min(NB, lo + per);
    uint32_t local = 0;
    for (int e = lo; e < hi; ++e) local += h[e];
    uint32_t below = block_exclusive_scan(local, sh32, nullptr);
    if (threadIdx.x == 0) {
        res[0] = -1;
        res[1] = 0;
    }
    __syncthreads();
    for (int e = lo; e < hi; ++e) {
        const uint32_t c = h[e];
        if (below < R && R <= below + c) {
            res[0] = e;
            res[1] = (int)below;
        }
        below += c;
    }
    __syncthreads();
    *out_d = res[0];
    *out_below = (uint32_t)res[1];
    __syncthreads();
}

// Descending digit search over T * NPT bins held in registers: thread t
// holds bins [T*NPT - (t+1)*NPT, T*NPT - t*NPT) as h[0..NPT) in ascending
// order (thread 0 holds the top bins).  Loaded straight from global memory,
// the bins need no shared-memory staging (no bank conflicts).
template <int NPT>
__device__ __forceinline__ void find_digit_desc_regs(const uint32_t (&h)[NPT], uint32_t K, uint32_t* sh32, int* res,
                                                     int* out_d, uint32_t* out_above) {
    const int t = threadIdx.x;
    uint32_t local = 0;
#pragma unroll
    for (int j = 0; j < NPT; ++j) local += h[j];
    if (t == 0) res[0] = -1;  // ordered before every write below by the scan's barriers
    uint32_t above = block_exclusive_scan(local, sh32, nullptr);  // keys in the bins above this range
    const int lo = ((int)blockDim.x - 1 - t) * NPT;
#pragma unroll
    for (int j = NPT - 1; j >= 0; --j) {
        if (above < K && K <= above + h[j]) {
            res[0] = lo + j;
            res[1] = (int)above;
        }
        above += h[j];
    }
    __syncthreads();
    *out_d = res[0];
    *out_above = (uint32_t)res[1];
    __syncthreads();
}

// Exclusive scans of two values at once (one set of barriers).
__device__ __forceinline__ void block_exclusive_scan2(uint32_t v0, uint32_t v1, uint32_t* sh64, uint32_t* e0,
                                                      uint32_t* e1, uint32_t* t0, uint32_t* t1) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t x0 = v0, x1 = v1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y0 = __shfl_up_sync(0xFFFFFFFFu, x0, o), y1 = __shfl_up_sync(0xFFFFFFFFu, x1, o);
        if (lane >= o) {
            x0 += y0;
            x1 += y1;
        }
    }
    if (lane == 31) {
        sh64[warp] = x0;
        sh64[32 + warp] = x1;
    }
    __syncthreads();
    if (warp == 0) {
        uint32_t w0 = lane < nw ? sh64[lane] : 0u, w1 = lane < nw ? sh64[32 + lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y0 = __shfl_up_sync(0xFFFFFFFFu, w0, o), y1 = __shfl_up_sync(0xFFFFFFFFu, w1, o);
            if (lane >= o) {
                w0 += y0;
                w1 += y1;
            }
        }
        sh64[lane] = w0;
        sh64[32 + lane] = w1;
    }
    __syncthreads();
    *e0 = (warp ? sh64[warp - 1] : 0u) + x0 - v0;
    *e1 = (warp ? sh64[32 + warp - 1] : 0u) + x1 - v1;
    *t0 = sh64[nw - 1];
    *t1 = sh64[32 + nw - 1];
    __syncthreads();
}

// Warp-aggregated shared-memory histogram increment (many equal bins).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool valid) {
    const uint32_t b = valid ? bin : 0xFFFFFFFFu;
    const uint32_t peers = __match_any_sync(0xFFFFFFFFu, b);
    const int leader = __ffs(peers) - 1;
    if (valid && (int)(threadIdx.x & 31) == leader) red_add_shared(&hist[bin], (uint32_t)__popc(peers));
}

// Among list entries (key[i], idx[i]), i < cnt, find the R-th largest by
// (key desc, idx asc): returns T and jmax such that exactly R entries satisfy
// key > T || (key == T && idx <= jmax).  hist: >= 2048 words of shared memory.
__device__ __forceinline__ void select_rank(const uint32_t* key, const int32_t* idx, uint32_t cnt, uint32_t R, uint32_t* hist,
                            uint32_t* sh32, int* res, uint32_t* T_out, int32_t* jmax_out) {
    const int shifts[3] = {21, 10, 0};
    const int widths[3] = {11, 11, 10};
    uint32_t prefix = 0, pmask = 0, rem = R;
    for (int p = 0; p < 3; ++p) {
        for (int i = threadIdx.x; i < kBins; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (uint32_t i0 = 0; i0 < cnt; i0 += blockDim.x) {  // warp-uniform trip count
            const uint32_t i = i0 + threadIdx.x;
            const uint32_t kk = i < cnt ? key[i] : 0u;
            hist_add(hist, (kk >> shifts[p]) & ((1u << widths[p]) - 1), i < cnt && (kk & pmask) == prefix);
        }
        __syncthreads();
        int d;
        uint32_t above;
        find_digit_desc<kBins>(hist, rem, sh32, &d, &above, res);
        if (d < 0) {
            if (threadIdx.x == 0) flag(DEV_LEN);  // inconsistent counts: cannot happen
            d = 0;
        }
        rem -= above;
        prefix |= (uint32_t)d << shifts[p];
        pmask |= ((1u << widths[p]) - 1) << shifts[p];
    }
    const uint32_t T = prefix;
    // ties at T: keep the rem with the lowest indices (indices < 2^31)
    uint32_t nties = 0;
    for (uint32_t i = threadIdx.x; i < cnt; i += blockDim.x) nties += key[i] == T;
    uint32_t total;
    block_exclusive_scan(nties, sh32, &total);
    int32_t jmax = 0x7FFFFFFF;
    if (rem < total) {
        const int ishift[3] = {20, 9, 0};
        const int iwidth[3] = {11, 11, 9};
        uint32_t ip = 0, im = 0, r2 = rem;
        for (int p = 0; p < 3; ++p) {
            for (int i = threadIdx.x; i < kBins; i += blockDim.x) hist[i] = 0;
            __syncthreads();
            for (uint32_t i0 = 0; i0 < cnt; i0 += blockDim.x) {
                const uint32_t i = i0 + threadIdx.x;
                const bool tie = i < cnt && key[i] == T;
                const uint32_t j = tie ? (uint32_t)idx[i] : 0u;
                hist_add(hist, (j >> ishift[p]) & ((1u << iwidth[p]) - 1), tie && (j & im) == ip);
            }
            __syncthreads();
            int d;
            uint32_t below;
            find_digit_asc<kBins>(hist, r2, sh32, &d, &below, res);
            if (d < 0) d = 0;
            r2 -= below;
            ip |= (uint32_t)d << ishift[p];
            im |= ((1u << iwidth[p]) - 1) << ishift[p];
        }
        jmax = (int32_t)ip;
    }
    *T_out = T;
    *jmax_out = jmax;
}

// The R-th largest key among cnt list keys, knowing that all of them except
// a rare fringe share the top 11 bits d1 (the candidates of a filter bin):
// keys above the bin are counted, the rest resolved with two digit passes
// (bits 20..10 and 9..0), whose bins are well spread, with plain shared
// atomics.  Returns false if the rank falls outside the bin (caller then
// uses the general select_rank).
__device__ __noinline__ bool rank_in_bin(const uint32_t* key, uint32_t cnt, uint32_t R, int d1, uint32_t* hist,
                                         uint32_t* sh32, int* res, uint32_t* T_out) {
    uint32_t above = 0, inbin = 0;
#pragma unroll 1
    for (uint32_t i = threadIdx.x; i < cnt; i += blockDim.x) {
        const int dig = (int)(key[i] >> 21);
        above += dig > d1;
        inbin += dig == d1;
    }
    uint32_t tot_above, tot_in;
    block_exclusive_scan(above, sh32, &tot_above);
    block_exclusive_scan(inbin, sh32, &tot_in);
    if (R <= tot_above || R > tot_above + tot_in) return false;
    uint32_t rem = R - tot_above;
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) hist[i] = 0;
    __syncthreads();
#pragma unroll 1
    for (uint32_t i = threadIdx.x; i < cnt; i += blockDim.x) {
        const uint32_t kk = key[i];
        if ((int)(kk >> 21) == d1) red_add_shared(&hist[(kk >> 10) & (kBins - 1)], 1u);
    }
    __syncthreads();
    int d2, d3;
    uint32_t ab;
    find_digit_desc<kBins>(hist, rem, sh32, &d2, &ab, res);
    rem -= ab;
    const uint32_t pre = ((uint32_t)d1 << 11) | (uint32_t)d2;
    for (int i = threadIdx.x; i < kBinsLow; i += blockDim.x) hist[i] = 0;
    __syncthreads();
#pragma unroll 1
    for (uint32_t i = threadIdx.x; i < cnt; i += blockDim.x) {
        const uint32_t kk = key[i];
        if ((kk >> 10) == pre) red_add_shared(&hist[kk & (kBinsLow - 1)], 1u);
    }
    __syncthreads();
    find_digit_desc<kBinsLow>(hist, rem, sh32, &d3, &ab, res);
    if (d2 < 0 || d3 < 0) return false;
    *T_out = (pre << 10) | (uint32_t)d3;
    return true;
}

// ------------------------------------------------------------ 1. scores ----
__global__ void __launch_bounds__(kScThreads, 3)
    score_decode_kernel(const __grid_constant__ CUtensorMap ic_map, TopkDecodeArgs a) {
    extern __shared__ uint8_t smem_raw[];
    // TMA with 128B swizzle needs a 1024-byte aligned destination
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* tiles = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kScStages * kScTileBytes);
    __shared__ float s_emax[kScThreads / 32];
    __shared__ uint32_t hist[kBins];  // top 11 key bits of this CTA's rows
    __shared__ uint32_t s_sh32[32];
    __shared__ int s_res[2];
    __shared__ uint32_t s_last;

    pdl_wait();
    pdl_release();
    SA_TRACE_MARK(TR_SCORE, 0);
    const int b = blockIdx.y;
    const int tid = threadIdx.x;
    const int row0 = blockIdx.x * a.chunk;
    // The first tiles go out before the length is known: rows below Ncap
    // exist in the cache whatever n is (rows at or past n are read, not used).
    // The map views Ic as [B][Ncap][64]: coordinates (dim, row, sequence).
    const int srows = max(0, min(row0 + a.chunk, a.Ncap) - row0);
    const int stiles = (srows + kScRows - 1) / kScRows;
    int issued = 0;
    if (tid == 0) {
        for (int s = 0; s < kScStages; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
        for (; issued < kScStages && issued < stiles; ++issued) {
            mbar_expect_tx(&full[issued], kScTileBytes);
            tma_load_3d(tiles + issued * kScTileBytes, &ic_map, 0, row0 + issued * kScRows, b, &full[issued]);
        }
    }
    const int n = clamp_n(a.n, b, a.Ncap);
    if (n <= a.k) {
        // everything visible is selected, nothing to score; the early copies
        // land before the CTA's shared memory goes away
        if (tid == 0)
            for (int i = 0; i < issued; ++i) mbar_wait(&full[i % kScStages], (i / kScStages) & 1);
        return;
    }
    const int row1 = min(row0 + a.chunk, n);
    // an empty chunk scans nothing but still takes part in the finish below
    const int ntiles = row1 > row0 ? (row1 - row0 + kScRows - 1) / kScRows : 0;

    float q[64];
    {
        const uint32_t* qw = reinterpret_cast<const uint32_t*>(a.q_idx + (size_t)b * 64);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const uint32_t w = __ldg(qw + i);
            q[2 * i] = bf16lo_f32(w);
            q[2 * i + 1] = bf16hi_f32(w);
        }
    }
    for (int i = tid; i < kBins; i += blockDim.x) hist[i] = 0;
    __syncthreads();

    int consumed = 0;
    bool timed_out = false;
    float emax = 0.f;
    for (int i = 0; i < ntiles; ++i) {
        const int s = i % kScStages;
        const bool ok = mbar_wait(&full[s], (i / kScStages) & 1);
        if (__syncthreads_or(!ok)) {
            timed_out = true;
            break;
        }
        consumed = i + 1;
        const int row = row0 + i * kScRows + tid;
        if (row < row1) {
            const uint8_t* rp = tiles + s * kScTileBytes + tid * 128;
            float acc = 0.f, aab = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 w = *reinterpret_cast<const uint4*>(rp + ((c ^ (tid & 7)) << 4));
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float k0 = bf16lo_f32(ws[h]), k1 = bf16hi_f32(ws[h]);
                    acc = fmaf(q[8 * c + 2 * h], k0, acc);
                    aab = fmaf(fabsf(q[8 * c + 2 * h]), fabsf(k0), aab);
                    acc = fmaf(q[8 * c + 2 * h + 1], k1, acc);
                    aab = fmaf(fabsf(q[8 * c + 2 * h + 1]), fabsf(k1), aab);
                }
            }
            const uint32_t key = score_key(acc);
            a.keys[(size_t)b * a.Ncap + row] = key;
            atomicAdd(&hist[key >> 21], 1u);
            emax = fmaxf(emax, fmaf(aab, 0x1p-16f, fmaf(fabsf(acc), 0x1p-22f, 0x1p-140f)));
        }
        __syncthreads();  // slot s is free again
        if (tid == 0 && issued < ntiles) {
            fence_proxy_async();
            mbar_expect_tx(&full[s], kScTileBytes);
            tma_load_3d(tiles + s * kScTileBytes, &ic_map, 0, row0 + issued * kScRows, b, &full[s]);
            ++issued;
        }
    }
    // copies not consumed (tiles issued past the chunk's end, or after a
    // timeout, which the device status records) land before the CTA's shared
    // memory goes away
    if (tid == 0)
        for (int i = consumed; i < issued; ++i) mbar_wait(&full[i % kScStages], (i / kScStages) & 1);
    if (timed_out) __syncthreads();
    // e_j is rounded to nearest in fp32: one more ulp keeps it an upper bound
    emax = __uint_as_float(__float_as_uint(emax) + 1u);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) emax = fmaxf(emax, __shfl_xor_sync(0xFFFFFFFFu, emax, o));
    if ((tid & 31) == 0) s_emax[tid >> 5] = emax;
    __syncthreads();
    if (tid == 0) {
        float m = s_emax[0];
        for (int w = 1; w < kScThreads / 32; ++w) m = fmaxf(m, s_emax[w]);
        a.emax_part[(size_t)b * a.nchunks + blockIdx.x] = m;
    }
    for (int i = tid; i < kBins; i += blockDim.x)
        if (hist[i]) atomicAdd(&a.hist1[(size_t)b * kBins + i], hist[i]);

    // The last CTA of the sequence to finish finds, once for every filter
    // CTA, the bin d1 of the k-th largest key, the count of keys above it
    // and the sequence's bound E.  (Ticket pattern: no CTA waits.  The
    // ticket is an acquire-release add after a barrier: it publishes this
    // CTA's histogram and bound, and the last CTA sees every other CTA's.)
    uint32_t* tot = a.totals + (size_t)b * kTotals;
    __syncthreads();
    SA_TRACE_MARK(TR_SCORE, 1);
    if (tid == 0) {
        uint32_t old;
        asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(old) : "l"(tot + kTotTicket) : "memory");
        s_last = old == gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last) return;
    constexpr int NPT = kBins / kScThreads;  // 16 bins per thread
    uint32_t hb[NPT];
    {
        const uint32_t* src = a.hist1 + (size_t)b * kBins + (kScThreads - 1 - tid) * NPT;
#pragma unroll
        for (int v = 0; v < NPT / 4; ++v) {
            const uint4 x = ld_cg_u32x4(src + 4 * v);
            hb[4 * v] = x.x;
            hb[4 * v + 1] = x.y;
            hb[4 * v + 2] = x.z;
            hb[4 * v + 3] = x.w;
        }
    }
    float e = 0.f;
    for (int q = tid; q < a.nchunks; q += blockDim.x) e = fmaxf(e, __ldcg(a.emax_part + (size_t)b * a.nchunks + q));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) e = fmaxf(e, __shfl_xor_sync(0xFFFFFFFFu, e, o));
    __syncthreads();  // every s_emax read above is done
    if ((tid & 31) == 0) s_emax[tid >> 5] = e;
    __syncthreads();
    float E = s_emax[0];
#pragma unroll
    for (int w = 1; w < kScThreads / 32; ++w) E = fmaxf(E, s_emax[w]);
    int d1;
    uint32_t above1;
    find_digit_desc_regs<NPT>(hb, (uint32_t)a.k, s_sh32, s_res, &d1, &above1);
    if (tid == 0) {
        if (d1 < 0) {  // cannot happen: the histogram counts all n > k keys
            flag(DEV_LEN);
            d1 = 0;
            above1 = 0;
        }
        tot[kTotBin] = (uint32_t)d1;
        tot[kTotE] = __float_as_uint(E);
        tot[kTotAbove] = above1;
    }
    SA_TRACE_MARK(TR_SCORE, 2);
}

// --------------------------------------------------------- 2. selection ----
constexpr int kSelThreads = 256;             // filter CTAs
constexpr int kFiltKPT = kFiltRows / kSelThreads;
constexpr int kResThreads = 1024;            // resolve CTA (one per sequence)
constexpr int kSelCap = 8192;                // candidates the resolving CTA holds in shared memory
constexpr int kSelSmem = kSelCap * 8;
constexpr int kSelMaxChunks = 1024;          // filter chunks per sequence
constexpr int kGatherJ = 4;                  // filter chunks per warp loaded ahead by the resolve
constexpr int kGatherS = 2;                  // ... and compact slots per lane of each
constexpr int kPf = 64;                      // index rows staged for the band
static_assert(kSelMaxChunks == kResThreads, "the resolve gives one thread to every chunk");
static_assert(kBins == 2 * kResThreads, "the resolve loads the second histogram two bins per thread");
static_assert(kFiltKPT * kSelThreads == kFiltRows, "one filter pass covers a chunk");
static_assert(32 * kGatherS <= kSlots, "preloaded slots are compact slots");

struct FilterBounds {
    float in_above;  // s~ > in_above  : surely selected
    float c_lo;      // c_lo <= s~ <= in_above : candidate
};

// The bin of the k-th largest screened key, widened by 2E on both sides.
__device__ __forceinline__ FilterBounds filter_bounds(int d1, float E) {
    float lo = key_to_float((uint32_t)d1 << 21);
    float hi = key_to_float(((uint32_t)d1 << 21) | 0x1FFFFFu);
    if (isnan(lo)) lo = -INFINITY;  // the outermost bins also hold the NaN key ranges
    if (isnan(hi)) hi = INFINITY;
    const float e2 = __fmul_ru(2.f, E);
    return {__fadd_ru(hi, e2), __fsub_rd(lo, e2)};
}

struct SelSmem {
    double q2[64];                  // qI * 2^768 for the exact rescoring
    uint32_t hist[kBins];           // digit histograms of the fallback searches
    uint32_t base[kSelMaxChunks];   // compact position of each filter chunk's candidates
    uint32_t ccnt[kSelMaxChunks];   // candidates per filter chunk
    uint32_t wcnt[kSelMaxChunks];   // winners among each chunk's candidates
    uint32_t sh64[64];
    int res[2];
    uint32_t f_cnt, found, tkey, amb_cnt, T2, pf_cnt;
    int32_t jmax2;
    uint32_t amb_key[kResThreads];  // the fine bin's keys, then the band's exact keys
    int32_t amb_idx[kResThreads];
    // index rows of the candidates within two fine bins of t~'s, staged for
    // the exact rescoring of the band
    uint32_t pf_key[kPf];
    int32_t pf_j[kPf];
    __align__(16) uint16_t pf_row[kPf][64];
};

// Filter: one CTA per kFiltRows (2048) rows.  Entries above the widened bin of t~ become
// bitmap bits (surely selected, counted), the rest of the widened bin become
// candidates in the chunk's own rows of the candidate arrays, and keys
// inside bin d1 feed the second histogram.  Integer compares on order keys.
__global__ void __launch_bounds__(kSelThreads) topk_filter_kernel(TopkDecodeArgs a) {
    __shared__ uint32_t s_cnt, s_in;
    pdl_wait();
    pdl_release();
    SA_TRACE_MARK(TR_FILTER, 0);
    const int b = blockIdx.y, c = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = a.k;
    const int row0 = c * a.fchunk;
    const int rcap = min(row0 + a.fchunk, a.Ncap);  // rows present in the arrays
    const uint32_t* keys = a.keys + (size_t)b * a.Ncap;
    const uint32_t* tot = a.totals + (size_t)b * kTotals;
    // every load goes out before the length is known: the first pass's keys
    // and the thresholds (one round trip; none of them depends on n)
    uint32_t kr[kFiltKPT];
#pragma unroll
    for (int i = 0; i < kFiltKPT; ++i) {
        const int row = row0 + i * kSelThreads + tid;
        kr[i] = row < rcap ? ld_cg_u32(keys + row) : 0u;
    }
    const int d1 = (int)ld_cg_u32(tot + kTotBin);
    const float E = __uint_as_float(ld_cg_u32(tot + kTotE));
    const int n = clamp_n(a.n, b, a.Ncap);
    if (n <= k) {
        if (c == 0) {
            int32_t* idx = a.idx + (size_t)b * k;
            for (int i = tid; i < k; i += blockDim.x) idx[i] = i < n ? i : -1;
            if (tid == 0) a.cnt[b] = n;
        }
        return;
    }
    const int row1 = min(row0 + a.fchunk, n);
    if (tid == 0) {
        s_cnt = 0;
        s_in = 0;
    }
    const FilterBounds fb = filter_bounds(d1, E);
    const uint32_t in_key = score_key(fb.in_above), lo_key = score_key(fb.c_lo);  // order-preserving
    uint2* cs = a.cslot + ((size_t)b * a.nfch + c) * kSlots;
    uint32_t* ck = a.cand_key + (size_t)b * a.Ncap + row0;
    int32_t* ci = a.cand_idx + (size_t)b * a.Ncap + row0;
    uint32_t* bm = a.bitmap + (size_t)b * a.Wcap;
    uint32_t* h2 = a.hist2 + (size_t)b * kBins;
    __syncthreads();
    uint32_t nin = 0;
#pragma unroll 1
    for (int p0 = row0; p0 < row1; p0 += kFiltRows) {  // one pass unless the chunk is larger
        if (p0 != row0) {
#pragma unroll
            for (int i = 0; i < kFiltKPT; ++i) {
                const int row = p0 + i * kSelThreads + tid;
                kr[i] = row < row1 ? __ldcg(keys + row) : 0u;
            }
        }
#pragma unroll
        for (int i = 0; i < kFiltKPT; ++i) {
            const int row = p0 + i * kSelThreads + tid;
            const int wrow = p0 + i * kSelThreads + warp * 32;  // this warp's 32 consecutive rows
            const bool valid = row < row1;
            const bool sel = valid && kr[i] > in_key;
            const uint32_t selm = __ballot_sync(0xFFFFFFFFu, sel);
            if (lane == 0 && wrow < row1) bm[wrow >> 5] = selm;  // row0 is a multiple of 32
            nin += __popc(selm);
            if (valid && !sel && kr[i] >= lo_key) {
                const uint32_t p = atom_add_shared(&s_cnt, 1u);
                if (p < (uint32_t)kSlots) {
                    cs[p] = make_uint2(kr[i], (uint32_t)row);
                } else {
                    ck[p] = kr[i];
                    ci[p] = row;
                }
                if ((int)(kr[i] >> 21) == d1) atomicAdd(h2 + ((kr[i] >> 10) & (kBins - 1)), 1u);
            }
        }
    }
    if (lane == 0 && nin) red_add_shared(&s_in, nin);  // every lane counted the same ballots
    __syncthreads();
    SA_TRACE_MARK(TR_FILTER, 1);
    if (tid == 0) {
        a.chunk_in[(size_t)b * a.nfch + c] = s_in;
        a.chunk_cnt[(size_t)b * a.nfch + c] = s_cnt;
    }
}

// The resolve once the counts are scanned, over the candidate list held in
// shared memory (SMEM, the usual case) or in global memory (overflow).
// Gathers the chunks' candidates into one list (collecting the keys of the
// fine bin of t~ and prefetching into L2 the index rows around it, which
// the exact rescoring of the band will read), finds t~, rescores the band
// exactly, cuts it by (s, -j), adds the winners to the bitmap and gives
// every chunk its output position.  EXACT: the keys are the exact scores
// already (E = 0, the band is the keys equal to t~'s), so nothing is staged
// or rescored.
template <bool SMEM, bool EXACT>
__device__ __forceinline__ void resolve_body(const TopkDecodeArgs& a, SelSmem& S, uint32_t* csm, int b, uint32_t C,
                                             uint32_t A, int d1, float E, int d2, uint32_t above2, uint32_t K2,
                                             const uint32_t (&pk)[kGatherJ * kGatherS],
                                             const int32_t (&pi)[kGatherJ * kGatherS],
                                             uint32_t cin) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = a.k, nfch = a.nfch;
    uint32_t* lk = SMEM ? csm : a.cmp_key + (size_t)b * a.Ncap;
    int32_t* li = SMEM ? reinterpret_cast<int32_t*>(csm + kSelCap) : a.cmp_idx + (size_t)b * a.Ncap;
    const uint2* cs = a.cslot + (size_t)b * nfch * kSlots;
    const uint32_t* gk = a.cand_key + (size_t)b * a.Ncap;
    const int32_t* gi = a.cand_idx + (size_t)b * a.Ncap;
    const uint16_t* icx = a.kidx + (size_t)b * a.Ncap * 64;
    const uint32_t pre = ((uint32_t)d1 << 11) | (uint32_t)(d2 < 0 ? 0 : d2);
    auto put = [&](uint32_t pos, uint32_t kk, int32_t j) {
        lk[pos] = kk;
        li[pos] = j;
        const uint32_t f = kk >> 10;
        if (d2 >= 0 && f + 2 >= pre && f <= pre + 2) {  // within two fine bins of t~'s
            const uint32_t q = atom_add_shared(&S.pf_cnt, 1u);
            if (q < (uint32_t)kPf) {
                S.pf_key[q] = kk;
                S.pf_j[q] = j;
                if (!EXACT) {
                    const uint16_t* row = icx + (size_t)j * 64;
#pragma unroll
                    for (int u = 0; u < 8; ++u) cp_async16(&S.pf_row[q][u * 8], row + u * 8);
                }
            }
            if (f == pre) {
                const uint32_t p = atom_add_shared(&S.f_cnt, 1u);
                if (p < (uint32_t)kResThreads) S.amb_key[p] = kk;
            }
        }
    };
#pragma unroll
    for (int j = 0; j < kGatherJ; ++j) {
        const int c = warp + 32 * j;
#pragma unroll
        for (int u = 0; u < kGatherS; ++u) {
            const uint32_t sl = (uint32_t)(lane + 32 * u);
            if (c < nfch && sl < S.ccnt[c]) put(S.base[c] + sl, pk[j * kGatherS + u], pi[j * kGatherS + u]);
        }
    }
#pragma unroll 1
    for (int c = warp; c < nfch; c += 32) {  // further slots, chunks beyond the first kGatherJ per warp
        const uint32_t cn = S.ccnt[c], cb = S.base[c];
        const uint32_t from = c < 32 * kGatherJ ? 32u * kGatherS : 0u;
        for (uint32_t i = from + lane; i < cn; i += 32) {
            if (i < (uint32_t)kSlots) {
                const uint2 e = cs[(size_t)c * kSlots + i];
                put(cb + i, e.x, (int32_t)e.y);
            } else {
                put(cb + i, __ldcg(gk + (size_t)c * a.fchunk + i), __ldcg(gi + (size_t)c * a.fchunk + i));
            }
        }
    }
    cp_async_commit();  // the staged rows are awaited just before the band
    if (!SMEM) __threadfence_block();
    __syncthreads();
    SA_TRACE_MARK(TR_RESOLVE, 2);

    // t~: the R3-th largest key of the fine bin (few keys: ranked pairwise)
    const uint32_t R1 = (uint32_t)k - A;  // rank of t~ among the candidates (>= 1)
    bool fast = false;
    if (d2 >= 0) {
        const uint32_t nf = S.f_cnt;
        const uint32_t R3 = K2 - above2;
        if (nf <= (uint32_t)kResThreads && R3 >= 1 && R3 <= nf) {
            if ((uint32_t)tid < nf) {
                const uint32_t mk = S.amb_key[tid];
                uint32_t gt = 0, ge = 0;
                for (uint32_t o = 0; o < nf; ++o) {
                    const uint32_t ok = S.amb_key[o];
                    gt += ok > mk;
                    ge += ok >= mk;
                }
                if (gt < R3 && R3 <= ge) {  // every thread holding t~ writes the same value
                    S.tkey = mk;
                    S.found = 1;
                }
            }
            __syncthreads();
            fast = S.found != 0;
        }
    }
    uint32_t tkey;
    if (fast) {
        tkey = S.tkey;
    } else if (!rank_in_bin(lk, C, R1, d1, S.hist, S.sh64, S.res, &tkey)) {
        int32_t jd;
        select_rank(lk, li, C, R1, S.hist, S.sh64, S.res, &tkey, &jd);
    }
    const float t = key_to_float(tkey);
    const float e2 = __fmul_ru(2.f, E);
    const uint32_t bhi_key = score_key(__fadd_ru(t, e2)), blo_key = score_key(__fsub_rd(t, e2));
    // the band list (global, used when the band is large)
    uint32_t* gak = a.amb_key + (size_t)b * a.Ncap;
    int32_t* gai = a.amb_idx + (size_t)b * a.Ncap;
    cp_async_wait<0>();
    __syncthreads();  // S.amb_key held the fine bin; the staged rows have landed
    SA_TRACE_MARK(TR_RESOLVE, 3);
    // when the band lies inside the staged window, its members are all staged
    const uint32_t lo_w = pre >= 2u ? (pre - 2u) << 10 : 0u;
    const bool win = fast && S.pf_cnt <= (uint32_t)kPf && blo_key >= lo_w && (bhi_key >> 10) <= pre + 2u;
    uint32_t my_in2 = 0;
    // candidates above the band are winners whatever the cut: marked here
    uint32_t* bm = a.bitmap + (size_t)b * a.Wcap;
    auto mark = [&](int32_t j) {
        atomicOr(&bm[j >> 5], 1u << (j & 31));
        red_add_shared(&S.wcnt[j / a.fchunk], 1u);
    };
    if (win) {
#pragma unroll 1
        for (uint32_t i = tid; i < C; i += kResThreads) {
            if (lk[i] > bhi_key) {
                ++my_in2;
                mark(li[i]);
            }
        }
        if ((uint32_t)tid < S.pf_cnt) {
            const uint32_t kk = S.pf_key[tid];
            if (kk >= blo_key && kk <= bhi_key) {
                const uint32_t p = atom_add_shared(&S.amb_cnt, 1u);
                S.amb_key[p] = EXACT ? kk : exact_key<true>(S.q2, S.pf_row[tid]);
                S.amb_idx[p] = S.pf_j[tid];
            }
        }
    } else {
#pragma unroll 1
        for (uint32_t i = tid; i < C; i += kResThreads) {
            const uint32_t kk = lk[i];
            if (kk > bhi_key) {
                ++my_in2;
                mark(li[i]);
            } else if (kk >= blo_key) {
                const int32_t j = li[i];
                const uint32_t p = atom_add_shared(&S.amb_cnt, 1u);
                const uint32_t ek = EXACT ? kk : exact_key(S.q2, icx + (size_t)j * 64);
                if (p < (uint32_t)kResThreads) {
                    S.amb_key[p] = ek;
                    S.amb_idx[p] = j;
                }
                gak[p] = ek;
                gai[p] = j;
            }
        }
    }
    uint32_t in2;
    block_exclusive_scan(my_in2, S.sh64, &in2);
    SA_TRACE_MARK(TR_RESOLVE, 4);
    const uint32_t na = S.amb_cnt;
    const uint32_t R2 = R1 - in2;  // winners to take from the band (1 <= R2 <= na)
    // the exact cut of the band: a member wins iff (key, -j) >= (T2, -jmax2)
    if (na <= (uint32_t)kResThreads) {
        if ((uint32_t)tid < na) {
            const uint32_t mk = S.amb_key[tid];
            const int32_t mj = S.amb_idx[tid];
            uint32_t rank = 0;
            for (uint32_t o = 0; o < na; ++o) {
                const uint32_t ok = S.amb_key[o];
                rank += (ok > mk) || (ok == mk && S.amb_idx[o] < mj);
            }
            if (rank == R2 - 1) {
                S.T2 = mk;
                S.jmax2 = mj;
            }
        }
        __syncthreads();
    } else {
        __threadfence_block();
        __syncthreads();
        uint32_t T2;
        int32_t jmax2;
        select_rank(gak, gai, na, R2, S.hist, S.sh64, S.res, &T2, &jmax2);
        if (tid == 0) {
            S.T2 = T2;
            S.jmax2 = jmax2;
        }
        __syncthreads();
    }
    const uint32_t T2 = S.T2;
    const int32_t jmax2 = S.jmax2;
    SA_TRACE_MARK(TR_RESOLVE, 5);
    // the band's winners
#pragma unroll 1
    for (uint32_t i = tid; i < na; i += kResThreads) {
        const uint32_t kk = na <= (uint32_t)kResThreads ? S.amb_key[i] : __ldcg(gak + i);
        const int32_t j = na <= (uint32_t)kResThreads ? S.amb_idx[i] : __ldcg(gai + i);
        if (kk > T2 || (kk == T2 && j <= jmax2)) mark(j);
    }
    __syncthreads();
    // output position of every chunk's first selected entry
    const uint32_t v = tid < nfch ? cin + S.wcnt[tid] : 0u;
    uint32_t total;
    const uint32_t pos = block_exclusive_scan(v, S.sh64, &total);
    if (tid < nfch) a.chunk_pos[(size_t)b * nfch + tid] = pos;
    if (tid == 0) {
        if (total != (uint32_t)k) flag(DEV_LEN);  // cannot happen
        a.cnt[b] = k;
    }
    SA_TRACE_MARK(TR_RESOLVE, 6);
}

// One CTA of 1024 threads per sequence.  One round trip brings the totals,
// every chunk's counts, the second histogram (two bins per thread, kept in
// registers) and, ahead of their counts, the first 32 candidate slots of
// each warp's first kGatherJ chunks; the fine bin of t~ then follows from
// the registers.
template <bool EXACT>
__global__ void __launch_bounds__(kResThreads, 1) topk_resolve_kernel(TopkDecodeArgs a) {
    extern __shared__ __align__(16) uint32_t csm[];  // [kSelCap] keys, [kSelCap] indices
    __shared__ SelSmem S;
    pdl_wait();
    pdl_release();
    SA_TRACE_MARK(TR_RESOLVE, 0);
    const int b = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = a.k;
    const int nfch = a.nfch;
    // every load goes out before the length is known (none depends on it)
    const uint32_t* tot = a.totals + (size_t)b * kTotals;
    const int d1 = (int)ld_cg_u32(tot + kTotBin);
    const float E = __uint_as_float(ld_cg_u32(tot + kTotE));
    const uint32_t above1 = ld_cg_u32(tot + kTotAbove);
    const uint32_t cin = tid < nfch ? ld_cg_u32(a.chunk_in + (size_t)b * nfch + tid) : 0u;
    const uint32_t ccn = tid < nfch ? ld_cg_u32(a.chunk_cnt + (size_t)b * nfch + tid) : 0u;
    uint32_t h2[2];
    {
        const uint2 x = ld_cg_u32x2(a.hist2 + (size_t)b * kBins + (kResThreads - 1 - tid) * 2);
        h2[0] = x.x;
        h2[1] = x.y;
    }
    const uint2* cs = a.cslot + (size_t)b * nfch * kSlots;
    uint32_t pk[kGatherJ * kGatherS];
    int32_t pi[kGatherJ * kGatherS];
#pragma unroll
    for (int j = 0; j < kGatherJ; ++j) {
        const int c = warp + 32 * j;
#pragma unroll
        for (int u = 0; u < kGatherS; ++u) {
            const uint2 e = c < nfch ? ld_cg_u32x2(cs + (size_t)c * kSlots + lane + 32 * u) : make_uint2(0u, 0u);
            pk[j * kGatherS + u] = e.x;
            pi[j * kGatherS + u] = (int32_t)e.y;
        }
    }
    const uint32_t qw = tid < 32 ? ld_cg_u32(reinterpret_cast<const uint32_t*>(a.q_idx + (size_t)b * 64) + tid) : 0u;
    const int n = clamp_n(a.n, b, a.Ncap);
    if (n <= k) return;  // the filter wrote the whole answer
    if (tid < 32) {  // qI * 2^768 in fp64 for the exact rescoring (see exact_key)
        S.q2[2 * tid] = (double)bf16lo_f32(qw) * 0x1p768;
        S.q2[2 * tid + 1] = (double)bf16hi_f32(qw) * 0x1p768;
    }
    if (tid == 0) {
        S.amb_cnt = 0;
        S.f_cnt = 0;
        S.found = 0;
        S.pf_cnt = 0;
    }
    S.wcnt[tid] = 0;  // kResThreads == kSelMaxChunks
    // the fine bin d2 of t~ inside bin d1 (rank K2 there)
    const uint32_t K2 = (uint32_t)k - above1;
    int d2;
    uint32_t above2;
    find_digit_desc_regs<2>(h2, K2, S.sh64, S.res, &d2, &above2);
    uint32_t base, ain, C, A;
    block_exclusive_scan2(ccn, cin, S.sh64, &base, &ain, &C, &A);
    if (tid < nfch) {
        S.base[tid] = base;
        S.ccnt[tid] = ccn;
    }
    __syncthreads();
    SA_TRACE_MARK(TR_RESOLVE, 1);
    if (C > (uint32_t)a.Ncap) {  // cannot happen: at most n candidates
        if (tid == 0) flag(DEV_LEN);
        C = a.Ncap;
    }
    if (C <= (uint32_t)kSelCap)
        resolve_body<true, EXACT>(a, S, csm, b, C, A, d1, E, d2, above2, K2, pk, pi, cin);
    else
        resolve_body<false, EXACT>(a, S, csm, b, C, A, d1, E, d2, above2, K2, pk, pi, cin);
    (void)ain;
}

// Emit: one CTA per filter chunk writes its selected indices, ascending,
// from its output position on.
constexpr int kEmitThreads = 256;
__global__ void __launch_bounds__(kEmitThreads) topk_emit_kernel(TopkDecodeArgs a) {
    __shared__ uint32_t sh32[32];
    pdl_wait();
    pdl_release();
    SA_TRACE_MARK(TR_EMIT, 0);
    const int b = blockIdx.y, c = blockIdx.x;
    const int row0 = c * a.fchunk;
    const uint32_t* bm = a.bitmap + (size_t)b * a.Wcap;
    // the first words and the position go out before the length is known
    const int wcap = (min(row0 + a.fchunk, a.Ncap) + 31) >> 5;
    const int wf = (row0 >> 5) + (int)threadIdx.x;
    const uint32_t word0 = wf < wcap ? ld_cg_u32(bm + wf) : 0u;
    uint32_t pos = ld_cg_u32(a.chunk_pos + (size_t)b * a.nfch + c);
    const int n = clamp_n(a.n, b, a.Ncap);
    if (n <= a.k) return;
    const int row1 = min(row0 + a.fchunk, n);
    if (row0 >= row1) return;
    int32_t* out = a.idx + (size_t)b * a.k;
    const int w0 = row0 >> 5, w1 = (row1 + 31) >> 5;
#pragma unroll 1
    for (int wb = w0; wb < w1; wb += kEmitThreads) {  // block-uniform trip count
        const int w = wb + threadIdx.x;
        uint32_t word = w < w1 ? (wb == w0 ? word0 : __ldcg(bm + w)) : 0u;
        uint32_t total;
        uint32_t p = pos + block_exclusive_scan(__popc(word), sh32, &total);
        while (word) {
            const int bit = __ffs(word) - 1;
            word &= word - 1;
            if (p < (uint32_t)a.k) out[p] = w * 32 + bit;
            else flag(DEV_LEN);  // cannot happen: exactly k bits are set
            ++p;
        }
        pos += total;
    }
    SA_TRACE_MARK(TR_EMIT, 1);
}

}  // namespace sa
