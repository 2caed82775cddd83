// topk_decode.cuh -- CSA indexer scores and exact top-k for decode (one query
// per sequence), "DeepSeek-V4 ... Review", section 3-2 (2) (CSA keeps a sparse
// top-k of the compressed entries) and 3-2 (4) (the CSA indexer QK path).
//
// score_j = fp32( fp64 sum_{i=0..63, ascending} qI[i] * Ic[j][i] ).  Each
// bf16 x bf16 product is exact in fp64, so the fp64 FMA chain in ascending i
// reproduces the definition bit for bit.  Selection keeps the k entries with
// the largest (score, -j) and reports them in ascending j.
//
// Three kernels, ordered on one stream:
//   1. score_decode_kernel   -- streams the indexer keys Ic (the dominant HBM
//      read of a decode step) through a TMA pipeline (128-byte rows, 128B
//      swizzle, 4 stages), one row per thread, writes a 32-bit order key per
//      entry and a histogram of the top 11 key bits (global atomics).
//   2. topk_filter_kernel    -- finds the 11-bit digit holding the k-th key;
//      writes a bitmap of entries whose digit is above it (surely selected),
//      and compacts the entries of that digit into a candidate list with a
//      histogram of their next 11 bits.
//   3. topk_resolve_kernel   -- one CTA per sequence: resolves the remaining
//      bits on the (small) candidate list, breaks ties at the threshold by
//      lowest index, marks the winners in the bitmap and compacts the bitmap
//      into ascending indices.
// No kernel waits on another CTA: every hand-off is a kernel boundary.
#pragma once
#include "sa_common.cuh"

namespace sa {

constexpr int kScRows = 128;      // rows per TMA tile (box height)
constexpr int kScStages = 4;      // TMA pipeline depth
constexpr int kScThreads = 128;   // one row per thread per tile
constexpr int kScTileBytes = kScRows * 128;
constexpr int kBins = 2048;       // 11-bit digits
constexpr int kBinsLow = 1024;    // last 10-bit digit

struct TopkDecodeArgs {
    const uint16_t* q_idx;  // [B][64]
    const int32_t* n;       // [B]
    uint32_t* keys;         // [B][Ncap]
    uint32_t* hist1;        // [B][2048]
    uint32_t* hist2;        // [B][2048]
    uint32_t* cand_cnt;     // [B]
    uint32_t* cand_key;     // [B][Ncap]
    int32_t* cand_idx;      // [B][Ncap]
    uint32_t* bitmap;       // [B][Wcap]
    int32_t* idx;           // [B][k]
    int32_t* cnt;           // [B]
    int Ncap, Wcap, chunk, k;
};

__device__ __forceinline__ int clamp_n(const int32_t* n, int b, int Ncap) {
    int v = n[b];
    if (v < 0 || v > Ncap) {
        flag(DEV_LEN);
        v = v < 0 ? 0 : Ncap;
    }
    return v;
}

// ------------------------------------------------------------ 1. scores ----
__global__ void __launch_bounds__(kScThreads, 3)
    score_decode_kernel(const __grid_constant__ CUtensorMap ic_map, TopkDecodeArgs a) {
    extern __shared__ uint8_t smem_raw[];
    // TMA with 128B swizzle needs a 1024-byte aligned destination
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* tiles = smem;
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + kScStages * kScTileBytes);
    uint64_t* full = reinterpret_cast<uint64_t*>(hist + kBins);

    const int b = blockIdx.y;
    const int n = clamp_n(a.n, b, a.Ncap);
    if (n <= a.k) return;  // everything visible is selected; nothing to score
    const int row0 = blockIdx.x * a.chunk;
    const int row1 = min(row0 + a.chunk, n);
    if (row0 >= row1) return;
    const int ntiles = (row1 - row0 + kScRows - 1) / kScRows;
    const int tid = threadIdx.x;

    // qI * 2^768 in fp64: with keys held as x * 2^-896, each product is
    // qI*k * 2^-128 exactly and no partial sum leaves the normal range.
    double q[64];
    {
        const uint32_t* qw = reinterpret_cast<const uint32_t*>(a.q_idx + (size_t)b * 64);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const uint32_t w = __ldg(qw + i);
            q[2 * i] = (double)bf16lo_f32(w) * 0x1p768;
            q[2 * i + 1] = (double)bf16hi_f32(w) * 0x1p768;
        }
    }
    for (int i = tid; i < kBins; i += blockDim.x) hist[i] = 0;
    if (tid == 0) {
        for (int s = 0; s < kScStages; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    __syncthreads();

    // the map views Ic as [B][Ncap][64]: coordinates (dim, row, sequence)
    int issued = 0;
    if (tid == 0) {
        for (; issued < kScStages && issued < ntiles; ++issued) {
            mbar_expect_tx(&full[issued], kScTileBytes);
            tma_load_3d(tiles + issued * kScTileBytes, &ic_map, 0, row0 + issued * kScRows, b, &full[issued]);
        }
    }
    int consumed = 0;
    bool timed_out = false;
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
            double acc = 0.0;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 w = *reinterpret_cast<const uint4*>(rp + ((c ^ (tid & 7)) << 4));
                acc = fma(q[8 * c + 0], bf16lo_scaled(w.x), acc);
                acc = fma(q[8 * c + 1], bf16hi_scaled(w.x), acc);
                acc = fma(q[8 * c + 2], bf16lo_scaled(w.y), acc);
                acc = fma(q[8 * c + 3], bf16hi_scaled(w.y), acc);
                acc = fma(q[8 * c + 4], bf16lo_scaled(w.z), acc);
                acc = fma(q[8 * c + 5], bf16hi_scaled(w.z), acc);
                acc = fma(q[8 * c + 6], bf16lo_scaled(w.w), acc);
                acc = fma(q[8 * c + 7], bf16hi_scaled(w.w), acc);
            }
            const uint32_t key = score_key(__double2float_rn(acc * 0x1p128));
            a.keys[(size_t)b * a.Ncap + row] = key;
            atomicAdd(&hist[key >> 21], 1u);
        }
        __syncthreads();  // slot s is free again
        if (tid == 0 && issued < ntiles) {
            fence_proxy_async();
            mbar_expect_tx(&full[s], kScTileBytes);
            tma_load_3d(tiles + s * kScTileBytes, &ic_map, 0, row0 + issued * kScRows, b, &full[s]);
            ++issued;
        }
    }
    if (timed_out) {
        // let copies still in flight land before the CTA's shared memory goes away
        if (tid == 0)
            for (int i = consumed; i < issued; ++i) mbar_wait(&full[i % kScStages], (i / kScStages) & 1);
        __syncthreads();
        return;
    }
    __syncthreads();
    for (int i = tid; i < kBins; i += blockDim.x)
        if (hist[i]) atomicAdd(&a.hist1[(size_t)b * kBins + i], hist[i]);
}

// --------------------------------------------------- digit search helpers --
// Descending: returns the digit d with  above(d) < K <= above(d) + h[d], where
// above(d) = sum of h[e] for e > d.  Every thread gets (d, above(d)).
template <int NB>
__device__ void find_digit_desc(const uint32_t* h, uint32_t K, uint32_t* sh32, int* out_d, uint32_t* out_above,
                                int* res) {
    const int T = blockDim.x;
    const int per = (NB + T - 1) / T;
    const int u = T - 1 - threadIdx.x;  // thread t handles the bins of thread u, so the scan runs high -> low
    const int lo = u * per, hi = min(NB, lo + per);
    uint32_t local = 0;
    for (int e = lo; e < hi; ++e) local += h[e];
    uint32_t above = block_exclusive_scan(local, sh32, nullptr);
    if (threadIdx.x == 0) {
        res[0] = -1;
        res[1] = 0;
    }
    __syncthreads();
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
__device__ void find_digit_asc(const uint32_t* h, uint32_t R, uint32_t* sh32, int* out_d, uint32_t* out_below,
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

// ------------------------------------------------------------ 2. filter ----
constexpr int kFiltThreads = 256;

__global__ void __launch_bounds__(kFiltThreads) topk_filter_kernel(TopkDecodeArgs a) {
    __shared__ uint32_t hsh[kBins];
    __shared__ uint32_t sh32[32];
    __shared__ int res[2];
    const int b = blockIdx.y;
    const int n = clamp_n(a.n, b, a.Ncap);
    if (n <= a.k) return;
    const int row0 = blockIdx.x * a.chunk;
    const int row1 = min(row0 + a.chunk, n);
    if (row0 >= row1) return;

    for (int i = threadIdx.x; i < kBins; i += blockDim.x) hsh[i] = a.hist1[(size_t)b * kBins + i];
    __syncthreads();
    int d1;
    uint32_t above1;
    find_digit_desc<kBins>(hsh, (uint32_t)a.k, sh32, &d1, &above1, res);
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) hsh[i] = 0;
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const uint32_t* keys = a.keys + (size_t)b * a.Ncap;
    // chunk and row0 are multiples of 32, so each warp owns whole bitmap words
    const int rend = row0 + ((row1 - row0 + 31) & ~31);
    for (int base = row0 + (threadIdx.x & ~31); base < rend; base += blockDim.x) {
        const int row = base + lane;
        const bool valid = row < row1;
        const uint32_t key = valid ? keys[row] : 0u;
        const int dig = (int)(key >> 21);
        const bool sel = valid && dig > d1;
        const bool cand = valid && dig == d1;
        const uint32_t selm = __ballot_sync(0xFFFFFFFFu, sel);
        const uint32_t candm = __ballot_sync(0xFFFFFFFFu, cand);
        if (lane == 0) a.bitmap[(size_t)b * a.Wcap + (row >> 5)] = selm;
        if (candm) {
            uint32_t basepos = 0;
            if (lane == 0) basepos = atomicAdd(&a.cand_cnt[b], (uint32_t)__popc(candm));
            basepos = __shfl_sync(0xFFFFFFFFu, basepos, 0);
            if (cand) {
                const uint32_t pos = basepos + __popc(candm & ((1u << lane) - 1u));
                if (pos < (uint32_t)a.Ncap) {
                    a.cand_key[(size_t)b * a.Ncap + pos] = key;
                    a.cand_idx[(size_t)b * a.Ncap + pos] = row;
                }
                atomicAdd(&hsh[(key >> 10) & (kBins - 1)], 1u);
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kBins; i += blockDim.x)
        if (hsh[i]) atomicAdd(&a.hist2[(size_t)b * kBins + i], hsh[i]);
}

// ----------------------------------------------------------- 3. resolve ----
constexpr int kResThreads = 1024;

// Writes the set bits of bm[0..nwords) as ascending indices into out[0..cap).
__device__ void compact_bitmap(const uint32_t* bm, int nwords, int32_t* out, uint32_t cap, uint32_t* sh32,
                               uint32_t* total_out) {
    uint32_t running = 0;
    for (int w0 = 0; w0 < nwords; w0 += blockDim.x) {
        const int w = w0 + threadIdx.x;
        uint32_t word = w < nwords ? bm[w] : 0u;
        uint32_t tot;
        uint32_t pos = running + block_exclusive_scan((uint32_t)__popc(word), sh32, &tot);
        while (word) {
            const int bit = __ffs(word) - 1;
            word &= word - 1;
            if (pos < cap) out[pos] = w * 32 + bit;
            ++pos;
        }
        running += tot;
    }
    *total_out = running;
}

__global__ void __launch_bounds__(kResThreads) topk_resolve_kernel(TopkDecodeArgs a) {
    __shared__ uint32_t hsh[kBins];
    __shared__ uint32_t sh32[32];
    __shared__ int res[2];
    const int b = blockIdx.x;
    const int n = clamp_n(a.n, b, a.Ncap);
    const int k = a.k;
    int32_t* idx = a.idx + (size_t)b * k;
    if (n <= k) {
        for (int i = threadIdx.x; i < k; i += blockDim.x) idx[i] = i < n ? i : -1;
        if (threadIdx.x == 0) a.cnt[b] = n;
        return;
    }
    // digit 1 (bits 31..21)
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) hsh[i] = a.hist1[(size_t)b * kBins + i];
    __syncthreads();
    int d1, d2, d3;
    uint32_t above;
    find_digit_desc<kBins>(hsh, (uint32_t)k, sh32, &d1, &above, res);
    uint32_t K1 = (uint32_t)k - above;
    // digit 2 (bits 20..10) among the candidates of digit 1
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) hsh[i] = a.hist2[(size_t)b * kBins + i];
    __syncthreads();
    find_digit_desc<kBins>(hsh, K1, sh32, &d2, &above, res);
    uint32_t K2 = K1 - above;
    // digit 3 (bits 9..0)
    uint32_t c1 = a.cand_cnt[b];
    if (c1 > (uint32_t)a.Ncap) {
        if (threadIdx.x == 0) flag(DEV_LEN);
        c1 = a.Ncap;
    }
    const uint32_t* ck = a.cand_key + (size_t)b * a.Ncap;
    const int32_t* ci = a.cand_idx + (size_t)b * a.Ncap;
    for (int i = threadIdx.x; i < kBinsLow; i += blockDim.x) hsh[i] = 0;
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < c1; i += blockDim.x) {
        const uint32_t key = ck[i];
        if ((int)((key >> 10) & (kBins - 1)) == d2) atomicAdd(&hsh[key & (kBinsLow - 1)], 1u);
    }
    __syncthreads();
    find_digit_desc<kBinsLow>(hsh, K2, sh32, &d3, &above, res);
    const uint32_t r = K2 - above;  // ties at the threshold key to keep (>= 1)
    const uint32_t nties = hsh[d3 < 0 ? 0 : d3];
    __syncthreads();
    const uint32_t T = ((uint32_t)d1 << 21) | ((uint32_t)d2 << 10) | (uint32_t)d3;
    if (d1 < 0 || d2 < 0 || d3 < 0) {
        if (threadIdx.x == 0) flag(DEV_LEN);  // inconsistent histograms: cannot happen
    }

    // lowest-index tie-break: jmax = the r-th smallest index among ties at T
    int32_t jmax = 0x7FFFFFFF;
    if (r < nties) {
        uint32_t prefix = 0, R = r;
        // indices < 2^31: digits of 11, 11 and 9 bits from the top
        const int shifts[3] = {20, 9, 0};
        const int widths[3] = {11, 11, 9};
        uint32_t pmask = 0;
        for (int p = 0; p < 3; ++p) {
            const int nb = 1 << widths[p];
            for (int i = threadIdx.x; i < kBins; i += blockDim.x) hsh[i] = 0;
            __syncthreads();
            for (uint32_t i = threadIdx.x; i < c1; i += blockDim.x) {
                if (ck[i] != T) continue;
                const uint32_t j = (uint32_t)ci[i];
                if ((j & pmask) != prefix) continue;
                atomicAdd(&hsh[(j >> shifts[p]) & (nb - 1)], 1u);
            }
            __syncthreads();
            int dd;
            uint32_t below;
            find_digit_asc<kBins>(hsh, R, sh32, &dd, &below, res);
            R -= below;
            prefix |= (uint32_t)dd << shifts[p];
            pmask |= (uint32_t)(nb - 1) << shifts[p];
        }
        jmax = (int32_t)prefix;
    }

    // mark winners among the candidates, then compact the bitmap in index order
    uint32_t* bm = a.bitmap + (size_t)b * a.Wcap;
    for (uint32_t i = threadIdx.x; i < c1; i += blockDim.x) {
        const uint32_t key = ck[i];
        const int32_t j = ci[i];
        if (key > T || (key == T && j <= jmax)) atomicOr(&bm[j >> 5], 1u << (j & 31));
    }
    __syncthreads();
    uint32_t total;
    compact_bitmap(bm, (n + 31) >> 5, idx, (uint32_t)k, sh32, &total);
    if (total != (uint32_t)k && threadIdx.x == 0) flag(DEV_LEN);  // cannot happen
    if (threadIdx.x == 0) a.cnt[b] = k;
}

}  // namespace sa
