// decode_fast.cuh -- the fast path of one hybrid decode step's CSA branch:
// indexer scores, exact top-k and the attention over the chosen entries,
// "DeepSeek-V4 ... Review", section 3-2 (2) (CSA keeps a sparse top-k of the
// compressed entries and attends over them) and 3-2 (4) (the indexer QK path).
//
// Three kernels for a bf16 cache, up to 64 heads and k <= 2048, then the
// split attention of attn.cuh over the selection:
//
//   1. topk_bound_kernel  -- one cluster of 8 CTAs per sequence screens a
//      strided sample of the indexer rows (at most 4096) and takes a sample
//      order statistic below the expected k-th largest score as a
//      provisional bound t_p, and the bin width of a candidate histogram.
//      The bound only steers how many candidates the scan keeps; the
//      exactness argument below does not depend on it.
//   2. score_fast_kernel  -- the indexer stream (TMA pipeline, fp32 screen
//      s~_j with its certified error bound e_j, as in topk_decode.cuh), which
//      writes every row with s~_j >= t_p to its chunk's candidate rows, in
//      ascending row order (ballots per tile), counts it in the sequence's
//      candidate histogram, and takes E = max e_j.  Every key is also
//      written, for the fallback below.
//   3. csa_select_fast_kernel -- one CTA per sequence: the candidate
//      histogram gives the bin of the k-th largest screened key t~; the
//      chunks' candidates are concatenated (ascending entry order) and t~ is
//      ranked inside its bin; the band |s~ - t~| <= 2E is rescored exactly
//      (the fp64 definition) and cut by (s, -j).  This is the exact selection
//      when at least k candidates were kept and t~ - 2E >= t_p: every entry
//      outside the list then has s~ < t~ - 2E and is surely not selected.
//      Otherwise (or when forced) the same selection runs over every key of
//      the sequence in global memory.  The ascending index list goes to the
//      caller's idx / cnt, which the attention reads.
//
// The scan waits for the bound kernel before it streams: sharing the SMs
// with the scan's FMA chains and the memory system with its TMA stream, the
// sample took longer than the whole prefix of the scan it was to overlap.
#pragma once
#include "topk_decode.cuh"

namespace sa {

constexpr int kFbCluster = 8;    // bound kernel: CTAs per sequence
constexpr int kFbThreads = 512;  // CTA 0's threads also run the order statistic
constexpr int kFbRowsPT = 1;     // sample rows per thread
constexpr int kFbSamp = kFbCluster * kFbThreads * kFbRowsPT;  // 4096 sample rows at most
constexpr int kFastCap = 8192;   // candidates the selecting CTA holds in shared memory
constexpr int kFastMaxK = 2048;
constexpr int kFaThreads = 512;  // the selection kernel's CTA (one per sequence)
constexpr int kFaBand = 1024;    // band members ranked in shared memory
constexpr int kCtl = 4;          // control words per sequence
constexpr int kCtlBound = 0, kCtlE = 1, kCtlShift = 2;
constexpr int kCH = 2048;        // bins of the candidate histogram: key offsets from t_p >> shift, the top bin clamped

// option values of the fast path (SA_OPT_DECODE_FAST)
constexpr int kFastOff = 0, kFastOn = 1, kFastForceGlobal = 2;

struct FastArgs {
    const uint16_t* q_idx;  // [B][64]
    const uint16_t* kidx;   // [B][Ncap][64]
    const int32_t* n;       // [B]
    uint32_t* ctrl;         // [B][kCtl]: the bound key t_p, E (fp32 bits, max over the scan's CTAs), histogram shift
    uint32_t* chist;        // [B][kCH] histogram of the candidates' keys (zeroed by the bound kernel)
    uint32_t* ccount;       // [B][nchunks] candidates of each scan chunk
    uint2* cand;            // [B][Ncap] (key, index): chunk c's candidates in the chunk's own rows
    uint32_t* keys;         // [B][Ncap] every screened key (the fallback selection)
    uint32_t* amb_key;      // [B][Ncap] exact keys of a band too large for shared memory
    int32_t* amb_idx;
    int32_t* idx;           // [B][k] out
    int32_t* cnt;           // [B] out
    int Ncap, k, chunk, nchunks, sstride, mode;
};

// The bound kernel's CTAs run beside the scan on SMs of their own (their
// shared memory leaves no room for a scan CTA) when there are few of them;
// the scan then awaits the bound only after its last tile.
constexpr int kFbReserveSmem = 190 * 1024;  // with the static ~33 KB: no 67 KB scan CTA fits beside it

// ------------------------------------------------------------- clusters ----
// The cluster barrier's ".aligned" forms need every thread of the warp to
// execute them together: each helper reconverges the warp first.
__device__ __forceinline__ void cluster_sync() {
    __syncwarp();
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// the two halves of a cluster barrier, to overlap its latency with other work
__device__ __forceinline__ void cluster_arrive_relaxed() {
    __syncwarp();
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    __syncwarp();
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared-memory address of the same variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_dsmem_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// The fp32 screen of one 128-byte indexer row held as eight 16-byte words
// (the same FMA chain as the scan's).
__device__ __forceinline__ float screen_row(const float* q, const uint4 (&w)[8]) {
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint32_t ws[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            acc = fmaf(q[8 * c + 2 * h], bf16lo_f32(ws[h]), acc);
            acc = fmaf(q[8 * c + 2 * h + 1], bf16hi_f32(ws[h]), acc);
        }
    }
    return acc;
}

constexpr int kDigBins = 256;  // 8-bit digits of the selection passes

// The K-th largest of a list of C keys (1 <= K <= C).  The digits are 8-bit
// slices of each key's offset from the list's smallest key, taken from the
// top of the list's own range down: a candidate list spans a narrow range of
// keys, which fixed top-bit digits would crowd into a few bins.  At most four
// passes.  Each warp counts into its own histogram, so shared-memory atomics
// contend only within a warp; the bins are then summed and searched.
// hist: kDigBins words per warp; sh32: at least 32 and 2 per warp.
// Keys below `floor` take no part (at least K keys must reach it).
template <typename KeyAt>
__device__ uint32_t kth_largest(KeyAt key_at, uint32_t C, uint32_t K, uint32_t* hist, uint32_t* sh32, int* res,
                                uint32_t floor = 0u) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    for (uint32_t i = tid; i < C; i += blockDim.x) {
        const uint32_t kk = key_at(i);
        if (kk >= floor) {
            lo = min(lo, kk);
            hi = max(hi, kk);
        }
    }
    lo = __reduce_min_sync(0xFFFFFFFFu, lo);
    hi = __reduce_max_sync(0xFFFFFFFFu, hi);
    if (lane == 0) {
        sh32[warp] = lo;
        sh32[nw + warp] = hi;
    }
    __syncthreads();
    for (int w = 0; w < nw; ++w) {
        lo = min(lo, sh32[w]);
        hi = max(hi, sh32[nw + w]);
    }
    __syncthreads();  // sh32 is reused below
    uint32_t* wh = hist + warp * kDigBins;
    // thread t holds `per` consecutive bins, the highest bins first
    const int per = max(1, kDigBins / (int)blockDim.x);
    const int nbt = kDigBins / per;  // threads that hold bins
    uint32_t base = lo, span1 = hi - lo, rem = K;  // the current range is [base, base + span1]
    while (span1 != 0) {                           // block-uniform
        const int bits = 32 - __clz((int)span1);
        const int shift = max(0, bits - 8);
        for (int i = tid; i < nw * kDigBins; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (uint32_t i = tid; i < C; i += blockDim.x) {
            const uint32_t off = key_at(i) - base;  // wraps past span1 for keys below the range
            if (off <= span1) red_add_shared(&wh[off >> shift], 1u);
        }
        __syncthreads();
        uint32_t cb[4] = {0u, 0u, 0u, 0u}, c = 0;  // per <= 4 (blockDim.x >= 64)
        const int top = kDigBins - 1 - tid * per;  // this thread's highest bin
        if (tid < nbt) {
            for (int j = 0; j < per; ++j)
                for (int w = 0; w < nw; ++w) cb[j] += hist[w * kDigBins + top - j];
            for (int j = 0; j < per; ++j) c += cb[j];
        }
        if (tid == 0) res[0] = -1;  // ordered before the writes below by the scan's barriers
        uint32_t above = block_exclusive_scan(c, sh32, nullptr);  // keys in the bins above this thread's
        if (tid < nbt) {
            for (int j = 0; j < per; ++j) {
                if (above < rem && rem <= above + cb[j]) {
                    res[0] = top - j;
                    res[1] = (int)above;
                }
                above += cb[j];
            }
        }
        __syncthreads();
        int d = res[0];
        const uint32_t ab = (uint32_t)res[1];
        __syncthreads();  // res is rewritten by the next pass
        if (d < 0) {
            if (tid == 0) flag(DEV_LEN);  // inconsistent counts: cannot happen
            return base;
        }
        rem -= ab;
        const uint32_t dlo = (uint32_t)d << shift;
        base += dlo;
        span1 = shift == 0 ? 0u : min(span1 - dlo, (1u << shift) - 1u);
    }
    return base;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
    return x;
}

// ------------------------------------------------------------ 1. bound ----
// Grid (kFbCluster, B), clusters of kFbCluster CTAs along x.
__global__ void __launch_bounds__(kFbThreads, 1) topk_bound_kernel(FastArgs a) {
    __shared__ float sq[64];
    __shared__ uint32_t skey[kFbSamp];  // CTA 0: every sample key of the sequence
    __shared__ uint32_t hist[kDigBins * kFbThreads / 32];
    __shared__ uint32_t sh32[32];
    __shared__ int res[2];
    pdl_wait();
    pdl_release();
    SA_TRACE_MARK(TR_BOUND, 0);
    const int b = blockIdx.y, tid = threadIdx.x;
    const uint32_t rank = cluster_rank();
    const int n = clamp_n(a.n, b, a.Ncap);
    uint32_t* ctl = a.ctrl + (size_t)b * kCtl;
    // a sequence with n <= k is answered whole; with n <= kFastCap every
    // entry is a candidate (bound key 0, below every real key)
    uint32_t* ch = a.chist + (size_t)b * kCH;
    if (n <= a.k || n <= kFastCap) {
        if (rank == 0) {
            if (tid == 0) {
                ctl[kCtlBound] = 0u;
                ctl[kCtlE] = 0u;
                ctl[kCtlShift] = 21u;  // every key falls into one of the histogram's bins
            }
            for (int i = tid; i < kCH; i += kFbThreads) ch[i] = 0u;
        }
        return;
    }
    // every CTA of the cluster has started before any remote store (the wait
    // below, after this CTA's loads are issued)
    cluster_arrive_relaxed();
    const int S = a.sstride;
    const int ns = (n + S - 1) / S;  // <= kFbSamp by the choice of S
    if (tid < 64) {
        const uint16_t* qp = a.q_idx + (size_t)b * 64;
        sq[tid] = __uint_as_float((uint32_t)qp[tid] << 16);
    }
    __syncthreads();
    const uint16_t* ic = a.kidx + (size_t)b * a.Ncap * 64;
    {
        uint4 w[kFbRowsPT][8];  // every row's loads in flight at once
        int si[kFbRowsPT];
#pragma unroll
        for (int u = 0; u < kFbRowsPT; ++u) {
            si[u] = (int)rank * (kFbThreads * kFbRowsPT) + u * kFbThreads + tid;
            const bool ok = si[u] < ns;
            const uint4* rp = reinterpret_cast<const uint4*>(ic + (size_t)(ok ? si[u] * S : 0) * 64);
#pragma unroll
            for (int c = 0; c < 8; ++c) w[u][c] = ok ? __ldg(rp + c) : make_uint4(0u, 0u, 0u, 0u);
        }
        cluster_wait();
#pragma unroll
        for (int u = 0; u < kFbRowsPT; ++u)  // into CTA 0's shared memory (a remote store for the other CTAs)
            if (si[u] < ns) st_dsmem_u32(dsmem_addr(&skey[si[u]], 0), score_key(screen_row(sq, w[u])));
    }
    SA_TRACE_MARK(TR_BOUND, 1);
    cluster_sync();  // every sample key is in CTA 0's shared memory
    if (rank == 0) {
        // expected sample count above the k-th largest score: mu = k ns / n;
        // the bound is the r-th largest sample with r about mu + 5 sqrt(mu) + 4
        const float mu = (float)a.k * (float)ns / (float)n;
        int r = (int)ceilf(mu + 5.f * sqrtf(mu) + 4.f);
        r = max(1, min(r, ns));
        // the r-th largest of the ns sample keys; only the samples above
        // mean + 1.5 sd (about 7% of a normal sample) enter the digit passes,
        // when at least r of them are there
        const int lane = tid & 31, warp = tid >> 5;
        float s1 = 0.f, s2 = 0.f;
        uint32_t smax = 0u;
        for (int i = tid; i < ns; i += kFbThreads) {
            const uint32_t kk = skey[i];
            const float x = key_to_float(kk);
            s1 += x;
            s2 = fmaf(x, x, s2);
            smax = max(smax, kk);
        }
        s1 = warp_sum(s1);
        s2 = warp_sum(s2);
        smax = __reduce_max_sync(0xFFFFFFFFu, smax);
        __shared__ float sf[2][kFbThreads / 32];
        __shared__ uint32_t su[kFbThreads / 32];
        if (lane == 0) {
            sf[0][warp] = s1;
            sf[1][warp] = s2;
            su[warp] = smax;
        }
        __syncthreads();
        s1 = s2 = 0.f;
        smax = 0u;
        for (int w = 0; w < kFbThreads / 32; ++w) {
            s1 += sf[0][w];
            s2 += sf[1][w];
            smax = max(smax, su[w]);
        }
        const float mean = s1 / (float)ns, var = fmaxf(0.f, s2 / (float)ns - mean * mean);
        const float cut = mean + 1.5f * sqrtf(var);
        uint32_t floor = isfinite(cut) ? score_key(cut) : 0u;
        // the samples at or above the cut, into a short list (hist's words)
        __shared__ uint32_t s_m, s_bound;
        if (tid == 0) {
            s_m = 0;
            s_bound = 0xFFFFFFFFu;
        }
        __syncthreads();
        uint32_t* L = hist;
        constexpr uint32_t kLcap = kDigBins * kFbThreads / 32;
        for (int i = tid; i < ns; i += kFbThreads) {
            const uint32_t kk = skey[i];
            if (kk >= floor) {
                const uint32_t q = atom_add_shared(&s_m, 1u);
                if (q < kLcap) L[q] = kk;
            }
        }
        __syncthreads();
        const uint32_t m = s_m;
        uint32_t bound;
        if (m >= (uint32_t)r && m <= kLcap && m <= 1024u) {
            // the r-th largest of the list by pairwise ranks
            for (uint32_t i = tid; i < m; i += kFbThreads) {
                const uint32_t mk = L[i];
                uint32_t gt = 0, ge = 0;
                for (uint32_t o = 0; o < m; ++o) {
                    const uint32_t ok = L[o];
                    gt += ok > mk;
                    ge += ok >= mk;
                }
                if (gt < (uint32_t)r && (uint32_t)r <= ge) s_bound = mk;  // every holder writes the same value
            }
            __syncthreads();
            bound = s_bound;
        } else {  // a sample far from normal: digit passes over every sample (or those above the cut)
            __syncthreads();  // the list's words are the passes' histograms
            if (m < (uint32_t)r) floor = 0u;
            bound = kth_largest([&](uint32_t i) { return skey[i]; }, (uint32_t)ns, (uint32_t)r, hist, sh32, res,
                                floor);
        }
        // candidate histogram bins: the sample maximum near the middle bin
        const uint32_t spread = (smax - bound) >> 10;
        const uint32_t shift = spread ? 32u - (uint32_t)__clz((int)spread) : 0u;
        if (tid == 0) {
            ctl[kCtlBound] = bound;
            ctl[kCtlE] = 0u;
            ctl[kCtlShift] = shift;
        }
        for (int i = tid; i < kCH; i += kFbThreads) ch[i] = 0u;
        SA_TRACE_MARK(TR_BOUND, 2);
    }
}

// ------------------------------------------------------------- 2. scan ----
// The indexer stream with candidate output.  Grid (nchunks, B), 128 threads.
// LATE: the bound kernel runs beside this one; the candidates are taken
// after the last tile, from the keys this CTA wrote (read back by the
// threads that wrote them), eight tiles per barrier.  Otherwise the bound
// is known before the first tile and every tile's candidates are written as
// it is scored.
template <bool LATE>
__global__ void __launch_bounds__(kScThreads, 4)
    score_fast_kernel(const __grid_constant__ CUtensorMap ic_map, FastArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* tiles = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kScStages * kScTileBytes);
    __shared__ float s_emax[kScThreads / 32];
    __shared__ uint32_t s_wc[2][kScThreads / 32];  // per-warp candidate counts of a tile
    __shared__ uint32_t s_ec[8][kScThreads / 32];  // ... of eight tiles (LATE)
    if (!LATE) pdl_wait();  // the bound first: nothing is loaded before it is known
    pdl_release();
    SA_TRACE_MARK(TR_SCORE, 0);
    const int b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row0 = blockIdx.x * a.chunk;
    const int n = clamp_n(a.n, b, a.Ncap);
    if (n <= a.k) {
        if (LATE) pdl_wait();  // completion stays transitive along the chain
        return;
    }
    const int row1 = min(row0 + a.chunk, n);
    const int ntiles = row1 > row0 ? (row1 - row0 + kScRows - 1) / kScRows : 0;
    int issued = 0;
    if (tid == 0) {
        for (int s = 0; s < kScStages; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
        for (; issued < kScStages && issued < ntiles; ++issued) {
            mbar_expect_tx(&full[issued], kScTileBytes);
            tma_load_3d(tiles + issued * kScTileBytes, &ic_map, 0, row0 + issued * kScRows, b, &full[issued]);
        }
    }
    const uint32_t* ctl = a.ctrl + (size_t)b * kCtl;
    uint32_t tp = 0, hsh = 0;
    if (!LATE) {
        tp = ld_cg_u32(ctl + kCtlBound);
        hsh = ld_cg_u32(ctl + kCtlShift);
    }
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
    uint32_t* kout = a.keys + (size_t)b * a.Ncap;
    uint2* cd = a.cand + (size_t)b * a.Ncap + row0;
    uint32_t* ch = a.chist + (size_t)b * kCH;
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t cbase = 0;
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
        const bool valid = row < row1;
        uint32_t key = 0;
        if (valid) {
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
            key = score_key(acc);
            kout[row] = key;
            emax = fmaxf(emax, fmaf(aab, 0x1p-16f, fmaf(fabsf(acc), 0x1p-22f, 0x1p-140f)));
        }
        const bool cand = !LATE && valid && key >= tp;
        const uint32_t bal = __ballot_sync(0xFFFFFFFFu, cand);
        if (!LATE && lane == 0) s_wc[i & 1][warp] = __popc(bal);
        __syncthreads();  // slot s is free again; this tile's warp counts are visible
        if (tid == 0 && issued < ntiles) {
            fence_proxy_async();
            mbar_expect_tx(&full[s], kScTileBytes);
            tma_load_3d(tiles + s * kScTileBytes, &ic_map, 0, row0 + issued * kScRows, b, &full[s]);
            ++issued;
        }
        if (!LATE) {
            uint32_t off = cbase, tot = 0;
#pragma unroll
            for (int w = 0; w < kScThreads / 32; ++w) {
                const uint32_t c = s_wc[i & 1][w];
                off += w < warp ? c : 0u;
                tot += c;
            }
            if (cand) {  // the candidate row and its histogram bin (a fire-and-forget add)
                cd[off + __popc(bal & lt)] = make_uint2(key, (uint32_t)row);
                const uint32_t bin = min((key - tp) >> hsh, (uint32_t)(kCH - 1));
                asm volatile("red.global.add.u32 [%0], 1;" ::"l"(ch + bin) : "memory");
            }
            cbase += tot;
        }
    }
    if (tid == 0)
        for (int i = consumed; i < issued; ++i) mbar_wait(&full[i % kScStages], (i / kScStages) & 1);
    if (timed_out) __syncthreads();
    if (LATE) {
        pdl_wait();
        tp = ld_cg_u32(ctl + kCtlBound);
        hsh = ld_cg_u32(ctl + kCtlShift);
#pragma unroll 1
        for (int g = 0; g < consumed; g += 8) {
            uint32_t kk[8], bal[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int row = row0 + (g + j) * kScRows + tid;
                const bool v = g + j < consumed && row < row1;
                kk[j] = v ? kout[row] : 0u;
                bal[j] = __ballot_sync(0xFFFFFFFFu, v && kk[j] >= tp);
                if (lane == 0) s_ec[j][warp] = __popc(bal[j]);
            }
            __syncthreads();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint32_t off = cbase, tot = 0;
#pragma unroll
                for (int w = 0; w < kScThreads / 32; ++w) {
                    const uint32_t c = s_ec[j][w];
                    off += w < warp ? c : 0u;
                    tot += c;
                }
                if ((bal[j] >> lane) & 1u) {
                    cd[off + __popc(bal[j] & lt)] = make_uint2(kk[j], (uint32_t)(row0 + (g + j) * kScRows + tid));
                    const uint32_t bin = min((kk[j] - tp) >> hsh, (uint32_t)(kCH - 1));
                    asm volatile("red.global.add.u32 [%0], 1;" ::"l"(ch + bin) : "memory");
                }
                cbase += tot;
            }
            __syncthreads();  // s_ec is rewritten by the next group
        }
    }
    emax = __uint_as_float(__float_as_uint(emax) + 1u);  // e_j rounded to nearest: one ulp up
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) emax = fmaxf(emax, __shfl_xor_sync(0xFFFFFFFFu, emax, o));
    if (lane == 0) s_emax[warp] = emax;
    __syncthreads();
    SA_TRACE_MARK(TR_SCORE, 1);
    if (tid == 0) {
        float m = s_emax[0];
        for (int w = 1; w < kScThreads / 32; ++w) m = fmaxf(m, s_emax[w]);
        a.ccount[(size_t)b * a.nchunks + blockIdx.x] = cbase;
        atomicMax(a.ctrl + (size_t)b * kCtl + kCtlE, __float_as_uint(m));  // positive floats order as integers
    }
}

// --------------------------------------------------------- 3. selection ----
// Shared memory of the selection kernel (dynamic, byte offsets).
constexpr int kFaLKey = 0;                          // candidate keys    [kFastCap]
constexpr int kFaLIdx = kFaLKey + kFastCap * 4;     // candidate indices [kFastCap]
constexpr int kFaHist = kFaLIdx + kFastCap * 4;     // digit histograms [16 warps][kDigBins] (or [kBins])
constexpr int kFaBase = kFaHist + 16 * kDigBins * 4;  // chunk positions [kSelMaxChunks + 1]
constexpr int kFaBKey = kFaBase + (kSelMaxChunks + 1) * 4 + 12;  // band exact keys [kFaBand]
constexpr int kFaBIdx = kFaBKey + kFaBand * 4;      // band indices    [kFaBand]
constexpr int kFaBPos = kFaBIdx + kFaBand * 4;      // band list positions [kFaBand]
constexpr int kStage = 256;                          // candidates of the bins around t~'s, staged for the band
constexpr int kFaSg = kFaBPos + kFaBand * 4;         // staged keys, indices, list positions, exact keys [4][kStage]
constexpr int kFaSmem = kFaSg + 4 * kStage * 4;
static_assert(kFaSmem <= 227 * 1024, "shared memory of one CTA");
static_assert((kFaBase & 15) == 0 && (kFaBKey & 15) == 0, "16-byte aligned scratch");

struct FaStatic {
    double q2[64];  // qI * 2^768 (exact rescoring)
    uint32_t sh64[64];
    int res[2];
    uint32_t nb, nd, a_cnt, tkey, nsg, hnext;
};

// The exact selection over a list of (screened key, index) pairs in
// ascending index order: GLOBAL = every key of the sequence in global memory
// (index = position), else the candidate list in shared memory.  Returns
// false (shared-memory list only) when the list cannot prove the selection:
// fewer than k entries, or the band reaching below the bound t_p, or a band
// larger than kFaBand.  On success the ascending selection is in the
// caller's idx / cnt.
// T_in: the k-th largest key when the caller found it (0xFFFFFFFF: not yet).
template <bool GLOBAL>
__device__ bool select_exact(const FastArgs& a, FaStatic& S, uint8_t* sm, int b, uint32_t C, uint32_t tp, float E,
                             uint32_t* lkey, int32_t* lidx, uint32_t T_in = 0xFFFFFFFFu) {
    const int tid = threadIdx.x;
    const uint32_t k = (uint32_t)a.k;
    uint32_t* hist = reinterpret_cast<uint32_t*>(sm + kFaHist);
    uint32_t* bkey = reinterpret_cast<uint32_t*>(sm + kFaBKey);
    int32_t* bidx = reinterpret_cast<int32_t*>(sm + kFaBIdx);
    uint32_t* bpos = reinterpret_cast<uint32_t*>(sm + kFaBPos);
    uint32_t* gkeys = a.keys + (size_t)b * a.Ncap;
    auto key_at = [&](uint32_t p) -> uint32_t { return GLOBAL ? __ldcg(gkeys + p) : lkey[p]; };
    auto idx_at = [&](uint32_t p) -> int32_t { return GLOBAL ? (int32_t)p : lidx[p]; };
    if (!GLOBAL && C < k) return false;
    const uint32_t T = T_in != 0xFFFFFFFFu ? T_in : kth_largest(key_at, C, k, hist, S.sh64, S.res);
    SA_TRACE_MARK(TR_FAST, 2);
    const float t = key_to_float(T);
    const float e2 = __fmul_ru(2.f, E);
    const uint32_t bhi = score_key(__fadd_ru(t, e2)), blo = score_key(__fsub_rd(t, e2));
    if (!GLOBAL && blo < tp) return false;
    // entries above the band are selected whatever the cut; the band's
    // members are collected (in shared memory while they fit)
    if (tid == 0) {
        S.nb = 0;
        S.a_cnt = 0;
    }
    __syncthreads();
    uint32_t* gak = a.amb_key + (size_t)b * a.Ncap;
    int32_t* gai = a.amb_idx + (size_t)b * a.Ncap;
    uint32_t my_above = 0;
    for (uint32_t p = tid; p < C; p += blockDim.x) {
        const uint32_t kk = key_at(p);
        if (kk > bhi) {
            ++my_above;
        } else if (kk >= blo) {
            const uint32_t slot = atom_add_shared(&S.nb, 1u);
            if (slot < (uint32_t)kFaBand) {
                bidx[slot] = idx_at(p);
                bpos[slot] = p;
            } else if (GLOBAL) {
                gai[slot] = idx_at(p);
            }
        }
    }
    my_above = __reduce_add_sync(0xFFFFFFFFu, my_above);
    if ((tid & 31) == 0) red_add_shared(&S.a_cnt, my_above);
    __syncthreads();
    const uint32_t nb = S.nb, A = S.a_cnt;
    if (!GLOBAL && nb > (uint32_t)kFaBand) return false;
    // exact rescoring of the band (the fp64 definition)
    const uint16_t* icx = a.kidx + (size_t)b * a.Ncap * 64;
    for (uint32_t i = tid; i < nb; i += blockDim.x) {
        if (i < (uint32_t)kFaBand) {
            const uint32_t ek = exact_key(S.q2, icx + (size_t)bidx[i] * 64);
            bkey[i] = ek;
            if (GLOBAL && nb > (uint32_t)kFaBand) {
                gak[i] = ek;
                gai[i] = bidx[i];
            }
        } else {
            gak[i] = exact_key(S.q2, icx + (size_t)__ldcg(gai + i) * 64);
        }
    }
    __threadfence_block();
    __syncthreads();
    SA_TRACE_MARK(TR_FAST, 3);
    // the cut: the R2 best band members by (exact key desc, index asc) win
    const uint32_t R2 = k - A;  // 1 <= R2 <= nb
    uint32_t T2;
    int32_t J2;
    if (nb <= (uint32_t)kFaBand) {
        for (uint32_t i = tid; i < nb; i += blockDim.x) {
            const uint32_t mk = bkey[i];
            const int32_t mj = bidx[i];
            uint32_t rank = 0;
            for (uint32_t o = 0; o < nb; ++o) {
                const uint32_t ok = bkey[o];
                rank += (ok > mk) || (ok == mk && bidx[o] < mj);
            }
            // a winner's key is raised above the band, a loser's put below it
            const uint32_t mark = rank < R2 ? 0xFFFFFFFFu : 0u;
            if (GLOBAL) gkeys[bidx[i]] = mark;
            else lkey[bpos[i]] = mark;
        }
    } else {  // a band larger than shared memory (global list only)
        select_rank(gak, gai, nb, R2, hist, S.sh64, S.res, &T2, &J2);
        for (uint32_t i = tid; i < nb; i += blockDim.x) {
            const uint32_t ek = __ldcg(gak + i);
            const int32_t j = __ldcg(gai + i);
            gkeys[j] = (ek > T2 || (ek == T2 && j <= J2)) ? 0xFFFFFFFFu : 0u;
        }
    }
    __threadfence_block();
    __syncthreads();
    SA_TRACE_MARK(TR_FAST, 4);
    // ordered compaction: entries with a key above the band, ascending
    int32_t* gout = a.idx + (size_t)b * a.k;
    const uint32_t per = (C + blockDim.x - 1) / blockDim.x;
    const uint32_t p0 = min(C, tid * per), p1 = min(C, p0 + per);
    uint32_t mine = 0;
    for (uint32_t p = p0; p < p1; ++p) mine += key_at(p) > bhi;
    uint32_t total;
    uint32_t o = block_exclusive_scan(mine, S.sh64, &total);
    for (uint32_t p = p0; p < p1; ++p) {
        if (key_at(p) > bhi) {
            const int32_t j = idx_at(p);
            if (o < k) gout[o] = j;
            ++o;
        }
    }
    if (tid == 0) {
        if (total != k) flag(DEV_LEN);  // cannot happen
        a.cnt[b] = (int32_t)k;
    }
    return true;
}

// Grid (B): one CTA per sequence.
__global__ void __launch_bounds__(kFaThreads, 1) csa_select_fast_kernel(FastArgs a) {
    extern __shared__ __align__(16) uint8_t sm[];
    __shared__ FaStatic S;
    const int b = blockIdx.x;
    const int tid = threadIdx.x;
    if (tid < 32) {  // qI * 2^768 in fp64 (exact rescoring); an input, read before the wait
        const uint32_t w = reinterpret_cast<const uint32_t*>(a.q_idx + (size_t)b * 64)[tid];
        S.q2[2 * tid] = (double)bf16lo_f32(w) * 0x1p768;
        S.q2[2 * tid + 1] = (double)bf16hi_f32(w) * 0x1p768;
    }
    pdl_wait();
    pdl_release();
    SA_TRACE_MARK(TR_FAST, 0);
    const int n = clamp_n(a.n, b, a.Ncap);
    {
        const uint32_t k = (uint32_t)a.k;
        if ((uint32_t)n <= k) {  // every visible entry, ascending
            int32_t* gout = a.idx + (size_t)b * a.k;
            for (int i = tid; i < a.k; i += kFaThreads) gout[i] = i < n ? i : -1;
            if (tid == 0) a.cnt[b] = n;
        } else {
            const uint32_t* ctl = a.ctrl + (size_t)b * kCtl;
            const uint32_t tp = ld_cg_u32(ctl + kCtlBound);
            const float E = __uint_as_float(ld_cg_u32(ctl + kCtlE));
            bool done = false;
            if (a.mode != kFastForceGlobal) {
                // One round trip: the chunks' candidate counts and the candidate
                // histogram; then the chunk positions and the histogram bin d
                // of the k-th largest key (bins held four per thread, the
                // highest first)
                uint32_t* base = reinterpret_cast<uint32_t*>(sm + kFaBase);
                const uint32_t* cc = a.ccount + (size_t)b * a.nchunks;
                const uint32_t* chg = a.chist + (size_t)b * kCH;
                const uint32_t hsh = ld_cg_u32(ctl + kCtlShift);
                constexpr int CPT = kSelMaxChunks / kFaThreads;  // chunks per thread (2)
                constexpr int HPT = kCH / kFaThreads;            // histogram bins per thread (4)
                uint32_t cv[CPT], sum = 0;
#pragma unroll
                for (int j = 0; j < CPT; ++j) {
                    const int c = tid * CPT + j;
                    cv[j] = c < a.nchunks ? ld_cg_u32(cc + c) : 0u;
                    sum += cv[j];
                }
                // ahead of the counts: the first kSpecS * 32 candidate slots of each
                // warp's first kSpecJ chunks (chunk c = warp + 16 j)
                constexpr int kSpecJ = 8, kSpecS = 2;
                const int lane = tid & 31, warp = tid >> 5;
                const uint2* cs = a.cand + (size_t)b * a.Ncap;
                uint2 spec[kSpecJ][kSpecS];
#pragma unroll
                for (int j = 0; j < kSpecJ; ++j) {
                    const int c = warp + 16 * j;
                    const int rows = c < a.nchunks ? min(a.chunk, a.Ncap - c * a.chunk) : 0;
#pragma unroll
                    for (int u = 0; u < kSpecS; ++u) {
                        const int slot = lane + 32 * u;
                        spec[j][u] = slot < rows ? __ldcg(cs + (size_t)c * a.chunk + slot) : make_uint2(0u, 0u);
                    }
                }
                const int htop = kCH - 1 - tid * HPT;  // this thread's highest bin
                const uint4 hv4 = ld_cg_u32x4(chg + htop - (HPT - 1));
                const uint32_t hv[HPT] = {hv4.w, hv4.z, hv4.y, hv4.x};  // descending bins
                const uint32_t hsum = hv[0] + hv[1] + hv[2] + hv[3];
                if (tid == 0) S.res[0] = -1;  // ordered before the writes below by the scans' barriers
                uint32_t pos, habove, C, htot;
                block_exclusive_scan2(sum, hsum, S.sh64, &pos, &habove, &C, &htot);
#pragma unroll
                for (int j = 0; j < CPT; ++j) {
                    const int c = tid * CPT + j;
                    if (c < a.nchunks) base[c] = pos;
                    pos += cv[j];
                }
#pragma unroll
                for (int j = 0; j < HPT; ++j) {
                    if (habove < k && k <= habove + hv[j]) {
                        S.res[0] = htop - j;
                        S.res[1] = (int)habove;
                    }
                    habove += hv[j];
                }
                if (tid == 0) {
                    base[a.nchunks] = C;
                    S.nd = 0;
                    S.nsg = 0;
                    S.hnext = 0;
                }
                __syncthreads();
                const int d = S.res[0];
                const uint32_t above_d = (uint32_t)S.res[1];
#pragma unroll
                for (int j = 0; j < HPT; ++j)  // the count of bin d + 1, for the band's count above it
                    if (htop - j == d + 1) S.hnext = hv[j];
                if (C >= k && C <= (uint32_t)kFastCap && htot == C && d >= 0) {
                    // The list: warp w copies chunks w, w + 16, ... (the first slots
                    // of its first chunks are in registers already).  The keys of
                    // bin d go to a short list, and the candidates of bins d - 1 ..
                    // d + 1 (where the band will lie) are staged.
                    uint32_t* lkey = reinterpret_cast<uint32_t*>(sm + kFaLKey);
                    int32_t* lidx = reinterpret_cast<int32_t*>(sm + kFaLIdx);
                    uint32_t* dkey = reinterpret_cast<uint32_t*>(sm + kFaBKey);  // the band's arrays, free until then
                    uint32_t* sg_key = reinterpret_cast<uint32_t*>(sm + kFaSg);
                    int32_t* sg_idx = reinterpret_cast<int32_t*>(sm + kFaSg + kStage * 4);
                    uint32_t* sg_pos = reinterpret_cast<uint32_t*>(sm + kFaSg + 2 * kStage * 4);
                    uint32_t* sg_ek = reinterpret_cast<uint32_t*>(sm + kFaSg + 3 * kStage * 4);
                    auto put = [&](uint32_t p, uint2 e) {
                        lkey[p] = e.x;
                        lidx[p] = (int32_t)e.y;
                        const int bin = (int)min((e.x - tp) >> hsh, (uint32_t)(kCH - 1));
                        if (bin == d) {
                            const uint32_t q = atom_add_shared(&S.nd, 1u);
                            if (q < (uint32_t)kFaBand) dkey[q] = e.x;
                        }
                        if (bin + 1 >= d && bin <= d + 1) {
                            const uint32_t q = atom_add_shared(&S.nsg, 1u);
                            if (q < (uint32_t)kStage) {
                                sg_key[q] = e.x;
                                sg_idx[q] = (int32_t)e.y;
                                sg_pos[q] = p;
                            }
                        }
                    };
#pragma unroll
                    for (int j = 0; j < kSpecJ; ++j) {
                        const int c = warp + 16 * j;
                        if (c < a.nchunks) {
                            const uint32_t cb = base[c], cn = base[c + 1] - cb;
#pragma unroll
                            for (int u = 0; u < kSpecS; ++u)
                                if ((uint32_t)(lane + 32 * u) < cn) put(cb + lane + 32 * u, spec[j][u]);
                        }
                    }
#pragma unroll 1
                    for (int c = warp; c < a.nchunks; c += 16) {  // slots not loaded ahead
                        const uint32_t cb = base[c], cn = base[c + 1] - cb;
                        const uint32_t from = c < 16 * kSpecJ ? 32u * kSpecS : 0u;
                        for (uint32_t i = from + lane; i < cn; i += 32) put(cb + i, __ldcg(cs + (size_t)c * a.chunk + i));
                    }
                    __syncthreads();
                    SA_TRACE_MARK(TR_FAST, 1);
                    // the k-th largest key (rank R = k - above_d inside bin d) by
                    // threads 0-255; the staged candidates' exact keys (the fp64
                    // definition) meanwhile by threads 256-511
                    uint32_t T = 0xFFFFFFFFu;
                    const uint32_t nd = S.nd, R = k - above_d, nsg = S.nsg;
                    if (tid == 0) S.tkey = 0xFFFFFFFFu;
                    __syncthreads();
                    const uint16_t* icx = a.kidx + (size_t)b * a.Ncap * 64;
                    if (tid >= kFaThreads - kStage) {
                        const int i = tid - (kFaThreads - kStage);
                        if ((uint32_t)i < nsg && nsg <= (uint32_t)kStage)
                            sg_ek[i] = exact_key(S.q2, icx + (size_t)sg_idx[i] * 64);
                    } else if (nd <= (uint32_t)kFaBand) {
                        for (uint32_t i = tid; i < nd; i += kFaThreads - kStage) {
                            const uint32_t mk = dkey[i];
                            uint32_t gt = 0, ge = 0;
                            for (uint32_t o = 0; o < nd; ++o) {
                                const uint32_t ok = dkey[o];
                                gt += ok > mk;
                                ge += ok >= mk;
                            }
                            if (gt < R && R <= ge) S.tkey = mk;  // every holder of the key writes the same value
                        }
                    }
                    __syncthreads();
                    T = S.tkey;
                    SA_TRACE_MARK(TR_FAST, 2);
                    // the band from the staged candidates when it lies inside their bins
                    bool staged = false;
                    uint32_t bhi = 0;
                    if (T != 0xFFFFFFFFu && nsg <= (uint32_t)kStage) {
                        const float t = key_to_float(T);
                        const float e2 = __fmul_ru(2.f, E);
                        bhi = score_key(__fadd_ru(t, e2));
                        const uint32_t blo = score_key(__fsub_rd(t, e2));
                        const unsigned long long lo_edge = (unsigned long long)tp + ((unsigned long long)max(d - 1, 0) << hsh);
                        const unsigned long long hi_edge =
                            d + 1 >= kCH - 1 ? 0xFFFFFFFFull
                                             : (unsigned long long)tp + ((unsigned long long)(d + 2) << hsh) - 1ull;
                        staged = blo >= tp && (unsigned long long)blo >= lo_edge && (unsigned long long)bhi <= hi_edge;
                        if (staged) {
                            // above the band: the bins above d + 1, and staged keys above bhi
                            const uint32_t hnext = d + 1 <= kCH - 1 ? S.hnext : 0u;
                            uint32_t A = above_d - hnext;
                            for (uint32_t o = 0; o < nsg; ++o) A += sg_key[o] > bhi;
                            const uint32_t R2 = k - A;  // band winners (>= 1)
                            // the cut among the staged band members by (exact key desc, index asc)
                            if ((uint32_t)tid < nsg) {
                                const uint32_t mk = sg_key[tid];
                                if (mk >= blo && mk <= bhi) {
                                    const uint32_t me = sg_ek[tid];
                                    const int32_t mj = sg_idx[tid];
                                    uint32_t rank = 0;
                                    for (uint32_t o = 0; o < nsg; ++o) {
                                        const uint32_t ok = sg_key[o];
                                        if (ok < blo || ok > bhi) continue;
                                        const uint32_t oe = sg_ek[o];
                                        rank += (oe > me) || (oe == me && sg_idx[o] < mj);
                                    }
                                    lkey[sg_pos[tid]] = rank < R2 ? 0xFFFFFFFFu : 0u;
                                }
                            }
                            __syncthreads();
                            SA_TRACE_MARK(TR_FAST, 4);
                            // ordered compaction: entries with a key above the band, ascending
                            int32_t* gout = a.idx + (size_t)b * a.k;
                            const uint32_t per = (C + kFaThreads - 1) / kFaThreads;
                            const uint32_t p0 = min(C, tid * per), p1 = min(C, p0 + per);
                            uint32_t mine = 0;
                            for (uint32_t p = p0; p < p1; ++p) mine += lkey[p] > bhi;
                            uint32_t total;
                            uint32_t o = block_exclusive_scan(mine, S.sh64, &total);
                            for (uint32_t p = p0; p < p1; ++p) {
                                if (lkey[p] > bhi) {
                                    if (o < k) gout[o] = lidx[p];
                                    ++o;
                                }
                            }
                            if (tid == 0) {
                                if (total != k) flag(DEV_LEN);  // cannot happen
                                a.cnt[b] = (int32_t)k;
                            }
                            done = true;
                        }
                    }
                    if (!done)
                    done = select_exact<false>(a, S, sm, b, C, tp, E, lkey, lidx, T);
                }
            }
            if (!done) select_exact<true>(a, S, sm, b, (uint32_t)n, tp, E, nullptr, nullptr);
        }
        __syncthreads();
    }
    SA_TRACE_MARK(TR_FAST, 5);
}

}  // namespace sa
