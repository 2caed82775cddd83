// decode_fast.cuh -- the fast path of one hybrid decode step's CSA branch:
// indexer scores, exact top-k and the attention over the chosen entries,
// "DeepSeek-V4 ... Review", section 3-2 (2) (CSA keeps a sparse top-k of the
// compressed entries and attends over them) and 3-2 (4) (the indexer QK path).
//
// Three kernels, chained by programmatic dependent launch, for a bf16 cache,
// up to 64 heads and k <= 2048:
//
//   1. topk_bound_kernel  -- one cluster of 16 CTAs per sequence screens a
//      strided sample of the indexer rows (at most 4096) and takes a sample
//      order statistic well below the expected k-th largest score as a
//      provisional bound t_p.  It only steers how many candidates the scan
//      keeps; the exactness argument below does not depend on it.
//   2. score_fast_kernel  -- the indexer stream (the decode_topk scan: TMA
//      pipeline, fp32 screen s~_j with its certified error bound e_j), which
//      also writes every row with s~_j >= t_p to its chunk's candidate rows,
//      in ascending row order (ballots per tile), and the sequence's
//      E = max e_j.  The bound is awaited only after the first tiles, so the
//      sample overlaps the stream.  Every key is also written, for the
//      fallback below.
//   3. csa_select_attend_kernel -- one cluster of 8 CTAs per sequence.  CTA 0
//      concatenates the chunks' candidates (ascending entry order), finds the
//      k-th largest screened key t~, rescores the band |s~ - t~| <= 2E exactly
//      (the fp64 definition) and cuts it by (s, -j).  This is the exact
//      selection when at least k candidates were kept and t~ - 2E >= t_p:
//      every entry outside the list then has s~ < t~ - 2E and is surely not
//      selected.  Otherwise (or when forced) CTA 0 runs the same selection
//      over all keys of the sequence in global memory.  The ascending index
//      list goes to the caller and, through distributed shared memory, to the
//      cluster: each CTA gathers up to 256 selected K / V rows and computes
//      its partial softmax attention on the tensor cores (tcgen05, TMEM
//      accumulators), transposed so that the MMA's 128 rows are entries:
//          S^T = K_sel Q^T        (M = 128 entries, N = 64 heads, K = 128)
//          O^T = V_sel^T P^T      (M = 128 dims,    N = 64 heads, K = entries)
//      The eight partials (o, max, sum per head) merge through distributed
//      shared memory, each CTA writing eight heads' outputs and lse.
#pragma once
#include "attn_prefill_tc.cuh"
#include "topk_decode.cuh"

namespace sa {

constexpr int kFbCluster = 16;   // bound kernel: CTAs per sequence (a non-portable cluster size)
constexpr int kFbThreads = 128;
constexpr int kFbRowsPT = 2;     // sample rows per thread, all loads in flight at once
constexpr int kFbSamp = kFbCluster * kFbThreads * kFbRowsPT;  // 4096 sample rows at most
constexpr int kFastCap = 8192;   // candidates the selecting CTA holds in shared memory
constexpr int kFastMaxK = 2048;
constexpr int kFaCluster = 8;    // selection + attention: CTAs per sequence
constexpr int kFaThreads = 512;  // 16 warps: all select; warps 0-7 run the softmax, 8 heads each merge
constexpr int kFaEntries = kFastMaxK / kFaCluster;  // 256 selected entries per CTA: two 128-row MMA tiles
constexpr int kFaEarly = 8;      // scan tiles streamed before the bound is awaited
constexpr int kFaBand = 1024;    // band members ranked in shared memory
constexpr int kCtl = 4;          // control words per sequence
constexpr int kCtlBound = 0, kCtlE = 1, kCtlShift = 2;
constexpr int kCH = 2048;        // bins of the candidate histogram: key offsets from t_p >> shift, the top bin clamped

// option values of the fast path (SA_OPT_DECODE_FAST)
constexpr int kFastOff = 0, kFastOn = 1, kFastForceGlobal = 2;

struct FastArgs {
    const uint16_t* q;      // [B][H][128]
    const uint16_t* q_idx;  // [B][64]
    const uint16_t* kidx;   // [B][Ncap][64]
    const uint16_t* K;      // [B][Ncap][128] bf16
    const uint16_t* V;
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
    uint16_t* out;          // [B][H][128] out
    float* lse;             // [B][H] out, or NULL
    int H, Ncap, k, chunk, nchunks, sstride, mode;
    float scale_log2;
};

// ------------------------------------------------------------- clusters ----
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// the two halves of a cluster barrier, to overlap its latency with other work
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }
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
__device__ __forceinline__ uint32_t ld_dsmem_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) { return __uint_as_float(ld_dsmem_u32(addr)); }
__device__ __forceinline__ void st_dsmem_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ float4 ld_dsmem_f32x4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
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
// Grid (kFbCluster, B), clusters of kFbCluster CTAs along x.  Small enough
// (registers, shared memory) to share an SM with three scan CTAs.
__global__ void __launch_bounds__(kFbThreads, 5) topk_bound_kernel(FastArgs a) {
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
#pragma unroll
    for (int h = 0; h < kFbRowsPT; h += 2) {
        uint4 w[2][8];
        int si[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            si[u] = (int)rank * (kFbThreads * kFbRowsPT) + (h + u) * kFbThreads + tid;
            const bool ok = si[u] < ns;
            const uint4* rp = reinterpret_cast<const uint4*>(ic + (size_t)(ok ? si[u] * S : 0) * 64);
#pragma unroll
            for (int c = 0; c < 8; ++c) w[u][c] = ok ? __ldg(rp + c) : make_uint4(0u, 0u, 0u, 0u);
        }
        if (h == 0) cluster_wait();
#pragma unroll
        for (int u = 0; u < 2; ++u)  // into CTA 0's shared memory (a remote store for the other CTAs)
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
        // the r-th largest of the ns sample keys (three digit passes over the
        // cluster's shared memory; keys of absent samples are 0 and there are
        // fewer than ns - r + 1 of them below any real key's rank)
        // only the samples above mean + 1.5 sd (about 7% of a normal sample)
        // enter the digit passes, when at least r of them are there
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
        __shared__ uint32_t su[2][kFbThreads / 32];
        if (lane == 0) {
            sf[0][warp] = s1;
            sf[1][warp] = s2;
            su[0][warp] = smax;
        }
        __syncthreads();
        s1 = s2 = 0.f;
        smax = 0u;
        for (int w = 0; w < kFbThreads / 32; ++w) {
            s1 += sf[0][w];
            s2 += sf[1][w];
            smax = max(smax, su[0][w]);
        }
        const float mean = s1 / (float)ns, var = fmaxf(0.f, s2 / (float)ns - mean * mean);
        const float cut = mean + 1.5f * sqrtf(var);
        uint32_t floor = isfinite(cut) ? score_key(cut) : 0u;
        uint32_t above = 0;
        for (int i = tid; i < ns; i += kFbThreads) above += skey[i] >= floor;
        above = __reduce_add_sync(0xFFFFFFFFu, above);
        if (lane == 0) su[1][warp] = above;
        __syncthreads();
        above = 0;
        for (int w = 0; w < kFbThreads / 32; ++w) above += su[1][w];
        if (above < (uint32_t)r) floor = 0u;
        const uint32_t bound =
            kth_largest([&](uint32_t i) { return skey[i]; }, (uint32_t)ns, (uint32_t)r, hist, sh32, res, floor);
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
__global__ void __launch_bounds__(kScThreads, 4)
    score_fast_kernel(const __grid_constant__ CUtensorMap ic_map, FastArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* tiles = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kScStages * kScTileBytes);
    __shared__ float s_emax[kScThreads / 32];
    __shared__ uint32_t s_wc[2][kScThreads / 32];        // per-warp candidate counts of a tile
    __shared__ uint32_t s_ec[kFaEarly][kScThreads / 32];  // ... of the early tiles
    // The selection kernel may begin launching: it waits for this grid.  This
    // kernel reads only the step's inputs and writes only its own rows before
    // it awaits the bound kernel (pdl_wait below).
    pdl_release();
    SA_TRACE_MARK(TR_SCORE, 0);
    const int b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row0 = blockIdx.x * a.chunk;
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
        if (tid == 0)
            for (int i = 0; i < issued; ++i) mbar_wait(&full[i % kScStages], (i / kScStages) & 1);
        pdl_wait();
        return;
    }
    const int row1 = min(row0 + a.chunk, n);
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
    uint32_t* kout = a.keys + (size_t)b * a.Ncap;
    uint2* cd = a.cand + (size_t)b * a.Ncap + row0;
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t tp = 0, cbase = 0, hsh = 0;
    uint32_t* ch = a.chist + (size_t)b * kCH;
    auto hist_add_key = [&](uint32_t key) {  // the candidate's histogram bin (a fire-and-forget add)
        const uint32_t bin = min((key - tp) >> hsh, (uint32_t)(kCH - 1));
        asm volatile("red.global.add.u32 [%0], 1;" ::"l"(ch + bin) : "memory");
    };
    // the early tiles' candidates, once the bound is known: this thread's own
    // keys of those tiles are read back (its own writes), ballots per tile and
    // warp, one barrier, then written in (tile, warp, lane) order
    auto early = [&](int ne) {
        pdl_wait();
        tp = ld_cg_u32(a.ctrl + (size_t)b * kCtl + kCtlBound);
        hsh = ld_cg_u32(a.ctrl + (size_t)b * kCtl + kCtlShift);
        uint32_t kk[kFaEarly], bal[kFaEarly];
#pragma unroll
        for (int j = 0; j < kFaEarly; ++j) {
            const int r = row0 + j * kScRows + tid;
            const bool v = j < ne && r < row1;
            kk[j] = v ? kout[r] : 0u;
            bal[j] = __ballot_sync(0xFFFFFFFFu, v && kk[j] >= tp);
            if (lane == 0 && j < ne) s_ec[j][warp] = __popc(bal[j]);
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kFaEarly; ++j) {
            if (j < ne) {
                uint32_t off = cbase, tot = 0;
#pragma unroll
                for (int w = 0; w < kScThreads / 32; ++w) {
                    const uint32_t c = s_ec[j][w];
                    off += w < warp ? c : 0u;
                    tot += c;
                }
                if ((bal[j] >> lane) & 1u) {
                    cd[off + __popc(bal[j] & lt)] = make_uint2(kk[j], (uint32_t)(row0 + j * kScRows + tid));
                    hist_add_key(kk[j]);
                }
                cbase += tot;
            }
        }
    };

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
        const bool late = i >= kFaEarly;  // block-uniform
        uint32_t bal = 0;
        if (late) {
            bal = __ballot_sync(0xFFFFFFFFu, valid && key >= tp);
            if (lane == 0) s_wc[i & 1][warp] = __popc(bal);
        }
        __syncthreads();  // slot s is free again; this tile's warp counts are visible
        if (tid == 0 && issued < ntiles) {
            fence_proxy_async();
            mbar_expect_tx(&full[s], kScTileBytes);
            tma_load_3d(tiles + s * kScTileBytes, &ic_map, 0, row0 + issued * kScRows, b, &full[s]);
            ++issued;
        }
        if (late) {
            uint32_t off = cbase, tot = 0;
#pragma unroll
            for (int w = 0; w < kScThreads / 32; ++w) {
                const uint32_t c = s_wc[i & 1][w];
                off += w < warp ? c : 0u;
                tot += c;
            }
            if ((bal >> lane) & 1u) {
                cd[off + __popc(bal & lt)] = make_uint2(key, (uint32_t)row);
                hist_add_key(key);
            }
            cbase += tot;
        }
        if (i + 1 == kFaEarly) early(kFaEarly);
    }
    if (tid == 0)
        for (int i = consumed; i < issued; ++i) mbar_wait(&full[i % kScStages], (i / kScStages) & 1);
    if (timed_out) {
        __syncthreads();
        pdl_wait();
    } else if (ntiles < kFaEarly) {
        early(ntiles);
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

// --------------------------------------------------- 3. select + attend ----
// Shared memory of the selection + attention kernel (offsets from a
// 1024-aligned base).  The selecting CTA's candidate list and scratch alias
// the K / V tiles, which are loaded only after the selection.
constexpr int kFaQ = 0;                          // Q: 64 heads x 128 dims, K-major SW128, halves 8 KB apart
constexpr int kFaK = kFaQ + 16384;               // K: two 128-row tiles of 32 KB (K-major SW128)
constexpr int kFaV = kFaK + 65536;               // V: two tiles, read as the MN-major A operand
constexpr int kFaP = kFaV + 65536;               // P^T: 256 entries x 64 heads, MN-major B operand
constexpr int kFaSel = kFaP + 32768;             // the selected list (CTA 0)
constexpr int kFaSmem = kFaSel + kFastMaxK * 4 + 1024;
// selection scratch, aliased onto K / V / P
constexpr int kFaLKey = kFaK;                    // candidate keys   [kFastCap]
constexpr int kFaLIdx = kFaK + kFastCap * 4;     // candidate indices [kFastCap]
constexpr int kFaHist = kFaV;                    // digit histograms [16 warps][kDigBins] (or [kBins])
constexpr int kFaBase = kFaV + 16 * kDigBins * 4;  // chunk positions [kSelMaxChunks + 1]
constexpr int kFaBKey = kFaBase + (kSelMaxChunks + 1) * 4 + 12;  // band exact keys [kFaBand]
constexpr int kFaBIdx = kFaBKey + kFaBand * 4;   // band indices    [kFaBand]
constexpr int kFaBPos = kFaBIdx + kFaBand * 4;   // band list positions [kFaBand]
constexpr int kFaPart = kFaK;                    // partial O: [64 heads][128 dims] fp32 (after the S MMAs)
static_assert(kFaBPos + kFaBand * 4 <= kFaP, "selection scratch fits in the V region");
static_assert(kFaLIdx + kFastCap * 4 <= kFaV, "the candidate list fits in the K region");
static_assert(kFaSmem <= 227 * 1024, "shared memory of one CTA");

struct FaStatic {
    double q2[64];     // qI * 2^768 (exact rescoring)
    float red[16][32];  // per-warp partial maxima / sums of its 32 heads
    float m[64];       // this CTA's partial: max of scale*log2e*s per head
    float l[64];       // ... and the sum of exp2(. - m)
    uint32_t sh64[64];
    int res[2];
    uint32_t nb, selcnt, nd, a_cnt, tkey;
    uint32_t tmem;
    uint64_t bar_s, bar_o;
};

// The exact selection over a list of (screened key, index) pairs in
// ascending index order: GLOBAL = every key of the sequence in global memory
// (index = position), else the candidate list in shared memory.  Returns
// false (shared-memory list only) when the list cannot prove the selection:
// fewer than k entries, or the band reaching below the bound t_p, or a band
// larger than kFaBand.  On success the ascending selection is in sel[0..k)
// and in the caller's idx / cnt.
// T_in: the k-th largest key when the caller found it (0xFFFFFFFF: not yet).
template <bool GLOBAL>
__device__ bool select_exact(const FastArgs& a, FaStatic& S, uint8_t* sm, int b, uint32_t C, uint32_t tp, float E,
                             uint32_t* lkey, int32_t* lidx, int32_t* sel, uint32_t T_in = 0xFFFFFFFFu) {
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
            if (o < k) {
                sel[o] = j;
                gout[o] = j;
            }
            ++o;
        }
    }
    if (tid == 0) {
        if (total != k) flag(DEV_LEN);  // cannot happen
        a.cnt[b] = (int32_t)k;
        S.selcnt = k;
    }
    return true;
}

// 2^x on the special-function unit (flushes subnormal results to zero: the
// softmax weights are at least 2^-126 wherever they matter, since the
// largest is 1)
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Transposed reduction of 32 values per lane over the warp's 32 lanes (max
// or sum per value index): at each of the five butterfly steps a lane keeps
// one half of its values and sends the other half to its partner, so that
// lane l ends with the reduction of value index l.
template <bool MAX>
__device__ __forceinline__ float head_reduce32(float (&v)[32], int lane) {
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int half = 16 >> step;
        const int o = 16 >> step;
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float keep = upper ? v[half + i] : v[i];
            const float send = upper ? v[i] : v[half + i];
            const float got = __shfl_xor_sync(0xFFFFFFFFu, send, o);
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
__device__ __forceinline__ uint32_t fa_idesc(uint32_t a_mn, uint32_t b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn << 15) | (b_mn << 16) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
}

// Grid (kFaCluster, B), clusters of kFaCluster CTAs along x.
__global__ void __launch_bounds__(kFaThreads, 1) csa_select_attend_kernel(FastArgs a) {
    extern __shared__ uint8_t fa_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fa_raw) + 1023) & ~uintptr_t(1023));
    __shared__ FaStatic S;
    const int b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t rank = cluster_rank();
    int32_t* sel = reinterpret_cast<int32_t*>(sm + kFaSel);
    const uint32_t sQ = smem_u32(sm + kFaQ), sK = smem_u32(sm + kFaK), sV = smem_u32(sm + kFaV),
                   sP = smem_u32(sm + kFaP);

    // Q (an input) before waiting for the scan: rows h < H, the rest zero
    {
        const int h = tid >> 3, c0 = (tid & 7) * 2;  // 64 rows x 16 chunks: 2 chunks per thread
        const bool ok = h < a.H;
        const uint16_t* src = a.q + ((size_t)b * a.H + (ok ? h : 0)) * 128;
#pragma unroll
        for (int c = c0; c < c0 + 2; ++c) cp_async16_zfill(sm + kFaQ + sw128_off(h, c, 8192), src + c * 8, ok);
        cp_async_commit();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S.tmem)),
                     "r"(256));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        mbar_init(&S.bar_s, 1);
        mbar_init(&S.bar_o, 1);
        fence_barrier_init();
    }
    if (rank == 0 && tid < 32) {  // qI * 2^768 in fp64 (exact rescoring)
        const uint32_t w = reinterpret_cast<const uint32_t*>(a.q_idx + (size_t)b * 64)[tid];
        S.q2[2 * tid] = (double)bf16lo_f32(w) * 0x1p768;
        S.q2[2 * tid + 1] = (double)bf16hi_f32(w) * 0x1p768;
    }
    pdl_wait();
    pdl_release();
    SA_TRACE_MARK(TR_FAST, 0);
    const int n = clamp_n(a.n, b, a.Ncap);

    // ---- the selection (CTA 0) ----
    if (rank == 0) {
        const uint32_t k = (uint32_t)a.k;
        if ((uint32_t)n <= k) {  // every visible entry, ascending
            int32_t* gout = a.idx + (size_t)b * a.k;
            for (int i = tid; i < a.k; i += kFaThreads) {
                const int32_t j = i < n ? i : -1;
                gout[i] = j;
                if (i < n) sel[i] = j;
            }
            if (tid == 0) {
                a.cnt[b] = n;
                S.selcnt = (uint32_t)n;
            }
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
                }
                __syncthreads();
                const int d = S.res[0];
                const uint32_t above_d = (uint32_t)S.res[1];
                if (C >= k && C <= (uint32_t)kFastCap && htot == C && d >= 0) {
                    // the list: thread t copies positions [t*per, (t+1)*per), finding its
                    // first chunk by binary search over the positions; the keys of
                    // bin d go to a short list as well
                    uint32_t* lkey = reinterpret_cast<uint32_t*>(sm + kFaLKey);
                    int32_t* lidx = reinterpret_cast<int32_t*>(sm + kFaLIdx);
                    uint32_t* dkey = reinterpret_cast<uint32_t*>(sm + kFaBKey);  // the band's arrays, free until then
                    constexpr int kPer = kFastCap / kFaThreads;  // positions per thread at most (16)
                    const uint32_t per = (C + kFaThreads - 1) / kFaThreads;
                    const uint32_t p0 = min(C, tid * per), p1 = min(C, p0 + per);
                    if (p0 < p1) {
                        int lo = 0, hi = a.nchunks - 1;  // the last chunk c with base[c] <= p0
                        while (lo < hi) {
                            const int mid = (lo + hi + 1) >> 1;
                            if (base[mid] <= p0) lo = mid;
                            else hi = mid - 1;
                        }
                        int c = lo;
                        const uint2* cs = a.cand + (size_t)b * a.Ncap;
                        uint2 e[kPer];  // every load in flight before the first store
#pragma unroll
                        for (int u = 0; u < kPer; ++u) {
                            const uint32_t p = p0 + u;
                            if (p < p1) {
                                while (p >= base[c + 1]) ++c;  // chunks with no candidates are skipped
                                e[u] = __ldcg(cs + (size_t)c * a.chunk + (p - base[c]));
                            }
                        }
#pragma unroll
                        for (int u = 0; u < kPer; ++u) {
                            if (p0 + u < p1) {
                                lkey[p0 + u] = e[u].x;
                                lidx[p0 + u] = (int32_t)e[u].y;
                                if ((int)min((e[u].x - tp) >> hsh, (uint32_t)(kCH - 1)) == d) {
                                    const uint32_t q = atom_add_shared(&S.nd, 1u);
                                    if (q < (uint32_t)kFaBand) dkey[q] = e[u].x;
                                }
                            }
                        }
                    }
                    __syncthreads();
                    SA_TRACE_MARK(TR_FAST, 1);
                    // the k-th largest key: rank R = k - above_d inside bin d
                    uint32_t T = 0xFFFFFFFFu;
                    const uint32_t nd = S.nd, R = k - above_d;
                    if (nd <= (uint32_t)kFaBand) {
                        if (tid == 0) S.tkey = 0xFFFFFFFFu;
                        __syncthreads();
                        for (uint32_t i = tid; i < nd; i += kFaThreads) {
                            const uint32_t mk = dkey[i];
                            uint32_t gt = 0, ge = 0;
                            for (uint32_t o = 0; o < nd; ++o) {
                                const uint32_t ok = dkey[o];
                                gt += ok > mk;
                                ge += ok >= mk;
                            }
                            if (gt < R && R <= ge) S.tkey = mk;  // every holder of the key writes the same value
                        }
                        __syncthreads();
                        T = S.tkey;
                    }
                    done = select_exact<false>(a, S, sm, b, C, tp, E, lkey, lidx, sel, T);
                }
            }
            if (!done) select_exact<true>(a, S, sm, b, (uint32_t)n, tp, E, nullptr, nullptr, sel);
        }
        __syncthreads();
    }
    SA_TRACE_MARK(TR_FAST, 5);
    cluster_sync();  // the selection is in CTA 0's shared memory

    // ---- this CTA's slice of the selection: gather, S^T, softmax, O^T ----
    const int p0 = (int)rank * kFaEntries;
    const int e_g = tid & (kFaEntries - 1);  // the slice entry this thread gathers (K: tid < 256, V: the rest)
    const uint32_t cnt = ld_dsmem_u32(dsmem_addr(&S.selcnt, 0));
    const int jl = (int)ld_dsmem_u32(dsmem_addr(&sel[p0 + e_g], 0));  // in the list's capacity; used below len
    const int len = max(0, min((int)cnt - p0, kFaEntries));
    {
        int j = 0;
        bool ok = e_g < len;
        if (ok) {
            j = jl;
            if (j < 0 || j >= n) {
                flag(DEV_INDEX);
                ok = false;
                j = 0;
            }
        }
        const bool isv = tid >= kFaEntries;
        const uint16_t* src = (isv ? a.V : a.K) + ((size_t)b * a.Ncap + j) * 128;
        uint8_t* dst = sm + (isv ? kFaV : kFaK) + (e_g >> 7) * 32768;
        const int r = e_g & 127;
#pragma unroll
        for (int c = 0; c < 16; ++c) cp_async16_zfill(dst + sw128_off(r, c, 16384), src + c * 8, ok);
        cp_async_commit();
    }
    cp_async_wait<0>();
    fence_async_smem();
    __syncthreads();
    SA_TRACE_MARK(TR_FAST, 6);
    tc_fence_after();
    const uint32_t tmem = S.tmem;
    const int ntile = (len + 127) >> 7;  // 0, 1 or 2 (block-uniform)
    int pend_s = 0, pend_o = 0;
    if (ntile > 0 && tid == 0) {
        const uint32_t id = fa_idesc(0, 0);
        for (int u = 0; u < ntile; ++u) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t ka = sK + u * 32768 + (ks >> 2) * 16384 + (ks & 3) * 32;
                const uint32_t qb = sQ + (ks >> 2) * 8192 + (ks & 3) * 32;
                tc_mma(tmem + 64 * u, tc_desc(ka, 16, 1024), tc_desc(qb, 16, 1024), id, ks > 0);
            }
        }
        tc_commit(&S.bar_s);
        pend_s = 1;
    }
    if (ntile > 0) {
        if (mbar_wait(&S.bar_s, 0) && tid == 0) pend_s = 0;  // a timeout is recorded in the status word
    }
    tc_fence_after();
    SA_TRACE_MARK(TR_FAST, 7);
    // softmax over this slice, per head: thread = (entry, half of the heads);
    // warp w takes TMEM lane quarter w % 4, tile (w / 4) % 2 and heads
    // 32 * (w / 8) .. +31, reading its 32 scores from TMEM twice (for the
    // maxima, then for the weights) rather than holding them across the
    // reduction
    const int u = (warp >> 2) & 1, quarter = warp & 3, hh = warp >> 3;
    const int e = u * 128 + quarter * 32 + lane;
    const bool valid = e < len;
    const uint32_t ta = tmem + ((uint32_t)(quarter * 32) << 16) + 64 * u + 32 * hh;
    float v[32];
    auto load_s = [&]() {
        uint32_t r[32];
        tc_ld32_nw(ta, r);
        tc_wait_ld();
#pragma unroll
        for (int h = 0; h < 32; ++h) v[h] = valid ? __uint_as_float(r[h]) * a.scale_log2 : -INFINITY;
    };
    if (u < ntile) {
        load_s();
    } else {
#pragma unroll
        for (int h = 0; h < 32; ++h) v[h] = -INFINITY;
    }
    S.red[warp][lane] = head_reduce32<true>(v, lane);  // head 32 * hh + lane
    __syncthreads();
    if (tid < 64) {  // head tid: the eight warps of its half
        const int w0 = (tid >> 5) * 8;
        float m = S.red[w0][tid & 31];
#pragma unroll
        for (int w = 1; w < 8; ++w) m = fmaxf(m, S.red[w0 + w][tid & 31]);
        S.m[tid] = m;
    }
    __syncthreads();
    if (u < ntile) load_s();
    // P^T row of this entry (bf16, heads contiguous): p = 2^(s - m), 0 off the slice
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t pk[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int h = c * 8 + w * 2;
            const float p0v = valid ? fast_exp2(v[h] - S.m[32 * hh + h]) : 0.f;  // valid: m is finite
            const float p1v = valid ? fast_exp2(v[h + 1] - S.m[32 * hh + h + 1]) : 0.f;
            v[h] = p0v;
            v[h + 1] = p1v;
            pk[w] = pack_bf16x2(p0v, p1v);
        }
        const int cc = 4 * hh + c;  // 16-byte chunk of the entry's 128-byte row
        *reinterpret_cast<uint4*>(sm + kFaP + (e >> 3) * 1024 + (e & 7) * 128 + ((cc ^ (e & 7)) << 4)) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    const float lsum = head_reduce32<false>(v, lane);
    __syncthreads();  // every read of the maxima in S.red is done
    S.red[warp][lane] = lsum;
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    SA_TRACE_MARK(TR_FAST, 8);
    if (tid < 64) {
        const int w0 = (tid >> 5) * 8;
        float l = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) l += S.red[w0 + w][tid & 31];
        S.l[tid] = l;
    }
    // O^T = V^T P^T over the slice's 16-entry steps
    const int nks = (len + 15) >> 4;
    if (nks > 0 && tid == 0) {
        tc_fence_after();
        const uint32_t id = fa_idesc(1, 1);
        for (int ks = 0; ks < nks; ++ks) {
            const uint32_t va = sV + (ks >> 3) * 32768 + (ks & 7) * 2048;
            tc_mma(tmem + 128, tc_desc(va, 16384, 1024), tc_desc(sP + ks * 2048, 16384, 1024), id, ks > 0);
        }
        tc_commit(&S.bar_o);
        pend_o = 1;
    }
    if (nks > 0) {
        if (mbar_wait(&S.bar_o, 0) && tid == 0) pend_o = 0;
    }
    tc_fence_after();
    SA_TRACE_MARK(TR_FAST, 9);
    // the partial O^T (lane = dim, column = head) into shared memory as [head][dim]
    float* part = reinterpret_cast<float*>(sm + kFaPart);
    if (warp < 8) {
        const int d = quarter * 32 + lane, ph = u;  // warps 4-7 take heads 32-63
        if (nks > 0) {
            uint32_t r0[32];
            tc_ld32_nw(tmem + ((uint32_t)(quarter * 32) << 16) + 128 + 32 * ph, r0);
            tc_wait_ld();
#pragma unroll
            for (int h = 0; h < 32; ++h) part[(32 * ph + h) * 128 + d] = __uint_as_float(r0[h]);
        } else {
#pragma unroll
            for (int h = 0; h < 32; ++h) part[(32 * ph + h) * 128 + d] = 0.f;
        }
    }
    if (tid == 0) {  // an MMA still in flight after a timeout is waited for before TMEM is freed
        if (pend_s) mbar_wait(&S.bar_s, 0);
        if (pend_o) mbar_wait(&S.bar_o, 0);
    }
    tc_fence_before();
    __syncthreads();
    SA_TRACE_MARK(TR_FAST, 10);
    cluster_sync();  // every CTA's partial is in its shared memory

    // ---- merge: CTA r writes heads 8r .. 8r+7 (warps 0-7, one head each) ----
    {
        const int h = (int)rank * 8 + (tid >> 5);
        const int d = (tid & 31) * 4;
        if (warp < 8 && h < a.H) {
            // every remote load is issued before the first use
            float mr[kFaCluster], lr[kFaCluster], M = -INFINITY;
            float4 xr[kFaCluster];
#pragma unroll
            for (int r = 0; r < kFaCluster; ++r) {
                mr[r] = ld_dsmem_f32(dsmem_addr(&S.m[h], (uint32_t)r));
                lr[r] = ld_dsmem_f32(dsmem_addr(&S.l[h], (uint32_t)r));
                xr[r] = ld_dsmem_f32x4(dsmem_addr(part + h * 128 + d, (uint32_t)r));
            }
#pragma unroll
            for (int r = 0; r < kFaCluster; ++r) M = fmaxf(M, mr[r]);
            float o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f, L = 0.f;
#pragma unroll
            for (int r = 0; r < kFaCluster; ++r) {
                if (mr[r] == -INFINITY) continue;  // an empty slice
                const float w = exp2f(mr[r] - M);
                const float4 x = xr[r];
                o0 = fmaf(w, x.x, o0);
                o1 = fmaf(w, x.y, o1);
                o2 = fmaf(w, x.z, o2);
                o3 = fmaf(w, x.w, o3);
                L = fmaf(w, lr[r], L);
            }
            const bool empty = !(L > 0.f);
            const float inv = empty ? 0.f : 1.f / L;
            uint2 pk;
            pk.x = pack_bf16x2(o0 * inv, o1 * inv);
            pk.y = pack_bf16x2(o2 * inv, o3 * inv);
            *reinterpret_cast<uint2*>(a.out + ((size_t)b * a.H + h) * 128 + d) = pk;
            if (a.lse && (tid & 31) == 0)
                a.lse[(size_t)b * a.H + h] = empty ? -INFINITY : (M + __log2f(L)) * 0.6931471805599453f;
        }
    }
    SA_TRACE_MARK(TR_FAST, 11);
    cluster_sync();  // no CTA leaves while others read its shared memory
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256));
    }
}

}  // namespace sa
