// topk_prefill.cuh -- CSA indexer scores and exact top-k for many queries at
// once (causal prefill), "DeepSeek-V4 ... Review", section 3-2 (2) and 3-2 (4).
//
// Query q at token position t sees entries c with (c + 1) * m <= t.  Scores
// are the same exact quantity as in decode (fp64 FMA chain in ascending i,
// rounded once to fp32).  Two kernels per block of queries:
//   1. score_prefill_kernel -- a register-tiled fp64 "GEMM": each CTA scores 64
//      queries x 128 entries.  The queries are staged as fp64 (q * 2^768), the
//      keys as packed bf16 pairs that each thread widens exactly (scaled-bf16
//      bit placement) right before use; every thread owns 4 x 8 independent
//      FMA chains.  Keys land in a [QB][KS] scratch block.
//   2. select_prefill_kernel -- one CTA per query: loads the query's visible
//      keys into shared memory, radix-selects the k-th largest (11/11/10-bit
//      digits), keeps ties at the threshold by lowest index, and writes the
//      chosen indices in ascending order with an ordered block compaction.
#pragma once
#include "sa_common.cuh"
#include "topk_decode.cuh"

namespace sa {

constexpr int kPsQ = 64;         // queries per score tile
constexpr int kPsE = 128;        // entries per score tile
constexpr int kPsThreads = 256;  // 16 x 16 threads, 4 queries x 8 entries each
constexpr int kPsSmem = 64 * kPsQ * 8 + 32 * kPsE * 4;  // fp64 queries + packed key pairs
constexpr int kPselThreads = 1024;
constexpr int kPselSmemKeys = 48 * 1024;  // keys held in shared memory (192 KB)

struct TopkPrefillArgs {
    const uint16_t* q_idx;  // [B][Tq][64]
    const uint16_t* kidx;   // [B][Ncap][64]
    const int32_t* pos;     // [B][Tq]
    const int32_t* n;       // [B]
    uint32_t* keys;         // [QB][KS] scratch for this block of queries
    int32_t* idx;           // [B][Tq][k]
    int32_t* cnt;           // [B][Tq]
    int Tq, Ncap, KS, k, log2m;
    int b, t0, qb;          // this launch: sequence b, queries t0 .. t0+qb-1
};

__device__ __forceinline__ int visible_entries(const TopkPrefillArgs& a, int t) {
    int nb = a.n[a.b];
    if (nb < 0 || nb > a.Ncap) {
        flag(DEV_LEN);
        nb = nb < 0 ? 0 : a.Ncap;
    }
    int p = a.pos[(size_t)a.b * a.Tq + t];
    if (p < 0) {
        flag(DEV_POS);
        p = 0;
    }
    return min(nb, p >> a.log2m);
}

__global__ void __launch_bounds__(kPsThreads, 2) score_prefill_kernel(TopkPrefillArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    double* sQ = reinterpret_cast<double*>(smem);                        // [64 dims][64 queries]
    uint32_t* sK = reinterpret_cast<uint32_t*>(smem + 64 * kPsQ * 8);    // [32 dim pairs][128 entries]
    __shared__ int s_maxvis;

    const int tid = threadIdx.x;
    const int e0 = blockIdx.x * kPsE;
    const int ql0 = blockIdx.y * kPsQ;  // first query of the tile, local to the block
    if (tid == 0) s_maxvis = 0;
    __syncthreads();
    if (tid < kPsQ && ql0 + tid < a.qb) atomicMax(&s_maxvis, visible_entries(a, a.t0 + ql0 + tid));
    __syncthreads();
    if (e0 >= s_maxvis) return;  // no query of this tile sees these entries
    SA_TRACE_MARK(TR_PSCORE, 0);

    {  // every load of the tile goes out at once, then the stores:
       // queries as q * 2^768 in fp64, dim-major; keys as packed bf16 pairs, [dim pair][entry]
        const int ql = tid & 63;
        const bool okq = ql0 + ql < a.qb;
        const uint4* srcq = reinterpret_cast<const uint4*>(a.q_idx + ((size_t)a.b * a.Tq + a.t0 + ql0 + ql) * 64);
        const int e = tid & 127;
        const bool okk = e0 + e < a.Ncap;
        const uint4* srck = reinterpret_cast<const uint4*>(a.kidx + ((size_t)a.b * a.Ncap + e0 + e) * 64);
        uint4 wq[2], wk[4];
#pragma unroll
        for (int v = 0; v < 2; ++v) wq[v] = okq ? __ldg(srcq + (tid >> 6) + 4 * v) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int v = 0; v < 4; ++v) wk[v] = okk ? __ldg(srck + (tid >> 7) + 2 * v) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int v = 0; v < 2; ++v) {
            const int c = (tid >> 6) + 4 * v;
            const uint32_t ws[4] = {wq[v].x, wq[v].y, wq[v].z, wq[v].w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                sQ[(8 * c + 2 * u) * kPsQ + ql] = (double)bf16lo_f32(ws[u]) * 0x1p768;
                sQ[(8 * c + 2 * u + 1) * kPsQ + ql] = (double)bf16hi_f32(ws[u]) * 0x1p768;
            }
        }
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int c = (tid >> 7) + 2 * v;
            sK[(4 * c + 0) * kPsE + e] = wk[v].x;
            sK[(4 * c + 1) * kPsE + e] = wk[v].y;
            sK[(4 * c + 2) * kPsE + e] = wk[v].z;
            sK[(4 * c + 3) * kPsE + e] = wk[v].w;
        }
    }
    __syncthreads();
    SA_TRACE_MARK(TR_PSCORE, 1);

    const int tq = tid >> 4, te = tid & 15;
    double acc[4][8];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[u][v] = 0.0;

#pragma unroll 2
    for (int i2 = 0; i2 < 32; ++i2) {
        const uint4 k0 = *reinterpret_cast<const uint4*>(sK + i2 * kPsE + te * 4);
        const uint4 k1 = *reinterpret_cast<const uint4*>(sK + i2 * kPsE + 64 + te * 4);
        const uint32_t kw[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // dim 2*i2 + h, ascending
            const double2 qa = *reinterpret_cast<const double2*>(sQ + (2 * i2 + h) * kPsQ + tq * 4);
            const double2 qb = *reinterpret_cast<const double2*>(sQ + (2 * i2 + h) * kPsQ + tq * 4 + 2);
            const double qv[4] = {qa.x, qa.y, qb.x, qb.y};
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const double kd = h ? bf16hi_scaled(kw[v]) : bf16lo_scaled(kw[v]);
#pragma unroll
                for (int u = 0; u < 4; ++u) acc[u][v] = fma(qv[u], kd, acc[u][v]);
            }
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int ql = ql0 + tq * 4 + u;
        if (ql >= a.qb) continue;
        uint32_t* row = a.keys + (size_t)ql * a.KS + e0;
        uint4 lo, hi;
        lo.x = score_key(__double2float_rn(acc[u][0] * 0x1p128));
        lo.y = score_key(__double2float_rn(acc[u][1] * 0x1p128));
        lo.z = score_key(__double2float_rn(acc[u][2] * 0x1p128));
        lo.w = score_key(__double2float_rn(acc[u][3] * 0x1p128));
        hi.x = score_key(__double2float_rn(acc[u][4] * 0x1p128));
        hi.y = score_key(__double2float_rn(acc[u][5] * 0x1p128));
        hi.z = score_key(__double2float_rn(acc[u][6] * 0x1p128));
        hi.w = score_key(__double2float_rn(acc[u][7] * 0x1p128));
        *reinterpret_cast<uint4*>(row + te * 4) = lo;       // KS is a multiple of 128: in bounds
        *reinterpret_cast<uint4*>(row + 64 + te * 4) = hi;
    }
    SA_TRACE_MARK(TR_PSCORE, 2);
}

__global__ void __launch_bounds__(kPselThreads, 1) select_prefill_kernel(TopkPrefillArgs a) {
    extern __shared__ __align__(16) uint32_t skeys[];  // [kPselSmemKeys]
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t sh32[32];
    __shared__ int res[2];
    const int ql = blockIdx.x;
    const int t = a.t0 + ql;
    const int k = a.k;
    const int nv = visible_entries(a, t);
    SA_TRACE_MARK(TR_PSELECT, 0);
    int32_t* idx = a.idx + ((size_t)a.b * a.Tq + t) * k;
    if (nv <= k) {
        for (int i = threadIdx.x; i < k; i += blockDim.x) idx[i] = i < nv ? i : -1;
        if (threadIdx.x == 0) a.cnt[(size_t)a.b * a.Tq + t] = nv;
        return;
    }
    const uint32_t* grow = a.keys + (size_t)ql * a.KS;
    const uint32_t* kp = grow;
    if (nv <= kPselSmemKeys) {
        const int n4 = (nv + 3) >> 2;  // rows are 16-byte aligned (KS multiple of 128)
        for (int i = threadIdx.x; i < n4; i += blockDim.x)
            reinterpret_cast<uint4*>(skeys)[i] = reinterpret_cast<const uint4*>(grow)[i];
        kp = skeys;
    }
    const int nround = (nv + blockDim.x - 1) / blockDim.x * blockDim.x;  // whole warps iterate together

    // digit 1
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    SA_TRACE_MARK(TR_PSELECT, 1);
    for (int j = threadIdx.x; j < nround; j += blockDim.x) {
        const bool v = j < nv;
        hist_add(hist, v ? kp[j] >> 21 : 0u, v);
    }
    __syncthreads();
    int d1, d2, d3;
    uint32_t above;
    find_digit_desc<kBins>(hist, (uint32_t)k, sh32, &d1, &above, res);
    SA_TRACE_MARK(TR_PSELECT, 2);
    const uint32_t K1 = (uint32_t)k - above;
    // digit 2
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < nround; j += blockDim.x) {
        const uint32_t key = j < nv ? kp[j] : 0u;
        const bool v = j < nv && (int)(key >> 21) == d1;
        hist_add(hist, (key >> 10) & (kBins - 1), v);
    }
    __syncthreads();
    find_digit_desc<kBins>(hist, K1, sh32, &d2, &above, res);
    SA_TRACE_MARK(TR_PSELECT, 3);
    const uint32_t K2 = K1 - above;
    // digit 3
    const uint32_t pre = ((uint32_t)d1 << 11) | (uint32_t)d2;
    for (int i = threadIdx.x; i < kBinsLow; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < nround; j += blockDim.x) {
        const uint32_t key = j < nv ? kp[j] : 0u;
        const bool v = j < nv && (key >> 10) == pre;
        hist_add(hist, key & (kBinsLow - 1), v);
    }
    __syncthreads();
    find_digit_desc<kBinsLow>(hist, K2, sh32, &d3, &above, res);
    const uint32_t r = K2 - above;
    const uint32_t nties = hist[d3 < 0 ? 0 : d3];
    __syncthreads();
    SA_TRACE_MARK(TR_PSELECT, 4);
    if ((d1 | d2 | d3) < 0 && threadIdx.x == 0) flag(DEV_LEN);  // inconsistent: cannot happen
    const uint32_t T = (pre << 10) | (uint32_t)d3;

    // lowest-index tie-break: the r-th tie in index order
    int jmax = 0x7FFFFFFF;
    if (r < nties) {
        uint32_t running = 0;
        for (int j0 = 0; j0 < nround; j0 += blockDim.x) {
            const int j = j0 + threadIdx.x;
            const bool tie = j < nv && kp[j] == T;
            uint32_t tot;
            const uint32_t before = running + block_exclusive_scan(tie ? 1u : 0u, sh32, &tot);
            if (tie && before + 1 == r) res[0] = j;
            running += tot;
            if (running >= r) break;  // uniform: every thread sees the same running
        }
        __syncthreads();
        jmax = res[0];
        __syncthreads();
    }
    SA_TRACE_MARK(TR_PSELECT, 5);
    // ordered compaction of the selection
    uint32_t running = 0;
    for (int j0 = 0; j0 < nround; j0 += blockDim.x) {
        const int j = j0 + threadIdx.x;
        const uint32_t key = j < nv ? kp[j] : 0u;
        const bool sel = j < nv && (key > T || (key == T && j <= jmax));
        uint32_t tot;
        const uint32_t p = running + block_exclusive_scan(sel ? 1u : 0u, sh32, &tot);
        if (sel && p < (uint32_t)k) idx[p] = j;
        running += tot;
    }
    if (threadIdx.x == 0) {
        if (running != (uint32_t)k) flag(DEV_LEN);  // cannot happen
        a.cnt[(size_t)a.b * a.Tq + t] = k;
    }
    SA_TRACE_MARK(TR_PSELECT, 6);
}

// ---------------------------------------------- selection, second form ----
// The same exact top-k of one query (ties at the threshold by lowest index,
// output ascending) in fewer passes and barriers:
//   pass 1  histogram of digit 1 (bits 31..21) over the query's keys;
//   pass 2  the keys of digit 1's bin go to a short list in shared memory
//           (a bin above kPsel2ListCap keys is ranked in place instead), and
//           digits 2 and 3 are found over that list alone: the threshold
//           key T and r, the number of keys equal to T that are taken;
//   pass 3  every warp counts, over its own contiguous run of keys, the keys
//           above T and those equal to T (ballots, one barrier);
//   pass 4  every warp writes its selected indices in ascending order at its
//           exclusive prefix, the ties at T taken in index order while their
//           running count is below r (ballots, no block scan).
// Two launch forms: NT = 1024 threads staging up to kPsel2SmemKeys keys in
// shared memory (one CTA per SM), or (STAGE = false) NT = 512 threads that
// read the keys from the scratch (L2) on every pass, with only the list and
// the histogram in shared memory, so that three queries share an SM.
constexpr int kPsel2SmemKeys = 40 * 1024;  // keys staged in shared memory (160 KB)
constexpr int kPsel2ListCap = 8192;        // keys of digit 1's bin held in shared memory (32 KB)
constexpr size_t kPsel2Smem = (size_t)(kPsel2SmemKeys + kPsel2ListCap) * 4;
constexpr size_t kPsel3Smem = (size_t)kPsel2ListCap * 4;
constexpr int kPsel3Threads = 512;

template <int NT, bool STAGE>
__global__ void __launch_bounds__(NT, STAGE ? 1 : 3) select_prefill_v2_kernel(TopkPrefillArgs a) {
    extern __shared__ __align__(16) uint32_t skeys2[];  // [kPsel2SmemKeys] keys (STAGE), [kPsel2ListCap] bin list
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t sh32[32];
    __shared__ int res[2];
    __shared__ uint32_t s_gt[32], s_eq[32];
    __shared__ uint32_t s_lcnt;
    static_assert(NT % 32 == 0 && NT <= 1024, "pass 3 reads one count per warp, at most one per lane");
    constexpr int nw = NT / 32;
    const int ql = blockIdx.x;
    const int t = a.t0 + ql;
    const int k = a.k;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nv = visible_entries(a, t);
    SA_TRACE_MARK(TR_PSELECT2, 0);
    int32_t* idx = a.idx + ((size_t)a.b * a.Tq + t) * k;
    if (nv <= k) {
        for (int i = threadIdx.x; i < k; i += blockDim.x) idx[i] = i < nv ? i : -1;
        if (threadIdx.x == 0) a.cnt[(size_t)a.b * a.Tq + t] = nv;
        return;
    }
    const uint32_t* grow = a.keys + (size_t)ql * a.KS;
    const uint32_t* kp = grow;
    uint32_t* list = STAGE ? skeys2 + kPsel2SmemKeys : skeys2;
    if (STAGE && nv <= kPsel2SmemKeys) {
        const int n4 = (nv + 3) >> 2;  // rows are 16-byte aligned (KS multiple of 128)
        for (int i = threadIdx.x; i < n4; i += blockDim.x)
            reinterpret_cast<uint4*>(skeys2)[i] = reinterpret_cast<const uint4*>(grow)[i];
        kp = skeys2;
    }
    const int nround = (nv + blockDim.x - 1) / blockDim.x * blockDim.x;  // whole warps iterate together

    // pass 1: digit 1
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) hist[i] = 0;
    if (threadIdx.x == 0) s_lcnt = 0;
    __syncthreads();
    SA_TRACE_MARK(TR_PSELECT2, 1);
    for (int j = threadIdx.x; j < nround; j += blockDim.x) {
        const bool v = j < nv;
        hist_add(hist, v ? kp[j] >> 21 : 0u, v);
    }
    __syncthreads();
    int d1, d2, d3;
    uint32_t above;
    find_digit_desc<kBins>(hist, (uint32_t)k, sh32, &d1, &above, res);
    SA_TRACE_MARK(TR_PSELECT2, 2);
    const uint32_t K1 = (uint32_t)k - above;
    const uint32_t c1 = d1 < 0 ? 0u : hist[d1];
    __syncthreads();  // every thread has read c1 before the histogram is cleared

    // pass 2: the keys of bin d1 into the list, then digits 2 and 3 over it
    const uint32_t* dk = kp;
    uint32_t dn = (uint32_t)nv;
    if (c1 <= (uint32_t)kPsel2ListCap) {
        for (int j0 = 0; j0 < nround; j0 += blockDim.x) {
            const int j = j0 + threadIdx.x;
            const uint32_t key = j < nv ? kp[j] : 0u;
            const bool in = j < nv && (int)(key >> 21) == d1;
            const uint32_t m = __ballot_sync(0xFFFFFFFFu, in);
            uint32_t base = 0u;
            if (lane == 0 && m) base = atom_add_shared(&s_lcnt, (uint32_t)__popc(m));
            base = __shfl_sync(0xFFFFFFFFu, base, 0);
            if (in) {
                const uint32_t p = base + (uint32_t)__popc(m & ((1u << lane) - 1u));
                if (p < (uint32_t)kPsel2ListCap) list[p] = key;
            }
        }
        __syncthreads();
        if (threadIdx.x == 0 && s_lcnt != c1) flag(DEV_LEN);  // cannot happen: the bin's own count
        dk = list;
        dn = min(s_lcnt, (uint32_t)kPsel2ListCap);
    }
    const uint32_t dround = (dn + blockDim.x - 1) / blockDim.x * blockDim.x;
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (uint32_t j = threadIdx.x; j < dround; j += blockDim.x) {
        const uint32_t key = j < dn ? dk[j] : 0u;
        const bool v = j < dn && (int)(key >> 21) == d1;
        hist_add(hist, (key >> 10) & (kBins - 1), v);
    }
    __syncthreads();
    find_digit_desc<kBins>(hist, K1, sh32, &d2, &above, res);
    SA_TRACE_MARK(TR_PSELECT2, 3);
    const uint32_t K2 = K1 - above;
    const uint32_t pre = ((uint32_t)d1 << 11) | (uint32_t)d2;
    for (int i = threadIdx.x; i < kBinsLow; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (uint32_t j = threadIdx.x; j < dround; j += blockDim.x) {
        const uint32_t key = j < dn ? dk[j] : 0u;
        const bool v = j < dn && (key >> 10) == pre;
        hist_add(hist, key & (kBinsLow - 1), v);
    }
    __syncthreads();
    find_digit_desc<kBinsLow>(hist, K2, sh32, &d3, &above, res);
    SA_TRACE_MARK(TR_PSELECT2, 4);
    const uint32_t r = K2 - above;  // keys equal to T that are taken (>= 1)
    if ((d1 | d2 | d3) < 0 && threadIdx.x == 0) flag(DEV_LEN);  // inconsistent: cannot happen
    const uint32_t T = (pre << 10) | (uint32_t)d3;

    // pass 3: per warp, over its own run of keys (whole 32-key groups)
    const uint32_t lt = (1u << lane) - 1u;
    const int run = ((nv + nw - 1) / nw + 31) & ~31;
    const int j_lo = warp * run, j_hi = min(nv, j_lo + run);
    uint32_t ngt = 0, neq = 0;
    for (int j0 = j_lo; j0 < j_hi; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t key = j < j_hi ? kp[j] : 0u;
        ngt += (uint32_t)__popc(__ballot_sync(0xFFFFFFFFu, j < j_hi && key > T));
        neq += (uint32_t)__popc(__ballot_sync(0xFFFFFFFFu, j < j_hi && key == T));
    }
    if (lane == 0) {
        s_gt[warp] = ngt;
        s_eq[warp] = neq;
    }
    __syncthreads();
    SA_TRACE_MARK(TR_PSELECT2, 5);
    uint32_t gt_before = lane < warp ? s_gt[lane] : 0u, eq_before = lane < warp ? s_eq[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        gt_before += __shfl_xor_sync(0xFFFFFFFFu, gt_before, o);
        eq_before += __shfl_xor_sync(0xFFFFFFFFu, eq_before, o);
    }
    // pass 4: this warp's selected entries, ascending, from its prefix on
    uint32_t pos = gt_before + min(eq_before, r);
    uint32_t eq_run = eq_before;  // keys equal to T before the current group
    for (int j0 = j_lo; j0 < j_hi; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t key = j < j_hi ? kp[j] : 0u;
        const bool gt = j < j_hi && key > T;
        const bool eq = j < j_hi && key == T;
        const uint32_t em = __ballot_sync(0xFFFFFFFFu, eq);
        const bool sel = gt || (eq && eq_run + (uint32_t)__popc(em & lt) < r);
        const uint32_t sm = __ballot_sync(0xFFFFFFFFu, sel);
        if (sel) {
            const uint32_t p = pos + (uint32_t)__popc(sm & lt);
            if (p < (uint32_t)k) idx[p] = j;
            else flag(DEV_LEN);  // cannot happen: exactly k are selected
        }
        pos += (uint32_t)__popc(sm);
        eq_run += (uint32_t)__popc(em);
    }
    if (threadIdx.x == blockDim.x - 1) {  // the last warp ends at the block's total
        if (pos != (uint32_t)k) flag(DEV_LEN);  // cannot happen
        a.cnt[(size_t)a.b * a.Tq + t] = k;
    }
    SA_TRACE_MARK(TR_PSELECT2, 6);
}

__global__ void fill_positions_kernel(int32_t* pos, int B, int T) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < (long long)B * T) pos[i] = (int32_t)(i % T);
}

}  // namespace sa
