// topk_prefill_fast.cuh -- the exact top-k of one causal-prefill query
// (SA_OPT_PREFILL_SELECT = 4), "DeepSeek-V4 ... Review", section 3-2 (2)
// (CSA keeps a sparse top-k of the compressed entries).  The keys are the
// exact fp32 scores (order keys) that score_prefill_kernel wrote; the result
// is the same as every other form: the k largest, ties at the threshold by
// lowest index, indices ascending.
//
// One CTA of 512 threads per query (two per SM), the keys staged in shared
// memory (the first 24K; a longer row is read from the scratch past them):
//   1. mean and standard deviation of the scores (one block reduction);
//   2. one histogram pass over 256 linear bins of the score on
//      [mean - 4 sd, mean + 4 sd] (clamped at both ends), counted in
//      per-warp histograms so that no shared-memory atomic contends across
//      warps: the bin d that holds the k-th largest key;
//   3. the keys of bin d go to a short list, and the threshold key T (the
//      k-th largest) is ranked there pairwise;
//   4. one pass counts, per thread's contiguous run of keys, the keys above
//      T and those equal to T; one block scan gives every run its output
//      position and its share of the ties (the lowest indices take them);
//      the indices are written in ascending order.
// When the bin is crowded (a narrow or far-from-normal distribution), T
// comes from byte-digit passes over all keys instead (kth_largest).
#pragma once
#include "decode_fast.cuh"
#include "topk_prefill.cuh"

namespace sa {

constexpr int kP4Threads = 512;     // two CTAs (queries) per SM
constexpr int kP4Keys = 24 * 1024;  // keys staged in shared memory (96 KB); the rest are read from the scratch
constexpr int kP4Bins = 256;        // linear score bins of the first pass
constexpr int kP4List = kP4Threads; // keys of the threshold's bin ranked pairwise (one per thread)
constexpr size_t kP4Smem = (size_t)kP4Keys * 4 + (size_t)(kP4Threads / 32) * kP4Bins * 4;

__global__ void __launch_bounds__(kP4Threads, 2) select_prefill_v4_kernel(TopkPrefillArgs a) {
    extern __shared__ __align__(16) uint32_t p4_sm[];  // [kP4Keys] keys, [16 warps][kP4Bins] histograms
    uint32_t* skeys = p4_sm;
    uint32_t* whist = p4_sm + kP4Keys;
    __shared__ float sf[2][32];
    __shared__ uint32_t sh64[64];
    __shared__ int res[2];
    __shared__ uint32_t s_nd, s_T;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ql = blockIdx.x;
    const int t = a.t0 + ql;
    const int k = a.k;
    const int nv = visible_entries(a, t);
    SA_TRACE_MARK(TR_PSELECT4, 0);
    int32_t* idx = a.idx + ((size_t)a.b * a.Tq + t) * k;
    if (nv <= k) {
        for (int i = tid; i < k; i += kP4Threads) idx[i] = i < nv ? i : -1;
        if (tid == 0) a.cnt[(size_t)a.b * a.Tq + t] = nv;
        return;
    }
    const uint32_t* grow = a.keys + (size_t)ql * a.KS;
    // the query's keys: the first kP4Keys staged in shared memory, the rest from the scratch
    auto kp = [&](int i) -> uint32_t { return i < kP4Keys ? skeys[i] : __ldg(grow + i); };
    // 1. stage the keys (16-byte rows: KS is a multiple of 128) and sum the scores
    float s1 = 0.f, s2 = 0.f;
    {
        const int n4 = (min(nv, kP4Keys) + 3) >> 2;
        // four 16-byte loads in flight per thread, then their stores and sums
        for (int i0 = tid; i0 < n4; i0 += 4 * kP4Threads) {
            uint4 w[4];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int i = i0 + v * kP4Threads;
                w[v] = i < n4 ? reinterpret_cast<const uint4*>(grow)[i] : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int i = i0 + v * kP4Threads;
                if (i >= n4) break;
                reinterpret_cast<uint4*>(skeys)[i] = w[v];
                const uint32_t ws[4] = {w[v].x, w[v].y, w[v].z, w[v].w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (4 * i + u < nv) {
                        const float x = key_to_float(ws[u]);
                        s1 += x;
                        s2 = fmaf(x, x, s2);
                    }
                }
            }
        }
        for (int i = kP4Keys + tid; i < nv; i += kP4Threads) {
            const float x = key_to_float(__ldg(grow + i));
            s1 += x;
            s2 = fmaf(x, x, s2);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, o);
        s2 += __shfl_xor_sync(0xFFFFFFFFu, s2, o);
    }
    if (lane == 0) {
        sf[0][warp] = s1;
        sf[1][warp] = s2;
    }
    for (int i = tid; i < (kP4Threads / 32) * kP4Bins; i += kP4Threads) whist[i] = 0;
    if (tid == 0) s_nd = 0;
    __syncthreads();
    SA_TRACE_MARK(TR_PSELECT4, 1);
    s1 = s2 = 0.f;
#pragma unroll
    for (int w = 0; w < kP4Threads / 32; ++w) {
        s1 += sf[0][w];
        s2 += sf[1][w];
    }
    const float mean = s1 / (float)nv, sd = sqrtf(fmaxf(0.f, s2 / (float)nv - mean * mean));
    const float lo = mean - 4.f * sd, w_inv = (float)kP4Bins / (8.f * sd);
    const bool linear = sd > 0.f && isfinite(w_inv) && isfinite(lo);
    uint32_t T = 0;
    bool found = false;
    if (linear) {
        // 2. the linear histogram (bins clamped to [0, 255])
        auto bin_of = [&](uint32_t key) -> int {
            const float f = (key_to_float(key) - lo) * w_inv;
            return f <= 0.f ? 0 : f >= (float)(kP4Bins - 1) ? kP4Bins - 1 : (int)f;
        };
        uint32_t* wh = whist + warp * kP4Bins;
        for (int i = tid; i < nv; i += kP4Threads) red_add_shared(&wh[bin_of(kp(i))], 1u);
        __syncthreads();
        // bins summed over the warps, the highest bin on thread 0; the bin d of the k-th largest
        uint32_t c = 0;
        const int bb = kP4Bins - 1 - tid;
        if (tid < kP4Bins)
            for (int w = 0; w < kP4Threads / 32; ++w) c += whist[w * kP4Bins + bb];
        if (tid == 0) res[0] = -1;  // ordered before the writes below by the scan's barriers
        const uint32_t above = block_exclusive_scan(c, sh64, nullptr);
        if (tid < kP4Bins && above < (uint32_t)k && (uint32_t)k <= above + c) {
            res[0] = bb;
            res[1] = (int)above;
        }
        __syncthreads();
        const int d = res[0];
        const uint32_t above_d = (uint32_t)res[1];
        // 3. the keys of bin d (the histogram region is free again)
        uint32_t* list = whist;
        if (d >= 0) {
            for (int i = tid; i < nv; i += kP4Threads) {
                const uint32_t key = kp(i);
                if (bin_of(key) == d) {
                    const uint32_t q = atom_add_shared(&s_nd, 1u);
                    if (q < (uint32_t)kP4List) list[q] = key;
                }
            }
        }
        __syncthreads();
        const uint32_t nd = s_nd, R = (uint32_t)k - above_d;
        if (d >= 0 && nd <= (uint32_t)kP4List && R >= 1 && R <= nd) {
            if (tid == 0) s_T = 0u;
            __syncthreads();
            if ((uint32_t)tid < nd) {
                const uint32_t mk = list[tid];
                uint32_t gt = 0, ge = 0;
                for (uint32_t o = 0; o < nd; ++o) {
                    const uint32_t ok = list[o];
                    gt += ok > mk;
                    ge += ok >= mk;
                }
                if (gt < R && R <= ge) s_T = mk;  // every holder of the key writes the same value
            }
            __syncthreads();
            T = s_T;
            found = true;
        }
    }
    SA_TRACE_MARK(TR_PSELECT4, 2);
    if (!found) {  // byte-digit passes over every key
        __syncthreads();
        T = kth_largest([&](uint32_t i) { return kp((int)i); }, (uint32_t)nv, (uint32_t)k, whist, sh64, res);
    }
    // 4. ordered output: each thread's contiguous run of keys
    const int per = (nv + kP4Threads - 1) / kP4Threads;
    const int j0 = min(nv, tid * per), j1 = min(nv, j0 + per);
    uint32_t n_above = 0, n_tie = 0;
    for (int j = j0; j < j1; ++j) {
        const uint32_t key = kp(j);
        n_above += key > T;
        n_tie += key == T;
    }
    uint32_t pa, pt, tot_a, tot_t;
    block_exclusive_scan2(n_above, n_tie, sh64, &pa, &pt, &tot_a, &tot_t);
    SA_TRACE_MARK(TR_PSELECT4, 3);
    const uint32_t take = (uint32_t)k > tot_a ? (uint32_t)k - tot_a : 0u;  // ties kept, lowest indices first
    if (tid == 0 && (tot_a >= (uint32_t)k || tot_a + tot_t < (uint32_t)k)) flag(DEV_LEN);  // cannot happen
    // the run's outputs start after the earlier runs' keys above T and kept ties
    uint32_t o = pa + min(pt, take);
    uint32_t ties_before = pt;
    for (int j = j0; j < j1; ++j) {
        const uint32_t key = kp(j);
        bool sel = key > T;
        if (key == T) {
            sel = ties_before < take;
            ++ties_before;
        }
        if (sel) {
            if (o < (uint32_t)k) idx[o] = j;
            ++o;
        }
    }
    if (tid == 0) a.cnt[(size_t)a.b * a.Tq + t] = k;
    SA_TRACE_MARK(TR_PSELECT4, 4);
}

}  // namespace sa
