// cp_decode.cuh -- context-parallel decode: the compressed entries of one
// sequence split over W ranks in contiguous shards (the review's section 3-2
// (4) names contextual parallelism among its infrastructure; the exchange
// below is this library's own).
//
// Exactness of the split selection: every entry of the global top-k (by
// score desc, index asc) is in the top-k of its own shard, so the global
// top-k is the top-k of the union of the W local top-k lists.  A step is
//   1. each rank: exact local top-k of its shard (the decode kernels), then
//      cp_candidates_kernel: the exact order key and the global index of each
//      local winner;
//   2. all-gather of the W candidate lists (k pairs per rank and sequence);
//   3. each rank: cp_merge_select_kernel cuts the union at the k-th largest
//      (key, -index) and keeps its own share of the winners;
//   4. each rank: attention over its share (CSA) and over its HCA shard, with
//      the log-sum-exp of each;
//   5. all-gather of the W partial (out, lse) and attn_lse_merge_n_kernel: the
//      attention over the union is the log-sum-exp merge of the partials.
// Gathered rank-major, the candidates are in ascending global index order
// (the shards are contiguous and each local list is ascending), which the
// merge uses for both its tie-break and its ordered outputs.
#pragma once
#include "sa_common.cuh"
#include "topk_decode.cuh"

namespace sa {

// ---------------------------------------------- 1. candidate keys ----------
struct CandArgs {
    const uint16_t* q_idx;  // [B][64] bf16
    const uint16_t* kidx;   // [B][Ncap][64] bf16: this rank's shard
    const int32_t* idx;     // [B][k] local winners (ascending, -1 padded)
    const int32_t* cnt;     // [B]
    const int32_t* base;    // [B] global index of the shard's entry 0
    uint32_t* keys;         // [B][k] out: exact order keys (0 past the count)
    int32_t* gidx;          // [B][k] out: global indices (-1 past the count)
    int32_t* gcnt;          // [B] out: the count
    int Ncap, k;
};

constexpr int kCandThreads = 256;

// grid (ceil(k / 256), B): one thread per list position.
__global__ void __launch_bounds__(kCandThreads) cp_candidates_kernel(CandArgs a) {
    __shared__ double q2[64];  // qI * 2^768 in fp64 (the layout exact_key reads)
    pdl_wait();
    pdl_release();
    const int b = blockIdx.y;
    const int tid = threadIdx.x;
    if (tid < 32) {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(a.q_idx + (size_t)b * 64) + tid);
        q2[2 * tid] = (double)bf16lo_f32(w) * 0x1p768;
        q2[2 * tid + 1] = (double)bf16hi_f32(w) * 0x1p768;
    }
    __syncthreads();
    int c = a.cnt[b];
    if (c < 0 || c > a.k) {
        if (blockIdx.x == 0 && tid == 0) flag(DEV_LEN);
        c = c < 0 ? 0 : a.k;
    }
    const int i = blockIdx.x * kCandThreads + tid;
    if (i >= a.k) return;
    if (i == 0) a.gcnt[b] = c;
    uint32_t key = 0u;
    int32_t g = -1;
    if (i < c) {
        const int j = a.idx[(size_t)b * a.k + i];
        if (j < 0 || j >= a.Ncap) {
            flag(DEV_INDEX);
        } else {
            key = exact_key(q2, a.kidx + ((size_t)b * a.Ncap + j) * 64);
            g = a.base[b] + j;
        }
    }
    a.keys[(size_t)b * a.k + i] = key;
    a.gidx[(size_t)b * a.k + i] = g;
}

// ------------------------------------------- 3. merge and select -----------
constexpr int kMergeThreads = 1024;
constexpr int kMergeCap = 16384;  // candidates of one sequence held in shared memory (W * k)
constexpr int kMergeMaxRanks = 64;
constexpr size_t kMergeSmem = (size_t)kMergeCap * 8;

struct MergeArgs {
    const uint32_t* keys;  // rank w's [B][k] candidate keys at keys + w * stride_list
    const int32_t* gidx;   // rank w's [B][k] at gidx + w * stride_list
    const int32_t* gcnt;   // rank w's [B] at gcnt + w * stride_cnt
    const int32_t* base;   // [B] this rank's shard start
    int32_t* local_idx;    // [B][k] out: this rank's winners, shard-local, ascending, -1 padded
    int32_t* local_cnt;    // [B] out
    int32_t* sel_idx;      // [B][k] out (or NULL): the global selection, ascending, -1 padded
    int32_t* sel_cnt;      // [B] out (or NULL)
    long long stride_list, stride_cnt;  // elements between consecutive ranks' arrays
    int W, B, k, rank;
};

// One CTA per sequence: the W candidate lists, rank-major, into shared
// memory; the exact cut at rank min(k, C) by (key desc, index asc); then
// the winners in list order (= ascending global index), globally and for
// this rank, written by warps over contiguous runs from their prefixes.
__global__ void __launch_bounds__(kMergeThreads, 1) cp_merge_select_kernel(MergeArgs a) {
    extern __shared__ __align__(16) uint32_t csm[];  // [kMergeCap] keys, [kMergeCap] global indices
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t sh64[64];
    __shared__ int res[2];
    __shared__ int s_off[kMergeMaxRanks + 1];
    __shared__ uint32_t s_win[32], s_mine[32], s_tot[2];
    static_assert(kMergeThreads == 1024, "one count per warp and lane");
    pdl_wait();
    pdl_release();
    const int b = blockIdx.x;
    const int tid = threadIdx.x;
    uint32_t* lk = csm;
    int32_t* li = reinterpret_cast<int32_t*>(csm + kMergeCap);
    if (tid == 0) {
        int o = 0;
        for (int w = 0; w < a.W; ++w) {
            int c = a.gcnt[(size_t)w * a.stride_cnt + b];
            if (c < 0 || c > a.k) {
                flag(DEV_LEN);
                c = c < 0 ? 0 : a.k;
            }
            s_off[w] = o;
            o += c;
        }
        s_off[a.W] = o;
    }
    __syncthreads();
    const uint32_t C = (uint32_t)s_off[a.W];  // <= W * k <= kMergeCap (checked on the host)
    for (uint32_t p = tid; p < C; p += kMergeThreads) {
        int w = 0;
        while (s_off[w + 1] <= (int)p) ++w;  // W is small
        const size_t src = (size_t)w * a.stride_list + (size_t)b * a.k + (p - (uint32_t)s_off[w]);
        lk[p] = __ldg(a.keys + src);
        li[p] = __ldg(a.gidx + src);
    }
    __syncthreads();
    const uint32_t R = min(C, (uint32_t)a.k);
    uint32_t T = 0u;
    int32_t jmax = 0x7FFFFFFF;
    const bool all = C <= (uint32_t)a.k;
    if (!all) select_rank(lk, li, C, R, hist, sh64, res, &T, &jmax);
    // winners in list order, globally and this rank's: every warp takes one
    // contiguous run of the list (whole 32-entry groups), counts its winners
    // by ballots, and after one barrier writes them from its exclusive prefix
    const uint32_t lo = (uint32_t)s_off[a.rank], hi = (uint32_t)s_off[a.rank + 1];
    const int32_t base = a.base[b];
    const int lane = tid & 31, warp = tid >> 5;
    const uint32_t lt = (1u << lane) - 1u;
    const uint32_t run = ((C + 31u) / 32u + 31u) & ~31u;
    const uint32_t p_lo = (uint32_t)warp * run, p_hi = min(C, p_lo + run);
    auto wins = [&](uint32_t p) {
        if (p >= p_hi) return false;
        const uint32_t kk = lk[p];
        return all || kk > T || (kk == T && li[p] <= jmax);
    };
    uint32_t nwin = 0, nmine = 0;
    for (uint32_t p0 = p_lo; p0 < p_hi; p0 += 32) {  // warp-uniform trip count
        const uint32_t p = p0 + lane;
        const bool win = wins(p);
        nwin += (uint32_t)__popc(__ballot_sync(0xFFFFFFFFu, win));
        nmine += (uint32_t)__popc(__ballot_sync(0xFFFFFFFFu, win && p >= lo && p < hi));
    }
    if (lane == 0) {
        s_win[warp] = nwin;
        s_mine[warp] = nmine;
    }
    __syncthreads();
    uint32_t gpos = lane < warp ? s_win[lane] : 0u, lpos = lane < warp ? s_mine[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        gpos += __shfl_xor_sync(0xFFFFFFFFu, gpos, o);
        lpos += __shfl_xor_sync(0xFFFFFFFFu, lpos, o);
    }
    for (uint32_t p0 = p_lo; p0 < p_hi; p0 += 32) {
        const uint32_t p = p0 + lane;
        const bool win = wins(p);
        const bool mine = win && p >= lo && p < hi;
        const uint32_t wm = __ballot_sync(0xFFFFFFFFu, win), mm = __ballot_sync(0xFFFFFFFFu, mine);
        // exactly R <= k winners (the cut's contract); a position past k is
        // flagged, never written
        if (win && a.sel_idx) {
            const uint32_t q = gpos + (uint32_t)__popc(wm & lt);
            if (q < (uint32_t)a.k) a.sel_idx[(size_t)b * a.k + q] = li[p];
            else flag(DEV_LEN);
        }
        if (mine) {
            const uint32_t q = lpos + (uint32_t)__popc(mm & lt);
            if (q < (uint32_t)a.k) a.local_idx[(size_t)b * a.k + q] = li[p] - base;
            else flag(DEV_LEN);
        }
        gpos += (uint32_t)__popc(wm);
        lpos += (uint32_t)__popc(mm);
    }
    if (tid == kMergeThreads - 1) {  // the last warp ends at the totals
        s_tot[0] = gpos;
        s_tot[1] = lpos;
    }
    __syncthreads();
    const uint32_t gtot = s_tot[0], ltot = s_tot[1];
    for (uint32_t i = gtot + tid; a.sel_idx && i < (uint32_t)a.k; i += kMergeThreads) a.sel_idx[(size_t)b * a.k + i] = -1;
    for (uint32_t i = ltot + tid; i < (uint32_t)a.k; i += kMergeThreads) a.local_idx[(size_t)b * a.k + i] = -1;
    if (tid == 0) {
        if (gtot != R) flag(DEV_LEN);  // cannot happen
        a.local_cnt[b] = (int32_t)min(ltot, (uint32_t)a.k);
        if (a.sel_cnt) a.sel_cnt[b] = (int32_t)R;
    }
}

// ------------------------------------------------- 5. W-way merge ----------
// Log-sum-exp merge of W attentions over disjoint key sets into the
// attention over their union: one warp per row, 4 dims a lane, fp32
// accumulation, one rounding to bf16.
__global__ void __launch_bounds__(256) attn_lse_merge_n_kernel(const uint16_t* outs, const float* lses, int W,
                                                               long long rows, long long stride_out,
                                                               long long stride_lse, uint16_t* out, float* lse) {
    pdl_wait();
    pdl_release();
    const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    float M = -INFINITY;
    for (int w = 0; w < W; ++w) M = fmaxf(M, lses[(size_t)w * stride_lse + r]);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    float ws = 0.f;
    for (int w = 0; w < W; ++w) {
        const float l = lses[(size_t)w * stride_lse + r];
        const float wt = l == -INFINITY ? 0.f : __expf(l - M);
        const uint2 v = *reinterpret_cast<const uint2*>(outs + (size_t)w * stride_out + (size_t)r * 128 + lane * 4);
        acc[0] += wt * bf16lo_f32(v.x);
        acc[1] += wt * bf16hi_f32(v.x);
        acc[2] += wt * bf16lo_f32(v.y);
        acc[3] += wt * bf16hi_f32(v.y);
        ws += wt;
    }
    const float inv = ws > 0.f ? 1.f / ws : 0.f;
    *reinterpret_cast<uint2*>(out + r * 128 + lane * 4) =
        make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv));
    if (lse && lane == 0) lse[r] = ws > 0.f ? M + __logf(ws) : -INFINITY;
}

}  // namespace sa
