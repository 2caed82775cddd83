// attn.cuh -- softmax attention of H query heads (one shared KV head) over a
// list of compressed entries: the CSA branch over the top-k entries
// (gathered rows) and the HCA branch over every visible entry (contiguous
// rows), "DeepSeek-V4 ... Review", section 3-2 (2) component table.
//
// out_h = sum_j softmax_j(scale * q_h . K_j) V_j,  lse_h = log sum_j exp(.)
//
// One CTA handles one query (all H heads: M = 16 rows per warp) and one split
// of its entry list, 64 entries per tile, pipelined with cp.async into
// XOR-swizzled shared memory (all tiles of a short split in flight).  In
// decode each tile is shared by two warp groups, 32 entries each, whose
// softmax states merge at the end.  QK^T and PV run on bf16 tensor-core MMAs
// (mma.sync) with fp32 accumulation (flash-decoding: online softmax in
// registers, P re-used from the S accumulators).  The dense path can keep
// only the last `win` visible rows: the sliding-window branch over raw
// tokens.  An fp8 cache is widened to bf16 in shared memory
// (every e4m3 value is exact in bf16); its per-64-entry scales multiply the S
// columns (K) and the P columns (V) in fp32.  A mixed cache (MIXED) keeps K's
// rotary dims 64..127 in bf16 after its 64 e4m3 codes (192-byte rows): the
// QK^T product runs over the widened e4m3 dims first, their S columns are
// scaled, and the bf16 dims then accumulate on top; V is e4m3.  With one split the CTA writes
// the bf16 output directly; otherwise it writes a normalised fp32 partial and
// its lse, merged by attn_combine_kernel in a fixed order (deterministic and
// independent of the batch: the split size depends only on the entry count).
#pragma once
#include <cooperative_groups.h>

#include "sa_common.cuh"

namespace sa {

constexpr int kTileN = 64;  // entries per tile

struct AttnArgs {
    const uint16_t* q;   // [BQ][H][128], BQ = B * Tq
    const void* K;       // [B][Ncap][128] bf16 or e4m3
    const void* V;
    const float* ks;     // [B][nG] (fp8)
    const float* vs;
    const int32_t* n;    // [B]
    const int32_t* idx;  // gather: [BQ][kmax]
    const int32_t* cnt;  // gather: [BQ]
    const int32_t* pos;  // dense: [BQ] token positions, or NULL (all n[b] visible)
    int Tq, H, Ncap, nG, kmax, m;
    int win;             // dense: keep only the last `win` visible rows (0: all)
    float scale_log2;    // softmax scale * log2(e)
    int tiles_per_split, splits;
    float* part_o;       // [BQ][splits][H][128]
    float* part_lse;     // [BQ][splits][H]
    uint16_t* out;       // [BQ][H][128]
    float* lse;          // [BQ][H] or NULL
};

__device__ __forceinline__ uint32_t swz(int r, int chunk) {  // byte offset in a [rows][128] bf16 tile
    return (uint32_t)(r * 256 + ((chunk ^ (r & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

constexpr int kMixedKRow = 192;  // mixed K row: 64 e4m3 codes, then 64 bf16 rotary dims

template <int NW, bool GATHER, bool FP8, int ST, bool MIXED = false>
struct AttnSmem {
    static constexpr int kQBytes = NW * 16 * 256;
    static constexpr int kKVBytes = kTileN * 256;                 // one bf16 tile
    static constexpr int kStageRaw = FP8 ? kTileN * 128 : kKVBytes;  // one raw tile (V, and K unless mixed)
    static constexpr int kStageRawK = MIXED ? kTileN * kMixedKRow : kStageRaw;  // one raw K tile
    static constexpr int kStagePair = kStageRawK + kStageRaw;
    static constexpr int kQ = 0;
    static constexpr int kRaw = kQ + kQBytes;                      // [ST stages][K, V] raw tiles
    static constexpr int kConv = kRaw + ST * kStagePair;           // fp8: widened K, V tiles
    static constexpr int kMeta = kConv + (FP8 ? 2 * kKVBytes : 0);  // [ST][64] valid + (fp8) scales
    static constexpr int kTotal = kMeta + ST * kTileN * 4 * 3;
};

constexpr int kAttnCluster = 8;  // splits of one query merged in shared memory (CLUSTER variant)

// ST = pipeline stages: ST - 1 tiles are in flight while one is computed.
// CLUSTER: the grid's x dimension is one cluster of kAttnCluster CTAs (the
// splits of one query); they merge their partials through distributed shared
// memory instead of a separate combine pass.
template <int NW, bool GATHER, bool FP8, int ST, bool CLUSTER, int EG, bool MIXED = false>
__global__ void __launch_bounds__(NW * EG * 32) attn_split_kernel(AttnArgs a) {
    using L = AttnSmem<NW, GATHER, FP8, ST, MIXED>;
    static_assert(!MIXED || FP8, "a mixed cache is widened like an e4m3 one");
    constexpr int NT = NW * EG * 32;  // threads
    constexpr int EPW = kTileN / EG;  // entries of a tile per warp
    constexpr int NJ = EPW / 8;       // 8-entry n-tiles per warp
    static_assert(EPW % 16 == 0, "an entry group is whole 16-entry k-steps");
    extern __shared__ __align__(128) uint8_t smem[];
    pdl_wait();
    pdl_release();
    SA_TRACE_MARK(TR_ATTN, 0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int hg = warp % NW, eg = warp / NW;  // head group (16 heads), entry group of each tile
    // grid: (splits, queries) in a cluster launch, else (queries, splits)
    const int split = CLUSTER ? blockIdx.x : blockIdx.y;
    const int bq = CLUSTER ? blockIdx.y : blockIdx.x;
    const int b = bq / a.Tq;
    constexpr int TPR = NT / kTileN;  // threads per row of a tile
    const int p_begin = split * a.tiles_per_split * kTileN;
    // the list entries of the first tiles go out before the counts are known
    int jpre[ST - 1];
#pragma unroll
    for (int s = 0; s < ST - 1; ++s) {
        const int p = p_begin + s * kTileN + tid / TPR;
        jpre[s] = GATHER && p < a.kmax ? (int)ld_cg_u32(a.idx + (size_t)bq * a.kmax + p) : 0;
    }
    int nb = a.n[b];
    if (nb < 0 || nb > a.Ncap) {
        if (tid == 0 && split == 0) flag(DEV_LEN);
        nb = nb < 0 ? 0 : a.Ncap;
    }
    // number of list positions for this query
    int R;
    if (GATHER) {
        R = a.cnt[bq];
        if (R < 0 || R > a.kmax) {
            if (tid == 0 && split == 0) flag(DEV_LEN);
            R = R < 0 ? 0 : a.kmax;
        }
    } else {
        R = nb;
        if (a.pos) {
            const int t = a.pos[bq];
            if (t < 0) {
                if (tid == 0 && split == 0) flag(DEV_POS);
                R = 0;
            } else {
                R = min(R, t / a.m);
            }
        }
    }
    // a sliding window keeps the last `win` visible rows: rbase .. rbase + R
    int rbase = 0;
    if (!GATHER && a.win > 0 && R > a.win) {
        rbase = R - a.win;
        R = a.win;
    }
    const int p_end = min(R, p_begin + a.tiles_per_split * kTileN);
    const int ntiles = p_end > p_begin ? (p_end - p_begin + kTileN - 1) / kTileN : 0;

    uint8_t* sQ = smem + L::kQ;
    uint8_t* sRaw = smem + L::kRaw;
    uint8_t* sConv = smem + L::kConv;
    int* sValid = reinterpret_cast<int*>(smem + L::kMeta);           // [ST][64]
    float* sKs = reinterpret_cast<float*>(sValid + ST * kTileN);      // [ST][64]
    float* sVs = sKs + ST * kTileN;                                   // [ST][64]

    const uint16_t* qp = a.q + (size_t)bq * a.H * 128;
    // Q tile: rows >= H are zero
    for (int c = tid; c < NW * 16 * 16; c += NT) {
        const int r = c >> 4, ch = c & 15;
        cp_async16_zfill(sQ + swz(r, ch), qp + (size_t)min(r, a.H - 1) * 128 + ch * 8, r < a.H);
    }
    cp_async_commit();

    const uint8_t* Kb = reinterpret_cast<const uint8_t*>(a.K);
    const uint8_t* Vb = reinterpret_cast<const uint8_t*>(a.V);
    const int rowBytes = FP8 ? 128 : 256;
    const size_t seqBase = (size_t)b * a.Ncap * rowBytes;

    // each thread copies CPT 16-byte chunks of one row, TPR apart, so that the
    // row's TPR threads read consecutive chunks in each instruction; a
    // gathered row costs one index load
    constexpr int cpr = FP8 ? 8 : 16;            // 16-byte chunks per row
    constexpr int CPT = cpr / TPR;               // chunks per thread
    static_assert(TPR >= 1 && CPT >= 1 && CPT * TPR == cpr, "tile mapping");
    auto load_tile = [&](int tile, int stage, int jv, bool have_j) {
        const int p0 = p_begin + tile * kTileN;
        uint8_t* rk = sRaw + stage * L::kStagePair;
        uint8_t* rv = rk + L::kStageRawK;
        const int r = tid / TPR, c0 = (tid % TPR) * CPT;
        const int p = p0 + r;
        int j = rbase + p;
        bool ok = p < p_end;
        if (GATHER && ok) {
            j = have_j ? jv : a.idx[(size_t)bq * a.kmax + p];
            if (j < 0 || j >= nb) {
                ok = false;
                if (c0 == 0) flag(DEV_INDEX);
            }
        }
        const size_t rowOff = seqBase + (size_t)(ok ? j : 0) * rowBytes;
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            const int ch = tid % TPR + c * TPR;
            const uint32_t doff = FP8 ? (uint32_t)(r * 128 + ch * 16) : swz(r, ch);
            if (!MIXED) cp_async16_zfill(rk + doff, Kb + rowOff + ch * 16, ok);
            cp_async16_zfill(rv + doff, Vb + rowOff + ch * 16, ok);
        }
        if (MIXED) {  // 12 chunks of a 192-byte K row, TPR threads per row
            const size_t rowOffK = ((size_t)b * a.Ncap + (size_t)(ok ? j : 0)) * kMixedKRow;
            for (int ch = tid % TPR; ch < kMixedKRow / 16; ch += TPR)
                cp_async16_zfill(rk + r * kMixedKRow + ch * 16, Kb + rowOffK + ch * 16, ok);
        }
        if (c0 == 0) {
            sValid[stage * kTileN + r] = ok;
            if (FP8) {
                const int g = ok ? j / 64 : 0;
                sKs[stage * kTileN + r] = ok ? a.ks[(size_t)b * a.nG + g] : 0.f;
                sVs[stage * kTileN + r] = ok ? a.vs[(size_t)b * a.nG + g] : 0.f;
            }
        }
    };

#pragma unroll
    for (int s = 0; s < ST - 1; ++s) {
        if (s < ntiles) load_tile(s, s, jpre[s], true);
        cp_async_commit();
    }

    // per-thread state: rows r0 = lane/4 and r1 = lane/4 + 8 of this warp's 16 heads
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
    uint32_t qf[8][4];

    for (int t = 0; t < ntiles; ++t) {
        const int stage = t % ST;
        if (t + ST - 1 < ntiles) load_tile(t + ST - 1, (t + ST - 1) % ST, 0, false);
        cp_async_commit();
        cp_async_wait<ST - 1>();  // Q (first group) and tile t have landed
        __syncthreads();
        if (t == 0) {
            const uint32_t qbase = smem_u32(sQ);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int r = hg * 16 + (lane & 15);
                const int ch = kk * 2 + (lane >> 4);
                ldsm_x4(qbase + swz(r, ch), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
            }
        }

        const uint8_t* tk;
        const uint8_t* tv;
        if (FP8) {
            // widen e4m3 codes to bf16 (exact), into swizzled tiles
            const uint8_t* rk = sRaw + stage * L::kStagePair;
            const uint8_t* rv = rk + L::kStageRawK;
            uint8_t* ck = sConv;
            uint8_t* cv = sConv + L::kKVBytes;
            for (int c = tid; c < kTileN * 16; c += NT) {  // 8 codes -> one 16-byte bf16 chunk
                const int r = c >> 4, ch = c & 15;
                const uint2 wk = MIXED ? (ch < 8 ? *reinterpret_cast<const uint2*>(rk + r * kMixedKRow + ch * 8)
                                                 : make_uint2(0u, 0u))
                                       : *reinterpret_cast<const uint2*>(rk + r * 128 + ch * 8);
                const uint2 wv = *reinterpret_cast<const uint2*>(rv + r * 128 + ch * 8);
                uint4 ok4, ov4;
                uint32_t* okp = &ok4.x;
                uint32_t* ovp = &ov4.x;
                const uint32_t kw[2] = {wk.x, wk.y}, vw[2] = {wv.x, wv.y};
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        okp[h * 2 + e] = pack_bf16x2(e4m3_to_f32((kw[h] >> (16 * e)) & 0xFF),
                                                     e4m3_to_f32((kw[h] >> (16 * e + 8)) & 0xFF));
                        ovp[h * 2 + e] = pack_bf16x2(e4m3_to_f32((vw[h] >> (16 * e)) & 0xFF),
                                                     e4m3_to_f32((vw[h] >> (16 * e + 8)) & 0xFF));
                    }
                if (MIXED && ch >= 8)  // rotary dims: already bf16
                    ok4 = *reinterpret_cast<const uint4*>(rk + r * kMixedKRow + 64 + (ch - 8) * 16);
                *reinterpret_cast<uint4*>(ck + swz(r, ch)) = ok4;
                *reinterpret_cast<uint4*>(cv + swz(r, ch)) = ov4;
            }
            __syncthreads();
            tk = ck;
            tv = cv;
        } else {
            tk = sRaw + stage * L::kStagePair;
            tv = tk + L::kStageRawK;
        }

        // S = Q K^T : 16 heads x EPW entries per warp
        float s[NJ][4];
#pragma unroll
        for (int j = 0; j < NJ; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
        const uint32_t kbase = smem_u32(tk);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            if (MIXED && kk == 4) {  // dims 0..63 (e4m3) done: scale them before the bf16 dims add in
#pragma unroll
                for (int j = 0; j < NJ; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        s[j][e] *= sKs[stage * kTileN + eg * EPW + j * 8 + (lane & 3) * 2 + (e & 1)];
            }
#pragma unroll
            for (int np = 0; np < NJ / 2; ++np) {  // pairs of 8-entry n-tiles
                const int r = eg * EPW + np * 16 + (lane & 7) + ((lane >> 4) << 3);
                const int ch = kk * 2 + ((lane >> 3) & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kbase + swz(r, ch), b0, b1, b2, b3);
                mma16816(s[2 * np], qf[kk], b0, b1);
                mma16816(s[2 * np + 1], qf[kk], b2, b3);
            }
        }
        // scales, masking, online softmax (log2 domain)
        const int* valid = sValid + stage * kTileN;
        float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < NJ; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int col = eg * EPW + j * 8 + (lane & 3) * 2 + (e & 1);
                float v = s[j][e];
                if (FP8 && !MIXED) v *= sKs[stage * kTileN + col];
                v = valid[col] ? v * a.scale_log2 : -INFINITY;
                s[j][e] = v;
                tmax[e >> 1] = fmaxf(tmax[e >> 1], v);
            }
        float alpha[2], mnew[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xFFFFFFFFu, tmax[h], 1));
            tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xFFFFFFFFu, tmax[h], 2));
            mnew[h] = fmaxf(mrow[h], tmax[h]);
            alpha[h] = (mnew[h] == -INFINITY) ? 1.f : exp2f(mrow[h] - mnew[h]);
            mrow[h] = mnew[h];
        }
        float lsum[2] = {0.f, 0.f};
        uint32_t pf[NJ / 2][4];  // P as bf16 A fragments, k-steps of 16 entries
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            float p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float mm = mnew[e >> 1];
                p[e] = (mm == -INFINITY) ? 0.f : exp2f(s[j][e] - mm);
                lsum[e >> 1] += p[e];
                if (FP8) p[e] *= sVs[stage * kTileN + eg * EPW + j * 8 + (lane & 3) * 2 + (e & 1)];
            }
            pf[j >> 1][(j & 1) * 2 + 0] = pack_bf16x2(p[0], p[1]);
            pf[j >> 1][(j & 1) * 2 + 1] = pack_bf16x2(p[2], p[3]);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) lrow[h] = lrow[h] * alpha[h] + lsum[h];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            o[i][0] *= alpha[0];
            o[i][1] *= alpha[0];
            o[i][2] *= alpha[1];
            o[i][3] *= alpha[1];
        }
        // O += P V
        const uint32_t vbase = smem_u32(tv);
#pragma unroll
        for (int kk = 0; kk < NJ / 2; ++kk) {
            // pf[kk] = {a0, a1, a2, a3} in mma order: rows r0/r1 x entries 16kk + {0..7, 8..15}
            const uint32_t af[4] = {pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3]};
#pragma unroll
            for (int dp = 0; dp < 8; ++dp) {  // pairs of 8-dim n-tiles
                const int r = eg * EPW + kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                const int ch = dp * 2 + (lane >> 4);
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vbase + swz(r, ch), b0, b1, b2, b3);
                mma16816(o[2 * dp], af, b0, b1);
                mma16816(o[2 * dp + 1], af, b2, b3);
            }
        }
        __syncthreads();  // this stage's buffers are reloaded next iteration
    }
    cp_async_wait<0>();

    // finish: row sums across the 4 lanes of a row
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        lrow[h] += __shfl_xor_sync(0xFFFFFFFFu, lrow[h], 1);
        lrow[h] += __shfl_xor_sync(0xFFFFFFFFu, lrow[h], 2);
    }
    if (EG > 1) {
        // merge the entry groups' softmax states into the group-0 warps (the
        // K/V buffers are free now); equal fragment layouts: lane-wise merge
        static_assert(L::kMeta - L::kRaw >= (EG - 1) * NW * 17 * 32 * 16, "entry-group merge buffer");
        float4* mb = reinterpret_cast<float4*>(smem + L::kRaw);
        __syncthreads();
        if (eg > 0) {
            float4* my = mb + (size_t)((eg - 1) * NW + hg) * 17 * 32 + lane;
#pragma unroll
            for (int i = 0; i < 16; ++i) my[i * 32] = make_float4(o[i][0], o[i][1], o[i][2], o[i][3]);
            my[16 * 32] = make_float4(mrow[0], mrow[1], lrow[0], lrow[1]);
        }
        __syncthreads();
        if (eg == 0) {
#pragma unroll 1
            for (int g = 1; g < EG; ++g) {
                const float4* ot = mb + (size_t)((g - 1) * NW + hg) * 17 * 32 + lane;
                const float4 ml = ot[16 * 32];
                const float m2[2] = {ml.x, ml.y}, l2[2] = {ml.z, ml.w};
                float al[2], be[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float M = fmaxf(mrow[h], m2[h]);
                    al[h] = mrow[h] == -INFINITY ? 0.f : exp2f(mrow[h] - M);
                    be[h] = m2[h] == -INFINITY ? 0.f : exp2f(m2[h] - M);
                    mrow[h] = M;
                    lrow[h] = lrow[h] * al[h] + l2[h] * be[h];
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float4 v = ot[i * 32];
                    o[i][0] = o[i][0] * al[0] + v.x * be[0];
                    o[i][1] = o[i][1] * al[0] + v.y * be[0];
                    o[i][2] = o[i][2] * al[1] + v.z * be[1];
                    o[i][3] = o[i][3] * al[1] + v.w * be[1];
                }
            }
        }
    }
    const float kLn2 = 0.6931471805599453f;
    float inv[2], lse_r[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const bool empty = !(lrow[h] > 0.f);
        inv[h] = empty ? 0.f : 1.f / lrow[h];
        lse_r[h] = empty ? -INFINITY : (mrow[h] + __log2f(lrow[h])) * kLn2;
    }
    const int hr[2] = {hg * 16 + (lane >> 2), hg * 16 + (lane >> 2) + 8};
    if (CLUSTER) {
        // partials into this CTA's shared memory (Q and the K/V buffers are free now)
        static_assert(L::kMeta >= NW * 16 * 129 * 4, "partial buffer");
        namespace cg = cooperative_groups;
        cg::cluster_group cluster = cg::this_cluster();
        __syncthreads();
        float* po = reinterpret_cast<float*>(smem);  // [NW*16][128]
        float* pl = po + NW * 16 * 128;                          // [NW*16]
#pragma unroll
        for (int h = 0; h < 2 && eg == 0; ++h) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int d = i * 8 + (lane & 3) * 2;
                *reinterpret_cast<float2*>(po + hr[h] * 128 + d) = make_float2(o[i][2 * h] * inv[h], o[i][2 * h + 1] * inv[h]);
            }
            if ((lane & 3) == 0) pl[hr[h]] = lse_r[h];
        }
        cluster.sync();
        // CTA r merges heads r, r + 8, ...: one warp per head, 4 dims per lane
        const int r = (int)cluster.block_rank();
        for (int h = r + kAttnCluster * warp; h < a.H; h += kAttnCluster * NW * EG) {
            float ls[kAttnCluster];
            float M = -INFINITY;
#pragma unroll
            for (int q = 0; q < kAttnCluster; ++q) {
                ls[q] = cluster.map_shared_rank(pl, q)[h];
                M = fmaxf(M, ls[q]);
            }
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            float ws = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int q = 0; q < kAttnCluster; ++q) {
                    const float w = ls[q] == -INFINITY ? 0.f : __expf(ls[q] - M);
                    const float4 v = *reinterpret_cast<const float4*>(cluster.map_shared_rank(po, q) + h * 128 + lane * 4);
                    acc.x += w * v.x;
                    acc.y += w * v.y;
                    acc.z += w * v.z;
                    acc.w += w * v.w;
                    ws += w;
                }
            }
            const float iw = ws > 0.f ? 1.f / ws : 0.f;
            uint16_t* op = a.out + ((size_t)bq * a.H + h) * 128 + lane * 4;
            *reinterpret_cast<uint2*>(op) =
                make_uint2(pack_bf16x2(acc.x * iw, acc.y * iw), pack_bf16x2(acc.z * iw, acc.w * iw));
            if (a.lse && lane == 0) a.lse[(size_t)bq * a.H + h] = ws > 0.f ? M + __logf(ws) : -INFINITY;
        }
        cluster.sync();  // no CTA leaves while others read its shared memory
        return;
    }
    if (eg != 0) return;  // group 0 holds the merged state
    if (a.splits == 1) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (hr[h] >= a.H) continue;
            uint16_t* op = a.out + ((size_t)bq * a.H + hr[h]) * 128;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int d = i * 8 + (lane & 3) * 2;
                *reinterpret_cast<uint32_t*>(op + d) = pack_bf16x2(o[i][2 * h] * inv[h], o[i][2 * h + 1] * inv[h]);
            }
            if (a.lse && (lane & 3) == 0) a.lse[(size_t)bq * a.H + hr[h]] = lse_r[h];
        }
    } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (hr[h] >= a.H) continue;
            float* op = a.part_o + (((size_t)bq * a.splits + split) * a.H + hr[h]) * 128;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int d = i * 8 + (lane & 3) * 2;
                *reinterpret_cast<float2*>(op + d) = make_float2(o[i][2 * h] * inv[h], o[i][2 * h + 1] * inv[h]);
            }
            if ((lane & 3) == 0) a.part_lse[((size_t)bq * a.splits + split) * a.H + hr[h]] = lse_r[h];
        }
    }
    SA_TRACE_MARK(TR_ATTN, 1);
}

// Merge the split partials of one (query, head): one CTA of 8 warps, warp w
// owns splits w, w+8, ...  The first four splits of every warp are loaded
// up front (one round trip for up to 32 splits) and merged against their
// max; further splits keep a running max.  The warps' states are then merged
// in a fixed order (deterministic).
constexpr int kCombThreads = 256;
constexpr int kCombWarps = kCombThreads / 32;
constexpr int kCombPre = 4;

__global__ void __launch_bounds__(kCombThreads) attn_combine_kernel(const float* part_o, const float* part_lse,
                                                                    int splits, int H, uint16_t* out, float* lse) {
    __shared__ float4 red[kCombWarps][32];
    __shared__ float wred[kCombWarps], mred[kCombWarps];
    pdl_wait();
    pdl_release();
    SA_TRACE_MARK(TR_COMBINE, 0);
    const int bh = blockIdx.x;  // bq * H + h
    const int bq = bh / H, h = bh - bq * H;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float* pl = part_lse + (size_t)bq * splits * H + h;
    const float* po = part_o + ((size_t)bq * splits * H + h) * 128 + lane * 4;
    const size_t so = (size_t)H * 128;  // split stride of part_o
    float ls[kCombPre];
    float4 v[kCombPre];
#pragma unroll
    for (int u = 0; u < kCombPre; ++u) {
        const int sp = warp + u * kCombWarps;
        ls[u] = sp < splits ? pl[(size_t)sp * H] : -INFINITY;
        v[u] = sp < splits ? *reinterpret_cast<const float4*>(po + sp * so) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float M = -INFINITY;
#pragma unroll
    for (int u = 0; u < kCombPre; ++u) M = fmaxf(M, ls[u]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
#pragma unroll
    for (int u = 0; u < kCombPre; ++u) {
        const float w = ls[u] == -INFINITY ? 0.f : __expf(ls[u] - M);
        acc.x += w * v[u].x;
        acc.y += w * v[u].y;
        acc.z += w * v[u].z;
        acc.w += w * v[u].w;
        wsum += w;
    }
#pragma unroll 1
    for (int sp = warp + kCombPre * kCombWarps; sp < splits; sp += kCombWarps) {
        const float l2 = pl[(size_t)sp * H];
        const float4 v2 = *reinterpret_cast<const float4*>(po + sp * so);
        if (l2 > M) {
            const float sc = M == -INFINITY ? 0.f : __expf(M - l2);
            acc.x *= sc;
            acc.y *= sc;
            acc.z *= sc;
            acc.w *= sc;
            wsum *= sc;
            M = l2;
        }
        const float w = l2 == -INFINITY ? 0.f : __expf(l2 - M);
        acc.x += w * v2.x;
        acc.y += w * v2.y;
        acc.z += w * v2.z;
        acc.w += w * v2.w;
        wsum += w;
    }
    red[warp][lane] = acc;
    if (lane == 0) {
        wred[warp] = wsum;
        mred[warp] = M;
    }
    __syncthreads();
    if (warp == 0) {
        float Mt = -INFINITY;
#pragma unroll
        for (int w = 0; w < kCombWarps; ++w) Mt = fmaxf(Mt, mred[w]);
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
        float ws = 0.f;
#pragma unroll
        for (int w = 0; w < kCombWarps; ++w) {
            const float sc = mred[w] == -INFINITY ? 0.f : __expf(mred[w] - Mt);
            t.x += sc * red[w][lane].x;
            t.y += sc * red[w][lane].y;
            t.z += sc * red[w][lane].z;
            t.w += sc * red[w][lane].w;
            ws += sc * wred[w];
        }
        const float inv = ws > 0.f ? 1.f / ws : 0.f;
        uint16_t* op = out + ((size_t)bq * H + h) * 128 + lane * 4;
        *reinterpret_cast<uint2*>(op) = make_uint2(pack_bf16x2(t.x * inv, t.y * inv), pack_bf16x2(t.z * inv, t.w * inv));
        if (lse && lane == 0) lse[(size_t)bq * H + h] = ws > 0.f ? Mt + __logf(ws) : -INFINITY;
    }
}

// Log-sum-exp merge of two attentions over disjoint key sets into the
// attention over their union: one warp per (query, head) row, 4 dims a lane.
__global__ void __launch_bounds__(256) attn_lse_merge_kernel(const uint16_t* oa, const float* la, const uint16_t* ob,
                                                             const float* lb, uint16_t* out, float* lse, long long rows) {
    pdl_wait();
    pdl_release();
    const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    const float x = la[r], y = lb[r];
    const float M = fmaxf(x, y);
    const float wa = x == -INFINITY ? 0.f : __expf(x - M), wb = y == -INFINITY ? 0.f : __expf(y - M);
    const float ws = wa + wb;
    const float inv = ws > 0.f ? 1.f / ws : 0.f;
    const uint2 va = *reinterpret_cast<const uint2*>(oa + r * 128 + lane * 4);
    const uint2 vb = *reinterpret_cast<const uint2*>(ob + r * 128 + lane * 4);
    const float a0 = bf16lo_f32(va.x), a1 = bf16hi_f32(va.x), a2 = bf16lo_f32(va.y), a3 = bf16hi_f32(va.y);
    const float b0 = bf16lo_f32(vb.x), b1 = bf16hi_f32(vb.x), b2 = bf16lo_f32(vb.y), b3 = bf16hi_f32(vb.y);
    *reinterpret_cast<uint2*>(out + r * 128 + lane * 4) =
        make_uint2(pack_bf16x2((wa * a0 + wb * b0) * inv, (wa * a1 + wb * b1) * inv),
                   pack_bf16x2((wa * a2 + wb * b2) * inv, (wa * a3 + wb * b3) * inv));
    if (lse && lane == 0) lse[r] = ws > 0.f ? M + __logf(ws) : -INFINITY;
}

}  // namespace sa
