// lowp_index.cuh -- the FP4 CSA indexer for decode, "DeepSeek-V4 ... Review",
// section 3-2 (4) (FP4 on the CSA indexer QK path) with the top-k of section
// 3-2 (2).  The review names the precision only; the format read here is
// MXFP4 (OCP Microscaling): e2m1 elements in blocks of 32 indexer dims, one
// E8M0 power-of-two scale per block, X = 2^(floor(log2 amax) - 2) with the
// exponent clamped to [-127, 127] (code 0 when amax == 0), element =
// e2m1 round-to-nearest-even of x / X, saturating at +-6.  Both the query and
// the compressed keys are quantized; the score is the correctly rounded fp32
// value of the exact sum over the two blocks of X_q * X_k * sum e2m1 * e2m1.
//
// Exactness without a screen: with every e2m1 value doubled (an integer in
// -12..12), a block's dot product is an integer A with |A| <= 32 * 144 < 2^13
// (dp4a on int8 operands), and its term A * 2^e (e >= -256 from the two
// E8M0 codes) is exact in fp64.  The two terms are added in fp64 (one
// rounding) and the sum rounded to fp32: rounding twice, first to 53 and
// then to 24 bits, gives the correctly rounded sum since 53 >= 2 * 24 + 2.
// (fp32 terms would round on their own once e < -149, when both blocks are
// tiny.)  The keys are therefore exact, the selection needs no rescoring
// band (bound E = 0), and the filter / resolve / emit kernels of the bf16
// path run unchanged (the resolve in its EXACT variant).
//
// Storage: codes [B][Ncap][32] bytes (element 2i in the low nibble of byte
// i), scales [B][Ncap][2] E8M0 bytes (block 0, block 1).  34 bytes per entry
// against 128 for the bf16 keys.
#pragma once
#include "sa_common.cuh"
#include "topk_decode.cuh"
#include "topk_prefill.cuh"

namespace sa {

// e2m1 code of an fp32 value: round to nearest, ties to the even fraction
// bit, saturating at 6; the sign bit is kept (also for zero).  The midpoints
// between consecutive magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6 are .25, .75,
// 1.25, 1.75, 2.5, 3.5 and 5; at a midpoint the magnitude with an even
// fraction bit (0, 1, 1, 2, 2, 4, 4) wins.
// 2^e as an fp64 bit pattern (exponent field e + 1023), for -1022 <= e <= 1023.
__device__ __forceinline__ double pow2_f64(int e) { return __longlong_as_double((long long)(e + 1023) << 52); }

// Order key of the score A0 * 2^e0 + A1 * 2^e1 (both terms exact in fp64):
// one fp64 addition, one rounding to fp32, -0 as +0 (score_key).
__device__ __noinline__ uint32_t mx_score_key_f64(int A0, int e0, int A1, int e1) {
    const double t = __dadd_rn((double)A0 * pow2_f64(e0), (double)A1 * pow2_f64(e1));
    return score_key(__double2float_rn(t));
}

// While both exponents lie in [-149, 114] the terms are exact and finite in
// fp32 too (A < 2^13 on the fp32 grid, |A * 2^e| < 2^127) and one fp32
// addition rounds their sum once; only blocks that small or that large take
// the fp64 routine (kept out of line: the common path keeps its registers).
__device__ __forceinline__ uint32_t mx_score_key(int A0, int e0, int A1, int e1) {
    if (min(e0, e1) >= -149 && max(e0, e1) <= 114)
        return score_key(__fadd_rn(ldexpf((float)A0, e0), ldexpf((float)A1, e1)));
    return mx_score_key_f64(A0, e0, A1, e1);
}

__device__ __forceinline__ uint32_t e2m1_code(float y) {
    const float a = fabsf(y);
    uint32_t c = (uint32_t)(a > 0.25f) + (uint32_t)(a >= 0.75f) + (uint32_t)(a > 1.25f) + (uint32_t)(a >= 1.75f) +
                 (uint32_t)(a > 2.5f) + (uint32_t)(a >= 3.5f) + (uint32_t)(a > 5.f);
    if (a != a) c = 7;  // e2m1 has no NaN: saturate
    return c | ((__float_as_uint(y) >> 28) & 8u);
}

// floor(log2 a) of a positive fp32 value (normal or subnormal).
__device__ __forceinline__ int floor_log2_f32(float a) {
    const uint32_t u = __float_as_uint(a);
    const int e = (int)((u >> 23) & 0xFFu);
    if (e != 0) return e - 127;
    return (31 - __clz((int)(u & 0x7FFFFFu))) - 149;
}

// The E8M0 exponent of a block with largest magnitude amax.
__device__ __forceinline__ int mx_scale_exp(float amax) {
    if (!(amax > 0.f)) return -127;
    return min(127, max(-127, floor_log2_f32(amax) - 2));
}

// 2^-se for se in [-127, 126] (a normal or the one subnormal power 2^-127).
__device__ __forceinline__ float mx_inv_scale(int se) {
    return 127 - se <= 254 ? __uint_as_float((uint32_t)(127 - se) << 23) : __uint_as_float(0x00400000u);
}

// ------------------------------------------------------- quantize keys ----
struct Mxfp4QuantArgs {
    const uint16_t* kidx;  // [B][Ncap][64] bf16 compressed indexer keys
    const int32_t* n;      // [B] entries present
    uint8_t* codes;        // [B][Ncap][32]
    uint8_t* scales;       // [B][Ncap][2]
    int Ncap, row_from;
};

constexpr int kQuantThreads = 256;

// One thread per (entry, block of 32 dims): entries row_from .. n-1 (grid:
// 2 * (Ncap - row_from) threads x B).
__global__ void __launch_bounds__(kQuantThreads) mxfp4_quantize_kernel(Mxfp4QuantArgs a) {
    const int b = blockIdx.y;
    const long long t = (long long)blockIdx.x * kQuantThreads + threadIdx.x;
    const long long r = (long long)a.row_from + (t >> 1);
    if (r >= a.Ncap) return;
    const int row = (int)r, blk = (int)(t & 1);
    const int n = clamp_n(a.n, b, a.Ncap);
    if (row < a.row_from || row >= n) return;
    const size_t e = (size_t)b * a.Ncap + row;
    const uint4* src = reinterpret_cast<const uint4*>(a.kidx + e * 64 + blk * 32);
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 v = __ldg(src + i);
        w[4 * i] = v.x;
        w[4 * i + 1] = v.y;
        w[4 * i + 2] = v.z;
        w[4 * i + 3] = v.w;
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16lo_f32(w[i])), fabsf(bf16hi_f32(w[i]))));
    const int se = mx_scale_exp(amax);
    const float inv = mx_inv_scale(se);  // x * 2^-se is exact (or below the smallest code's midpoint)
    uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t byte = e2m1_code(bf16lo_f32(w[i]) * inv) | (e2m1_code(bf16hi_f32(w[i]) * inv) << 4);
        out[i >> 2] |= byte << (8 * (i & 3));
    }
    *reinterpret_cast<uint4*>(a.codes + e * 32 + blk * 16) = make_uint4(out[0], out[1], out[2], out[3]);
    a.scales[e * 2 + blk] = (uint8_t)(se + 127);
}

// ------------------------------------------------------------ FP4 scores ---
constexpr int kF4Threads = 256;
constexpr int kF4Batch = 4;                       // entries per thread with loads in flight together
constexpr int kF4Rows = kF4Threads * kF4Batch;    // entries per CTA pass
// doubled e2m1 magnitudes by 3-bit code: 0 1 2 3 4 6 8 12 (bytes)
constexpr uint32_t kE2m1LutLo = 0x03020100u, kE2m1LutHi = 0x0C080604u;

// Signed dot product of eight doubled key elements (one 32-bit word of
// codes, element j in nibble j) with the matching eight doubled query
// elements, given as (qp, qn) = +q and -q for elements 0..3 and (qp2, qn2)
// for 4..7.  The key's magnitudes come from a byte permute of the table, its
// signs pick +q or -q byte by byte.
__device__ __forceinline__ int dot8_e2m1(uint32_t x, uint32_t qp, uint32_t qn, uint32_t qp2, uint32_t qn2, int acc) {
    const uint32_t m0 = __byte_perm(kE2m1LutLo, kE2m1LutHi, x & 0x7777u);
    const uint32_t s0 = __byte_perm(qp, qn, 0x3210u | ((x >> 1) & 0x4444u));
    const uint32_t m1 = __byte_perm(kE2m1LutLo, kE2m1LutHi, (x >> 16) & 0x7777u);
    const uint32_t s1 = __byte_perm(qp2, qn2, 0x3210u | ((x >> 17) & 0x4444u));
    acc = __dp4a((int)m0, (int)s0, acc);
    return __dp4a((int)m1, (int)s1, acc);
}

// Order keys of the FP4 scores of a.chunk entries per CTA (grid: chunks x B),
// their top-11-bit histogram, and, from the sequence's last CTA, the bin of
// the k-th largest key, the count above it and E = 0, in the layout the
// filter and resolve kernels read.
__global__ void __launch_bounds__(kF4Threads) score_decode_mxfp4_kernel(TopkDecodeArgs a,
                                                                        const uint8_t* __restrict__ codes,
                                                                        const uint8_t* __restrict__ scales) {
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t s_qp[16], s_qn[16];
    __shared__ int s_qe[2];
    __shared__ uint32_t s_sh32[32];
    __shared__ int s_res[2];
    __shared__ uint32_t s_last;
    pdl_wait();
    pdl_release();
    SA_TRACE_MARK(TR_SCORE_FP4, 0);
    const int b = blockIdx.y;
    const int tid = threadIdx.x;
    const int n = clamp_n(a.n, b, a.Ncap);
    if (n <= a.k) return;  // the filter answers this sequence
    const int row0 = blockIdx.x * a.chunk;
    const int row1 = min(row0 + a.chunk, n);

    // the query, quantized like the keys: warp 0, two elements per lane
    if (tid < 32) {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(a.q_idx + (size_t)b * 64) + tid);
        const float x0 = bf16lo_f32(w), x1 = bf16hi_f32(w);
        float m = fmaxf(fabsf(x0), fabsf(x1));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));  // 16 lanes = 32 dims
        const int se = mx_scale_exp(m);
        const float inv = mx_inv_scale(se);
        // doubled signed values as int8: e2m1 code -> +-{0,1,2,3,4,6,8,12}
        const uint32_t c0 = e2m1_code(x0 * inv), c1 = e2m1_code(x1 * inv);
        const int v0 = (int)((__byte_perm(kE2m1LutLo, kE2m1LutHi, c0 & 7u)) & 0xFFu) * ((c0 & 8u) ? -1 : 1);
        const int v1 = (int)((__byte_perm(kE2m1LutLo, kE2m1LutHi, c1 & 7u)) & 0xFFu) * ((c1 & 8u) ? -1 : 1);
        const uint32_t pair = ((uint32_t)v0 & 0xFFu) | (((uint32_t)v1 & 0xFFu) << 8);
        const uint32_t npair = ((uint32_t)(-v0) & 0xFFu) | (((uint32_t)(-v1) & 0xFFu) << 8);
        const uint32_t hi = __shfl_down_sync(0xFFFFFFFFu, pair, 1), nhi = __shfl_down_sync(0xFFFFFFFFu, npair, 1);
        if ((tid & 1) == 0) {  // elements 4m..4m+3 in word m = tid / 2
            s_qp[tid >> 1] = pair | (hi << 16);
            s_qn[tid >> 1] = npair | (nhi << 16);
        }
        if ((tid & 15) == 0) s_qe[tid >> 4] = se + 127;
    }
    for (int i = tid; i < kBins; i += kF4Threads) hist[i] = 0;
    __syncthreads();
    uint32_t qp[16], qn[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        qp[i] = s_qp[i];
        qn[i] = s_qn[i];
    }
    // block b of an entry scores A_b * 2^(ek_b - 127) * 2^(eq_b - 127) / 4,
    // with ek_b, eq_b the E8M0 codes: the exponent is ek_b + (eq_b - 254) - 2
    const int eq0 = s_qe[0] - 254, eq1 = s_qe[1] - 254;

    const uint4* c4 = reinterpret_cast<const uint4*>(codes + (size_t)b * a.Ncap * 32);
    const uint16_t* s2 = reinterpret_cast<const uint16_t*>(scales + (size_t)b * a.Ncap * 2);
    uint32_t* keys = a.keys + (size_t)b * a.Ncap;
#pragma unroll 1
    for (int p0 = row0; p0 < row1; p0 += kF4Rows) {
        uint4 lo[kF4Batch], hi[kF4Batch];
        uint32_t sc[kF4Batch];
#pragma unroll
        for (int u = 0; u < kF4Batch; ++u) {
            const int row = p0 + u * kF4Threads + tid;
            if (row < row1) {
                lo[u] = __ldg(c4 + 2 * (size_t)row);
                hi[u] = __ldg(c4 + 2 * (size_t)row + 1);
                sc[u] = __ldg(s2 + row);
            }
        }
#pragma unroll
        for (int u = 0; u < kF4Batch; ++u) {
            const int row = p0 + u * kF4Threads + tid;
            if (row >= row1) continue;
            int A0 = 0, A1 = 0;
            A0 = dot8_e2m1(lo[u].x, qp[0], qn[0], qp[1], qn[1], A0);
            A0 = dot8_e2m1(lo[u].y, qp[2], qn[2], qp[3], qn[3], A0);
            A0 = dot8_e2m1(lo[u].z, qp[4], qn[4], qp[5], qn[5], A0);
            A0 = dot8_e2m1(lo[u].w, qp[6], qn[6], qp[7], qn[7], A0);
            A1 = dot8_e2m1(hi[u].x, qp[8], qn[8], qp[9], qn[9], A1);
            A1 = dot8_e2m1(hi[u].y, qp[10], qn[10], qp[11], qn[11], A1);
            A1 = dot8_e2m1(hi[u].z, qp[12], qn[12], qp[13], qn[13], A1);
            A1 = dot8_e2m1(hi[u].w, qp[14], qn[14], qp[15], qn[15], A1);
            const uint32_t key = mx_score_key(A0, (int)(sc[u] & 0xFFu) + eq0 - 2, A1, (int)(sc[u] >> 8) + eq1 - 2);
            keys[row] = key;
            atomicAdd(&hist[key >> 21], 1u);
        }
    }
    __syncthreads();
    for (int i = tid; i < kBins; i += kF4Threads)
        if (hist[i]) atomicAdd(&a.hist1[(size_t)b * kBins + i], hist[i]);

    // the sequence's last CTA finds the bin d1 of the k-th largest key and
    // the count above it; E = 0 (the keys are exact)
    uint32_t* tot = a.totals + (size_t)b * kTotals;
    __threadfence();
    __syncthreads();
    SA_TRACE_MARK(TR_SCORE_FP4, 1);
    if (tid == 0) s_last = atomicAdd(tot + kTotTicket, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    constexpr int NPT = kBins / kF4Threads;  // 8 bins per thread
    uint32_t hb[NPT];
    {
        const uint32_t* src = a.hist1 + (size_t)b * kBins + (kF4Threads - 1 - tid) * NPT;
#pragma unroll
        for (int v = 0; v < NPT / 4; ++v) {
            const uint4 x = ld_cg_u32x4(src + 4 * v);
            hb[4 * v] = x.x;
            hb[4 * v + 1] = x.y;
            hb[4 * v + 2] = x.z;
            hb[4 * v + 3] = x.w;
        }
    }
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
        tot[kTotE] = __float_as_uint(0.f);
        tot[kTotAbove] = above1;
    }
    SA_TRACE_MARK(TR_SCORE_FP4, 2);
}

// ------------------------------------------------- FP4 prefill scores ---
// The causal-prefill counterpart: order keys of the FP4 scores of a block of
// queries against every entry, in the key block select_prefill_kernel reads.
// A CTA takes 64 queries x 128 entries (the bf16 kernel's tiling); each
// thread owns 4 queries x 8 entries and one exact int32 accumulator per
// 32-dim block.  The queries are quantized here by the rule of the keys;
// the keys' codes are widened once per tile to doubled signed int8 values
// (+-{0,1,2,3,4,6,8,12}) in shared memory, four per 32-bit word.
constexpr int kPf4Smem = kPsQ * 16 * 4 + 16 * kPsE * 4;  // query words [64][16] + key words [16][128]

__device__ __forceinline__ uint32_t e2m1_doubled_s8(uint32_t code) {  // signed doubled value as a byte
    const int m = (int)(__byte_perm(kE2m1LutLo, kE2m1LutHi, code & 7u) & 0xFFu);
    return (uint32_t)((code & 8u) ? -m : m) & 0xFFu;
}

__global__ void __launch_bounds__(kPsThreads, 2) score_prefill_mxfp4_kernel(TopkPrefillArgs a,
                                                                           const uint8_t* __restrict__ codes,
                                                                           const uint8_t* __restrict__ scales) {
    extern __shared__ __align__(16) uint32_t smem_w[];
    uint32_t* sQ = smem_w;                 // [64 queries][16 words]
    uint32_t* sK = smem_w + kPsQ * 16;     // [16 words][128 entries]
    __shared__ int sQe[kPsQ][2];           // E8M0 codes of the queries' blocks
    __shared__ uint8_t sKe[kPsE][2];       // ... and of the entries'
    __shared__ int s_maxvis;

    const int tid = threadIdx.x;
    const int e0 = blockIdx.x * kPsE;
    const int ql0 = blockIdx.y * kPsQ;
    if (tid == 0) s_maxvis = 0;
    __syncthreads();
    if (tid < kPsQ && ql0 + tid < a.qb) atomicMax(&s_maxvis, visible_entries(a, a.t0 + ql0 + tid));
    __syncthreads();
    if (e0 >= s_maxvis) return;  // no query of this tile sees these entries
    SA_TRACE_MARK(TR_PSCORE_FP4, 0);

    if (tid < 2 * kPsQ) {  // one thread per (query, 32-dim block): quantize
        const int ql = tid >> 1, blk = tid & 1;
        const bool ok = ql0 + ql < a.qb;
        uint32_t w[16];
        const uint4* src = reinterpret_cast<const uint4*>(a.q_idx + ((size_t)a.b * a.Tq + a.t0 + ql0 + ql) * 64 +
                                                          blk * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = ok ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
            w[4 * i] = v.x;
            w[4 * i + 1] = v.y;
            w[4 * i + 2] = v.z;
            w[4 * i + 3] = v.w;
        }
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16lo_f32(w[i])), fabsf(bf16hi_f32(w[i]))));
        const int se = mx_scale_exp(amax);
        const float inv = mx_inv_scale(se);
#pragma unroll
        for (int i = 0; i < 8; ++i) {  // word i: elements 4i .. 4i+3 of the block
            const uint32_t b0 = e2m1_doubled_s8(e2m1_code(bf16lo_f32(w[2 * i]) * inv));
            const uint32_t b1 = e2m1_doubled_s8(e2m1_code(bf16hi_f32(w[2 * i]) * inv));
            const uint32_t b2 = e2m1_doubled_s8(e2m1_code(bf16lo_f32(w[2 * i + 1]) * inv));
            const uint32_t b3 = e2m1_doubled_s8(e2m1_code(bf16hi_f32(w[2 * i + 1]) * inv));
            sQ[ql * 16 + blk * 8 + i] = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
        }
        sQe[ql][blk] = se + 127;
    }
    {  // keys: one thread per (entry, 16-byte half of its codes)
        const int e = tid >> 1, half = tid & 1;
        const bool ok = e0 + e < a.Ncap;
        const size_t row = (size_t)a.b * a.Ncap + e0 + e;
        const uint4 c = ok ? __ldg(reinterpret_cast<const uint4*>(codes + row * 32) + half) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // 8 codes -> two words of 4 doubled int8
            uint32_t lo = 0u, hi = 0u;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                lo |= e2m1_doubled_s8((cw[i] >> (4 * j)) & 0xFu) << (8 * j);
                hi |= e2m1_doubled_s8((cw[i] >> (4 * (j + 4))) & 0xFu) << (8 * j);
            }
            sK[(half * 8 + 2 * i) * kPsE + e] = lo;
            sK[(half * 8 + 2 * i + 1) * kPsE + e] = hi;
        }
        if (half == 0) {
            const uint16_t sc = ok ? __ldg(reinterpret_cast<const uint16_t*>(scales + row * 2)) : (uint16_t)0x7F7F;
            sKe[e][0] = (uint8_t)(sc & 0xFFu);
            sKe[e][1] = (uint8_t)(sc >> 8);
        }
    }
    __syncthreads();
    SA_TRACE_MARK(TR_PSCORE_FP4, 1);

    const int tq = tid >> 4, te = tid & 15;
    int acc[2][4][8];
#pragma unroll
    for (int g = 0; g < 2; ++g)
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 8; ++v) acc[g][u][v] = 0;
#pragma unroll
    for (int g = 0; g < 2; ++g) {  // the two 32-dim blocks
#pragma unroll 2
        for (int i = 0; i < 8; ++i) {
            const int wi = g * 8 + i;
            const uint4 k0 = *reinterpret_cast<const uint4*>(sK + wi * kPsE + te * 4);
            const uint4 k1 = *reinterpret_cast<const uint4*>(sK + wi * kPsE + 64 + te * 4);
            const uint32_t kw[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
            uint32_t qw[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) qw[u] = sQ[(tq * 4 + u) * 16 + wi];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 8; ++v) acc[g][u][v] = __dp4a((int)qw[u], (int)kw[v], acc[g][u][v]);
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int ql = ql0 + tq * 4 + u;
        if (ql >= a.qb) continue;
        uint32_t kk[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const int e = (v < 4 ? te * 4 + v : 64 + te * 4 + v - 4);
            // block b scores A_b * 2^(cq_b - 127) * 2^(ck_b - 127) / 4
            kk[v] = mx_score_key(acc[0][u][v], sQe[tq * 4 + u][0] + (int)sKe[e][0] - 256, acc[1][u][v],
                                 sQe[tq * 4 + u][1] + (int)sKe[e][1] - 256);
        }
        uint32_t* row = a.keys + (size_t)ql * a.KS + e0;
        *reinterpret_cast<uint4*>(row + te * 4) = make_uint4(kk[0], kk[1], kk[2], kk[3]);
        *reinterpret_cast<uint4*>(row + 64 + te * 4) = make_uint4(kk[4], kk[5], kk[6], kk[7]);
    }
    SA_TRACE_MARK(TR_PSCORE_FP4, 2);
}

}  // namespace sa
