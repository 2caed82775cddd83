// compress.cuh -- sequence-dimension KV compression (CSA m = 4, HCA m = 128).
//
// "DeepSeek-V4 ... Review", section 3-2 (2), component table: CSA turns every
// 4 tokens into one compressed entry, HCA every 128 tokens.  The entry is the
// mean of its aligned block: fp64 sum in ascending token order, times 1/m
// (m a power of two, so exact), rounded once to bf16 with ties to even.  FP8
// caches ("Mixed KV storage" row) then get one fp32 scale per 64 consecutive
// entries, scale = fp32(amax / 448), and codes e4m3_rne_satfinite(x / scale).
//
// Append (compress-when-ready): once more raw tokens are present, only the
// group holding the first new entry and the groups after it are computed;
// the result is bit-identical to compressing the whole sequence again.
//
// Mixed storage (MIXED): K keeps its rotary dims 64..127 in bf16 and stores
// dims 0..63 as e4m3, in one 192-byte row per entry (codes, then the bf16
// dims); the group scale of K covers dims 0..63 only.  V is stored as e4m3.
//
// One CTA compresses one group of 64 entries of one sequence for every tensor
// (k, v and optionally the indexer keys).  Each thread owns one 16-byte chunk
// (8 dims) of one entry and streams the m tokens of its block; the sums run in
// the scaled-fp64 representation of sa_common.cuh, which needs no conversion
// instructions.  The kernel is HBM-bound: every raw byte is read exactly once.
#pragma once
#include "sa_common.cuh"

namespace sa {

struct CompressArgs {
    const uint16_t* src[3];  // raw k, v, kidx: [B][Lcap][D]
    void* dst[3];            // cache k, v (bf16 or e4m3), kidx (bf16)
    float* scale[2];         // fp8 scales of k, v: [B][nG]
    int dims[3];             // D of each tensor
    int ntensors;            // 2 (HCA) or 3 (CSA)
    const int32_t* len;      // [B]
    int32_t* n_out;          // [B] (full compression only)
    const int32_t* n_from;   // [B] entries already in the cache (append), or NULL
    int Lcap, Ncap, nG, m, log2m, fp8;
};

constexpr int kCompThreads = 256;

__device__ __forceinline__ void acc8(double (&a)[8], const uint4 w) {
    a[0] += bf16lo_scaled(w.x);
    a[1] += bf16hi_scaled(w.x);
    a[2] += bf16lo_scaled(w.y);
    a[3] += bf16hi_scaled(w.y);
    a[4] += bf16lo_scaled(w.z);
    a[5] += bf16hi_scaled(w.z);
    a[6] += bf16lo_scaled(w.w);
    a[7] += bf16hi_scaled(w.w);
}

constexpr int kMixedRowBytes = 192;  // mixed K row: 64 e4m3 codes + 64 bf16 rotary dims
constexpr int kMixedFp8Chunks = 8;   // 16-byte bf16 chunks of K (8 dims each) stored as e4m3

template <bool MIXED>
__global__ void __launch_bounds__(kCompThreads) compress_kernel(CompressArgs a) {
    __shared__ __align__(16) uint16_t stage[64 * 128];  // bf16 entries of one fp8 group
    __shared__ float red[kCompThreads / 32];

    const int b = blockIdx.y;
    int len = a.len[b];
    if (len < 0 || len > a.Lcap) {
        if (blockIdx.x == 0 && threadIdx.x == 0) flag(DEV_LEN);
        len = len < 0 ? 0 : a.Lcap;
    }
    const int n = len >> a.log2m;
    int g = blockIdx.x;
    if (a.n_from) {
        // append: start at the group holding the first new entry; that group is
        // recomputed whole (an fp8 group's scale covers all its present entries;
        // bf16 entries recompute to the same bits)
        int n0 = a.n_from[b];
        n0 = n0 < 0 ? 0 : min(n0, n);
        g += n0 >> 6;
        if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0 && (g + 1) * 64 < n) flag(DEV_LEN);  // bound exceeded
    } else if (g == 0 && threadIdx.x == 0) {
        a.n_out[b] = n;
    }
    const int e0 = g * 64;
    if (e0 >= n) return;
    const int ne = min(64, n - e0);
    const double inv_m = 1.0 / (double)a.m;  // a power of two: exact

    for (int t = 0; t < a.ntensors; ++t) {
        const int D = a.dims[t];
        const int cpe = D / 8;  // 16-byte chunks per entry
        const bool to_fp8 = a.fp8 && t < 2;
        const bool mixed_k = MIXED && t == 0;  // rotary chunks c >= 8 stay bf16
        const uint4* src = reinterpret_cast<const uint4*>(a.src[t]) + (size_t)b * a.Lcap * cpe;
        float amax = 0.f;
        for (int task = threadIdx.x; task < ne * cpe; task += blockDim.x) {
            const int el = task / cpe, c = task - el * cpe;
            const int e = e0 + el;
            const uint4* p = src + (size_t)e * a.m * cpe + c;
            double acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.0;
            int tok = 0;
            for (; tok + 4 <= a.m; tok += 4) {  // ascending token order
                const uint4 w0 = __ldg(p + (size_t)(tok + 0) * cpe);
                const uint4 w1 = __ldg(p + (size_t)(tok + 1) * cpe);
                const uint4 w2 = __ldg(p + (size_t)(tok + 2) * cpe);
                const uint4 w3 = __ldg(p + (size_t)(tok + 3) * cpe);
                acc8(acc, w0);
                acc8(acc, w1);
                acc8(acc, w2);
                acc8(acc, w3);
            }
            for (; tok < a.m; ++tok) acc8(acc, __ldg(p + (size_t)tok * cpe));
            uint32_t r[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                r[i] = (uint32_t)scaled_to_bf16_rne(acc[2 * i] * inv_m) |
                       ((uint32_t)scaled_to_bf16_rne(acc[2 * i + 1] * inv_m) << 16);
            if (!to_fp8) {
                uint4* dst = reinterpret_cast<uint4*>(a.dst[t]) + ((size_t)b * a.Ncap + e) * cpe + c;
                *dst = make_uint4(r[0], r[1], r[2], r[3]);
            } else if (mixed_k && c >= kMixedFp8Chunks) {
                uint8_t* row = reinterpret_cast<uint8_t*>(a.dst[t]) + ((size_t)b * a.Ncap + e) * kMixedRowBytes;
                *reinterpret_cast<uint4*>(row + 64 + (c - kMixedFp8Chunks) * 16) = make_uint4(r[0], r[1], r[2], r[3]);
            } else {
                *reinterpret_cast<uint4*>(&stage[el * 128 + c * 8]) = make_uint4(r[0], r[1], r[2], r[3]);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    amax = fmaxf(amax, fmaxf(fabsf(bf16lo_f32(r[i])), fabsf(bf16hi_f32(r[i]))));
            }
        }
        if (to_fp8) {
            // group amax over the valid entries of this group
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
            if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
            __syncthreads();
            float gmax = 0.f;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) gmax = fmaxf(gmax, red[w]);
            const float s = (gmax == 0.f) ? 1.0f : __fdiv_rn(gmax, 448.0f);
            if (threadIdx.x == 0) a.scale[t][(size_t)b * a.nG + g] = s;
            const int qcpe = mixed_k ? kMixedFp8Chunks : cpe;  // chunks stored as e4m3
            for (int task = threadIdx.x; task < ne * qcpe; task += blockDim.x) {
                const int el = task / qcpe, c = task - el * qcpe;
                const uint4 w = *reinterpret_cast<const uint4*>(&stage[el * 128 + c * 8]);
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
                uint32_t codes[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t c01 = f32x2_to_e4m3x2(__fdiv_rn(bf16lo_f32(ws[2 * h]), s),
                                                         __fdiv_rn(bf16hi_f32(ws[2 * h]), s));
                    const uint32_t c23 = f32x2_to_e4m3x2(__fdiv_rn(bf16lo_f32(ws[2 * h + 1]), s),
                                                         __fdiv_rn(bf16hi_f32(ws[2 * h + 1]), s));
                    codes[h] = c01 | (c23 << 16);
                }
                const int rowBytes = mixed_k ? kMixedRowBytes : D;
                uint2* dst = reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(a.dst[t]) +
                                                      ((size_t)b * a.Ncap + e0 + el) * rowBytes + c * 8);
                *dst = make_uint2(codes[0], codes[1]);
            }
            __syncthreads();  // `stage` and `red` are reused by the next tensor
        }
    }
}

// After an append: the entry counts follow the raw lengths, up to the groups
// the append computed (`groups` from the one holding the old count).
__global__ void set_counts_kernel(const int32_t* len, int32_t* n, int B, int Lcap, int log2m, int groups) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    int l = len[b];
    l = l < 0 ? 0 : min(l, Lcap);
    const int full = l >> log2m;
    int n0 = n[b];
    n0 = n0 < 0 ? 0 : min(n0, full);
    n[b] = min(full, ((n0 >> 6) + groups) * 64);
}

}  // namespace sa
