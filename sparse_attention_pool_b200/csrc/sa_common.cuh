// sa_common.cuh -- device helpers shared by the sm_100a kernels of
// libsparse_attn.so: number-format bit manipulation, the per-device status
// word, bounded mbarrier waits and TMA bulk-tensor copies.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sa {

// ---------------------------------------------------------------- status --
// Device-side anomalies are OR-ed into one word per device; the host reads and
// clears it with sa_read_device_status().  Kernels never trap.
enum : uint32_t {
    DEV_TIMEOUT = 1u,   // a bounded mbarrier / flag wait ran out
    DEV_LEN = 2u,       // a length or count outside its capacity (clamped)
    DEV_INDEX = 4u,     // an entry index outside 0..n-1 (skipped)
    DEV_POS = 8u,       // a query position outside its range (clamped)
};

__device__ uint32_t g_status = 0;  // one translation unit holds all device code

__device__ __forceinline__ void flag(uint32_t f) { atomicOr(&g_status, f); }

// --------------------------------------------------------------- tracing --
// Per-CTA phase marks for device timelines, compiled in only when the library
// is built with -DSA_TRACE (the default build has none).  Thread 0 of a CTA
// appends one 16-byte record -- the global nanosecond timer, the kernel, the
// phase, the SM and the CTA's linear index -- to a device buffer the host
// installs with sa_trace_install; marks past the buffer's capacity are
// counted and dropped.  Marks sit after a barrier where they stand for the
// whole CTA.
enum : uint32_t {
    TR_SCORE = 1, TR_FILTER = 2, TR_RESOLVE = 3, TR_EMIT = 4, TR_ATTN = 5, TR_COMBINE = 6, TR_SCORE_FP4 = 7,
    TR_PSCORE = 8, TR_PSELECT = 9, TR_PSCORE_FP4 = 10, TR_PSELECT2 = 11, TR_BOUND = 12, TR_FAST = 13, TR_PSELECT4 = 14,
    TR_PATTN = 15,
};
#ifdef SA_TRACE
struct TraceRec {
    unsigned long long t;
    uint16_t kernel, phase, sm, cta;
};
__device__ TraceRec* g_trace_buf = nullptr;
__device__ uint32_t g_trace_cap = 0;
__device__ uint32_t g_trace_n = 0;
// Marks stand at CTA-uniform points; the warp reconverges after thread 0's
// record, since a warp-wide ".aligned" instruction (a cluster barrier, a
// tensor-memory load) may follow.
__device__ __forceinline__ void trace_mark(uint32_t kernel, uint32_t phase) {
    if (threadIdx.x == 0 && g_trace_buf != nullptr) {
        unsigned long long t;
        uint32_t sm;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
        const uint32_t i = atomicAdd(&g_trace_n, 1u);
        if (i < g_trace_cap)
            g_trace_buf[i] = {t, (uint16_t)kernel, (uint16_t)phase, (uint16_t)sm,
                              (uint16_t)(blockIdx.x + gridDim.x * blockIdx.y)};
    }
    __syncwarp();
}
#define SA_TRACE_MARK(kernel, phase) ::sa::trace_mark((kernel), (phase))
// Marks inside a tight loop: the time is read into a register or shared
// memory (SA_TRACE_NOW) and the record is written later by one thread
// (SA_TRACE_PUT), with `unit` in the record's CTA field (a tile, say).
__device__ __forceinline__ unsigned long long trace_now() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void trace_put(unsigned long long t, uint32_t kernel, uint32_t phase, uint32_t unit) {
    if (g_trace_buf == nullptr) return;
    uint32_t sm;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
    const uint32_t i = atomicAdd(&g_trace_n, 1u);
    if (i < g_trace_cap) g_trace_buf[i] = {t, (uint16_t)kernel, (uint16_t)phase, (uint16_t)sm, (uint16_t)unit};
}
#define SA_TRACE_NOW() ::sa::trace_now()
#define SA_TRACE_PUT(t, kernel, phase, unit) ::sa::trace_put((t), (kernel), (phase), (unit))
#else
#define SA_TRACE_MARK(kernel, phase) ((void)0)
#define SA_TRACE_NOW() 0ull
#define SA_TRACE_PUT(t, kernel, phase, unit) ((void)0)
#endif

// Iteration limit of every spin on an mbarrier: each try_wait may itself
// suspend for a while, so this is far above any legitimate copy latency.
constexpr uint32_t kWaitLimit = 1u << 22;

// ---------------------------------------------------------- bf16 <-> fp64 --
// A bf16 pattern placed in the top bits of an fp64 pattern, with the exponent
// field left as is (no re-biasing), is the exact fp64 value  x * 2^-896: the
// bf16 exponent field e (bias 127) becomes an fp64 exponent field e (bias
// 1023), and bf16 subnormals land on fp64 subnormals of the same scaled value.
// Sums of such values are exact scalings of the unscaled sums (no rounding in
// the subnormal range is possible: every partial sum is a multiple of the
// scaled bf16 quantum 2^-1029).  This avoids 64-bit conversion instructions.
__device__ __forceinline__ double bf16lo_scaled(uint32_t w) {
    uint32_t hi = ((w << 16) & 0x80000000u) | ((w << 13) & 0x0FFFE000u);
    return __hiloint2double((int)hi, 0);
}
__device__ __forceinline__ double bf16hi_scaled(uint32_t w) {
    uint32_t hi = (w & 0x80000000u) | ((w >> 3) & 0x0FFFE000u);
    return __hiloint2double((int)hi, 0);
}

// Nearest-even bf16 of a scaled fp64 value x' = x * 2^-896 (|x| < 2^128 keeps
// the exponent field below 256, so the bf16 is simply the top bits rounded).
__device__ __forceinline__ uint16_t scaled_to_bf16_rne(double xs) {
    unsigned long long u = (unsigned long long)__double_as_longlong(xs);
    unsigned long long mag = u & 0x7FFFFFFFFFFFFFFFull;
    unsigned long long r = (mag + 0x00000FFFFFFFFFFFull + ((mag >> 45) & 1ull)) >> 45;
    if (r > 0x7F80ull) r = 0x7F80ull;  // (unreachable for finite bf16 inputs)
    return (uint16_t)(((u >> 48) & 0x8000ull) | r);
}

__device__ __forceinline__ float bf16lo_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Nearest-even bf16 of an fp32 value (finite inputs), two values packed.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// e4m3 (OCP "fn") -> fp32: every e4m3 value is exact in bf16 and fp32.
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
    uint32_t s = (c & 0x80u) << 24;
    uint32_t e = (c >> 3) & 0xFu;
    uint32_t f = c & 7u;
    float v;
    if (e == 0) v = (float)f * 0.001953125f;  // f * 2^-9, subnormal
    else v = __uint_as_float(((e + 120u) << 23) | (f << 20));
    return __uint_as_float(__float_as_uint(v) | s);
}

// Two fp32 values -> two e4m3 codes, nearest even, saturating to +-448.
// PTX places the first source operand in the upper byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return (uint32_t)r;
}

// Order-preserving 32-bit key of an fp32 score: larger score -> larger key.
// -0 is folded onto +0 first.
__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s);
    if ((u & 0x7FFFFFFFu) == 0) u = 0;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// --------------------------------------------------------------- mbarrier --
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Returns false (and records DEV_TIMEOUT) if the phase did not complete in time.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit = kWaitLimit) {
    uint32_t addr = smem_u32(bar);
    for (uint32_t it = 0; it < limit; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(addr), "r"(parity)
            : "memory");
        if (done) return true;
    }
    flag(DEV_TIMEOUT);
    return false;
}

// 2-D tiled TMA load of box {x .. x+bx-1} x {y .. y+by-1} into shared memory,
// completing on `bar`.  x is in elements of the innermost dimension and must
// be a multiple of 16 bytes' worth of elements (all call sites use x = 0).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
            "r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------------- cp.async ----
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Shared-memory atomics through explicit shared-space addresses (a generic
// pointer into shared memory would otherwise compile to a generic atomic).
__device__ __forceinline__ uint32_t atom_add_shared(uint32_t* p, uint32_t v) {
    uint32_t old;
    asm volatile("atom.shared.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(smem_u32(p)), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void red_add_shared(uint32_t* p, uint32_t v) {
    asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

// L2 loads kept where they are written: issued early, consumed later (the
// compiler may otherwise sink an ordinary load to its first use).
__device__ __forceinline__ uint32_t ld_cg_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint2 ld_cg_u32x2(const void* p) {
    uint2 v;
    asm volatile("ld.global.cg.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}
__device__ __forceinline__ uint4 ld_cg_u32x4(const void* p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while its predecessor on the stream is still
// running; pdl_wait() returns once that predecessor has completed and its
// writes are visible (for an ordinary launch it returns at once).  Every
// kernel calls it before it touches global memory another kernel may write
// or read, and before any early return, so completion stays transitive along
// a chain.  pdl_release() lets the next kernel on the stream begin launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------ block scans --
// Exclusive prefix sum over the block (blockDim.x multiple of 32, <= 1024).
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* sh32, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh32[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = lane < nw ? sh32[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(0xFFFFFFFFu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < nw) sh32[lane] = w;
    }
    __syncthreads();
    uint32_t base = warp ? sh32[warp - 1] : 0;
    if (total) *total = sh32[nw - 1];
    __syncthreads();
    return base + x - v;
}

}  // namespace sa
