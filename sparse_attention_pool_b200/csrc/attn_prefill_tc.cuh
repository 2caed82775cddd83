// attn_prefill_tc.cuh -- causal prefill attention of the CSA and HCA branches
// on the 5th-generation tensor cores (tcgen05 + tensor memory),
// "DeepSeek-V4 ... Review", section 3-2 (2) component table.
//
// One CTA takes two consecutive query positions of one sequence: its 128
// MMA rows are (query, head) pairs, 64 heads each, all sharing the single
// compressed KV head.  Entries stream through in tiles of 128:
//   * HCA (dense): a tile is 128 consecutive entries, shared by both
//     queries; a column is masked where it lies past the row's query's
//     visible count floor(t / m).
//   * CSA (gathered): a tile holds 64 entries of each query's top-k list
//     (rows 0-63 of the tile from query 0's list, 64-127 from query 1's);
//     a row sees only its own query's half (block-diagonal mask).  This
//     variant wastes half of every MMA and is not dispatched: the mma.sync
//     kernel is faster for the gathered lists; the dense one is used.
// Per tile: S = Q K^T (tcgen05.mma, M=128 N=128, fp32 in tensor memory),
// the softmax reads S with tcgen05.ld (one thread per row), writes P in
// bf16 to shared memory, then PV = P V (tcgen05.mma, V as an MN-major
// operand) lands in tensor memory and is folded into the row's output in
// registers with the online-softmax rescale.  Operands sit in shared memory
// in the 128-byte-swizzled canonical layout, loaded by cp.async (gathered
// rows need per-row addresses).  Completion of each MMA group is signalled
// through tcgen05.commit on an mbarrier; every wait is bounded.
#pragma once
#include "sa_common.cuh"

namespace sa {

constexpr int kTcThreads = 128;          // 4 warps: one TMEM lane quarter each
constexpr int kTcRows = 128;             // MMA M: 2 queries x 64 heads
constexpr int kTcTileN = 128;            // entries per tile (MMA N of QK^T, K of PV)
constexpr int kTcOpBytes = 128 * 256;    // one 128 x 128 bf16 operand: 32 KB
constexpr int kTcQ = 0;
constexpr int kTcK = kTcQ + kTcOpBytes;          // [2] stages
constexpr int kTcV = kTcK + 2 * kTcOpBytes;      // [2] stages
constexpr int kTcP = kTcV + 2 * kTcOpBytes;
constexpr int kTcBar = kTcP + kTcOpBytes;        // mbarriers + the TMEM address
constexpr int kTcSmem = kTcBar + 64 + 1024;      // + alignment slack
constexpr uint32_t kTcCols = 256;                // TMEM columns: S [0,128), PV [128,256)

// Byte offset of (row r, 16-byte chunk c) of a 128 x 128 bf16 operand in the
// canonical SW128 layout: two 64-element halves of 16 KB, 8-row atoms of
// 1 KB, chunk index XOR (row % 8).  The same bytes serve as a K-major
// operand (rows = M or N, chunks along K) and, for V, as an MN-major one
// (rows = K = entries, chunks along N = dims).
__device__ __forceinline__ uint32_t tc_off(int r, int c) {
    return (uint32_t)((c >> 3) * 16384 + (r >> 3) * 1024 + (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Shared-memory matrix descriptor: start, leading / stride byte offsets,
// version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: D f32, A and B bf16, A K-major, B
// K-major (b_mn = 0) or MN-major (b_mn = 1), M = 128, N = 128.
__device__ __forceinline__ uint32_t tc_idesc(uint32_t b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn << 16) | ((uint32_t)(kTcTileN >> 3) << 17) |
           ((uint32_t)(kTcRows >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0));
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane, without the wait
// (tc_wait_ld completes every load issued before it).
__device__ __forceinline__ void tc_ld32_nw(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

struct TcArgs {
    const uint16_t* q;   // [B][T][64][128]
    const uint16_t* K;   // [B][Ncap][128] bf16
    const uint16_t* V;
    const int32_t* n;    // [B]
    const int32_t* pos;  // [B][T] query positions
    const int32_t* idx;  // gather: [B][T][kmax]
    const int32_t* cnt;  // gather: [B][T]
    int T, Ncap, kmax, m;
    float scale_log2;
    uint16_t* out;       // [B][T][64][128]
    float* lse;          // [B][T][64] or NULL
};

template <bool GATHER>
__global__ void __launch_bounds__(kTcThreads, 1) attn_prefill_tc_kernel(TcArgs a) {
    extern __shared__ uint8_t tc_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bar_s = reinterpret_cast<uint64_t*>(sm + kTcBar);
    uint64_t* bar_o = bar_s + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_s + 2);
    pdl_wait();
    pdl_release();
    const int tid = threadIdx.x, warp = tid >> 5;
    const int b = blockIdx.y;
    const int t0 = blockIdx.x * 2;
    const uint32_t sQ = smem_u32(sm + kTcQ), sK = smem_u32(sm + kTcK), sV = smem_u32(sm + kTcV), sP = smem_u32(sm + kTcP);

    // tensor memory: one warp allocates, everyone reads the address
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTcCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        mbar_init(bar_s, 1);
        mbar_init(bar_o, 1);
        fence_barrier_init();
    }

    // the two queries: visible / listed counts
    int nb = a.n[b];
    if (nb < 0 || nb > a.Ncap) {
        if (tid == 0) flag(DEV_LEN);
        nb = nb < 0 ? 0 : a.Ncap;
    }
    int R[2];
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) {
        const int t = t0 + qq;
        int r = 0;
        if (t < a.T) {
            const size_t bq = (size_t)b * a.T + t;
            if (GATHER) {
                r = a.cnt[bq];
                if (r < 0 || r > a.kmax) {
                    if (tid == 0) flag(DEV_LEN);
                    r = r < 0 ? 0 : a.kmax;
                }
            } else {
                const int tp = a.pos[bq];
                r = tp < 0 ? 0 : min(nb, tp / a.m);
            }
        }
        R[qq] = r;
    }
    const int per_tile = GATHER ? kTcTileN / 2 : kTcTileN;  // list positions per tile and query
    const int rmax = max(R[0], R[1]);
    const int ntiles = (rmax + per_tile - 1) / per_tile;

    // Copies of 128-row operands: warp w takes rows 32w .. 32w + 31, two
    // rows per instruction (16 lanes a row, 512 contiguous bytes when the
    // rows are consecutive).
    const int lane = tid & 31, gchunk = lane & 15;
    // Q: row (qq * 64 + h), 16 chunks of 8 dims; rows of a missing second query are zero
#pragma unroll
    for (int p = 0; p < 16; ++p) {
        const int r = 32 * warp + 2 * p + (lane >> 4);
        const int qq = r >> 6, h = r & 63;
        const bool ok = t0 + qq < a.T;
        const uint16_t* src = a.q + (((size_t)b * a.T + (ok ? t0 + qq : t0)) * 64 + h) * 128 + gchunk * 8;
        cp_async16_zfill(sm + kTcQ + tc_off(r, gchunk), src, ok);
    }
    cp_async_commit();

    // one tile of K and V; thread tid knows the entry of tile row tid (a
    // gathered row's list entry is fetched one tile ahead by ld_idx, so the
    // copies of a tile never wait for it) and hands it to the lanes copying it
    auto ld_idx = [&](int i) -> int {
        if (!GATHER) return 0;
        const int qq = tid >> 6;
        const int p = i * per_tile + (tid & 63);
        return i < ntiles && t0 + qq < a.T && p < R[qq]
                   ? (int)ld_cg_u32(a.idx + ((size_t)b * a.T + t0 + qq) * a.kmax + p)
                   : 0;
    };
    auto load_tile = [&](int i, int stage, int jg) {
        int jo;  // tile row tid: its entry, or -1 (past the list, or out of range and flagged)
        if (GATHER) {
            const int qq = tid >> 6;
            const int p = i * per_tile + (tid & 63);
            bool ok = t0 + qq < a.T && p < R[qq];
            if (ok && (jg < 0 || jg >= nb)) {
                flag(DEV_INDEX);
                ok = false;
            }
            jo = ok ? jg : -1;
        } else {
            const int j = i * per_tile + tid;
            jo = j < rmax ? j : -1;
        }
        uint8_t* dk = sm + kTcK + stage * kTcOpBytes;
        uint8_t* dv = sm + kTcV + stage * kTcOpBytes;
#pragma unroll
        for (int p = 0; p < 16; ++p) {
            const int r = 32 * warp + 2 * p + (lane >> 4);
            const int j = __shfl_sync(0xFFFFFFFFu, jo, 2 * p + (lane >> 4));  // the lane of row r
            const bool ok = j >= 0;
            const size_t off = ((size_t)b * a.Ncap + (ok ? j : 0)) * 128 + gchunk * 8;
            cp_async16_zfill(dk + tc_off(r, gchunk), a.K + off, ok);
            cp_async16_zfill(dv + tc_off(r, gchunk), a.V + off, ok);
        }
    };
    const int j0 = ld_idx(0);
    int jn = ld_idx(1);  // tile 1's entry, consumed by the first iteration
    if (ntiles > 0) load_tile(0, 0, j0);
    cp_async_commit();
    __syncthreads();  // TMEM address and barrier init visible
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_s = tmem, t_pv = tmem + kTcTileN;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;  // this warp's TMEM lane quarter

    const int row = tid, qq = row >> 6;  // this thread's MMA row
    float o[128];
#pragma unroll
    for (int c = 0; c < 128; ++c) o[c] = 0.f;
    float mrow = -INFINITY, lrow = 0.f;
    const uint32_t id_qk = tc_idesc(0), id_pv = tc_idesc(1);
    uint32_t ph_s = 0, ph_o = 0;
    int pend_s = 0, pend_o = 0;  // (thread 0) commits not yet observed complete
    bool bad = false;

    for (int i = 0; i < ntiles; ++i) {
        const int stage = i & 1;
        if (i + 1 < ntiles) load_tile(i + 1, stage ^ 1, jn);
        jn = ld_idx(i + 2);
        cp_async_commit();
        cp_async_wait<1>();  // Q and tile i have landed (this thread's copies)
        fence_async_smem();  // ... and are visible to the tensor cores
        __syncthreads();
        // S = Q K^T over 8 k-steps of 16 dims
        if (tid == 0) {
            tc_fence_after();
            const uint32_t kb = sK + stage * kTcOpBytes;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                tc_mma(t_s, tc_desc(sQ + off, 16, 1024), tc_desc(kb + off, 16, 1024), id_qk, ks > 0);
            }
            tc_commit(bar_s);
            ++pend_s;
        }
        if (mbar_wait(bar_s, ph_s)) {
            ph_s ^= 1;
            if (tid == 0) --pend_s;
        } else {
            bad = true;
        }
        tc_fence_after();
        // softmax of this row: masked max, then P in bf16 into shared memory
        const int cbase = GATHER ? qq * 64 : 0;  // the row's columns
        const int ncol = GATHER ? 64 : 128;
        const int rvis = R[qq] - i * per_tile;  // columns of this tile the row may see
        // the row's columns come in halves of 64 (two TMEM loads, one wait);
        // a gathered row owns one half, whose scores stay in registers
        float mx = -INFINITY;
        uint32_t sv[2][32];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int cb = hh * 64;
            if (cb < cbase || cb >= cbase + ncol) continue;  // warp-uniform (rows of a warp share a query)
            tc_ld32_nw(t_s + lane_base + cb, sv[0]);
            tc_ld32_nw(t_s + lane_base + cb + 32, sv[1]);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 64; ++e)
                if (cb - cbase + e < rvis) mx = fmaxf(mx, __uint_as_float(sv[e >> 5][e & 31]) * a.scale_log2);
        }
        const float mnew = fmaxf(mrow, mx);
        const float alpha = mnew == -INFINITY ? 1.f : exp2f(mrow - mnew);
        float lsum = 0.f;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int cb = hh * 64;
            const bool mine = !(cb < cbase || cb >= cbase + ncol);
            if (mine && !GATHER) {  // the dense rows own both halves: reload this one
                tc_ld32_nw(t_s + lane_base + cb, sv[0]);
                tc_ld32_nw(t_s + lane_base + cb + 32, sv[1]);
                tc_wait_ld();
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {  // 8 chunks of 8 columns
                uint32_t pk[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const int e = u * 8 + w * 2;
                    float p0 = 0.f, p1 = 0.f;
                    if (mine && cb - cbase + e < rvis)
                        p0 = exp2f(__uint_as_float(sv[e >> 5][e & 31]) * a.scale_log2 - mnew);
                    if (mine && cb - cbase + e + 1 < rvis)
                        p1 = exp2f(__uint_as_float(sv[(e + 1) >> 5][(e + 1) & 31]) * a.scale_log2 - mnew);
                    lsum += p0 + p1;
                    pk[w] = pack_bf16x2(p0, p1);
                }
                *reinterpret_cast<uint4*>(sm + kTcP + tc_off(row, (cb >> 3) + u)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
        }
        mrow = mnew;
        lrow = lrow * alpha + lsum;
        tc_fence_before();
        fence_async_smem();
        __syncthreads();
        // PV = P V over 8 k-steps of 16 entries (V: MN-major, dims contiguous)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t vb = sV + stage * kTcOpBytes;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t aoff = (ks >> 2) * 16384 + (ks & 3) * 32;
                tc_mma(t_pv, tc_desc(sP + aoff, 16, 1024), tc_desc(vb + ks * 2048, 16384, 1024), id_pv, ks > 0);
            }
            tc_commit(bar_o);
            ++pend_o;
        }
        if (mbar_wait(bar_o, ph_o)) {
            ph_o ^= 1;
            if (tid == 0) --pend_o;
        } else {
            bad = true;
        }
        tc_fence_after();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            tc_ld32_nw(t_pv + lane_base + hh * 64, sv[0]);
            tc_ld32_nw(t_pv + lane_base + hh * 64 + 32, sv[1]);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 64; ++e) o[hh * 64 + e] = o[hh * 64 + e] * alpha + __uint_as_float(sv[e >> 5][e & 31]);
        }
        tc_fence_before();
        if (__syncthreads_or(bad)) break;  // a wait ran out (recorded); stop issuing
    }
    cp_async_wait<0>();

    // epilogue: this row's output and lse
    const int t = t0 + qq, h = row & 63;
    if (t < a.T) {
        const size_t bq = (size_t)b * a.T + t;
        const bool empty = !(lrow > 0.f);
        const float inv = empty ? 0.f : 1.f / lrow;
        uint16_t* op = a.out + (bq * 64 + h) * 128;
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
            uint4 w;
            w.x = pack_bf16x2(o[c] * inv, o[c + 1] * inv);
            w.y = pack_bf16x2(o[c + 2] * inv, o[c + 3] * inv);
            w.z = pack_bf16x2(o[c + 4] * inv, o[c + 5] * inv);
            w.w = pack_bf16x2(o[c + 6] * inv, o[c + 7] * inv);
            *reinterpret_cast<uint4*>(op + c) = w;
        }
        if (a.lse) a.lse[bq * 64 + h] = empty ? -INFINITY : (mrow + __log2f(lrow)) * 0.6931471805599453f;
    }
    // an MMA still in flight after a timeout is waited for (bounded) before
    // its tensor memory is released
    if (tid == 0) {
        if (pend_s > 0) mbar_wait(bar_s, ph_s);
        if (pend_o > 0) mbar_wait(bar_o, ph_o);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcCols));
    }
}

}  // namespace sa
