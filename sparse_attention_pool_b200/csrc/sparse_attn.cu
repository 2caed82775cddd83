// sparse_attn.cu -- the C ABI of libsparse_attn.so (declared in
// include/sparse_attn.h): argument checks, workspace layout and the launch
// sequence of every operation.  All device code lives in the *.cuh files
// included below, compiled as one translation unit for sm_100a.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <functional>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <utility>

#include "../../include/sparse_attn.h"
#include "attn.cuh"
#include "attn_prefill_tc.cuh"
#include "attn_prefill_tr.cuh"
#include "compress.cuh"
#include "cp_decode.cuh"
#include "decode_fast.cuh"
#include "lowp_index.cuh"
#include "sa_common.cuh"
#include "topk_decode.cuh"
#include "topk_prefill.cuh"
#include "topk_prefill_fast.cuh"

namespace {

thread_local char g_err[512] = "";
thread_local uint64_t g_launches = 0;
thread_local cudaEvent_t g_stage_ev[SA_NUM_STAGES][2] = {};
std::atomic<int> g_prefill_select{4};  // SA_OPT_PREFILL_SELECT
std::atomic<int> g_decode_fast{0};      // SA_OPT_DECODE_FAST
std::atomic<int> g_hca_prefill{0};      // SA_OPT_HCA_PREFILL

// Inside a stream capture the record must become a graph node of its own
// (an "external" record), so that replays re-record the event.
inline void stage_mark(int stage, int which, cudaStream_t st) {
    cudaEvent_t ev = g_stage_ev[stage][which];
    if (!ev) return;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(st, &cs);
    if (cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
    else
        cudaEventRecord(ev, st);
}

// Programmatic dependent launch joins the library's own consecutive kernels
// of one call (never a call's first kernel, whose predecessor may be any
// stream work), and is off while stage events are set: their record nodes
// sit between the kernels.
bool pdl_on() {
    for (const auto& e : g_stage_ev)
        if (e[0] || e[1]) return false;
    return true;
}

// Scheduling priority of the kernels launched through launch_k while set
// (0: none).  The CSA chain of a hybrid decode step runs at the device's
// highest priority, so that its latency-bound kernels take SMs ahead of the
// concurrent HCA branch's CTAs as those drain.
thread_local int g_launch_priority = 0;
struct PriorityScope {
    int old;
    explicit PriorityScope(int p) : old(g_launch_priority) { g_launch_priority = p; }
    ~PriorityScope() { g_launch_priority = old; }
};
int highest_priority() {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return 0;
    return greatest;
}

// cudaLaunchKernelEx with optional programmatic stream serialization, an
// optional cluster shape and the current launch priority.
template <typename... P, typename... A>
cudaError_t launch_k(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                     unsigned cluster_x, A&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[3];
    unsigned na = 0;
    if (g_launch_priority != 0) {
        attr[na].id = cudaLaunchAttributePriority;
        attr[na].val.priority = g_launch_priority;
        ++na;
    }
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (cluster_x > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = cluster_x;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

sa_status fail(sa_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

#define SA_CHECK(cond, ...)                                  \
    do {                                                     \
        if (!(cond)) return fail(SA_ERR_INVALID_ARG, __VA_ARGS__); \
    } while (0)

#define SA_LAUNCHED()                                                                          \
    do {                                                                                       \
        cudaError_t e_ = cudaGetLastError();                                                   \
        if (e_ != cudaSuccess) return fail(SA_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(e_)); \
        ++g_launches;                                                                          \
    } while (0)

#define SA_CUDA(call)                                                                              \
    do {                                                                                           \
        cudaError_t e_ = (call);                                                                   \
        if (e_ != cudaSuccess) return fail(SA_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
    } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
inline int cdiv(long long a, long long b) { return (int)((a + b - 1) / b); }

// Kernel attributes are set once per device: `done` holds one bit per device.
inline int cur_device() {
    int dev = 0;
    cudaGetDevice(&dev);
    return dev;
}
inline bool attr_done(const std::atomic<uint64_t>& done) {
    const int dev = cur_device();
    return dev >= 0 && dev < 64 && (done.load() >> dev & 1u);
}
inline void attr_set(std::atomic<uint64_t>& done) {
    const int dev = cur_device();
    if (dev >= 0 && dev < 64) done.fetch_or(uint64_t(1) << dev);
}

int num_sms() {
    static int sms[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (!sms[dev]) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        sms[dev] = v > 0 ? v : 148;
    }
    return sms[dev];
}

sa_status check_cache(const sa_cache* c, bool need_kidx, const char* what) {
    SA_CHECK(c != nullptr, "%s: cache descriptor is NULL", what);
    SA_CHECK(c->B >= 1 && c->B <= 65535, "%s: B=%d outside 1..65535", what, c->B);
    SA_CHECK(c->Ncap >= 0 && c->Ncap <= (1 << 24), "%s: Ncap=%d outside 0..2^24", what, c->Ncap);
    SA_CHECK(c->d == 128, "%s: head dim d=%d (only 128 is supported)", what, c->d);
    SA_CHECK(c->m >= 1 && c->m <= 1024 && (c->m & (c->m - 1)) == 0, "%s: m=%d is not a power of two in 1..1024",
             what, c->m);
    SA_CHECK(c->dtype == SA_BF16 || c->dtype == SA_FP8_E4M3 || c->dtype == SA_KV_MIXED, "%s: dtype=%d", what,
             c->dtype);
    SA_CHECK(c->k && c->v && c->n, "%s: k, v and n must be non-NULL", what);
    SA_CHECK(aligned16(c->k) && aligned16(c->v) && aligned16(c->n), "%s: k, v, n must be 16-byte aligned", what);
    if (c->dtype != SA_BF16) {
        SA_CHECK(c->k_scale && c->v_scale, "%s: fp8 cache needs k_scale and v_scale", what);
        SA_CHECK(aligned16(c->k_scale) && aligned16(c->v_scale), "%s: scales must be 16-byte aligned", what);
    }
    if (need_kidx) {
        SA_CHECK(c->kidx != nullptr, "%s: CSA cache needs indexer keys (kidx)", what);
        SA_CHECK(c->d_idx == 64, "%s: indexer dim d_idx=%d (only 64 is supported)", what, c->d_idx);
        SA_CHECK(aligned16(c->kidx), "%s: kidx must be 16-byte aligned", what);
    }
    return SA_OK;
}

inline int ilog2(int v) {
    int r = 0;
    while ((1 << r) < v) ++r;
    return r;
}

// --------------------------------------------------------------- TMA map --
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Indexer keys [B][Ncap][64] bf16 as a 3-D tensor map, box 64 x kScRows x 1, 128B swizzle.
sa_status make_ic_map(CUtensorMap* map, const void* kidx, int B, int Ncap) {
    auto enc = get_encode();
    if (!enc) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t dims[3] = {64, (cuuint64_t)Ncap, (cuuint64_t)B};
    cuuint64_t strides[2] = {128, (cuuint64_t)Ncap * 128};
    cuuint32_t box[3] = {64, (cuuint32_t)sa::kScRows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kidx), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return SA_OK;
}

// ------------------------------------------------------- workspace layout --
struct TopkDecodeWs {
    size_t hist, hist2, totals, zero_end, keys, emax, chunk_in, chunk_cnt, chunk_pos, cslot, cand_key, cand_idx, cmp_key,
        cmp_idx, amb_key, amb_idx, bitmap, idx, cnt, total;
    size_t fctrl = 0, fccount = 0, fchist = 0, fcand = 0;  // the fast hybrid path's control words, chunk
                                                          // counts, candidate histogram, candidates
    int maxchunks, fchunk, nfch, Wcap;
};

// Rows per filter / emit CTA: kFiltRows (2048), or a multiple of it once a sequence
// would need more than kSelMaxChunks filter chunks.
int filter_chunk(int Ncap) {
    const long long per = (long long)sa::kFiltRows * sa::kSelMaxChunks;
    const long long m = std::max<long long>(1, (Ncap + per - 1) / per);
    return (int)(m * sa::kFiltRows);
}

// Rows per score CTA: about three CTAs per SM over the whole batch, whole tiles.
int score_chunk(int B, int Ncap) {
    const long long target = (long long)num_sms() * 3;
    long long chunk = ((long long)B * Ncap + target - 1) / target;
    chunk = ((chunk + sa::kScRows - 1) / sa::kScRows) * sa::kScRows;
    return (int)std::max<long long>(chunk, sa::kScRows);
}

// Small per-call arrays first, so that the latency-bound selection kernels
// touch few pages: [reserved 256 B][histograms][second histograms][totals]
// (zeroed per call) [per-score-chunk max error][per-filter-chunk sure-ins,
// candidates, output positions][compact candidate slots][bitmap], then the
// large ones: [keys][further candidates key/idx][compact list key/idx]
// [band key/idx][idx][cnt].  `fast` adds the arrays of the fast hybrid
// decode path: per sequence its control words and per scan chunk its
// candidate count (small), and a (key, index) candidate row per entry.
TopkDecodeWs topk_decode_layout(int B, int Ncap, int k, bool own_idx, bool fast = false) {
    TopkDecodeWs w{};
    w.maxchunks = std::max(1, cdiv(Ncap, sa::kScRows));
    w.fchunk = filter_chunk(Ncap);
    w.nfch = std::max(1, cdiv(Ncap, w.fchunk));
    w.Wcap = ((Ncap + 31) / 32 + 1) & ~1;
    size_t o = 256;
    w.hist = o;
    o += (size_t)B * sa::kBins * 4;
    w.hist2 = o;
    o += (size_t)B * sa::kBins * 4;
    w.totals = o;
    o += (size_t)B * sa::kTotals * 4;
    w.zero_end = o;
    o = up256(o);
    if (fast) {
        w.fctrl = o;
        o += up256((size_t)B * sa::kCtl * 4);
        w.fccount = o;
        o += up256((size_t)B * w.maxchunks * 4);
        w.fchist = o;
        o += up256((size_t)B * sa::kCH * 4);
    }
    const size_t col = up256((size_t)B * Ncap * 4);
    const size_t per_fch = up256((size_t)B * w.nfch * 4);
    w.emax = o;
    o += up256((size_t)B * w.maxchunks * 4);
    w.chunk_in = o;
    o += per_fch;
    w.chunk_cnt = o;
    o += per_fch;
    w.chunk_pos = o;
    o += per_fch;
    w.cslot = o;
    o += up256((size_t)B * w.nfch * sa::kSlots * 8);
    w.bitmap = o;
    o += up256((size_t)B * w.Wcap * 4);
    w.keys = o;
    o += col;
    w.cand_key = o;
    o += col;
    w.cand_idx = o;
    o += col;
    w.cmp_key = o;
    o += col;
    w.cmp_idx = o;
    o += col;
    w.amb_key = o;
    o += col;
    w.amb_idx = o;
    o += col;
    w.idx = o;
    if (own_idx) o += up256((size_t)B * k * 4);
    w.cnt = o;
    if (own_idx) o += up256((size_t)B * 4);
    if (fast) {
        w.fcand = o;
        o += up256((size_t)B * Ncap * 8);
    }
    w.total = o;
    return w;
}

// Workspace of hybrid_attn_decode_swa: the hybrid step's, then the window
// attention's (partials for the most splits a decode list takes, so the size
// does not depend on the window), the window's output and lse, and the two
// branches' lse when the caller keeps none.
struct SwaDecodeWs {
    size_t hybrid, win_ws, win_out, win_lse, lse_c, lse_h, total;
};
SwaDecodeWs swa_decode_layout(int B, int H, int Ncap_csa, int Ncap_hca, int k);

// Split rule of the attention kernels: depends only on the list capacity, never
// on the batch, so a sequence's result does not depend on its batch-mates.
struct Split {
    int tps, splits;
};
Split attn_split(int rows_cap, bool prefill, bool gather = false) {
    const int tiles = cdiv(rows_cap > 0 ? rows_cap : 1, sa::kTileN);
    if (prefill) return {tiles, 1};
    (void)gather;  // both lists split the same way (measured: 32 one-tile splits and a merge kernel beat
                   // 8 four-tile splits merged in a cluster for a 2048-entry list)
    const int tps = cdiv(tiles, 32);  // at most 32 splits, merged by the combine kernel
    return {tps, cdiv(tiles, tps)};
}

size_t attn_partial_bytes(long long BQ, int splits, int H) {
    if (splits <= 1) return 0;
    return up256((size_t)BQ * splits * H * 128 * 4) + up256((size_t)BQ * splits * H * 4);
}

size_t hybrid_decode_bytes(int B, int H, int Ncap_csa, int Ncap_hca, int k) {
    TopkDecodeWs w = topk_decode_layout(B, Ncap_csa, k, true, true);
    Split sc = attn_split(k, false, true), sh = attn_split(Ncap_hca, false);
    return w.total + attn_partial_bytes(B, sc.splits, H) + attn_partial_bytes(B, sh.splits, H);
}

SwaDecodeWs swa_decode_layout(int B, int H, int Ncap_csa, int Ncap_hca, int k) {
    SwaDecodeWs w{};
    size_t o = up256(hybrid_decode_bytes(B, H, Ncap_csa, Ncap_hca, k));
    w.hybrid = o;
    w.win_ws = o;
    o += 256 + attn_partial_bytes(B, 32, H);  // decode lists take at most 32 splits
    o = up256(o);
    w.win_out = o;
    o += up256((size_t)B * H * 128 * 2);
    w.win_lse = o;
    o += up256((size_t)B * H * 4);
    w.lse_c = o;
    o += up256((size_t)B * H * 4);
    w.lse_h = o;
    o += up256((size_t)B * H * 4);
    w.total = o;
    return w;
}

// ------------------------------------------------------------ launchers ----
template <int NW, bool G, bool F, int ST, bool CL, int EG, bool MX = false>
sa_status launch_attn_t(const sa::AttnArgs& a, dim3 grid, cudaStream_t st, bool pdl) {
    using L = sa::AttnSmem<NW, G, F, ST, MX>;
    static std::atomic<uint64_t> init{0};
    if (!attr_done(init)) {
        SA_CUDA(cudaFuncSetAttribute(sa::attn_split_kernel<NW, G, F, ST, CL, EG, MX>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal));
        attr_set(init);
    }
    SA_CUDA(launch_k(sa::attn_split_kernel<NW, G, F, ST, CL, EG, MX>, grid, dim3(NW * EG * 32), L::kTotal, st, pdl,
                     CL ? (unsigned)sa::kAttnCluster : 1u, a));
    SA_LAUNCHED();
    return SA_OK;
}

// kv: 0 = bf16 cache, 1 = e4m3 K and V, 2 = mixed K (e4m3 + bf16 rotary dims) and e4m3 V.
template <int NW, int ST, bool CL, int EG>
sa_status launch_attn_nw(const sa::AttnArgs& a, bool gather, int kv, dim3 grid, cudaStream_t st, bool pdl) {
    if (gather) {
        if (kv == 2) return launch_attn_t<NW, true, true, ST, CL, EG, true>(a, grid, st, pdl);
        return kv == 1 ? launch_attn_t<NW, true, true, ST, CL, EG>(a, grid, st, pdl)
                       : launch_attn_t<NW, true, false, ST, CL, EG>(a, grid, st, pdl);
    }
    if (kv == 2) return launch_attn_t<NW, false, true, ST, CL, EG, true>(a, grid, st, pdl);
    return kv == 1 ? launch_attn_t<NW, false, true, ST, CL, EG>(a, grid, st, pdl)
                   : launch_attn_t<NW, false, false, ST, CL, EG>(a, grid, st, pdl);
}

// Splits of up to 4 tiles keep all of them in flight (4 or 5 stages);
// longer lists (prefill) stream through a 2-stage pipeline.  A query split
// exactly kAttnCluster ways merges inside a cluster.  Decode with up to 64
// heads splits every tile between two warp groups (8 warps), which halves
// the serial work per warp; prefill and more heads keep one group.
sa_status launch_attn(const sa::AttnArgs& a, bool gather, int kv, long long BQ, cudaStream_t st, bool pdl,
                      bool decode) {
    const bool cl = a.splits == sa::kAttnCluster && BQ <= 65535;
    if (BQ > 2147483647LL || a.splits > 65535) return fail(SA_ERR_INVALID_ARG, "too many queries or splits");
    const dim3 grid = cl ? dim3(a.splits, (unsigned)BQ) : dim3((unsigned)BQ, a.splits);
    const bool deep = a.tiles_per_split >= 2 && a.tiles_per_split <= 4;
    if (a.H <= 64 && decode) {
        // splits of 4 tiles keep all four in flight (5 stages)
        const bool d5 = a.tiles_per_split == 4;
        if (cl)
            return d5 ? launch_attn_nw<4, 5, true, 2>(a, gather, kv, grid, st, pdl)
                      : deep ? launch_attn_nw<4, 4, true, 2>(a, gather, kv, grid, st, pdl)
                             : launch_attn_nw<4, 2, true, 2>(a, gather, kv, grid, st, pdl);
        return d5 ? launch_attn_nw<4, 5, false, 2>(a, gather, kv, grid, st, pdl)
                  : deep ? launch_attn_nw<4, 4, false, 2>(a, gather, kv, grid, st, pdl)
                         : launch_attn_nw<4, 2, false, 2>(a, gather, kv, grid, st, pdl);
    }
    if (a.H <= 64) {  // prefill: long lists, one warp group measured faster
        if (cl)
            return deep ? launch_attn_nw<4, 4, true, 1>(a, gather, kv, grid, st, pdl)
                        : launch_attn_nw<4, 2, true, 1>(a, gather, kv, grid, st, pdl);
        return deep ? launch_attn_nw<4, 4, false, 1>(a, gather, kv, grid, st, pdl)
                    : launch_attn_nw<4, 2, false, 1>(a, gather, kv, grid, st, pdl);
    }
    if (cl)
        return deep ? launch_attn_nw<8, 4, true, 1>(a, gather, kv, grid, st, pdl)
                    : launch_attn_nw<8, 2, true, 1>(a, gather, kv, grid, st, pdl);
    return deep ? launch_attn_nw<8, 4, false, 1>(a, gather, kv, grid, st, pdl)
                : launch_attn_nw<8, 2, false, 1>(a, gather, kv, grid, st, pdl);
}

// Causal prefill with 64 heads over a bf16 cache: the tensor-memory kernel
// (two query positions per CTA, 128-row MMAs).
sa_status launch_prefill_tc(const sa::AttnArgs& aa, const sa_cache* c, bool gather, cudaStream_t st) {
    sa::TcArgs a{};
    a.q = aa.q;
    a.K = static_cast<const uint16_t*>(c->k);
    a.V = static_cast<const uint16_t*>(c->v);
    a.n = c->n;
    a.pos = aa.pos;
    a.idx = aa.idx;
    a.cnt = aa.cnt;
    a.T = aa.Tq;
    a.Ncap = c->Ncap;
    a.kmax = aa.kmax;
    a.m = c->m;
    a.scale_log2 = aa.scale_log2;
    a.out = aa.out;
    a.lse = aa.lse;
    static std::atomic<uint64_t> init{0};
    if (!attr_done(init)) {
        SA_CUDA(cudaFuncSetAttribute(sa::attn_prefill_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     sa::kTcSmem));
        SA_CUDA(cudaFuncSetAttribute(sa::attn_prefill_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     sa::kTcSmem));
        attr_set(init);
    }
    const dim3 grid((unsigned)((a.T + 1) / 2), (unsigned)c->B);
    if (grid.y > 65535) return fail(SA_ERR_INVALID_ARG, "too many sequences");
    if (gather)
        sa::attn_prefill_tc_kernel<true><<<grid, sa::kTcThreads, sa::kTcSmem, st>>>(a);
    else
        sa::attn_prefill_tc_kernel<false><<<grid, sa::kTcThreads, sa::kTcSmem, st>>>(a);
    SA_LAUNCHED();
    return SA_OK;
}

// Causal prefill with at most 64 heads over a bf16 cache on the transposed
// tensor-memory kernel, a persistent grid of one CTA per SM: the gathered
// lists (CSA) or every visible entry (HCA, needs the query positions).
sa_status launch_prefill_tr(const sa::AttnArgs& aa, const sa_cache* c, bool gather, long long BQ, cudaStream_t st) {
    sa::CtArgs a{};
    a.q = aa.q;
    a.K = static_cast<const uint16_t*>(c->k);
    a.V = static_cast<const uint16_t*>(c->v);
    a.n = c->n;
    a.idx = aa.idx;
    a.cnt = aa.cnt;
    a.pos = aa.pos;
    a.m = c->m;
    a.BQ = BQ;
    a.T = aa.Tq;
    a.H = aa.H;
    a.Ncap = c->Ncap;
    a.kmax = aa.kmax;
    a.scale_log2 = aa.scale_log2;
    a.out = aa.out;
    a.lse = aa.lse;
    static std::atomic<uint64_t> init{0};
    if (!attr_done(init)) {
        SA_CUDA(cudaFuncSetAttribute(sa::attn_prefill_tr_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     sa::kCtSmem));
        SA_CUDA(cudaFuncSetAttribute(sa::attn_prefill_tr_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     sa::kCtSmem));
        SA_CUDA(cudaFuncSetAttribute(sa::attn_prefill_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     sa::kPrSmem));
        attr_set(init);
    }
    if (!gather && aa.H == 64 && (c->m & 1) == 0 && g_hca_prefill.load() == 0) {
        // dense, 64 heads: two query positions per tile
        const long long pairs = (long long)c->B * ((aa.Tq + 1) / 2);
        const long long grid = std::min<long long>(pairs, (long long)num_sms());
        if (grid < 1) return SA_OK;
        sa::attn_prefill_pair_kernel<<<(unsigned)grid, sa::kPrThreads, sa::kPrSmem, st>>>(a);
        SA_LAUNCHED();
        return SA_OK;
    }
    const long long grid = std::min<long long>(BQ, (long long)num_sms());
    if (grid < 1) return SA_OK;
    if (gather)
        sa::attn_prefill_tr_kernel<true><<<(unsigned)grid, sa::kCtThreads, sa::kCtSmem, st>>>(a);
    else
        sa::attn_prefill_tr_kernel<false><<<(unsigned)grid, sa::kCtThreads, sa::kCtSmem, st>>>(a);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        cudaFuncAttributes fa{};
        cudaFuncGetAttributes(&fa, gather ? (const void*)sa::attn_prefill_tr_kernel<true>
                                          : (const void*)sa::attn_prefill_tr_kernel<false>);
        return fail(SA_ERR_CUDA, "kernel launch: %s (transposed prefill kernel: %d threads, %d registers, "
                    "%zu + %d bytes of shared memory; the kernel allows %d threads, %d bytes dynamic)",
                    cudaGetErrorString(e), sa::kCtThreads, fa.numRegs, fa.sharedSizeBytes, sa::kCtSmem,
                    fa.maxThreadsPerBlock, fa.maxDynamicSharedSizeBytes);
    }
    ++g_launches;
    return SA_OK;
}

// The merge follows its split kernel on the same stream: always chained.
sa_status launch_combine(const float* po, const float* pl, int splits, int H, long long BQ, uint16_t* out, float* lse,
                         cudaStream_t st) {
    if (BQ * H > 2147483647LL) return fail(SA_ERR_INVALID_ARG, "too many queries");
    SA_CUDA(launch_k(sa::attn_combine_kernel, dim3((unsigned)(BQ * H)), dim3(sa::kCombThreads), 0, st, pdl_on(), 1u,
                     po, pl, splits, H, out, lse));
    SA_LAUNCHED();
    return SA_OK;
}

// A side stream (per host thread and device) on which the HCA branch of a
// hybrid decode step runs concurrently with the CSA chain.  Created by the
// first hybrid call on a device, which should precede any stream capture.
struct SideStream {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
thread_local SideStream g_side[64];

sa_status side_stream(SideStream** out) {
    int dev = 0;
    SA_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return fail(SA_ERR_UNSUPPORTED, "device ordinal %d", dev);
    SideStream& ss = g_side[dev];
    if (!ss.s) {
        SA_CUDA(cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking));
        SA_CUDA(cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming));
        SA_CUDA(cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming));
    }
    *out = &ss;
    return SA_OK;
}

// Shared body of csa_sparse_attn / hca_dense_attn / the hybrid calls.
sa_status run_attn(const void* q, int Tq, int H, const sa_cache* c, bool gather, const int32_t* idx,
                   const int32_t* cnt, int kmax, const int32_t* pos, float scale, void* out, float* lse, void* ws,
                   size_t ws_off, cudaStream_t st, bool chained = false, int win = 0) {
    const long long BQ = (long long)c->B * Tq;
    const bool prefill = (Tq > 1) || (pos != nullptr);
    const Split sp = attn_split(gather ? kmax : (win > 0 ? std::min(win, c->Ncap) : c->Ncap), prefill, gather);
    sa::AttnArgs a{};
    a.q = static_cast<const uint16_t*>(q);
    a.K = c->k;
    a.V = c->v;
    a.ks = c->k_scale;
    a.vs = c->v_scale;
    a.n = c->n;
    a.idx = idx;
    a.cnt = cnt;
    a.pos = pos;
    a.Tq = Tq;
    a.H = H;
    a.Ncap = c->Ncap;
    a.nG = (c->Ncap + 63) / 64;
    a.kmax = kmax;
    a.m = c->m;
    a.win = win;
    const float s = scale == 0.f ? 1.0f / sqrtf(128.0f) : scale;
    a.scale_log2 = s * 1.4426950408889634f;
    a.tiles_per_split = sp.tps;
    a.splits = sp.splits;
    a.out = static_cast<uint16_t*>(out);
    a.lse = lse;
    if (sp.splits > 1) {
        uint8_t* base = static_cast<uint8_t*>(ws) + ws_off;
        a.part_o = reinterpret_cast<float*>(base);
        a.part_lse = reinterpret_cast<float*>(base + up256((size_t)BQ * sp.splits * H * 128 * 4));
    }
    // causal prefill on the tensor cores: the gathered lists (CSA) on the
    // transposed kernel; the dense branch (HCA) on it too, or, with
    // SA_OPT_HCA_PREFILL = 1, on the two-query kernel.  (The gathered variant
    // of the two-query kernel is not dispatched: its block-diagonal tiles,
    // two queries' lists in one 128-row MMA, waste half of every MMA.)
    if (prefill && !gather && win == 0 && c->dtype == SA_BF16 && pos) {
        if (g_hca_prefill.load() == 1 && H == 64) return launch_prefill_tc(a, c, false, st);
        if (H <= 64) return launch_prefill_tr(a, c, false, BQ, st);
    }
    if (prefill && gather && H <= 64 && c->dtype == SA_BF16) return launch_prefill_tr(a, c, true, BQ, st);
    const int kv = c->dtype == SA_KV_MIXED ? 2 : c->dtype == SA_FP8_E4M3 ? 1 : 0;
    sa_status r = launch_attn(a, gather, kv, BQ, st, chained && pdl_on(), !prefill);
    if (r != SA_OK) return r;
    // a query split kAttnCluster ways was merged inside its cluster
    if (sp.splits > 1 && !(sp.splits == sa::kAttnCluster && BQ <= 65535))
        return launch_combine(a.part_o, a.part_lse, sp.splits, H, BQ, a.out, lse, st);
    return SA_OK;
}

// Rows per FP4 score CTA: about four CTAs per SM over the whole batch, whole
// passes of the CTA.
int fp4_score_chunk(int B, int Ncap) {
    const long long target = (long long)num_sms() * 4;
    long long chunk = ((long long)B * Ncap + target - 1) / target;
    chunk = ((chunk + sa::kF4Rows - 1) / sa::kF4Rows) * sa::kF4Rows;
    return (int)std::max<long long>(chunk, sa::kF4Rows);
}

// The indexer + top-k of a decode step: the score kernel (the HBM stream),
// the filter, the resolve and the emit.  `between` runs after the filter is
// queued (the hybrid step forks its HCA branch there).  With MXFP4 keys
// (codes4 / scales4 non-NULL) the FP4 score kernel writes exact keys and the
// resolve runs its EXACT variant; the bf16 keys are then not read.
template <typename F>
sa_status run_topk_decode(const void* q_idx, const sa_cache* c, int k, int32_t* idx, int32_t* cnt, void* ws,
                          const TopkDecodeWs& w, cudaStream_t st, F&& between, const uint8_t* codes4 = nullptr,
                          const uint8_t* scales4 = nullptr) {
    const bool fp4 = codes4 != nullptr;
    const int B = c->B, Ncap = c->Ncap;
    uint8_t* base = static_cast<uint8_t*>(ws);
    sa::TopkDecodeArgs a{};
    a.q_idx = static_cast<const uint16_t*>(q_idx);
    a.kidx = static_cast<const uint16_t*>(c->kidx);
    a.n = c->n;
    a.keys = reinterpret_cast<uint32_t*>(base + w.keys);
    a.hist1 = reinterpret_cast<uint32_t*>(base + w.hist);
    a.hist2 = reinterpret_cast<uint32_t*>(base + w.hist2);
    a.emax_part = reinterpret_cast<float*>(base + w.emax);
    a.chunk_in = reinterpret_cast<uint32_t*>(base + w.chunk_in);
    a.chunk_cnt = reinterpret_cast<uint32_t*>(base + w.chunk_cnt);
    a.chunk_pos = reinterpret_cast<uint32_t*>(base + w.chunk_pos);
    a.cslot = reinterpret_cast<uint2*>(base + w.cslot);
    a.cand_key = reinterpret_cast<uint32_t*>(base + w.cand_key);
    a.cand_idx = reinterpret_cast<int32_t*>(base + w.cand_idx);
    a.cmp_key = reinterpret_cast<uint32_t*>(base + w.cmp_key);
    a.cmp_idx = reinterpret_cast<int32_t*>(base + w.cmp_idx);
    a.amb_key = reinterpret_cast<uint32_t*>(base + w.amb_key);
    a.amb_idx = reinterpret_cast<int32_t*>(base + w.amb_idx);
    a.totals = reinterpret_cast<uint32_t*>(base + w.totals);
    a.bitmap = reinterpret_cast<uint32_t*>(base + w.bitmap);
    a.idx = idx;
    a.cnt = cnt;
    a.Ncap = Ncap;
    a.Wcap = w.Wcap;
    a.k = k;
    a.chunk = fp4 ? fp4_score_chunk(B, Ncap) : score_chunk(B, Ncap);
    a.nchunks = Ncap > 0 ? cdiv(Ncap, a.chunk) : 1;
    a.fchunk = w.fchunk;
    a.nfch = w.nfch;
    if (a.nchunks > w.maxchunks || a.nfch > sa::kSelMaxChunks)
        return fail(SA_ERR_WORKSPACE, "internal: chunk count above the workspace bound");
    static std::atomic<uint64_t> init{0};
    const size_t smem = sa::kScStages * sa::kScTileBytes + sa::kScStages * 8 + 1024;
    if (!attr_done(init)) {
        SA_CUDA(cudaFuncSetAttribute(sa::score_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        SA_CUDA(cudaFuncSetAttribute(sa::topk_resolve_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     sa::kSelSmem));
        SA_CUDA(cudaFuncSetAttribute(sa::topk_resolve_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     sa::kSelSmem));
        attr_set(init);
    }
    if (Ncap > 0 && fp4) {
        SA_CUDA(cudaMemsetAsync(a.hist1, 0, w.zero_end - w.hist, st));
        stage_mark(SA_STAGE_INDEX_SCORE, 0, st);
        sa::score_decode_mxfp4_kernel<<<dim3(a.nchunks, B), sa::kF4Threads, 0, st>>>(a, codes4, scales4);
        SA_LAUNCHED();
        stage_mark(SA_STAGE_INDEX_SCORE, 1, st);
    } else if (Ncap > 0) {
        CUtensorMap map;
        sa_status r = make_ic_map(&map, c->kidx, B, Ncap);
        if (r != SA_OK) return r;
        SA_CUDA(cudaMemsetAsync(a.hist1, 0, w.zero_end - w.hist, st));
        stage_mark(SA_STAGE_INDEX_SCORE, 0, st);
        sa::score_decode_kernel<<<dim3(a.nchunks, B), sa::kScThreads, smem, st>>>(map, a);
        SA_LAUNCHED();
        stage_mark(SA_STAGE_INDEX_SCORE, 1, st);
    }
    stage_mark(SA_STAGE_TOPK_SELECT, 0, st);
    // a sequence with n <= k visible entries (every one, when Ncap is 0) is
    // answered by the filter's first CTA; the other kernels skip it
    const bool pdl = pdl_on();
    SA_CUDA(launch_k(sa::topk_filter_kernel, dim3(a.nfch, B), dim3(sa::kSelThreads), 0, st, pdl && Ncap > 0, 1u, a));
    SA_LAUNCHED();
    // `between` runs here: the many small filter CTAs have the SMs to
    // themselves, and what it queues overlaps the latency-bound rest
    sa_status r = between();
    if (r != SA_OK) return r;
    SA_CUDA(launch_k(fp4 ? sa::topk_resolve_kernel<true> : sa::topk_resolve_kernel<false>, dim3(B),
                     dim3(sa::kResThreads), sa::kSelSmem, st, pdl, 1u, a));
    SA_LAUNCHED();
    SA_CUDA(launch_k(sa::topk_emit_kernel, dim3(a.nfch, B), dim3(sa::kEmitThreads), 0, st, pdl, 1u, a));
    SA_LAUNCHED();
    stage_mark(SA_STAGE_TOPK_SELECT, 1, st);
    return SA_OK;
}

// ---------------------------------------------------- fast hybrid decode --
// Sample stride of the bound kernel: about 32 expected sample hits above the
// k-th largest score (k / 32), and at most kFbSamp sample rows.
int fast_stride(int Ncap, int k) { return std::max(1, std::max(k / 32, cdiv(Ncap, sa::kFbSamp))); }

// With few sequences the bound kernel runs beside the scan on SMs of its own
// (late candidates); the scan then has three CTAs on every other SM.
bool fast_late(int B) {
    (void)B;
    return false;
}
int fast_chunk(int B, int Ncap) {
    const long long target = 3LL * (fast_late(B) ? num_sms() - B * sa::kFbCluster : num_sms());
    long long chunk = ((long long)B * Ncap + target - 1) / target;
    chunk = ((chunk + sa::kScRows - 1) / sa::kScRows) * sa::kScRows;
    return (int)std::max<long long>(chunk, sa::kScRows);
}

// The fast selection serves bf16 indexer keys with k <= 2048 (twice k fits
// the selecting CTA's candidate list); other calls take the general kernels.
bool fast_decode_ok(const sa_cache* c, int H, int k) {
    (void)H;
    if (g_decode_fast.load() == sa::kFastOff || k > sa::kFastMaxK || c->Ncap < 1) return false;
    return cdiv(c->Ncap, fast_chunk(c->B, c->Ncap)) <= sa::kSelMaxChunks;
}

// The indexer + top-k of a hybrid decode step on the fast path: the bound
// kernel, the indexer scan with candidate output, and the selection kernel.
// `between` runs once the scan is queued (the HCA branch forks there).
template <typename F>
sa_status run_fast_topk(const void* q_idx, const sa_cache* c, int k, int32_t* idx, int32_t* cnt, void* ws,
                        const TopkDecodeWs& w, cudaStream_t st, F&& between) {
    const int B = c->B, Ncap = c->Ncap;
    uint8_t* base = static_cast<uint8_t*>(ws);
    sa::FastArgs a{};
    a.q_idx = static_cast<const uint16_t*>(q_idx);
    a.kidx = static_cast<const uint16_t*>(c->kidx);
    a.n = c->n;
    a.ctrl = reinterpret_cast<uint32_t*>(base + w.fctrl);
    a.chist = reinterpret_cast<uint32_t*>(base + w.fchist);
    a.ccount = reinterpret_cast<uint32_t*>(base + w.fccount);
    a.cand = reinterpret_cast<uint2*>(base + w.fcand);
    a.keys = reinterpret_cast<uint32_t*>(base + w.keys);
    a.amb_key = reinterpret_cast<uint32_t*>(base + w.amb_key);
    a.amb_idx = reinterpret_cast<int32_t*>(base + w.amb_idx);
    a.idx = idx;
    a.cnt = cnt;
    a.Ncap = Ncap;
    a.k = k;
    a.chunk = fast_chunk(B, Ncap);
    a.nchunks = cdiv(Ncap, a.chunk);
    a.sstride = fast_stride(Ncap, k);
    const bool late = fast_late(B);
    a.mode = g_decode_fast.load();
    if (a.nchunks > w.maxchunks || a.nchunks > sa::kSelMaxChunks)
        return fail(SA_ERR_WORKSPACE, "internal: chunk count above the workspace bound");
    const size_t smem = sa::kScStages * sa::kScTileBytes + sa::kScStages * 8 + 1024;
    static std::atomic<uint64_t> init{0};
    if (!attr_done(init)) {
        SA_CUDA(cudaFuncSetAttribute(sa::score_fast_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem));
        SA_CUDA(cudaFuncSetAttribute(sa::score_fast_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem));
        SA_CUDA(cudaFuncSetAttribute(sa::topk_bound_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     sa::kFbReserveSmem));
        SA_CUDA(cudaFuncSetAttribute(sa::csa_select_fast_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     sa::kFaSmem));
        SA_CUDA(cudaFuncSetAttribute(sa::topk_bound_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
        attr_set(init);
    }
    CUtensorMap map;
    sa_status r = make_ic_map(&map, c->kidx, B, Ncap);
    if (r != SA_OK) return r;
    const bool pdl = pdl_on();
    stage_mark(SA_STAGE_INDEX_SCORE, 0, st);
    // (the reserved shared memory is not used: it keeps the scan's CTAs off
    // the bound kernel's SMs while both run)
    SA_CUDA(launch_k(sa::topk_bound_kernel, dim3(sa::kFbCluster, B), dim3(sa::kFbThreads),
                     late ? (size_t)sa::kFbReserveSmem : 0, st, false, (unsigned)sa::kFbCluster, a));
    SA_LAUNCHED();
    SA_CUDA(launch_k(late ? sa::score_fast_kernel<true> : sa::score_fast_kernel<false>, dim3(a.nchunks, B),
                     dim3(sa::kScThreads), smem, st, pdl, 1u, map, a));
    SA_LAUNCHED();
    stage_mark(SA_STAGE_INDEX_SCORE, 1, st);
    r = between();
    if (r != SA_OK) return r;
    stage_mark(SA_STAGE_TOPK_SELECT, 0, st);
    SA_CUDA(launch_k(sa::csa_select_fast_kernel, dim3(B), dim3(sa::kFaThreads), sa::kFaSmem, st, pdl, 1u, a));
    SA_LAUNCHED();
    stage_mark(SA_STAGE_TOPK_SELECT, 1, st);
    return SA_OK;
}

sa_status check_ws(void* ws, size_t have, size_t need) {
    if (need == 0) return SA_OK;
    if (!ws) return fail(SA_ERR_WORKSPACE, "workspace is NULL but %zu bytes are needed", need);
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(SA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    if (have < need) return fail(SA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", have, need);
    return SA_OK;
}

// ---------------------------------------------------------------- prefill --
constexpr int kPrefillQB = 1024;  // queries per score block

inline int keys_stride(int Ncap) { return std::max(1, cdiv(Ncap, sa::kPsE)) * sa::kPsE; }

size_t prefill_pos_off() { return 256; }
size_t prefill_keys_off(int B, int T) { return 256 + up256((size_t)B * T * 4); }

size_t prefill_topk_bytes(int B, int T, int Ncap, int k) {
    (void)k;
    const int qb = std::min(T, kPrefillQB);
    return prefill_keys_off(B, T) + up256((size_t)qb * keys_stride(Ncap) * 4);
}

const int32_t* prefill_positions(void* ws, int B, int T, cudaStream_t st) {
    int32_t* pos = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + prefill_pos_off());
    const long long total = (long long)B * T;
    sa::fill_positions_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(pos, B, T);
    if (cudaGetLastError() != cudaSuccess) return nullptr;
    ++g_launches;
    return pos;
}

// With MXFP4 keys (codes4 / scales4 non-NULL) the FP4 score kernel writes the
// key block; the selection is the same.
sa_status run_topk_prefill(const void* q_idx, int Tq, const int32_t* pos, const sa_cache* c, int k, int32_t* idx,
                           int32_t* cnt, void* ws, cudaStream_t st, const uint8_t* codes4 = nullptr,
                           const uint8_t* scales4 = nullptr) {
    sa::TopkPrefillArgs a{};
    a.q_idx = static_cast<const uint16_t*>(q_idx);
    a.kidx = static_cast<const uint16_t*>(c->kidx);
    a.pos = pos;
    a.n = c->n;
    a.keys = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + prefill_keys_off(c->B, Tq));
    a.idx = idx;
    a.cnt = cnt;
    a.Tq = Tq;
    a.Ncap = c->Ncap;
    a.KS = keys_stride(c->Ncap);
    a.k = k;
    a.log2m = ilog2(c->m);
    static std::atomic<uint64_t> init{0};
    if (!attr_done(init)) {
        SA_CUDA(cudaFuncSetAttribute(sa::score_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     sa::kPsSmem));
        SA_CUDA(cudaFuncSetAttribute(sa::select_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     sa::kPselSmemKeys * 4));
        SA_CUDA(cudaFuncSetAttribute(sa::select_prefill_v2_kernel<sa::kPselThreads, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sa::kPsel2Smem));
        SA_CUDA(cudaFuncSetAttribute(sa::select_prefill_v4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)sa::kP4Smem));
        attr_set(init);
    }
    const int etiles = std::max(1, cdiv(c->Ncap, sa::kPsE));
    const int select_form = g_prefill_select.load();
    for (int b = 0; b < c->B; ++b) {
        for (int t0 = 0; t0 < Tq; t0 += kPrefillQB) {
            a.b = b;
            a.t0 = t0;
            a.qb = std::min(kPrefillQB, Tq - t0);
            if (c->Ncap > 0 && codes4) {
                sa::score_prefill_mxfp4_kernel<<<dim3(etiles, cdiv(a.qb, sa::kPsQ)), sa::kPsThreads, sa::kPf4Smem,
                                                 st>>>(a, codes4, scales4);
                SA_LAUNCHED();
            } else if (c->Ncap > 0) {
                sa::score_prefill_kernel<<<dim3(etiles, cdiv(a.qb, sa::kPsQ)), sa::kPsThreads, sa::kPsSmem, st>>>(a);
                SA_LAUNCHED();
            }
            if (select_form == 4)
                sa::select_prefill_v4_kernel<<<a.qb, sa::kP4Threads, sa::kP4Smem, st>>>(a);
            else if (select_form == 2)
                sa::select_prefill_v2_kernel<sa::kPselThreads, true><<<a.qb, sa::kPselThreads, sa::kPsel2Smem, st>>>(a);
            else if (select_form == 3)
                sa::select_prefill_v2_kernel<sa::kPsel3Threads, false>
                    <<<a.qb, sa::kPsel3Threads, sa::kPsel3Smem, st>>>(a);
            else
                sa::select_prefill_kernel<<<a.qb, sa::kPselThreads, sa::kPselSmemKeys * 4, st>>>(a);
            SA_LAUNCHED();
        }
    }
    return SA_OK;
}

// ------------------------------------------------------- static scratch --
// The scratch of csa_index_topk_noalloc: a device array owned by the library,
// resident on every GPU that loads it.  In host code the name is only a
// stand-in for the symbol; kernels get its device address, looked up once per
// device with that device current.
static __device__ __align__(256) uint8_t g_noalloc_scratch[SA_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

sa_status noalloc_scratch(void** out) {
    int dev = 0;
    SA_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return fail(SA_ERR_UNSUPPORTED, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p)
            return fail(SA_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(e));
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return SA_OK;
}

}  // namespace

namespace sa {
// Failure-detection self-test: one CTA waits on an mbarrier that nothing
// arrives at.  The bounded wait gives up after `limit` tries, records
// DEV_TIMEOUT in the status word and returns; no copy is in flight, so the
// CTA exits cleanly and the context stays usable.
__global__ void selftest_wait_kernel(uint32_t limit) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, limit);
}
}  // namespace sa

namespace sa {
// Copies n 16-byte words from a pinned host buffer (read through its device
// mapping, fetched again every time: no stale cached line of it is used).
__global__ void __launch_bounds__(256) copy_in_kernel(const uint4* src, uint4* __restrict__ dst, uint32_t n) {
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) dst[i] = __ldcv(src + i);
}
}  // namespace sa

// =========================================================== public ABI ====
extern "C" {

int32_t sa_abi_version(void) { return SA_ABI_VERSION; }

uint64_t sa_launch_count(void) { return g_launches; }

sa_status sa_set_option(int32_t option, int64_t value) {
    switch (option) {
        case SA_OPT_PREFILL_SELECT:
            SA_CHECK(value >= 1 && value <= 4, "sa_set_option: SA_OPT_PREFILL_SELECT=%lld (1 to 4)",
                     (long long)value);
            g_prefill_select.store((int)value);
            return SA_OK;
        case SA_OPT_DECODE_FAST:
            SA_CHECK(value >= 0 && value <= 2, "sa_set_option: SA_OPT_DECODE_FAST=%lld (0, 1 or 2)", (long long)value);
            g_decode_fast.store((int)value);
            return SA_OK;
        case SA_OPT_HCA_PREFILL:
            SA_CHECK(value >= 0 && value <= 2, "sa_set_option: SA_OPT_HCA_PREFILL=%lld (0, 1 or 2)", (long long)value);
            g_hca_prefill.store((int)value);
            return SA_OK;
        default:
            return fail(SA_ERR_INVALID_ARG, "sa_set_option: unknown option %d", option);
    }
}

sa_status sa_get_option(int32_t option, int64_t* value) {
    SA_CHECK(value != nullptr, "sa_get_option: value is NULL");
    switch (option) {
        case SA_OPT_PREFILL_SELECT:
            *value = g_prefill_select.load();
            return SA_OK;
        case SA_OPT_DECODE_FAST:
            *value = g_decode_fast.load();
            return SA_OK;
        case SA_OPT_HCA_PREFILL:
            *value = g_hca_prefill.load();
            return SA_OK;
        default:
            return fail(SA_ERR_INVALID_ARG, "sa_get_option: unknown option %d", option);
    }
}

sa_status sa_set_stage_events(int32_t stage, void* before, void* after) {
    SA_CHECK(stage >= 0 && stage < SA_NUM_STAGES, "sa_set_stage_events: stage=%d", stage);
    SA_CHECK((before == nullptr) == (after == nullptr), "sa_set_stage_events: give both events or neither");
    g_stage_ev[stage][0] = static_cast<cudaEvent_t>(before);
    g_stage_ev[stage][1] = static_cast<cudaEvent_t>(after);
    return SA_OK;
}

const char* sa_last_error(void) { return g_err; }

sa_status sa_trace_install(void* buf, uint32_t capacity, void* stream) {
#ifdef SA_TRACE
    SA_CHECK(capacity == 0 || (buf != nullptr && aligned16(buf)),
             "sa_trace_install: buf must be non-NULL and 16-byte aligned when capacity > 0");
    SA_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    sa::TraceRec* p = capacity ? static_cast<sa::TraceRec*>(buf) : nullptr;
    const uint32_t zero = 0;
    SA_CUDA(cudaMemcpyToSymbol(sa::g_trace_buf, &p, sizeof(p)));
    SA_CUDA(cudaMemcpyToSymbol(sa::g_trace_cap, &capacity, sizeof(capacity)));
    SA_CUDA(cudaMemcpyToSymbol(sa::g_trace_n, &zero, sizeof(zero)));
    return SA_OK;
#else
    (void)buf;
    (void)capacity;
    (void)stream;
    return fail(SA_ERR_UNSUPPORTED, "sa_trace_install: this library was built without SA_TRACE");
#endif
}

sa_status sa_trace_count(uint32_t* n, void* stream) {
    SA_CHECK(n != nullptr, "sa_trace_count: n is NULL");
#ifdef SA_TRACE
    SA_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    SA_CUDA(cudaMemcpyFromSymbol(n, sa::g_trace_n, sizeof(*n)));
    return SA_OK;
#else
    (void)stream;
    *n = 0;
    return fail(SA_ERR_UNSUPPORTED, "sa_trace_count: this library was built without SA_TRACE");
#endif
}

sa_status sa_selftest_wait_timeout(uint32_t wait_tries, void* stream) {
    SA_CHECK(wait_tries >= 1 && wait_tries <= sa::kWaitLimit, "sa_selftest_wait_timeout: wait_tries=%u outside 1..%u",
             wait_tries, sa::kWaitLimit);
    sa::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(wait_tries);
    SA_LAUNCHED();
    return SA_OK;
}

static sa_status check_common_q(const void* q, int H, const char* what);

static sa_status compress_common(const sa_raw* raw, const sa_cache* out, void* stream, bool csa,
                                 int32_t max_new_tokens = -1) {
    const bool append = max_new_tokens >= 0;
    const char* what = append ? (csa ? "csa_append" : "hca_append") : (csa ? "csa_compress" : "hca_compress");
    SA_CHECK(raw != nullptr, "%s: raw descriptor is NULL", what);
    sa_status r = check_cache(out, csa, what);
    if (r != SA_OK) return r;
    SA_CHECK(raw->B == out->B, "%s: raw B=%d but cache B=%d", what, raw->B, out->B);
    SA_CHECK(raw->d == 128, "%s: raw d=%d (only 128)", what, raw->d);
    SA_CHECK(raw->Lcap >= 0, "%s: Lcap=%d", what, raw->Lcap);
    SA_CHECK(raw->k && raw->v && raw->len, "%s: raw k, v, len must be non-NULL", what);
    SA_CHECK(aligned16(raw->k) && aligned16(raw->v) && aligned16(raw->len), "%s: raw pointers must be 16-byte aligned",
             what);
    SA_CHECK((long long)out->Ncap >= (long long)raw->Lcap / out->m, "%s: Ncap=%d < Lcap/m=%d", what, out->Ncap,
             raw->Lcap / out->m);
    if (csa) {
        SA_CHECK(raw->kidx != nullptr && aligned16(raw->kidx), "%s: raw kidx must be non-NULL and aligned", what);
        SA_CHECK(raw->d_idx == 64, "%s: raw d_idx=%d (only 64)", what, raw->d_idx);
    }
    sa::CompressArgs a{};
    a.src[0] = static_cast<const uint16_t*>(raw->k);
    a.src[1] = static_cast<const uint16_t*>(raw->v);
    a.src[2] = csa ? static_cast<const uint16_t*>(raw->kidx) : nullptr;
    a.dst[0] = out->k;
    a.dst[1] = out->v;
    a.dst[2] = csa ? out->kidx : nullptr;
    a.scale[0] = out->k_scale;
    a.scale[1] = out->v_scale;
    a.dims[0] = 128;
    a.dims[1] = 128;
    a.dims[2] = 64;
    a.ntensors = csa ? 3 : 2;
    a.len = raw->len;
    a.n_out = out->n;
    a.Lcap = raw->Lcap;
    a.Ncap = out->Ncap;
    a.nG = (out->Ncap + 63) / 64;
    a.m = out->m;
    a.log2m = ilog2(out->m);
    a.fp8 = out->dtype != SA_BF16;  // e4m3 K and V, or mixed K + e4m3 V
    const bool mixed = out->dtype == SA_KV_MIXED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!append) {
        const int groups = std::max(1, cdiv(raw->Lcap / out->m, 64));
        if (mixed)
            sa::compress_kernel<true><<<dim3(groups, raw->B), sa::kCompThreads, 0, st>>>(a);
        else
            sa::compress_kernel<false><<<dim3(groups, raw->B), sa::kCompThreads, 0, st>>>(a);
        SA_LAUNCHED();
        return SA_OK;
    }
    // new entries: at most (max_new_tokens + m - 1) / m (a partial block may
    // complete); groups: those, plus the partly filled group they join
    a.n_from = out->n;
    const long long new_entries = ((long long)max_new_tokens + out->m - 1) / out->m;
    const long long groups = std::min<long long>((new_entries + 63) / 64 + 1, cdiv(out->Ncap, 64) + 1LL);
    if (mixed)
        sa::compress_kernel<true><<<dim3((unsigned)groups, raw->B), sa::kCompThreads, 0, st>>>(a);
    else
        sa::compress_kernel<false><<<dim3((unsigned)groups, raw->B), sa::kCompThreads, 0, st>>>(a);
    SA_LAUNCHED();
    sa::set_counts_kernel<<<cdiv(raw->B, 128), 128, 0, st>>>(raw->len, out->n, raw->B, raw->Lcap, a.log2m,
                                                               (int)groups);
    SA_LAUNCHED();
    return SA_OK;
}

sa_status csa_compress(const sa_raw* raw, const sa_cache* out, void* stream) {
    return compress_common(raw, out, stream, true);
}

sa_status hca_compress(const sa_raw* raw, const sa_cache* out, void* stream) {
    return compress_common(raw, out, stream, false);
}

sa_status csa_append(const sa_raw* raw, const sa_cache* cache, int32_t max_new_tokens, void* stream) {
    SA_CHECK(max_new_tokens >= 0, "csa_append: max_new_tokens=%d", max_new_tokens);
    return compress_common(raw, cache, stream, true, max_new_tokens);
}

sa_status hca_append(const sa_raw* raw, const sa_cache* cache, int32_t max_new_tokens, void* stream) {
    SA_CHECK(max_new_tokens >= 0, "hca_append: max_new_tokens=%d", max_new_tokens);
    return compress_common(raw, cache, stream, false, max_new_tokens);
}

sa_status swa_attn(const void* q, int32_t Tq, int32_t H, const int32_t* q_pos, const sa_raw* raw, int32_t window,
                   float scale, void* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
    SA_CHECK(raw != nullptr, "swa_attn: raw descriptor is NULL");
    sa_status r = check_common_q(q, H, "swa_attn");
    if (r != SA_OK) return r;
    SA_CHECK(raw->B >= 1 && raw->Lcap >= 0 && raw->d == 128, "swa_attn: raw B=%d Lcap=%d d=%d", raw->B, raw->Lcap,
             raw->d);
    SA_CHECK(raw->k && raw->v && raw->len && aligned16(raw->k) && aligned16(raw->v) && aligned16(raw->len),
             "swa_attn: raw k, v, len must be non-NULL and 16-byte aligned");
    SA_CHECK(window >= 1, "swa_attn: window=%d", window);
    SA_CHECK(Tq >= 1, "swa_attn: Tq=%d", Tq);
    SA_CHECK(q_pos != nullptr || Tq == 1, "swa_attn: decode (q_pos == NULL) needs Tq == 1");
    SA_CHECK(!q_pos || aligned16(q_pos), "swa_attn: q_pos must be 16-byte aligned");
    SA_CHECK(out && aligned16(out), "swa_attn: out must be non-NULL and 16-byte aligned");
    SA_CHECK(!lse || aligned16(lse), "swa_attn: lse must be 16-byte aligned");
    SA_CHECK(std::isfinite(scale) && scale >= 0.f, "swa_attn: scale must be finite and >= 0");
    r = check_ws(ws, ws_bytes, sa_workspace_size(SA_OP_WINDOW_ATTN, raw->B, Tq, H, 0, 0, window));
    if (r != SA_OK) return r;
    // the raw tokens as a cache of single-token entries (m = 1): entry t is token t
    sa_cache view{};
    view.k = const_cast<void*>(raw->k);
    view.v = const_cast<void*>(raw->v);
    view.n = const_cast<int32_t*>(raw->len);
    view.B = raw->B;
    view.Ncap = raw->Lcap;
    view.d = 128;
    view.d_idx = 64;
    view.m = 1;
    view.dtype = SA_BF16;
    return run_attn(q, Tq, H, &view, false, nullptr, nullptr, 0, q_pos, scale, out, lse, ws, 256,
                    static_cast<cudaStream_t>(stream), false, window);
}

sa_status attn_lse_merge(const void* out_a, const float* lse_a, const void* out_b, const float* lse_b, int64_t rows,
                         void* out, float* lse, void* stream) {
    SA_CHECK(rows >= 0, "attn_lse_merge: rows=%lld", (long long)rows);
    SA_CHECK(out_a && out_b && lse_a && lse_b && out, "attn_lse_merge: inputs and out must be non-NULL");
    SA_CHECK(aligned16(out_a) && aligned16(out_b) && aligned16(out) && aligned16(lse_a) && aligned16(lse_b) &&
                 (!lse || aligned16(lse)),
             "attn_lse_merge: pointers must be 16-byte aligned");
    if (rows == 0) return SA_OK;
    const long long blocks = (rows + 7) / 8;
    SA_CHECK(blocks <= 2147483647LL, "attn_lse_merge: too many rows");
    sa::attn_lse_merge_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint16_t*>(out_a), lse_a, static_cast<const uint16_t*>(out_b), lse_b,
        static_cast<uint16_t*>(out), lse, rows);
    SA_LAUNCHED();
    return SA_OK;
}

size_t sa_workspace_size(int32_t op, int32_t B, int32_t Tq, int32_t H, int32_t Ncap_csa, int32_t Ncap_hca,
                         int32_t k) {
    if (B < 1 || Tq < 1 || H < 1 || H > 128 || Ncap_csa < 0 || Ncap_hca < 0 || k < 0) return 0;
    const long long BQ = (long long)B * Tq;
    const bool prefill = Tq > 1;
    switch (op) {
        case SA_OP_INDEX_TOPK:
            if (k < 1) return 0;
            if (prefill) return prefill_topk_bytes(B, Tq, Ncap_csa, k);
            return topk_decode_layout(B, Ncap_csa, k, false).total;
        case SA_OP_SPARSE_ATTN: {
            if (k < 1) return 0;
            Split s = attn_split(k, prefill, true);
            return 256 + attn_partial_bytes(BQ, s.splits, H);
        }
        case SA_OP_DENSE_ATTN: {
            Split s = attn_split(Ncap_hca, prefill);
            return 256 + attn_partial_bytes(BQ, s.splits, H);
        }
        case SA_OP_HYBRID_DECODE: {
            if (k < 1 || Tq != 1) return 0;
            return hybrid_decode_bytes(B, H, Ncap_csa, Ncap_hca, k);
        }
        case SA_OP_HYBRID_PREFILL:
            if (k < 1) return 0;
            return prefill_topk_bytes(B, Tq, Ncap_csa, k);
        case SA_OP_WINDOW_ATTN: {  // k = the window
            if (k < 1) return 0;
            Split s = attn_split(k, prefill);
            return 256 + attn_partial_bytes(BQ, s.splits, H);
        }
        case SA_OP_CP_CANDIDATES:
            if (k < 1 || Tq != 1) return 0;
            return topk_decode_layout(B, Ncap_csa, k, true).total;
        case SA_OP_HYBRID_DECODE_SWA:
            if (k < 1 || Tq != 1) return 0;
            return swa_decode_layout(B, H, Ncap_csa, Ncap_hca, k).total;
        default:
            return 0;
    }
}

sa_status sa_read_device_status(void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    SA_CUDA(cudaStreamSynchronize(st));
    uint32_t v = 0, zero = 0;
    SA_CUDA(cudaMemcpyFromSymbol(&v, sa::g_status, sizeof(v)));
    SA_CUDA(cudaMemcpyToSymbol(sa::g_status, &zero, sizeof(zero)));
    if (v & sa::DEV_TIMEOUT) return fail(SA_ERR_TIMEOUT, "device status 0x%x: a bounded wait ran out", v);
    if (v) return fail(SA_ERR_DEVICE, "device status 0x%x (2: length/count out of range, 4: bad index, 8: bad position)", v);
    return SA_OK;
}

static sa_status check_common_q(const void* q, int H, const char* what) {
    SA_CHECK(q != nullptr && aligned16(q), "%s: q must be non-NULL and 16-byte aligned", what);
    SA_CHECK(H >= 1 && H <= 128, "%s: H=%d outside 1..128", what, H);
    return SA_OK;
}

sa_status csa_index_topk(const void* q_idx, int32_t Tq, const int32_t* q_pos, const sa_cache* csa, int32_t k,
                         int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes, void* stream) {
    sa_status r = check_cache(csa, true, "csa_index_topk");
    if (r != SA_OK) return r;
    SA_CHECK(q_idx && aligned16(q_idx), "csa_index_topk: q_idx must be non-NULL and 16-byte aligned");
    SA_CHECK(idx && cnt && aligned16(idx) && aligned16(cnt), "csa_index_topk: idx/cnt must be non-NULL and aligned");
    SA_CHECK(k >= 1 && k <= 65536, "csa_index_topk: k=%d outside 1..65536", k);
    SA_CHECK(Tq >= 1, "csa_index_topk: Tq=%d", Tq);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (q_pos == nullptr) {
        SA_CHECK(Tq == 1, "csa_index_topk: decode (q_pos == NULL) needs Tq == 1, got %d", Tq);
        TopkDecodeWs w = topk_decode_layout(csa->B, csa->Ncap, k, false);
        r = check_ws(ws, ws_bytes, w.total);
        if (r != SA_OK) return r;
        return run_topk_decode(q_idx, csa, k, idx, cnt, ws, w, st, [] { return SA_OK; });
    }
    SA_CHECK(aligned16(q_pos), "csa_index_topk: q_pos must be 16-byte aligned");
    r = check_ws(ws, ws_bytes, prefill_topk_bytes(csa->B, Tq, csa->Ncap, k));
    if (r != SA_OK) return r;
    return run_topk_prefill(q_idx, Tq, q_pos, csa, k, idx, cnt, ws, st);
}

sa_status csa_index_topk_noalloc(const void* q_idx, const sa_cache* csa, int32_t k, int32_t* idx, int32_t* cnt,
                                 void* stream) {
    sa_status r = check_cache(csa, true, "csa_index_topk_noalloc");
    if (r != SA_OK) return r;
    SA_CHECK(q_idx && aligned16(q_idx), "csa_index_topk_noalloc: q_idx must be non-NULL and 16-byte aligned");
    SA_CHECK(idx && cnt && aligned16(idx) && aligned16(cnt),
             "csa_index_topk_noalloc: idx/cnt must be non-NULL and aligned");
    SA_CHECK(k >= 1 && k <= 65536, "csa_index_topk_noalloc: k=%d outside 1..65536", k);
    const TopkDecodeWs w = topk_decode_layout(csa->B, csa->Ncap, k, false);
    if (w.total > (size_t)SA_NOALLOC_SCRATCH_BYTES)
        return fail(SA_ERR_UNSUPPORTED,
                    "csa_index_topk_noalloc: B=%d, Ncap=%d, k=%d need %zu bytes of scratch; the static scratch "
                    "holds %u (use csa_index_topk with a workspace)",
                    csa->B, csa->Ncap, k, w.total, (unsigned)SA_NOALLOC_SCRATCH_BYTES);
    void* scratch = nullptr;
    r = noalloc_scratch(&scratch);
    if (r != SA_OK) return r;
    return run_topk_decode(q_idx, csa, k, idx, cnt, scratch, w, static_cast<cudaStream_t>(stream),
                           [] { return SA_OK; });
}

sa_status csa_index_quantize_mxfp4(const sa_cache* csa, int32_t row_from, uint8_t* codes, uint8_t* scales,
                                   void* stream) {
    sa_status r = check_cache(csa, true, "csa_index_quantize_mxfp4");
    if (r != SA_OK) return r;
    SA_CHECK(row_from >= 0, "csa_index_quantize_mxfp4: row_from=%d", row_from);
    SA_CHECK(codes && scales && aligned16(codes) && aligned16(scales),
             "csa_index_quantize_mxfp4: codes and scales must be non-NULL and 16-byte aligned");
    if (row_from >= csa->Ncap) return SA_OK;
    sa::Mxfp4QuantArgs a{};
    a.kidx = static_cast<const uint16_t*>(csa->kidx);
    a.n = csa->n;
    a.codes = codes;
    a.scales = scales;
    a.Ncap = csa->Ncap;
    a.row_from = row_from;
    const long long threads = 2LL * (csa->Ncap - row_from);
    sa::mxfp4_quantize_kernel<<<dim3((unsigned)cdiv(threads, sa::kQuantThreads), csa->B), sa::kQuantThreads, 0,
                                 static_cast<cudaStream_t>(stream)>>>(a);
    SA_LAUNCHED();
    return SA_OK;
}

sa_status csa_index_topk_mxfp4(const void* q_idx, int32_t Tq, const int32_t* q_pos, const sa_cache* csa,
                               const uint8_t* codes, const uint8_t* scales, int32_t k, int32_t* idx, int32_t* cnt,
                               void* ws, size_t ws_bytes, void* stream) {
    sa_status r = check_cache(csa, false, "csa_index_topk_mxfp4");
    if (r != SA_OK) return r;
    SA_CHECK(q_idx && aligned16(q_idx), "csa_index_topk_mxfp4: q_idx must be non-NULL and 16-byte aligned");
    SA_CHECK(codes && scales && aligned16(codes) && aligned16(scales),
             "csa_index_topk_mxfp4: codes and scales must be non-NULL and 16-byte aligned");
    SA_CHECK(idx && cnt && aligned16(idx) && aligned16(cnt),
             "csa_index_topk_mxfp4: idx/cnt must be non-NULL and aligned");
    SA_CHECK(k >= 1 && k <= 65536, "csa_index_topk_mxfp4: k=%d outside 1..65536", k);
    SA_CHECK(Tq >= 1, "csa_index_topk_mxfp4: Tq=%d", Tq);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (q_pos == nullptr) {
        SA_CHECK(Tq == 1, "csa_index_topk_mxfp4: decode (q_pos == NULL) needs Tq == 1, got %d", Tq);
        const TopkDecodeWs w = topk_decode_layout(csa->B, csa->Ncap, k, false);
        r = check_ws(ws, ws_bytes, w.total);
        if (r != SA_OK) return r;
        return run_topk_decode(q_idx, csa, k, idx, cnt, ws, w, st, [] { return SA_OK; }, codes, scales);
    }
    SA_CHECK(aligned16(q_pos), "csa_index_topk_mxfp4: q_pos must be 16-byte aligned");
    r = check_ws(ws, ws_bytes, prefill_topk_bytes(csa->B, Tq, csa->Ncap, k));
    if (r != SA_OK) return r;
    return run_topk_prefill(q_idx, Tq, q_pos, csa, k, idx, cnt, ws, st, codes, scales);
}

sa_status cp_decode_candidates(const void* q_idx, const sa_cache* csa, int32_t k, const int32_t* base,
                               uint32_t* keys, int32_t* gidx, int32_t* gcnt, void* ws, size_t ws_bytes,
                               void* stream) {
    sa_status r = check_cache(csa, true, "cp_decode_candidates");
    if (r != SA_OK) return r;
    SA_CHECK(q_idx && aligned16(q_idx), "cp_decode_candidates: q_idx must be non-NULL and 16-byte aligned");
    SA_CHECK(base && keys && gidx && gcnt, "cp_decode_candidates: base, keys, gidx, gcnt must be non-NULL");
    SA_CHECK(((reinterpret_cast<uintptr_t>(base) | reinterpret_cast<uintptr_t>(keys) |
               reinterpret_cast<uintptr_t>(gidx) | reinterpret_cast<uintptr_t>(gcnt)) & 3u) == 0,
             "cp_decode_candidates: base, keys, gidx, gcnt must be 4-byte aligned");
    SA_CHECK(k >= 1 && k <= 65536, "cp_decode_candidates: k=%d outside 1..65536", k);
    const TopkDecodeWs w = topk_decode_layout(csa->B, csa->Ncap, k, true);
    r = check_ws(ws, ws_bytes, w.total);
    if (r != SA_OK) return r;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    int32_t* idx = reinterpret_cast<int32_t*>(wsb + w.idx);
    int32_t* cnt = reinterpret_cast<int32_t*>(wsb + w.cnt);
    r = run_topk_decode(q_idx, csa, k, idx, cnt, ws, w, st, [] { return SA_OK; });
    if (r != SA_OK) return r;
    sa::CandArgs a{};
    a.q_idx = static_cast<const uint16_t*>(q_idx);
    a.kidx = static_cast<const uint16_t*>(csa->kidx);
    a.idx = idx;
    a.cnt = cnt;
    a.base = base;
    a.keys = keys;
    a.gidx = gidx;
    a.gcnt = gcnt;
    a.Ncap = csa->Ncap;
    a.k = k;
    SA_CUDA(launch_k(sa::cp_candidates_kernel, dim3((unsigned)cdiv(k, sa::kCandThreads), csa->B),
                     dim3(sa::kCandThreads), 0, st, pdl_on(), 1u, a));
    SA_LAUNCHED();
    return SA_OK;
}

sa_status cp_decode_merge_select(const uint32_t* keys, const int32_t* gidx, const int32_t* gcnt, int64_t stride_list,
                                 int64_t stride_cnt, int32_t W, int32_t B, int32_t k, int32_t rank,
                                 const int32_t* base, int32_t* local_idx, int32_t* local_cnt, int32_t* sel_idx,
                                 int32_t* sel_cnt, void* stream) {
    SA_CHECK(W >= 1 && W <= sa::kMergeMaxRanks, "cp_decode_merge_select: W=%d outside 1..%d", W, sa::kMergeMaxRanks);
    SA_CHECK(rank >= 0 && rank < W, "cp_decode_merge_select: rank=%d outside 0..W-1", rank);
    SA_CHECK(B >= 1 && B <= 65535, "cp_decode_merge_select: B=%d outside 1..65535", B);
    SA_CHECK(k >= 1 && k <= 65536, "cp_decode_merge_select: k=%d outside 1..65536", k);
    if ((long long)W * k > sa::kMergeCap)
        return fail(SA_ERR_UNSUPPORTED, "cp_decode_merge_select: W*k=%lld candidates exceed %d", (long long)W * k,
                    sa::kMergeCap);
    SA_CHECK(keys && gidx && gcnt && base && local_idx && local_cnt,
             "cp_decode_merge_select: keys, gidx, gcnt, base, local_idx, local_cnt must be non-NULL");
    SA_CHECK(stride_list >= (int64_t)B * k && stride_cnt >= B,
             "cp_decode_merge_select: stride_list=%lld must be >= B*k and stride_cnt=%lld >= B",
             (long long)stride_list, (long long)stride_cnt);
    SA_CHECK((sel_idx == nullptr) == (sel_cnt == nullptr), "cp_decode_merge_select: give sel_idx and sel_cnt or neither");
    SA_CHECK(((reinterpret_cast<uintptr_t>(keys) | reinterpret_cast<uintptr_t>(gidx) |
               reinterpret_cast<uintptr_t>(gcnt) | reinterpret_cast<uintptr_t>(base) |
               reinterpret_cast<uintptr_t>(local_idx) | reinterpret_cast<uintptr_t>(local_cnt) |
               reinterpret_cast<uintptr_t>(sel_idx) | reinterpret_cast<uintptr_t>(sel_cnt)) & 3u) == 0,
             "cp_decode_merge_select: pointers must be 4-byte aligned");
    static std::atomic<uint64_t> init{0};
    if (!attr_done(init)) {
        SA_CUDA(cudaFuncSetAttribute(sa::cp_merge_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)sa::kMergeSmem));
        attr_set(init);
    }
    sa::MergeArgs a{};
    a.keys = keys;
    a.gidx = gidx;
    a.gcnt = gcnt;
    a.base = base;
    a.local_idx = local_idx;
    a.local_cnt = local_cnt;
    a.sel_idx = sel_idx;
    a.sel_cnt = sel_cnt;
    a.stride_list = stride_list;
    a.stride_cnt = stride_cnt;
    a.W = W;
    a.B = B;
    a.k = k;
    a.rank = rank;
    sa::cp_merge_select_kernel<<<B, sa::kMergeThreads, sa::kMergeSmem, static_cast<cudaStream_t>(stream)>>>(a);
    SA_LAUNCHED();
    return SA_OK;
}

sa_status attn_lse_merge_n(const void* outs, const float* lses, int32_t W, int64_t rows, int64_t stride_out,
                           int64_t stride_lse, void* out, float* lse, void* stream) {
    SA_CHECK(W >= 1 && W <= 1024, "attn_lse_merge_n: W=%d outside 1..1024", W);
    SA_CHECK(rows >= 0, "attn_lse_merge_n: rows=%lld", (long long)rows);
    SA_CHECK(outs && lses && out, "attn_lse_merge_n: outs, lses and out must be non-NULL");
    SA_CHECK(stride_out >= rows * 128 && stride_out % 8 == 0 && stride_lse >= rows,
             "attn_lse_merge_n: stride_out=%lld (>= rows*128, a multiple of 8) / stride_lse=%lld (>= rows)",
             (long long)stride_out, (long long)stride_lse);
    SA_CHECK(aligned16(outs) && aligned16(out) && (!lse || (reinterpret_cast<uintptr_t>(lse) & 3u) == 0) &&
                 (reinterpret_cast<uintptr_t>(lses) & 3u) == 0,
             "attn_lse_merge_n: outs and out must be 16-byte aligned, lses and lse 4-byte");
    if (rows == 0) return SA_OK;
    const long long blocks = (rows + 7) / 8;
    SA_CHECK(blocks <= 2147483647LL, "attn_lse_merge_n: too many rows");
    sa::attn_lse_merge_n_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint16_t*>(outs), lses, W, rows, stride_out, stride_lse, static_cast<uint16_t*>(out), lse);
    SA_LAUNCHED();
    return SA_OK;
}

sa_status csa_sparse_attn(const void* q, int32_t Tq, int32_t H, const sa_cache* csa, const int32_t* idx,
                          const int32_t* cnt, int32_t k, float scale, void* out, float* lse, void* ws,
                          size_t ws_bytes, void* stream) {
    sa_status r = check_cache(csa, false, "csa_sparse_attn");
    if (r != SA_OK) return r;
    r = check_common_q(q, H, "csa_sparse_attn");
    if (r != SA_OK) return r;
    SA_CHECK(Tq >= 1, "csa_sparse_attn: Tq=%d", Tq);
    SA_CHECK(k >= 1 && k <= 65536, "csa_sparse_attn: k=%d outside 1..65536", k);
    SA_CHECK(idx && cnt && aligned16(idx) && aligned16(cnt), "csa_sparse_attn: idx/cnt must be non-NULL and aligned");
    SA_CHECK(out && aligned16(out), "csa_sparse_attn: out must be non-NULL and 16-byte aligned");
    SA_CHECK(!lse || aligned16(lse), "csa_sparse_attn: lse must be 16-byte aligned");
    SA_CHECK(std::isfinite(scale) && scale >= 0.f, "csa_sparse_attn: scale must be finite and >= 0");
    r = check_ws(ws, ws_bytes, sa_workspace_size(SA_OP_SPARSE_ATTN, csa->B, Tq, H, csa->Ncap, 0, k));
    if (r != SA_OK) return r;
    return run_attn(q, Tq, H, csa, true, idx, cnt, k, nullptr, scale, out, lse, ws, 256,
                    static_cast<cudaStream_t>(stream));
}

sa_status hca_dense_attn(const void* q, int32_t Tq, int32_t H, const int32_t* q_pos, const sa_cache* hca, float scale,
                         void* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
    sa_status r = check_cache(hca, false, "hca_dense_attn");
    if (r != SA_OK) return r;
    r = check_common_q(q, H, "hca_dense_attn");
    if (r != SA_OK) return r;
    SA_CHECK(Tq >= 1, "hca_dense_attn: Tq=%d", Tq);
    SA_CHECK(q_pos != nullptr || Tq == 1, "hca_dense_attn: decode (q_pos == NULL) needs Tq == 1");
    SA_CHECK(!q_pos || aligned16(q_pos), "hca_dense_attn: q_pos must be 16-byte aligned");
    SA_CHECK(out && aligned16(out), "hca_dense_attn: out must be non-NULL and 16-byte aligned");
    SA_CHECK(!lse || aligned16(lse), "hca_dense_attn: lse must be 16-byte aligned");
    SA_CHECK(std::isfinite(scale) && scale >= 0.f, "hca_dense_attn: scale must be finite and >= 0");
    const bool prefill = (Tq > 1) || q_pos;
    const Split sp = attn_split(hca->Ncap, prefill);
    r = check_ws(ws, ws_bytes, 256 + attn_partial_bytes((long long)hca->B * Tq, sp.splits, H));
    if (r != SA_OK) return r;
    return run_attn(q, Tq, H, hca, false, nullptr, nullptr, 0, q_pos, scale, out, lse, ws, 256,
                    static_cast<cudaStream_t>(stream));
}

// One decode step of both branches; with MXFP4 indexer keys (codes4 /
// scales4 non-NULL) the CSA selection runs on FP4 scores.
// `side_extra`, when given, queues more independent work on the side stream
// after the HCA branch (it joins the caller's stream with it).
static sa_status hybrid_decode_impl(const char* what, const void* q, const void* q_idx, int32_t H,
                                    const sa_cache* csa, const sa_cache* hca, const uint8_t* codes4,
                                    const uint8_t* scales4, int32_t k, float scale, void* out_csa, void* out_hca,
                                    float* lse_csa, float* lse_hca, int32_t* idx_out, int32_t* cnt_out, void* ws,
                                    size_t ws_bytes, void* stream,
                                    const std::function<sa_status(cudaStream_t)>& side_extra = nullptr) {
    const bool fp4 = codes4 != nullptr || scales4 != nullptr;
    sa_status r = check_cache(csa, !fp4, fp4 ? "hybrid_attn_decode_mxfp4(csa)" : "hybrid_attn_decode(csa)");
    if (r != SA_OK) return r;
    r = check_cache(hca, false, fp4 ? "hybrid_attn_decode_mxfp4(hca)" : "hybrid_attn_decode(hca)");
    if (r != SA_OK) return r;
    r = check_common_q(q, H, what);
    if (r != SA_OK) return r;
    if (fp4)
        SA_CHECK(codes4 && scales4 && aligned16(codes4) && aligned16(scales4),
                 "%s: codes and scales must be non-NULL and 16-byte aligned", what);
    SA_CHECK(csa->B == hca->B, "%s: csa B=%d != hca B=%d", what, csa->B, hca->B);
    SA_CHECK(q_idx && aligned16(q_idx), "%s: q_idx must be non-NULL and aligned", what);
    SA_CHECK(k >= 1 && k <= 65536, "%s: k=%d outside 1..65536", what, k);
    SA_CHECK(out_csa && out_hca && aligned16(out_csa) && aligned16(out_hca), "%s: outputs must be aligned", what);
    SA_CHECK((!lse_csa || aligned16(lse_csa)) && (!lse_hca || aligned16(lse_hca)), "%s: lse alignment", what);
    SA_CHECK((idx_out == nullptr) == (cnt_out == nullptr), "%s: give both idx_out and cnt_out or neither", what);
    SA_CHECK((!idx_out || aligned16(idx_out)) && (!cnt_out || aligned16(cnt_out)), "%s: idx/cnt alignment", what);
    SA_CHECK(std::isfinite(scale) && scale >= 0.f, "%s: scale must be finite and >= 0", what);
    const size_t need = sa_workspace_size(SA_OP_HYBRID_DECODE, csa->B, 1, H, csa->Ncap, hca->Ncap, k);
    r = check_ws(ws, ws_bytes, need);
    if (r != SA_OK) return r;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    TopkDecodeWs w = topk_decode_layout(csa->B, csa->Ncap, k, true, true);
    uint8_t* base = static_cast<uint8_t*>(ws);
    int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(base + w.idx);
    int32_t* cnt = cnt_out ? cnt_out : reinterpret_cast<int32_t*>(base + w.cnt);
    const Split sc = attn_split(k, false, true);
    // HCA needs neither the indexer nor the top-k: once the indexer stream and
    // the filter are queued, fork it onto the side stream so that it overlaps
    // the latency-bound resolve, emit and CSA attention instead of competing
    // with the indexer stream or the filter's many CTAs.
    SideStream* side = nullptr;
    r = side_stream(&side);
    if (r != SA_OK) return r;
    auto fork_hca = [&]() -> sa_status {
        PriorityScope normal(0);  // the HCA branch keeps the default priority
        SA_CUDA(cudaEventRecord(side->fork, st));
        SA_CUDA(cudaStreamWaitEvent(side->s, side->fork, 0));
        stage_mark(SA_STAGE_HCA_ATTN, 0, side->s);
        sa_status rr = run_attn(q, 1, H, hca, false, nullptr, nullptr, 0, nullptr, scale, out_hca, lse_hca, ws,
                                w.total + attn_partial_bytes(csa->B, sc.splits, H), side->s);
        if (rr != SA_OK) return rr;
        stage_mark(SA_STAGE_HCA_ATTN, 1, side->s);
        if (side_extra) {
            rr = side_extra(side->s);
            if (rr != SA_OK) return rr;
        }
        SA_CUDA(cudaEventRecord(side->join, side->s));
        return SA_OK;
    };
    PriorityScope high(highest_priority());
    if (!fp4 && fast_decode_ok(csa, H, k))
        r = run_fast_topk(q_idx, csa, k, idx, cnt, ws, w, st, fork_hca);
    else
        r = run_topk_decode(q_idx, csa, k, idx, cnt, ws, w, st, fork_hca, codes4, scales4);
    if (r != SA_OK) return r;
    stage_mark(SA_STAGE_CSA_ATTN, 0, st);
    r = run_attn(q, 1, H, csa, true, idx, cnt, k, nullptr, scale, out_csa, lse_csa, ws, w.total, st, true);
    if (r != SA_OK) return r;
    stage_mark(SA_STAGE_CSA_ATTN, 1, st);
    SA_CUDA(cudaStreamWaitEvent(st, side->join, 0));
    return SA_OK;
}

sa_status hybrid_attn_decode(const void* q, const void* q_idx, int32_t H, const sa_cache* csa, const sa_cache* hca,
                             int32_t k, float scale, void* out_csa, void* out_hca, float* lse_csa, float* lse_hca,
                             int32_t* idx_out, int32_t* cnt_out, void* ws, size_t ws_bytes, void* stream) {
    return hybrid_decode_impl("hybrid_attn_decode", q, q_idx, H, csa, hca, nullptr, nullptr, k, scale, out_csa,
                              out_hca, lse_csa, lse_hca, idx_out, cnt_out, ws, ws_bytes, stream);
}

sa_status hybrid_attn_decode_swa(const void* q, const void* q_idx, int32_t H, const sa_cache* csa,
                                 const sa_cache* hca, const sa_raw* raw, int32_t window, int32_t k, float scale,
                                 void* out_csa, void* out_hca, float* lse_csa, float* lse_hca, int32_t* idx_out,
                                 int32_t* cnt_out, void* ws, size_t ws_bytes, void* stream) {
    SA_CHECK(csa != nullptr && hca != nullptr, "hybrid_attn_decode_swa: cache descriptors must be non-NULL");
    SA_CHECK(raw != nullptr, "hybrid_attn_decode_swa: raw descriptor is NULL");
    SA_CHECK(raw->B == csa->B, "hybrid_attn_decode_swa: raw B=%d != csa B=%d", raw->B, csa->B);
    SA_CHECK(window >= 1, "hybrid_attn_decode_swa: window=%d", window);
    // every check of the window call, here: it runs on the side stream once the
    // step is queued, where a refusal would leave that stream unjoined
    SA_CHECK(raw->Lcap >= 0 && raw->d == 128, "hybrid_attn_decode_swa: raw Lcap=%d d=%d", raw->Lcap, raw->d);
    SA_CHECK(raw->k && raw->v && raw->len && aligned16(raw->k) && aligned16(raw->v) && aligned16(raw->len),
             "hybrid_attn_decode_swa: raw k, v, len must be non-NULL and 16-byte aligned");
    SA_CHECK(std::isfinite(scale) && scale >= 0.f, "hybrid_attn_decode_swa: scale must be finite and >= 0");
    SA_CHECK(q != nullptr && aligned16(q), "hybrid_attn_decode_swa: q must be non-NULL and 16-byte aligned");
    SA_CHECK(H >= 1 && H <= 128, "hybrid_attn_decode_swa: H=%d outside 1..128", H);
    SA_CHECK(k >= 1 && k <= 65536, "hybrid_attn_decode_swa: k=%d outside 1..65536", k);
    const SwaDecodeWs w = swa_decode_layout(csa->B, H, csa->Ncap, hca->Ncap, k);
    sa_status r = check_ws(ws, ws_bytes, w.total);
    if (r != SA_OK) return r;
    uint8_t* base = static_cast<uint8_t*>(ws);
    float* lc = lse_csa ? lse_csa : reinterpret_cast<float*>(base + w.lse_c);
    float* lh = lse_hca ? lse_hca : reinterpret_cast<float*>(base + w.lse_h);
    // the window over the raw tokens, once for both layers: it needs neither
    // the indexer nor the top-k, so it runs on the side stream after the HCA
    // branch, beside the CSA chain; then one merge each on the caller's stream
    void* wo = base + w.win_out;
    float* wl = reinterpret_cast<float*>(base + w.win_lse);
    auto window_attn = [&](cudaStream_t s) -> sa_status {
        return swa_attn(q, 1, H, nullptr, raw, window, scale, wo, wl, base + w.win_ws, w.win_out - w.win_ws, s);
    };
    r = hybrid_decode_impl("hybrid_attn_decode_swa", q, q_idx, H, csa, hca, nullptr, nullptr, k, scale, out_csa,
                           out_hca, lc, lh, idx_out, cnt_out, ws, w.win_ws, stream, window_attn);
    if (r != SA_OK) return r;
    const int64_t rows = (int64_t)csa->B * H;
    r = attn_lse_merge(out_csa, lc, wo, wl, rows, out_csa, lc, stream);
    if (r != SA_OK) return r;
    return attn_lse_merge(out_hca, lh, wo, wl, rows, out_hca, lh, stream);
}

sa_status hybrid_attn_decode_mxfp4(const void* q, const void* q_idx, int32_t H, const sa_cache* csa,
                                   const sa_cache* hca, const uint8_t* codes, const uint8_t* scales, int32_t k,
                                   float scale, void* out_csa, void* out_hca, float* lse_csa, float* lse_hca,
                                   int32_t* idx_out, int32_t* cnt_out, void* ws, size_t ws_bytes, void* stream) {
    SA_CHECK(codes && scales, "hybrid_attn_decode_mxfp4: codes and scales must be non-NULL");
    return hybrid_decode_impl("hybrid_attn_decode_mxfp4", q, q_idx, H, csa, hca, codes, scales, k, scale, out_csa,
                              out_hca, lse_csa, lse_hca, idx_out, cnt_out, ws, ws_bytes, stream);
}

sa_status sa_decode_io_layout(int32_t B, int32_t H, sa_decode_io* io) {
    SA_CHECK(io != nullptr, "sa_decode_io_layout: io must be non-NULL");
    SA_CHECK(B >= 1 && H >= 1 && H <= 128, "sa_decode_io_layout: B=%d H=%d outside B >= 1, H 1..128", B, H);
    const size_t rows = (size_t)B * H;
    io->q_idx_off = 0;
    io->q_off = up256((size_t)B * 64 * 2);
    io->in_bytes = io->q_off + up256(rows * 128 * 2);
    io->out_hca_off = 0;
    io->lse_hca_off = up256(rows * 128 * 2);
    io->out_csa_off = io->lse_hca_off + up256(rows * 4);
    io->lse_csa_off = io->out_csa_off + up256(rows * 128 * 2);
    io->out_bytes = io->lse_csa_off + up256(rows * 4);
    return SA_OK;
}

struct sa_decode_graph {
    cudaGraphExec_t exec = nullptr;
    uint64_t kernels = 0;  // kernels one step launches (for sa_launch_count)
};

// The device's view of a pinned host buffer (NULL when it has none), after
// checking that `p` is pinned host memory.
static sa_status host_mapping(const void* p, const char* what, const char* name, void** dev_view) {
    cudaPointerAttributes a{};
    SA_CUDA(cudaPointerGetAttributes(&a, p));
    SA_CHECK(a.type == cudaMemoryTypeHost, "%s: %s must be pinned host memory", what, name);
    *dev_view = a.devicePointer;
    return SA_OK;
}

static sa_status check_device_mem(const void* p, const char* what, const char* name) {
    cudaPointerAttributes a{};
    SA_CUDA(cudaPointerGetAttributes(&a, p));
    SA_CHECK(a.type == cudaMemoryTypeDevice, "%s: %s must be device memory", what, name);
    return SA_OK;
}

sa_status sa_decode_graph_create(const sa_cache* csa, const sa_cache* hca, int32_t H, int32_t k, float scale,
                                 const uint8_t* codes, const uint8_t* scales, void* host_in, void* host_out,
                                 void* dev_in, void* dev_out, int32_t* idx_out, int32_t* cnt_out, void* ws,
                                 size_t ws_bytes, uint32_t flags, sa_decode_graph** graph) {
    const char* what = "sa_decode_graph_create";
    SA_CHECK(graph != nullptr, "%s: graph must be non-NULL", what);
    *graph = nullptr;
    SA_CHECK(csa != nullptr && hca != nullptr, "%s: caches must be non-NULL", what);
    SA_CHECK((codes == nullptr) == (scales == nullptr), "%s: give both codes and scales or neither", what);
    SA_CHECK((flags & ~(SA_DG_KERNEL_IN | SA_DG_DIRECT_OUT)) == 0, "%s: unknown flags 0x%x", what, flags);
    const bool kin = flags & SA_DG_KERNEL_IN, dout_direct = flags & SA_DG_DIRECT_OUT;
    sa_decode_io io;
    sa_status r = sa_decode_io_layout(csa->B, H, &io);
    if (r != SA_OK) return r;
    SA_CHECK(host_in && host_out && dev_in && (dev_out || dout_direct), "%s: I/O buffers must be non-NULL", what);
    SA_CHECK(aligned16(host_in) && aligned16(host_out) && aligned16(dev_in) && aligned16(dev_out),
             "%s: I/O buffers must be 16-byte aligned", what);
    void *map_in = nullptr, *map_out = nullptr;
    if ((r = host_mapping(host_in, what, "host_in", &map_in)) != SA_OK) return r;
    if ((r = host_mapping(host_out, what, "host_out", &map_out)) != SA_OK) return r;
    SA_CHECK(!kin || (map_in && aligned16(map_in)), "%s: SA_DG_KERNEL_IN needs host_in mapped into the device", what);
    SA_CHECK(!dout_direct || (map_out && aligned16(map_out)),
             "%s: SA_DG_DIRECT_OUT needs host_out mapped into the device", what);
    if ((r = check_device_mem(dev_in, what, "dev_in")) != SA_OK) return r;
    if (!dout_direct && (r = check_device_mem(dev_out, what, "dev_out")) != SA_OK) return r;
    const bool fp4 = codes != nullptr;
    uint8_t* di = static_cast<uint8_t*>(dev_in);
    uint8_t* hout = static_cast<uint8_t*>(host_out);
    // where the kernels write the outputs: the device buffer, or the host
    // buffer's device mapping
    uint8_t* dout = static_cast<uint8_t*>(dout_direct ? map_out : dev_out);
    // One step: the packed queries in, both branches, the HCA half of the
    // outputs back from the HCA branch (overlapping the CSA branch), the CSA
    // half at the end.  The eager pass (kernel attributes, the side stream)
    // zeroes the queries instead of copying them and copies nothing back.
    auto body = [&](cudaStream_t cs, bool eager) -> sa_status {
        if (eager) {
            SA_CUDA(cudaMemsetAsync(di, 0, io.in_bytes, cs));
        } else if (kin) {
            const uint32_t n16 = (uint32_t)(io.in_bytes / 16);
            sa::copy_in_kernel<<<std::min(cdiv(n16, 256), 2 * num_sms()), 256, 0, cs>>>(
                static_cast<const uint4*>(map_in), reinterpret_cast<uint4*>(di), n16);
            SA_LAUNCHED();
        } else {
            SA_CUDA(cudaMemcpyAsync(di, host_in, io.in_bytes, cudaMemcpyHostToDevice, cs));
        }
        const bool copy_back = !eager && !dout_direct;
        std::function<sa_status(cudaStream_t)> hca_back = nullptr;
        if (copy_back)
            hca_back = [&](cudaStream_t s) -> sa_status {
                SA_CUDA(cudaMemcpyAsync(hout, dout, io.out_csa_off, cudaMemcpyDeviceToHost, s));
                return SA_OK;
            };
        // the eager pass writes to the device buffer when there is one
        uint8_t* o = eager && dev_out ? static_cast<uint8_t*>(dev_out) : dout;
        sa_status rr = hybrid_decode_impl(fp4 ? "hybrid_attn_decode_mxfp4" : "hybrid_attn_decode", di + io.q_off,
                                          di + io.q_idx_off, H, csa, hca, codes, scales, k, scale,
                                          o + io.out_csa_off, o + io.out_hca_off,
                                          reinterpret_cast<float*>(o + io.lse_csa_off),
                                          reinterpret_cast<float*>(o + io.lse_hca_off), idx_out, cnt_out, ws,
                                          ws_bytes, cs, hca_back);
        if (rr != SA_OK) return rr;
        if (copy_back)
            SA_CUDA(cudaMemcpyAsync(hout + io.out_csa_off, dout + io.out_csa_off, io.out_bytes - io.out_csa_off,
                                    cudaMemcpyDeviceToHost, cs));
        return SA_OK;
    };
    cudaStream_t cs = nullptr;
    SA_CUDA(cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking));
    cudaGraph_t g = nullptr;
    cudaGraphExec_t exec = nullptr;
    uint64_t kernels = 0;
    r = body(cs, true);
    cudaError_t e = cudaStreamSynchronize(cs);
    if (r == SA_OK && e != cudaSuccess) r = fail(SA_ERR_CUDA, "%s: eager step: %s", what, cudaGetErrorString(e));
    if (r == SA_OK) {
        e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
        if (e != cudaSuccess) {
            r = fail(SA_ERR_CUDA, "%s: begin capture: %s", what, cudaGetErrorString(e));
        } else {
            const uint64_t n0 = g_launches;
            r = body(cs, false);
            kernels = g_launches - n0;
            e = cudaStreamEndCapture(cs, &g);  // always ends the capture, also after an error
            if (r == SA_OK && e != cudaSuccess) r = fail(SA_ERR_CUDA, "%s: end capture: %s", what, cudaGetErrorString(e));
        }
    }
    if (r == SA_OK) {
        e = cudaGraphInstantiate(&exec, g, 0);
        if (e != cudaSuccess) r = fail(SA_ERR_CUDA, "%s: instantiate: %s", what, cudaGetErrorString(e));
    }
    if (g) cudaGraphDestroy(g);
    cudaStreamDestroy(cs);
    if (r != SA_OK) {
        if (exec) cudaGraphExecDestroy(exec);
        return r;
    }
    sa_decode_graph* h = new (std::nothrow) sa_decode_graph;
    if (!h) {
        cudaGraphExecDestroy(exec);
        return fail(SA_ERR_UNSUPPORTED, "%s: out of host memory", what);
    }
    h->exec = exec;
    h->kernels = kernels;
    *graph = h;
    return SA_OK;
}

sa_status sa_decode_graph_step(sa_decode_graph* graph, void* stream) {
    SA_CHECK(graph != nullptr && graph->exec != nullptr, "sa_decode_graph_step: graph must be a created graph");
    SA_CUDA(cudaGraphLaunch(graph->exec, static_cast<cudaStream_t>(stream)));
    g_launches += graph->kernels;
    return SA_OK;
}

sa_status sa_decode_graph_destroy(sa_decode_graph* graph) {
    if (!graph) return SA_OK;
    const cudaError_t e = graph->exec ? cudaGraphExecDestroy(graph->exec) : cudaSuccess;
    delete graph;
    if (e != cudaSuccess) return fail(SA_ERR_CUDA, "sa_decode_graph_destroy: %s", cudaGetErrorString(e));
    return SA_OK;
}

// Causal prefill of both branches; with MXFP4 indexer keys (codes4 /
// scales4 non-NULL) the CSA selection runs on FP4 scores.
static sa_status hybrid_prefill_impl(const char* what, const void* q, const void* q_idx, int32_t T, int32_t H,
                                     const sa_cache* csa, const sa_cache* hca, const uint8_t* codes4,
                                     const uint8_t* scales4, int32_t k, float scale, void* out_csa, void* out_hca,
                                     float* lse_csa, float* lse_hca, int32_t* idx_out, int32_t* cnt_out, void* ws,
                                     size_t ws_bytes, void* stream) {
    const bool fp4 = codes4 != nullptr || scales4 != nullptr;
    sa_status r = check_cache(csa, !fp4, fp4 ? "hybrid_attn_prefill_mxfp4(csa)" : "hybrid_attn_prefill(csa)");
    if (r != SA_OK) return r;
    r = check_cache(hca, false, fp4 ? "hybrid_attn_prefill_mxfp4(hca)" : "hybrid_attn_prefill(hca)");
    if (r != SA_OK) return r;
    r = check_common_q(q, H, what);
    if (r != SA_OK) return r;
    if (fp4)
        SA_CHECK(codes4 && scales4 && aligned16(codes4) && aligned16(scales4),
                 "%s: codes and scales must be non-NULL and 16-byte aligned", what);
    SA_CHECK(csa->B == hca->B, "%s: csa B=%d != hca B=%d", what, csa->B, hca->B);
    SA_CHECK(T >= 1, "%s: T=%d", what, T);
    SA_CHECK(q_idx && aligned16(q_idx), "%s: q_idx must be non-NULL and aligned", what);
    SA_CHECK(k >= 1 && k <= 65536, "%s: k=%d outside 1..65536", what, k);
    SA_CHECK(out_csa && out_hca && aligned16(out_csa) && aligned16(out_hca), "%s: outputs must be aligned", what);
    SA_CHECK((!lse_csa || aligned16(lse_csa)) && (!lse_hca || aligned16(lse_hca)), "%s: lse alignment", what);
    SA_CHECK(idx_out && cnt_out && aligned16(idx_out) && aligned16(cnt_out),
             "%s: idx_out and cnt_out are required and must be aligned", what);
    SA_CHECK(std::isfinite(scale) && scale >= 0.f, "%s: scale must be finite and >= 0", what);
    r = check_ws(ws, ws_bytes, sa_workspace_size(SA_OP_HYBRID_PREFILL, csa->B, T, H, csa->Ncap, hca->Ncap, k));
    if (r != SA_OK) return r;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // positions 0..T-1 for every sequence live in the workspace
    const int32_t* pos = prefill_positions(ws, csa->B, T, st);
    if (!pos) return fail(SA_ERR_CUDA, "could not write query positions");
    r = run_topk_prefill(q_idx, T, pos, csa, k, idx_out, cnt_out, ws, st, codes4, scales4);
    if (r != SA_OK) return r;
    r = run_attn(q, T, H, csa, true, idx_out, cnt_out, k, pos, scale, out_csa, lse_csa, ws, 0, st);
    if (r != SA_OK) return r;
    return run_attn(q, T, H, hca, false, nullptr, nullptr, 0, pos, scale, out_hca, lse_hca, ws, 0, st);
}

sa_status hybrid_attn_prefill(const void* q, const void* q_idx, int32_t T, int32_t H, const sa_cache* csa,
                              const sa_cache* hca, int32_t k, float scale, void* out_csa, void* out_hca,
                              float* lse_csa, float* lse_hca, int32_t* idx_out, int32_t* cnt_out, void* ws,
                              size_t ws_bytes, void* stream) {
    return hybrid_prefill_impl("hybrid_attn_prefill", q, q_idx, T, H, csa, hca, nullptr, nullptr, k, scale, out_csa,
                               out_hca, lse_csa, lse_hca, idx_out, cnt_out, ws, ws_bytes, stream);
}

sa_status hybrid_attn_prefill_mxfp4(const void* q, const void* q_idx, int32_t T, int32_t H, const sa_cache* csa,
                                    const sa_cache* hca, const uint8_t* codes, const uint8_t* scales, int32_t k,
                                    float scale, void* out_csa, void* out_hca, float* lse_csa, float* lse_hca,
                                    int32_t* idx_out, int32_t* cnt_out, void* ws, size_t ws_bytes, void* stream) {
    SA_CHECK(codes && scales, "hybrid_attn_prefill_mxfp4: codes and scales must be non-NULL");
    return hybrid_prefill_impl("hybrid_attn_prefill_mxfp4", q, q_idx, T, H, csa, hca, codes, scales, k, scale,
                               out_csa, out_hca, lse_csa, lse_hca, idx_out, cnt_out, ws, ws_bytes, stream);
}

}  // extern "C"
