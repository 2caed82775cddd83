/*
 * sparse_attn.h -- C ABI of libsparse_attn.so: CSA + HCA hybrid attention on
 * one NVIDIA B200 (sm_100a).
 *
 * The method is the hybrid attention of "DeepSeek-V4: Towards Highly Efficient
 * Million-Token Context Intelligence Review" (dimensionstp.github.io),
 * section 3-2 (2) "Hybrid attention with CSA and HCA":
 *   - CSA (compressed sparse attention) pools every 4 tokens of K/V into one
 *     compressed entry, scores every entry with an indexer, keeps the top-k
 *     entries and attends over them only;
 *   - HCA (heavily compressed attention) pools every 128 tokens into one entry
 *     and attends densely over all entries;
 *   - the layers interleave the two, so one "hybrid" step returns both outputs;
 *   - compressed KV may be stored in FP8 (the "Mixed KV storage" row).
 * Where the page leaves the arithmetic open, this library implements:
 *   pooling  = fp64 sum of each aligned, complete block of m tokens in
 *              ascending token order, times 1/m, rounded once to bf16 (RNE);
 *              an incomplete tail block is not compressed;
 *   fp8      = e4m3 codes, one fp32 scale per 64 consecutive entries,
 *              scale = fp32(amax / 448) (1 when amax == 0),
 *              code = e4m3_rne_satfinite(fp32(x / scale));
 *   score    = fp32( fp64 sum over i = 0..63, ascending, of q_idx[i]*kidx[j][i] ),
 *              -0 -> +0; one 64-dim indexer query per token, shared by heads;
 *   top-k    = the k entries with the largest (score, -index); indices are
 *              returned in ascending order, padded with -1;
 *   attention= per head softmax(scale * q . K^T) V over the chosen entries,
 *              fp32 accumulation, bf16 output (RNE), fp32 natural-log lse;
 *              scale = 1/sqrt(128) when 0 is passed; an empty set gives a
 *              zero output and lse = -inf;
 *   causality= a query at token position t sees entry c iff (c + 1) * m <= t;
 *              in decode the query follows the cached tokens, t = length.
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; each must
 *     be 16-byte aligned.  bf16 tensors are raw IEEE bfloat16, e4m3 tensors
 *     are raw OCP FP8 E4M3 ("fn") bytes.  Layouts are dense, row-major, in
 *     the order written next to each argument.
 *   - The library never allocates, frees or synchronises device memory; all
 *     work is queued on `stream` (a cudaStream_t passed as void*, NULL = the
 *     legacy default stream) and returns before it runs.
 *   - Argument errors are detected on the host before anything is launched
 *     and return a non-zero sa_status; sa_last_error() then gives the reason.
 *   - Errors that only the device can see (a length above its capacity, a
 *     bounded wait that ran out) never trap: kernels record them in a
 *     per-device status word and carry on with clamped values.
 *     sa_read_device_status() reports and clears it.
 *   - head_dim d must be 128 and the indexer dim d_idx 64.  H is 1..128.
 *   - Results are deterministic run to run and do not depend on the batch a
 *     sequence is in (the split of every reduction is fixed per sequence).
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SA_ABI_VERSION 1

typedef enum {
    SA_OK = 0,
    SA_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, bad size or shape      */
    SA_ERR_UNSUPPORTED = 2,  /* a valid request the library does not implement     */
    SA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than sa_workspace_size */
    SA_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, memset, ...)   */
    SA_ERR_TIMEOUT = 5,      /* device status: a bounded wait ran out              */
    SA_ERR_DEVICE = 6        /* device status: a length exceeded its capacity, ... */
} sa_status;

/* Storage of the compressed K and V ("Mixed KV storage" row of the review's
 * section 3-2 (2) table: rotary dims in BF16, the rest in FP8).
 *   SA_BF16:     K, V [B][Ncap][d] bf16.
 *   SA_FP8_E4M3: K, V [B][Ncap][d] e4m3 codes; k_scale / v_scale
 *                [B][ceil(Ncap/64)] fp32, one per 64 consecutive entries,
 *                scale = fp32(amax / 448) (1 when amax == 0).
 *   SA_KV_MIXED: K [B][Ncap][192] bytes per entry: dims 0..63 as e4m3 codes
 *                (bytes 0..63) then the rotary dims 64..127 as bf16 (bytes
 *                64..191); k_scale over dims 0..63 only.  V as SA_FP8_E4M3.
 *                The page gives no rotary width; the last 64 of the 128 dims
 *                is the reading taken here.                                   */
typedef enum { SA_BF16 = 0, SA_FP8_E4M3 = 1, SA_KV_MIXED = 2 } sa_kv_dtype;

/* Raw (uncompressed) tokens of B sequences, padded to Lcap tokens each. */
typedef struct {
    const void* k;         /* [B][Lcap][d] bf16                                   */
    const void* v;         /* [B][Lcap][d] bf16                                   */
    const void* kidx;      /* [B][Lcap][d_idx] bf16 indexer keys (CSA), or NULL   */
    const int32_t* len;    /* device [B]: tokens of each sequence, 0..Lcap        */
    int32_t B, Lcap, d, d_idx;
} sa_raw;

/* A compressed cache (CSA: m = 4 with indexer keys; HCA: m = 128 without). */
typedef struct {
    void* k;               /* [B][Ncap][d] bf16 or e4m3, or [B][Ncap][192] mixed    */
    void* v;               /* [B][Ncap][d] bf16, or e4m3 codes                     */
    float* k_scale;        /* [B][ceil(Ncap/64)] fp32 unless dtype == SA_BF16       */
    float* v_scale;        /* same for v; both NULL for bf16                        */
    void* kidx;            /* [B][Ncap][d_idx] bf16 (needed by the CSA indexer)     */
    int32_t* n;            /* device [B]: complete entries per sequence             */
    int32_t B, Ncap, d, d_idx;
    int32_t m;             /* tokens per entry: a power of two, 1..1024            */
    int32_t dtype;         /* sa_kv_dtype                                           */
} sa_cache;

/* Operation codes for sa_workspace_size. */
typedef enum {
    SA_OP_INDEX_TOPK = 1,
    SA_OP_SPARSE_ATTN = 2,
    SA_OP_DENSE_ATTN = 3,
    SA_OP_HYBRID_DECODE = 4,
    SA_OP_HYBRID_PREFILL = 5,
    SA_OP_WINDOW_ATTN = 6,  /* k = the window */
    SA_OP_CP_CANDIDATES = 7, /* cp_decode_candidates (Tq = 1) */
    SA_OP_HYBRID_DECODE_SWA = 8 /* hybrid_attn_decode_swa (Tq = 1; any window) */
} sa_op;

/* Compression, section 3-2 (2) component table, CSA row ("every 4 tokens ->
 * 1 compressed entry").  Pools raw k, v and kidx of every sequence into
 * `out` (out->m tokens per entry, normally 4) and writes out->n[b] =
 * floor(len[b] / m).  Needs out->kidx != NULL and raw->kidx != NULL.
 * Entries at or beyond n[b] are left untouched.  fp8 caches also get their
 * per-64-entry scales.  Requires out->Ncap >= Lcap / m.                       */
sa_status csa_compress(const sa_raw* raw, const sa_cache* out, void* stream);

/* Compression, HCA row ("every 128 tokens -> 1 compressed entry"): as
 * csa_compress for k and v only (kidx ignored); out->m is normally 128.      */
sa_status hca_compress(const sa_raw* raw, const sa_cache* out, void* stream);

/* Compress-when-ready, section 3-2 (4) (the state cache holds the tail until
 * a block is complete): the raw sequences have grown since the cache was last
 * brought up to date (cache->n[b] entries).  Computes the entries
 * cache->n[b] .. floor(len[b] / m) - 1, recomputes the partly filled group of
 * 64 entries they join (an fp8 group's scale covers every entry present) and
 * sets cache->n[b] = floor(len[b] / m).  The result is bit-identical to
 * csa_compress / hca_compress of the new lengths.
 *   max_new_tokens: an upper bound, per sequence, on the raw tokens added
 *   since cache->n[b] was set (the launch is sized from it).  A sequence that
 *   grew by more is completed only as far as the launch reaches (cache->n[b]
 *   says how far) and flagged in the device status (SA_ERR_DEVICE from
 *   sa_read_device_status).
 * Other arguments and requirements as for csa_compress / hca_compress.        */
sa_status csa_append(const sa_raw* raw, const sa_cache* cache, int32_t max_new_tokens, void* stream);
sa_status hca_append(const sa_raw* raw, const sa_cache* cache, int32_t max_new_tokens, void* stream);

/* Sliding-window branch, section 3-2 (2) (a small window of the latest
 * uncompressed tokens beside the compressed branches).  Softmax attention of
 * the H query heads over the last `window` raw tokens visible to the query:
 * tokens max(0, T - window) .. T - 1 with T = len[b] (decode, q_pos NULL,
 * Tq 1) or T = min(len[b], t) for a query at position t (q_pos [B][Tq]).
 *   q [B][Tq][H][128] bf16; raw->k, raw->v [B][Lcap][128] bf16, raw->len [B].
 *   out [B][Tq][H][128] bf16; lse [B][Tq][H] fp32 (natural log) or NULL.
 * ws / ws_bytes: at least sa_workspace_size(SA_OP_WINDOW_ATTN, B, Tq, H, 0, 0,
 * window).  No visible token: out 0, lse -inf.                               */
sa_status swa_attn(const void* q, int32_t Tq, int32_t H, const int32_t* q_pos, const sa_raw* raw,
                   int32_t window, float scale, void* out, float* lse, void* ws, size_t ws_bytes,
                   void* stream);

/* Merges two attentions over disjoint key sets (for instance a compressed
 * branch and the window branch) into the attention over their union:
 * lse = log(e^lse_a + e^lse_b), out = (e^lse_a out_a + e^lse_b out_b) / e^lse.
 * rows = B * Tq * H; out_* [rows][128] bf16, lse_* [rows] fp32; out may alias
 * out_a or out_b (each row is read before it is written); lse may be NULL.
 * A row whose lse_a and lse_b are both -inf gets out 0, lse -inf.            */
sa_status attn_lse_merge(const void* out_a, const float* lse_a, const void* out_b, const float* lse_b,
                         int64_t rows, void* out, float* lse, void* stream);

/* CSA indexer + top-k, section 3-2 (2) (CSA "sparse top-k selection") and
 * 3-2 (4) ("CSA indexer QK path").
 *   q_idx [B][Tq][d_idx] bf16: indexer queries.
 *   q_pos [B][Tq] int32 device token positions, or NULL for decode (Tq must
 *         then be 1 and every complete entry is visible).
 *   idx   [B][Tq][k] int32 out: chosen entries, ascending, -1 padded.
 *   cnt   [B][Tq] int32 out: min(k, visible entries).
 * ws / ws_bytes: scratch of at least sa_workspace_size(SA_OP_INDEX_TOPK, ...).
 * k: 1..65536.                                                               */
sa_status csa_index_topk(const void* q_idx, int32_t Tq, const int32_t* q_pos,
                         const sa_cache* csa, int32_t k, int32_t* idx, int32_t* cnt,
                         void* ws, size_t ws_bytes, void* stream);

/* FP4 indexer keys, section 3-2 (4) ("FP4 quantization-aware training ... in
 * the CSA indexer QK path"; the page names the precision only).  Format read
 * here: MXFP4 of the OCP Microscaling specification.  Each compressed
 * indexer key (64 bf16 dims, as csa_compress writes them) becomes two blocks
 * of 32 e2m1 elements with one E8M0 scale per block:
 *   X = 2^(floor(log2 amax) - 2), exponent clamped to [-127, 127], E8M0 code
 *       0 when amax == 0;  element = e2m1 round-to-nearest-even of x / X,
 *       saturating at +-6, sign kept.
 *   codes  [B][Ncap][32] uint8 out: element 2i in the low nibble of byte i,
 *          element 2i+1 in the high nibble.
 *   scales [B][Ncap][2] uint8 out: E8M0 codes of blocks 0 (dims 0..31) and 1.
 * Entries row_from .. n[b]-1 of every sequence are (re)written; the others
 * are left alone (after an append, pass the smallest old n to refresh the new
 * entries only).  Both buffers are the caller's, 16-byte aligned.            */
sa_status csa_index_quantize_mxfp4(const sa_cache* csa, int32_t row_from, uint8_t* codes, uint8_t* scales,
                                   void* stream);

/* Top-k on FP4 indexer scores (same section), in decode and in causal
 * prefill.  The queries q_idx [B][Tq][d_idx] bf16 are quantized in the kernel
 * by the rule above; the score of entry j is the fp32 value, rounded to
 * nearest even once, of the exact sum over the two blocks of
 * X_q * X_k * sum_i e2m1(q_i) * e2m1(k_ji) (-0 -> +0).  Tq, q_pos,
 * visibility, selection, order, padding and count are those of
 * csa_index_topk.  codes / scales as written by csa_index_quantize_mxfp4 for
 * the entries 0..n[b]-1; the bf16 indexer keys of the cache are not read.
 * ws / ws_bytes: at least sa_workspace_size(SA_OP_INDEX_TOPK, B, Tq, ...).    */
sa_status csa_index_topk_mxfp4(const void* q_idx, int32_t Tq, const int32_t* q_pos, const sa_cache* csa,
                               const uint8_t* codes, const uint8_t* scales, int32_t k, int32_t* idx, int32_t* cnt,
                               void* ws, size_t ws_bytes, void* stream);

/* CSA attention over the chosen entries, section 3-2 (2) (CSA attends over
 * the selected entries only).
 *   q   [B][Tq][H][d] bf16; idx / cnt as produced by csa_index_topk (an index
 *       outside 0..n[b]-1 is skipped and flagged in the device status).
 *   out [B][Tq][H][d] bf16; lse [B][Tq][H] fp32 or NULL.                     */
sa_status csa_sparse_attn(const void* q, int32_t Tq, int32_t H, const sa_cache* csa,
                          const int32_t* idx, const int32_t* cnt, int32_t k, float scale,
                          void* out, float* lse, void* ws, size_t ws_bytes, void* stream);

/* HCA dense attention over every visible entry, section 3-2 (2) (HCA keeps
 * dense attention, no selection).  q_pos as in csa_index_topk (NULL = decode,
 * all n[b] entries visible).  Shapes as csa_sparse_attn.                     */
sa_status hca_dense_attn(const void* q, int32_t Tq, int32_t H, const int32_t* q_pos,
                         const sa_cache* hca, float scale, void* out, float* lse,
                         void* ws, size_t ws_bytes, void* stream);

/* One decode step of both branches for B sequences (one new query each):
 * indexer + top-k + CSA attention, and HCA attention.
 *   q [B][H][d] bf16, q_idx [B][d_idx] bf16.
 *   out_csa, out_hca [B][H][d] bf16; lse_csa, lse_hca [B][H] fp32 or NULL.
 *   idx_out [B][k] / cnt_out [B] int32, or NULL to keep them in the workspace. */
sa_status hybrid_attn_decode(const void* q, const void* q_idx, int32_t H,
                             const sa_cache* csa, const sa_cache* hca, int32_t k, float scale,
                             void* out_csa, void* out_hca, float* lse_csa, float* lse_hca,
                             int32_t* idx_out, int32_t* cnt_out,
                             void* ws, size_t ws_bytes, void* stream);

/* hybrid_attn_prefill with the CSA selection on FP4 indexer scores (the
 * prefill selection of csa_index_topk_mxfp4; codes / scales as written by
 * csa_index_quantize_mxfp4).  Same workspace, shapes and outputs; the bf16
 * indexer keys of the CSA cache are not read and may be NULL.               */
sa_status hybrid_attn_prefill_mxfp4(const void* q, const void* q_idx, int32_t T, int32_t H,
                                    const sa_cache* csa, const sa_cache* hca,
                                    const uint8_t* codes, const uint8_t* scales, int32_t k, float scale,
                                    void* out_csa, void* out_hca, float* lse_csa, float* lse_hca,
                                    int32_t* idx_out, int32_t* cnt_out,
                                    void* ws, size_t ws_bytes, void* stream);

/* A hybrid decode step captured once into a CUDA graph together with its
 * host copies, for a serving loop that decodes the same batch step after
 * step: one cudaGraphLaunch per step copies the new queries in from pinned
 * host memory, runs hybrid_attn_decode (or hybrid_attn_decode_mxfp4) and
 * copies both outputs and both lse back to pinned host memory.  The review
 * (section 3-2 (2)) defines the step; the graph and the packed copies are
 * this library's own serving form of it, with no counterpart on the page.
 *
 * Packed I/O, the same layout on the host and on the device (byte offsets
 * from sa_decode_io_layout, each a multiple of 256):
 *   in:  q_idx [B][d_idx] bf16 at q_idx_off, q [B][H][d] bf16 at q_off;
 *   out: out_hca [B][H][d] bf16, lse_hca [B][H] fp32, out_csa, lse_csa.
 * The HCA half of `out` (out_hca, lse_hca) is copied back as soon as the
 * HCA branch ends, overlapping the CSA branch; the CSA half at the end.     */
typedef struct {
    size_t in_bytes, q_idx_off, q_off;
    size_t out_bytes, out_hca_off, lse_hca_off, out_csa_off, lse_csa_off;
} sa_decode_io;

/* Fills *io for B sequences and H heads (B >= 1, H 1..128).                */
sa_status sa_decode_io_layout(int32_t B, int32_t H, sa_decode_io* io);

typedef struct sa_decode_graph sa_decode_graph;

/* How the step moves its I/O (flags of sa_decode_graph_create):
 *   0                    copy-engine copies: host_in -> dev_in before the
 *                        step, dev_out -> host_out after each branch;
 *   SA_DG_KERNEL_IN      the queries are copied by a kernel that reads
 *                        host_in through its device mapping;
 *   SA_DG_DIRECT_OUT     the attention kernels write both outputs and both
 *                        lse straight into host_out through its device
 *                        mapping (no copy after the step; dev_out unused).
 * The mapped forms need host buffers that the device can address (pinned
 * memory on a system with unified addressing, where cudaHostAlloc memory is
 * mapped); otherwise SA_ERR_INVALID_ARG.                                     */
#define SA_DG_KERNEL_IN 1u
#define SA_DG_DIRECT_OUT 2u

/* Captures the step.  The caller owns every buffer and keeps it alive (and
 * at the same address) until sa_decode_graph_destroy:
 *   host_in, host_out: PINNED host memory (cudaHostAlloc or
 *     cudaHostRegister) of io.in_bytes / io.out_bytes; pageable memory is
 *     rejected with SA_ERR_INVALID_ARG;
 *   dev_in, dev_out: device memory of the same sizes (dev_out may be NULL
 *     with SA_DG_DIRECT_OUT);
 *   idx_out [B][k] / cnt_out [B] int32 device, or both NULL;
 *   ws / ws_bytes as for hybrid_attn_decode;
 *   codes / scales: the MXFP4 indexer (as for hybrid_attn_decode_mxfp4), or
 *     both NULL for the bf16 indexer keys;
 *   flags: 0 or an OR of SA_DG_KERNEL_IN and SA_DG_DIRECT_OUT.
 * The caches are read in place at every step, so appends between steps are
 * seen; their struct fields (pointers, capacities) are fixed at capture, and
 * so are the library options.  Unlike the other calls, this one runs the
 * step once eagerly and synchronises the device before capturing (on a
 * stream of its own).  On success *graph receives the handle.               */
sa_status sa_decode_graph_create(const sa_cache* csa, const sa_cache* hca, int32_t H, int32_t k, float scale,
                                 const uint8_t* codes, const uint8_t* scales, void* host_in, void* host_out,
                                 void* dev_in, void* dev_out, int32_t* idx_out, int32_t* cnt_out, void* ws,
                                 size_t ws_bytes, uint32_t flags, sa_decode_graph** graph);

/* Launches one captured step on `stream`.  host_in must hold the step's
 * queries when the launch runs; host_out holds the results once `stream`
 * has reached the end of the step (synchronise or wait on an event).       */
sa_status sa_decode_graph_step(sa_decode_graph* graph, void* stream);

/* Frees the graph (not the caller's buffers).  NULL is accepted.           */
sa_status sa_decode_graph_destroy(sa_decode_graph* graph);

/* hybrid_attn_decode with the sliding-window branch of both layers: the
 * review (section 3-2 (2)) adds a window of recent uncompressed tokens to CSA
 * and to HCA alike.  out_csa is the attention over the CSA selection joined
 * with the last `window` raw tokens, out_hca over the HCA entries joined with
 * the same window (one softmax over each union: the log-sum-exp merge of the
 * branch and the window, as attn_lse_merge computes it).
 *   raw: the raw tokens (k, v [B][Lcap][d] bf16, len [B]) as for swa_attn;
 *        its B must equal the caches'.
 *   lse_csa / lse_hca: the lse of each union, or NULL.
 * ws / ws_bytes: at least sa_workspace_size(SA_OP_HYBRID_DECODE_SWA, B, 1, H,
 * Ncap_csa, Ncap_hca, k) (independent of the window).                      */
sa_status hybrid_attn_decode_swa(const void* q, const void* q_idx, int32_t H,
                                 const sa_cache* csa, const sa_cache* hca, const sa_raw* raw, int32_t window,
                                 int32_t k, float scale, void* out_csa, void* out_hca, float* lse_csa,
                                 float* lse_hca, int32_t* idx_out, int32_t* cnt_out,
                                 void* ws, size_t ws_bytes, void* stream);

/* hybrid_attn_decode with the CSA selection on FP4 indexer scores (the
 * selection of csa_index_topk_mxfp4; codes / scales as written by
 * csa_index_quantize_mxfp4).  Same workspace, shapes and outputs; the bf16
 * indexer keys of the CSA cache are not read and may be NULL.               */
sa_status hybrid_attn_decode_mxfp4(const void* q, const void* q_idx, int32_t H,
                                   const sa_cache* csa, const sa_cache* hca,
                                   const uint8_t* codes, const uint8_t* scales, int32_t k, float scale,
                                   void* out_csa, void* out_hca, float* lse_csa, float* lse_hca,
                                   int32_t* idx_out, int32_t* cnt_out,
                                   void* ws, size_t ws_bytes, void* stream);

/* Causal prefill of both branches: T queries per sequence at token positions
 * 0..T-1 over caches compressed from those same tokens.
 *   q [B][T][H][d] bf16, q_idx [B][T][d_idx] bf16.
 *   out_csa, out_hca [B][T][H][d] bf16; lse_* [B][T][H] fp32 or NULL.
 *   idx_out [B][T][k] and cnt_out [B][T] int32 are required.                  */
sa_status hybrid_attn_prefill(const void* q, const void* q_idx, int32_t T, int32_t H,
                              const sa_cache* csa, const sa_cache* hca, int32_t k, float scale,
                              void* out_csa, void* out_hca, float* lse_csa, float* lse_hca,
                              int32_t* idx_out, int32_t* cnt_out,
                              void* ws, size_t ws_bytes, void* stream);

/* Bytes of scratch an operation needs (0 on invalid sizes).  Ncap_csa /
 * Ncap_hca are the capacities of the two caches (pass 0 for one that the
 * operation does not use).  The scratch must be device memory, 256-byte
 * aligned, zeroed once before its first use; calls sharing one scratch
 * buffer must be ordered on one stream.                                      */
size_t sa_workspace_size(int32_t op, int32_t B, int32_t Tq, int32_t H,
                         int32_t Ncap_csa, int32_t Ncap_hca, int32_t k);

/* Synchronises `stream`, reads the device status word that every kernel of
 * the library records its device-side anomalies in (one word per device,
 * shared by all callers in the process), clears it, and returns SA_OK,
 * SA_ERR_TIMEOUT or SA_ERR_DEVICE.                                           */
sa_status sa_read_device_status(void* stream);

/* Failure-detection self-test.  Every cross-CTA wait in the library is
 * bounded: a wait that runs out records a timeout in the device status word
 * and its kernel returns instead of hanging or trapping.  This launches one
 * small kernel whose wait on a barrier that nothing completes gives up after
 * wait_tries polls (1..4194304; 65536 takes well under a second); the next
 * sa_read_device_status then returns SA_ERR_TIMEOUT, and the context stays
 * usable.  A diagnostic only: the method has no counterpart.               */
sa_status sa_selftest_wait_timeout(uint32_t wait_tries, void* stream);

/* Device timelines (a profiling build only).  A library compiled with
 * -DSA_TRACE (libsparse_attn_trace.so) has per-CTA phase marks in its
 * decode-path kernels and in the prefill indexer's score and selection
 * kernels: thread 0 of a CTA appends a 16-byte record
 *   { uint64 t_ns (%globaltimer); uint16 kernel; uint16 phase; uint16 sm;
 *     uint16 cta (blockIdx.x + gridDim.x * blockIdx.y, mod 2^16) }
 * kernel: 1 indexer score, 2 filter, 3 resolve, 4 emit, 5 attention split,
 * 6 split merge, 7 FP4 indexer score, 8 prefill indexer score, 9 prefill
 * selection, 10 FP4 prefill indexer score, 11 prefill selection (second
 * form, SA_OPT_PREFILL_SELECT = 2), 12 sampled bound and 13 fast selection
 * (SA_OPT_DECODE_FAST = 1), 14 prefill selection (fourth form, the
 * default), 15 prefill attention on the transposed kernel (per tile of the
 * gathered lists of CTA 0's last two queries; the record's cta field holds
 * the tile: 16 * (query parity) + tile).  Phases: score 0 start, 1 scan
 * done, 2 threshold found (last CTA); filter 0 start, 1 rows done; resolve 0
 * start, 1 counts scanned, 2 candidates gathered, 3 t~ known, 4 band done,
 * 5 cut done, 6 positions written; emit, attention 0 start, 1 end; merge 0;
 * prefill scores (CTAs whose tile some query sees) 0 start, 1 operands
 * staged, 2 end; prefill selection (one CTA per query) 0 start, then, when
 * the query sees more than k entries, 1 keys staged, 2..4 digits 1..3
 * found, 5 ties resolved (second form: per-warp counts done), 6 end;
 * fourth form 0 start, 1 keys staged, 2 threshold found, 3 runs counted,
 * 4 end; prefill attention 0 tile start, 1 scores ready, 2 softmax done,
 * 3 copies landed (barrier), 4 MMAs issued, 5 next copies out.
 * sa_trace_install(buf, capacity) waits for `stream`, then makes buf (device
 * memory, 16-byte aligned, capacity records) the destination and resets the
 * count; capacity 0 switches tracing off.  sa_trace_count waits for `stream`
 * and returns the records written (marks past capacity are dropped but
 * counted).  The default library returns SA_ERR_UNSUPPORTED from both.    */
sa_status sa_trace_install(void* buf, uint32_t capacity, void* stream);
sa_status sa_trace_count(uint32_t* n, void* stream);

/* Text for the last non-OK status returned on the calling host thread.      */
const char* sa_last_error(void);

/* SA_ABI_VERSION of the loaded library.                                      */
int32_t sa_abi_version(void);

/* Stages of a decode step, for sa_set_stage_events.                          */
typedef enum {
    SA_STAGE_INDEX_SCORE = 0,  /* indexer score kernel (streams the indexer keys) */
    SA_STAGE_TOPK_SELECT = 1,  /* threshold search + ordered selection kernels    */
    SA_STAGE_CSA_ATTN = 2,     /* CSA attention (+ its split merge)                */
    SA_STAGE_HCA_ATTN = 3,     /* HCA attention (+ its split merge)                */
    SA_NUM_STAGES = 4
} sa_stage;

/* Tracing hook: while set, every decode-path call made on the calling host
 * thread records `before` and `after` (cudaEvent_t passed as void*) on its
 * stream immediately around the kernels of `stage`.  NULL, NULL switches the
 * stage off.  The events are the caller's; the library only records them.   */
sa_status sa_set_stage_events(int32_t stage, void* before, void* after);

/* Maximum scratch of csa_index_topk_noalloc, per device.                    */
#define SA_NOALLOC_SCRATCH_BYTES (32u << 20)

/* csa_index_topk for callers that cannot allocate device memory.  (The paper
 * has no counterpart: this is a deployment convenience.)  Some callers cannot
 * give the library a workspace: a C caller that only holds its input and
 * output buffers, or a serving loop whose device memory is entirely owned by
 * another allocator and which may not call cudaMalloc (that call can also
 * synchronise the device, which such a loop cannot afford).  This entry point
 * computes the same decode top-k as csa_index_topk with q_pos == NULL and
 * Tq == 1, bit for bit, but takes its scratch from a static device array of
 * SA_NOALLOC_SCRATCH_BYTES that the library owns: every GPU that loads the
 * library holds that array until the process exits.  It allocates and frees
 * nothing.  The first call on a device looks the array's address up
 * (cudaGetSymbolAddress) and should therefore come before any stream capture.
 * All calls on a device share the one array, which keeps the last call's
 * contents (each call clears what it needs): calls whose work overlaps on the
 * GPU, on different streams or host threads, race and must not be issued.
 * Returns SA_ERR_UNSUPPORTED when B, Ncap and k need more scratch than the
 * array holds (for example B = 4, Ncap = 262144, k = 2048 needs about 21 MB).
 *   q_idx [B][d_idx] bf16; idx [B][k] and cnt [B] int32 out, as csa_index_topk. */
sa_status csa_index_topk_noalloc(const void* q_idx, const sa_cache* csa, int32_t k, int32_t* idx, int32_t* cnt,
                                 void* stream);

/* ---- Context-parallel decode -------------------------------------------
 * The review's section 3-2 (4) lists contextual parallelism among the
 * inference infrastructure without describing it; the exchange here is this
 * library's own.  One sequence's compressed entries are split over W ranks in
 * contiguous shards, rank w holding global entries base[b] .. base[b] +
 * n[b] - 1 of sequence b (shards in rank order, shard boundaries on whole
 * HCA blocks).  Because every entry of the global top-k is in the top-k of
 * its own shard, a step is exact:
 *   1. cp_decode_candidates on every rank;
 *   2. all-gather of (keys, gidx, gcnt) in rank order (W x the arrays);
 *   3. cp_decode_merge_select on every rank: its share of the global top-k;
 *   4. csa_sparse_attn over that share and hca_dense_attn over the HCA
 *      shard, each with its lse;
 *   5. all-gather of the partial (out, lse) and attn_lse_merge_n.
 * The collectives are the caller's (NCCL through torch.distributed in the
 * Python binding); these calls are the per-rank compute.                   */

/* Exact local top-k of this rank's CSA shard for B decode queries, then the
 * exact order key and global index of each winner (the four int32 arrays
 * need 4-byte alignment: they may sit packed in one buffer).
 *   base  [B] int32: global index of the shard's entry 0.
 *   keys  [B][k] uint32 out: order key of the winner's fp32 score s: the
 *         bits of s with the sign bit set for s >= 0, all bits flipped for
 *         s < 0 (-0 counts as +0); 0 past the count.
 *   gidx  [B][k] int32 out: global indices, ascending, -1 past the count.
 *   gcnt  [B] int32 out: min(k, n[b]).
 * ws / ws_bytes: at least sa_workspace_size(SA_OP_CP_CANDIDATES, B, 1, H,
 * Ncap, 0, k).                                                              */
sa_status cp_decode_candidates(const void* q_idx, const sa_cache* csa, int32_t k, const int32_t* base,
                               uint32_t* keys, int32_t* gidx, int32_t* gcnt, void* ws, size_t ws_bytes,
                               void* stream);

/* The global top-k from the gathered candidates of all W ranks and this
 * rank's share of it.
 *   keys, gidx, gcnt: rank w's candidate arrays ([B][k], [B][k], [B]) start
 *              at keys + w * stride_list, gidx + w * stride_list and
 *              gcnt + w * stride_cnt (elements): arrays stacked in rank order
 *              (stride_list = B*k, stride_cnt = B), or one packed
 *              [keys | gidx | gcnt] int32 buffer per rank gathered whole
 *              (both strides = 2*B*k + B), which needs one all-gather.
 *   base [B]: this rank's shard start (as given to cp_decode_candidates).
 *   local_idx [B][k] int32 out: this rank's winners as shard-local indices,
 *              ascending, -1 padded; local_cnt [B] out: their count.
 *   sel_idx [B][k] / sel_cnt [B] out, or both NULL: the global selection,
 *              ascending, -1 padded, and min(k, total candidates).
 * W * k must be at most 16384 (SA_ERR_UNSUPPORTED otherwise).              */
sa_status cp_decode_merge_select(const uint32_t* keys, const int32_t* gidx, const int32_t* gcnt, int64_t stride_list,
                                 int64_t stride_cnt, int32_t W, int32_t B, int32_t k, int32_t rank,
                                 const int32_t* base, int32_t* local_idx, int32_t* local_cnt, int32_t* sel_idx,
                                 int32_t* sel_cnt, void* stream);

/* W-way log-sum-exp merge of attentions over disjoint key sets:
 * lse = log sum_w e^lse_w, out = sum_w e^lse_w out_w / e^lse.
 *   part w's [rows][128] bf16 outputs start at outs + w * stride_out and its
 *   [rows] fp32 lse at lses + w * stride_lse (elements; stride_out a multiple
 *   of 8): stacked arrays, or one gathered byte buffer per part.
 *   out [rows][128] bf16, lse [rows] fp32 or NULL.  A row whose lses are all
 *   -inf gets 0, -inf.                                                        */
sa_status attn_lse_merge_n(const void* outs, const float* lses, int32_t W, int64_t rows, int64_t stride_out,
                           int64_t stride_lse, void* out, float* lse, void* stream);

/* Number of kernels this library has launched from the calling host thread
 * since the process started (a diagnostic counter; memsets are not kernels). */
uint64_t sa_launch_count(void);

/* Library options: process-wide, read when a call enqueues its kernels (so a
 * CUDA graph keeps the choice it was captured with).  Host-only: no device
 * work, callable without a GPU.
 *   SA_OPT_PREFILL_SELECT  the selection kernel of the causal prefill top-k
 *     (csa_index_topk / csa_index_topk_mxfp4 with Tq > 1, and the hybrid
 *     prefill calls).  Every form gives the same indices, the exact top-k of
 *     section 3-2 (4) of the review with the lowest-index tie-break:
 *       1            one 1024-thread CTA per query: three radix-digit
 *                    passes over the query's keys, a tie pass and an
 *                    ordered block-scan compaction;
 *       2            the first digit over the keys, the second and third
 *                    over the threshold bin's keys only (a short list in
 *                    shared memory), then warp-chunked counting and ordered
 *                    output with the ties taken in the same pass;
 *       3            form 2 in 512-thread CTAs that read the keys from the
 *                    scratch on every pass instead of staging them, so
 *                    that three queries share an SM;
 *       4 (default)  one 512-thread CTA per query, two per SM: the
 *                    scores' mean and deviation, one pass over 256 linear
 *                    score bins counted in per-warp histograms, the
 *                    threshold ranked inside its bin, then one counting
 *                    pass and an ordered output by contiguous runs (28 ms
 *                    of selection became 12 ms on the 128K-token prefill
 *                    with k = 2048).
 *   SA_OPT_DECODE_FAST  the indexer and top-k of the hybrid decode calls
 *     (hybrid_attn_decode, hybrid_attn_decode_swa) with bf16 indexer keys
 *     and k <= 2048.  Every value gives the same indices (the exact top-k)
 *     and the same outputs:
 *       1            three kernels: a sampled bound on the k-th score, the
 *                    indexer scan keeping the entries above that bound as
 *                    candidates (with a histogram of their scores), and one
 *                    CTA per sequence that selects exactly from the
 *                    candidates (or, when they cannot prove the selection,
 *                    from every score);
 *       2            the same kernels, the selection always from every
 *                    score (the fallback, for testing);
 *       0 (default)  the general kernels (scan, filter, resolve, emit), as
 *                    for csa_index_topk; on a B200 they measured faster
 *                    at a 1M-token context (64 us per step against 67).
 *   SA_OPT_HCA_PREFILL  the kernel of the dense (HCA) causal prefill with
 *     query positions and a bf16 cache (hca_dense_attn with q_pos, the
 *     hybrid prefill calls).  Same outputs up to the order of the fp32
 *     sums (both within the bf16 tolerance of the definition):
 *       0 (default)  the transposed tensor-memory kernel (128 entries per
 *                    MMA): with exactly 64 heads and an even m, two query
 *                    positions per tile (2 x 64 heads as the MMA's N);
 *                    otherwise one query at a time (<= 64 heads);
 *       1            the two-query kernel (2 queries x 64 heads per 128-row
 *                    MMA; exactly 64 heads);
 *       2            the transposed kernel one query at a time.
 * sa_set_option returns SA_ERR_INVALID_ARG for an unknown option or value;
 * sa_get_option writes the current value to *value.                        */
typedef enum { SA_OPT_PREFILL_SELECT = 1, SA_OPT_DECODE_FAST = 2, SA_OPT_HCA_PREFILL = 3 } sa_option;
sa_status sa_set_option(int32_t option, int64_t value);
sa_status sa_get_option(int32_t option, int64_t* value);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_H */
