/*
 * absp.h -- C ABI of the adaptive-block sparse decode attention library
 * (libabsp.so, CUDA, sm_100a).
 *
 * The method is AB-Sparse: Sparse Attention with Adaptive Block Size
 * (arXiv 2605.12110).  Its decode path, as its review page describes it:
 *   - Fig. 1: keys are grouped into blocks; each block is represented by a
 *     centroid; a query-centroid dot product scores each block; the top-K
 *     blocks are selected; attention runs over their keys only.
 *   - Fig. 3 / Fig. 5: each KV head has its own block size in {16, 32, 64},
 *     fixed offline, so centroids are built once over all keys.
 *   - Fig. 8 / abstract: centroids are kept as INT4 codes, asymmetric,
 *     with per-channel parameters.
 *   - Fig. 9: logical blocks are runs of consecutive 16-token physical
 *     pages (block size / 16 pages per block); every head reads the same
 *     number of pages, i.e. the budget is in tokens.
 *
 * Conventions shared by every call:
 *   - All buffers are owned by the caller.  Pointers marked "device" must
 *     be device memory of the current CUDA device; "host" means host memory.
 *     The library never allocates device memory.
 *   - Every call that launches work is asynchronous on `stream` (a
 *     cudaStream_t passed as void*; NULL is the legacy default stream).
 *   - Host-side argument checks return an error status before anything is
 *     launched.  Faults detected on the device (a page id or block index
 *     out of range, a length beyond the page table, a wait that timed out)
 *     are recorded in the first bytes of the workspace and reported by
 *     absp_check_device_error(); kernels never trap.
 *   - head_dim must be 128 and page_size 16 (ABSP_ERR_UNSUPPORTED otherwise).
 *   - Calls that only launch work on `stream` may be captured into a CUDA
 *     graph, in any capture mode, including the first launch of a kernel in
 *     the process (its one-time set-up never touches the capturing
 *     stream).  Not capturable: absp_check_device_error (it waits for the
 *     stream) and the first absp_build_quantize_noalloc call per device.
 *   - No call throws; every call returns an absp_status.
 */
#ifndef ABSP_H_
#define ABSP_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ABSP_API __attribute__((visibility("default")))
#else
#define ABSP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t absp_status;
#define ABSP_OK 0
#define ABSP_ERR_INVALID_ARG 1   /* null pointer, bad size, misalignment   */
#define ABSP_ERR_UNSUPPORTED 2   /* head_dim != 128, page_size != 16, ... */
#define ABSP_ERR_CUDA 3          /* a CUDA runtime call failed            */
#define ABSP_ERR_DEVICE_FAULT 4  /* a device-side bounds check fired      */
#define ABSP_ERR_TIMEOUT 5       /* a device-side bounded wait gave up    */

#define ABSP_HEAD_DIM 128
#define ABSP_PAGE_SIZE 16
#define ABSP_CODE_ROW_BYTES 64           /* 128 INT4 codes per centroid    */
#define ABSP_MAX_KV_HEADS 64
#define ABSP_MAX_GROUP 16                /* query heads per KV head        */
#define ABSP_MAX_BLOCKS_PER_HEAD 16384   /* centroid rows per (seq, head)  */
#define ABSP_MAX_BUDGET 65536            /* token budget per KV head       */

/* One attention layer's paged KV cache (Fig. 9: physical pages, logical
 * blocks).  Token t of sequence s lives in physical page
 * page_table[s * max_pages_per_seq + t / 16], slot t % 16.  A page holds all
 * KV heads: k_pages[page][kv_head][slot][channel], bf16, so one
 * (page, head) slice is 4 KiB contiguous.  Query head j belongs to KV head
 * j / (num_q_heads / num_kv_heads) (contiguous GQA grouping). */
typedef struct absp_layer_kv {
    int32_t num_seqs;            /* S >= 1                                  */
    int32_t num_q_heads;         /* Hq, a multiple of Hkv, Hq/Hkv <= 16     */
    int32_t num_kv_heads;        /* Hkv, 1..64                              */
    int32_t head_dim;            /* must be 128                             */
    int32_t page_size;           /* must be 16                              */
    int32_t max_pages_per_seq;   /* page-table row stride (>= 1)            */
    int64_t num_phys_pages;      /* pages in k_pages / v_pages (>= 1)       */
    const int32_t* seq_lens;     /* device [S]; 0 <= len <= 16*max_pages    */
    const int32_t* page_table;   /* device [S][max_pages_per_seq]           */
    const void* k_pages;         /* device bf16, 256-byte aligned           */
    const void* v_pages;         /* device bf16, 256-byte aligned           */
    const int32_t* block_size;   /* HOST [Hkv], each 16, 32 or 64           */
} absp_layer_kv;

/* INT4 centroid store of one layer (Fig. 8: asymmetric, per channel).
 * Head h of sequence s has capacity cap_h = ceil(16*max_pages_per_seq/bs_h)
 * rows; its rows start at row  s * rows_per_seq + base_h  where
 * base_h = sum_{h' < h} cap_h' and rows_per_seq = sum_h cap_h (see
 * absp_centroid_row_offset).  Row b (block b of the head) holds 64 bytes:
 * channel 2i in the low nibble of byte i, channel 2i+1 in the high nibble.
 * Dequantised centroid = (code - zp[s][h][c]) * scale[s][h][c]. */
typedef struct absp_centroids {
    uint8_t* codes;              /* device, 256-byte aligned               */
    float* scale;                /* device [S][Hkv][128]                   */
    int32_t* zp;                 /* device [S][Hkv][128]                   */
    int32_t format;              /* ABSP_CENTROIDS_INT4 (0) or _BF16 (1)   */
} absp_centroids;

/* Centroid storage formats (the precision comparison of Fig. 13: INT4
 * codes vs unquantised BF16 centroids).
 *   ABSP_CENTROIDS_INT4: as above, 64-byte rows of packed nibbles plus
 *     per-channel scale / zp.
 *   ABSP_CENTROIDS_BF16: 256-byte rows, channel c as the bf16 nearest to
 *     the fp64 mean (ties to even, no intermediate rounding); scale and zp
 *     are neither read nor written (may be NULL). */
#define ABSP_CENTROIDS_INT4 0
#define ABSP_CENTROIDS_BF16 1

/* Human-readable name of a status code (static string, never NULL). */
ABSP_API const char* absp_status_string(absp_status status);

/* Identity of the sources this library was compiled from: the first 16 hex
 * digits of a SHA-256 over its CUDA sources, headers, build script and
 * compile flags ("unknown" for a build that did not define it).  Static
 * string, host only, never fails.  The paper has no counterpart: it lets a
 * record of a run name the exact sources that ran. */
ABSP_API const char* absp_build_id(void);

/* Bytes of the three centroid buffers for `kv` (host only, no launch). */
ABSP_API absp_status absp_centroid_sizes(const absp_layer_kv* kv, size_t* codes_bytes,
                                size_t* scale_bytes, size_t* zp_bytes);

/* Bytes of the centroid buffers for a given format (ABSP_CENTROIDS_*);
 * scale / zp bytes are 0 for ABSP_CENTROIDS_BF16. */
ABSP_API absp_status absp_centroid_sizes_fmt(const absp_layer_kv* kv, int32_t format,
                                             size_t* codes_bytes, size_t* scale_bytes,
                                             size_t* zp_bytes);

/* First code row of (seq, kv_head) in absp_centroids.codes (host only);
 * rows are 64 bytes (INT4) or 256 bytes (BF16). */
ABSP_API absp_status absp_centroid_row_offset(const absp_layer_kv* kv, int32_t seq,
                                     int32_t kv_head, int64_t* row);

/* Workspace bytes for absp_build_centroids + absp_quantize_centroids (and
 * absp_build_quantize_centroids): 256 B header + per-channel min/max +
 * fp64 centroids (1 KiB per row). */
ABSP_API absp_status absp_build_workspace_size(const absp_layer_kv* kv, size_t* bytes);

/* Workspace bytes for the decode calls (score/select, sparse decode,
 * decode step, and the host-buffer decode step). */
ABSP_API absp_status absp_decode_workspace_size(const absp_layer_kv* kv,
                                       int32_t budget_tokens, size_t* bytes);

/* Row stride of the block-index list `sel`: max over heads of
 * K_h = max(1, budget / bs_h) (Fig. 9 equal token budget). */
ABSP_API absp_status absp_select_capacity(const absp_layer_kv* kv, int32_t budget_tokens,
                                 int32_t* kmax);

/* Zero-fill a workspace (its error word must start at 0).  Call once per
 * workspace before its first use. */
ABSP_API absp_status absp_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Step 1 (Fig. 1 "block representation", Fig. 5 "centroids over all key
 * vectors"): for every (seq, kv_head, block b) the mean of the block's
 * valid keys, c[b][ch] = (sum_t K[t][ch]) / cnt_b, summed in token order in
 * fp64 (a ragged last block averages its valid tokens only).  Writes the
 * fp64 centroids and the per-channel min/max into `ws` (size from
 * absp_build_workspace_size).  Reads every key of the layer once.
 * Layout of `ws` afterwards: a 256-byte header (the error word), then
 * S * Hkv * 128 * 2 order-mapped 8-byte min / max keys, then the fp64
 * centroids, 128 doubles per row, block b of (seq, kv_head) at row
 * absp_centroid_row_offset(seq, kv_head) + b.
 * The sums are exact whenever a block's nonzero keys span at most 39
 * binades, so the kernel may add them in any exact way (fp32 page sums
 * proved exact by rounding down and up); blocks outside that condition,
 * or holding a zero, subnormal, infinite or NaN key, are summed in token
 * order.  The results are the token-order sums either way. */
ABSP_API absp_status absp_build_centroids(const absp_layer_kv* kv, void* ws,
                                 size_t ws_bytes, void* stream);

/* Step 2 (Fig. 8: INT4 asymmetric per-channel): from the workspace filled by
 * absp_build_centroids, per (seq, kv_head, channel):
 *   scale = fp32((max - min) / 15), zp = rint(-min / scale) (int32, not
 *   clamped to 4 bits), code = clamp(rint(c / scale) + zp, 0, 15),
 * rint = round half to even, all in fp64 except the stored scale; a channel
 * with max == min gets scale 0, zp 0, codes 0.  Writes `out`.  With
 * out->format == ABSP_CENTROIDS_BF16 it writes the bf16-rounded centroids
 * instead (no quantisation). */
ABSP_API absp_status absp_quantize_centroids(const absp_layer_kv* kv, void* ws,
                                    size_t ws_bytes, const absp_centroids* out,
                                    void* stream);

/* Steps 1-2 in one call, with the results of absp_build_centroids followed
 * by absp_quantize_centroids (bit for bit): for INT4 those two steps'
 * launches; for BF16 one launch of the build kernel writing the bf16 rows
 * directly (no fp64 rows, no min / max).  `ws` is sized by
 * absp_build_workspace_size. */
ABSP_API absp_status absp_build_quantize_centroids(const absp_layer_kv* kv, void* ws,
                                                   size_t ws_bytes, const absp_centroids* out,
                                                   void* stream);

/* Incremental update during decode (Fig. 5: block sizes are fixed, so the
 * store is kept up to date instead of rebuilt).  Call after the caller has
 * written the new tokens' K/V into the pages and raised seq_lens.  For every
 * (seq, kv_head) the centroid of the block holding the last token is
 * recomputed from that block's keys (token-order fp64 mean, the value a
 * full rebuild gives) and stored under the EXISTING per-channel scale / zp
 * (INT4: code = clamp(rint(c/scale) + zp, 0, 15)) or as bf16 (BF16 format).
 * The per-channel parameters are not changed.  exceeded (optional, device
 * int32 [S][Hkv]) receives, per (seq, head), the number of channels whose
 * unclamped code left 0..15 (channels with scale 0 are not counted): a
 * non-zero count means the parameters no longer cover the range and a
 * rebuild (steps 1-2) is due.  ws: any decode workspace (error word). */
ABSP_API absp_status absp_append_centroids(const absp_layer_kv* kv, const absp_centroids* cent,
                                           int32_t* exceeded, void* ws, size_t ws_bytes,
                                           void* stream);

/* Steps 3-4 (Fig. 1 "dot product estimation", "importance score",
 * "top-K selection"): for every (seq, kv_head), qbar = sum of the GQA
 * group's queries (q: device bf16 [S][Hq][128]), score[b] =
 * sum_ch qbar[ch] * (code[b][ch] - zp[ch]) * scale[ch] (fp32; with BF16
 * centroids sum_ch qbar[ch] * centroid[b][ch]), then the
 * K_h = min(n_h, max(1, budget / bs_h)) highest scores, ties to the lower
 * block index.  Writes sel[(s*Hkv + h) * kmax + i], i < K_h, ascending
 * block indices (kmax from absp_select_capacity), and sel_count[s*Hkv + h]
 * = K_h.  sel: device int32 [S][Hkv][kmax]; sel_count: device int32
 * [S][Hkv]. */
ABSP_API absp_status absp_score_select(const absp_layer_kv* kv, const absp_centroids* cent,
                              const void* q, int32_t budget_tokens, int32_t* sel,
                              int32_t* sel_count, void* ws, size_t ws_bytes,
                              void* stream);

/* Step 5 (Fig. 1 "sparse attention"): for every query head j of KV head h,
 * out[s][j] = softmax_t(q_j . K_t / sqrt(128)) V over the valid tokens of
 * the blocks listed in sel / sel_count (layout as written by
 * absp_score_select for the same budget_tokens), gathered through the page
 * table.  bf16 in, fp32 accumulation, bf16 out (device [S][Hq][128]).  A
 * head with no valid token gets a zero output.  Block indices out of range
 * are skipped and reported as ABSP_ERR_DEVICE_FAULT. */
ABSP_API absp_status absp_sparse_decode(const absp_layer_kv* kv, const void* q,
                               const int32_t* sel, const int32_t* sel_count,
                               int32_t budget_tokens, void* out, void* ws,
                               size_t ws_bytes, void* stream);

/* Steps 3-5 in one launch: score, select and attend, with the selection
 * kept on chip.  Same results as absp_score_select followed by
 * absp_sparse_decode. */
ABSP_API absp_status absp_decode_step(const absp_layer_kv* kv, const absp_centroids* cent,
                             const void* q, int32_t budget_tokens, void* out,
                             void* ws, size_t ws_bytes, void* stream);

/* Flags of absp_decode_step_ex / absp_score_select_ex. */
#define ABSP_STEP_EARLY_PREFETCH 1u
#define ABSP_STEP_GROUP_MAX 2u
/* ABSP_STEP_GROUP_MAX: the variant aggregation of a GQA group's queries: a
 * block's score is max_j q_j . centroid over the group's query heads
 * (fp32 per head) instead of qbar . centroid with qbar the group sum. */
/* ABSP_STEP_EARLY_PREFETCH: the launch overlaps the tail of the preceding
 * kernel in `stream` (programmatic dependent launch) and, before waiting for
 * it, already reads the sequence lengths, page table, centroid codes and
 * per-channel parameters; only the query is read after the wait.  The
 * caller guarantees that the kernel issued immediately before this call in
 * `stream` writes none of those buffers (it may write `q`).  This is the
 * decode-loop case: the cache and centroids of a layer were written by
 * earlier steps, the query by the kernel just before.  Without the flag
 * nothing is read before the preceding kernel has completed. */

/* ABSP_STEP_DIAG_WAIT_TIMEOUT: a diagnostic of the failure path, not a
 * decode variant (the paper has no counterpart).  The launch runs a kernel
 * instance whose score-exchange barrier expects 16 bytes more than the
 * cluster sends and whose bounded waits give up after 1 ms instead of 1 s:
 * that wait runs out, the kernel records ABSP_ERR_TIMEOUT (detail 4, the
 * score wait) in the workspace, carries on to its normal end and returns.
 * Its selection and output are then meaningless; the next call on the same
 * workspace, after absp_check_device_error has read and cleared the error
 * word, runs normally.  Only with INT4 centroids, sum aggregation, a GQA
 * group of at most 8 and without ABSP_STEP_EARLY_PREFETCH
 * (ABSP_ERR_UNSUPPORTED otherwise). */
#define ABSP_STEP_DIAG_WAIT_TIMEOUT 0x100u
/* ABSP_STEP_THROUGHPUT: a hint that the caller overlaps this launch with
 * other independent launches (separate requests on several streams, no
 * dependency between them).  Each (seq, kv_head) then gets half as many
 * CTAs, each doing twice the work, so that more launches are resident at
 * once: longer per launch, more launches per second in aggregate.  The
 * selection is the same; the output differs from the default only in the
 * order of the softmax merge's partial sums (fp32 rounding). */
#define ABSP_STEP_THROUGHPUT 0x4u

/* absp_decode_step with flags (ABSP_STEP_EARLY_PREFETCH, ABSP_STEP_GROUP_MAX,
 * ABSP_STEP_THROUGHPUT, ABSP_STEP_DIAG_WAIT_TIMEOUT; other bits are
 * rejected).  Without ABSP_STEP_GROUP_MAX, ABSP_STEP_THROUGHPUT and the
 * diagnostic, same results as absp_decode_step. */
ABSP_API absp_status absp_decode_step_ex(const absp_layer_kv* kv, const absp_centroids* cent,
                                         const void* q, int32_t budget_tokens, void* out,
                                         void* ws, size_t ws_bytes, uint32_t flags,
                                         void* stream);

/* absp_score_select with flags (0, ABSP_STEP_GROUP_MAX or
 * ABSP_STEP_DIAG_WAIT_TIMEOUT). */
ABSP_API absp_status absp_score_select_ex(const absp_layer_kv* kv, const absp_centroids* cent,
                                          const void* q, int32_t budget_tokens, int32_t* sel,
                                          int32_t* sel_count, void* ws, size_t ws_bytes,
                                          uint32_t flags, void* stream);

/* absp_decode_step with HOST query and output buffers (bf16 [S][Hq][128]).
 * When both are pinned and mapped into the device address space (pinned
 * allocations are, under unified addressing), the kernel reads q_host and
 * writes out_host directly across the host link; otherwise q_host is copied
 * into the workspace, the step runs, and the result is copied back to
 * out_host, all on `stream` (pin the buffers for true asynchrony).  The
 * caller synchronises `stream` before reading out_host. */
ABSP_API absp_status absp_decode_step_host(const absp_layer_kv* kv,
                                  const absp_centroids* cent, const void* q_host,
                                  int32_t budget_tokens, void* out_host, void* ws,
                                  size_t ws_bytes, void* stream);

/* absp_decode_step_host with the flags of absp_decode_step_ex
 * (ABSP_STEP_EARLY_PREFETCH, ABSP_STEP_GROUP_MAX; other bits are rejected).
 * With ABSP_STEP_EARLY_PREFETCH the cache-side reads (lengths, page table,
 * centroid codes and parameters) start before the preceding launch on
 * `stream` has completed; only the query is read after it. */
ABSP_API absp_status absp_decode_step_host_ex(const absp_layer_kv* kv,
                                     const absp_centroids* cent, const void* q_host,
                                     int32_t budget_tokens, void* out_host, void* ws,
                                     size_t ws_bytes, uint32_t flags, void* stream);

/* Allocation-free steps 1-2.  The paper has no counterpart to this call;
 * it exists for callers that cannot allocate device memory where they build
 * a layer's centroids (code inside a framework that owns all device memory
 * through its own pool, or on a path where cudaMalloc is forbidden or would
 * synchronise the device).  Same results as absp_build_centroids followed
 * by absp_quantize_centroids, but the workspace is a static array of
 * ABSP_NOALLOC_BUILD_WS_BYTES bytes inside the library instead of a caller
 * buffer; the caller passes only the layer and the centroid buffers.
 *   - Layers whose absp_build_workspace_size exceeds that size are
 *     rejected with ABSP_ERR_UNSUPPORTED before anything is launched.
 *   - No device memory is allocated by the call.  The array itself is held
 *     on every GPU where the library's module is loaded, until the process
 *     exits: from the first call on that GPU under lazy module loading (the
 *     CUDA default), from context creation on every GPU the process uses
 *     under CUDA_MODULE_LOADING=EAGER.
 *   - The first call on each device looks the array's device address up on
 *     the host (with that device current), and so does the first call after
 *     the device's context changed (after a cudaDeviceReset, say); make such
 *     a call before any stream capture.
 *   - All calls on a GPU share the array; each call clears what must start
 *     at zero.  Calls whose GPU work can overlap (unordered streams) race on
 *     the array and must be ordered by the caller.
 *   - device_status (optional, device memory, 2 x int32, may be NULL)
 *     receives {error code, detail} of the device-side checks when the work
 *     completes: 0 or ABSP_ERR_DEVICE_FAULT / ABSP_ERR_TIMEOUT. */
#define ABSP_NOALLOC_BUILD_WS_BYTES (16u << 20)
ABSP_API absp_status absp_build_quantize_noalloc(const absp_layer_kv* kv,
                                                 const absp_centroids* out,
                                                 int32_t* device_status, void* stream);

/* Synchronises `stream`, reads the workspace's error word and clears it.
 * Returns ABSP_OK, ABSP_ERR_DEVICE_FAULT or ABSP_ERR_TIMEOUT; *detail (if
 * not NULL) receives the first faulting sequence/unit index. */
ABSP_API absp_status absp_check_device_error(void* ws, size_t ws_bytes, void* stream,
                                    int32_t* detail);

/* The CUDA error behind the most recent ABSP_ERR_CUDA that a call of this
 * library returned on the calling thread (0 if none yet): a cudaError_t, or
 * for a tensor-map encoding failure the driver's CUresult (the two agree on
 * the common codes).  Host only, never launches, never fails. */
ABSP_API int absp_last_cuda_error(void);

/* cudaGetErrorString of absp_last_cuda_error(), "no error" when it is 0.
 * The string is static; do not free it. */
ABSP_API const char* absp_last_cuda_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* ABSP_H_ */
