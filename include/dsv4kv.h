/*
 * dsv4kv — decode attention over DeepSeek-V4-style hybrid compressed KV caches
 * on NVIDIA B200 (sm_100a).  C ABI.
 *
 * Sources the operations follow (web pages, cited by title and section):
 *  [P1] "How DeepSeek V4 Uses Less Memory: KV Cache Explained"
 *  [P2] "DeepSeek V4 KV Cache" visual walkthrough
 *  [P3] "KV cache at 890 bytes per token: how DeepSeek squeezed attention memory"
 *
 * Conventions shared by every call
 *  - Every pointer argument that names tensor data is DEVICE memory owned by
 *    the caller (for example allocated through PyTorch).  The library keeps
 *    no pointer after a call returns and allocates no device memory on any
 *    call path; scratch memory is the caller's workspace.  The one exception
 *    is dsv4kv_index_topk_noalloc, whose scratch is a library-owned static
 *    device array shared by all its calls (calls to it that overlap on the
 *    GPU race).
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream) and never synchronises the host.
 *  - Tensors are dense and row-major with the shapes given below.
 *  - bf16 data is passed as 16-bit words (IEEE binary32 upper halves).
 *  - Return value: DSV4KV_OK or an error code; on an error nothing was
 *    launched (DSV4KV_ERR_CUDA: a launch failed — the text is in
 *    dsv4kv_last_error(), and the workspace must be zero-filled again).
 *  - Workspaces: `*_workspace_bytes` gives the size; a workspace is 16-byte
 *    aligned (as every cudaMalloc'd block is; the decode calls return
 *    DSV4KV_ERR_INVALID_ARG otherwise), and it must be
 *    zero-filled once before its first use and is left in that state by every
 *    successful call, so it can be reused by the next call on the same stream.
 *    Calls that run concurrently need separate workspaces.  The first 4 bytes
 *    of a workspace are a sticky device status word: kernels OR the
 *    DSV4KV_DEV_* flags below into it and never trap or hang; the caller
 *    reads and clears it.
 */
#ifndef DSV4KV_H_
#define DSV4KV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSV4KV_OK = 0,
  DSV4KV_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer  */
  DSV4KV_ERR_UNSUPPORTED = 2,  /* a format or dimension the library lacks    */
  DSV4KV_ERR_WORKSPACE = 3,    /* workspace null or smaller than required     */
  DSV4KV_ERR_CUDA = 4          /* CUDA runtime/driver error at launch         */
} dsv4kv_status;

/* Device status flags (OR-ed into the first word of a workspace). */
#define DSV4KV_DEV_BAD_INDEX 0x1u  /* a selected index was outside [0, n): row skipped */
#define DSV4KV_DEV_TIMEOUT 0x2u    /* a bounded wait gave up: outputs are invalid       */
#define DSV4KV_DEV_INCONSISTENT 0x4u /* selection counts disagreed: outputs are invalid */
#define DSV4KV_DEV_BAD_POOL 0x8u     /* a candidate pool was not ascending: ties may differ */
#define DSV4KV_DEV_BAD_PAGE 0x10u    /* a block-table page number was outside the pool: its rows skipped */
#define DSV4KV_DEV_BAD_LENGTH 0x20u  /* a sequence length was < 0 or > t_max: clamped into [0, t_max] */

/* Cache row formats.
 *  DSV4KV_BF16:          codes = bf16 [B][rows][dim]; scales = NULL.
 *  DSV4KV_FP8_E4M3_ROW:  codes = u8 [B][rows][dim] (OCP E4M3); scales = float [B][rows];
 *                        value = E4M3(code) * scale.  ([P1] "the attention cache uses fp8",
 *                        "decode uses partly token-wise fp8")
 *  DSV4KV_FP4_E2M1_G16:  codes = u8 [B][rows][dim/2], two OCP E2M1 codes per byte, the
 *                        even channel in the low nibble; scales = u8 [B][rows][dim/16] E4M3,
 *                        one per 16 channels; value = E2M1(code) * E4M3(scale).
 *                        ([P3] "storing the main KV in FP4"; [P1] "indexer cache uses fp4")
 *  DSV4KV_FP8_E4M3_ROW_ROPE_BF16: the last 64 (rotary) channels kept in bf16, the other
 *                        dim - 64 in fp8 under one fp32 scale per row.  codes = u8
 *                        [B][rows][dim + 64]: dim - 64 OCP E4M3 codes, then the 64 bf16
 *                        values (little-endian, 128 bytes); scales = float [B][rows];
 *                        value = E4M3(code) * scale for channels < dim - 64, the bf16 value
 *                        for the rest.  ([P1] quantisation paragraph: fp8 for most of the
 *                        attention cache, the RoPE dimensions in bf16.)  With this format
 *                        the decode calls require rope_dim == 64; they stage the rotary
 *                        values as f16 of value / scale, accurate while a row's rotary
 *                        values stay below 146 x the largest magnitude of its other
 *                        channels (the f16 range).
 */
typedef enum {
  DSV4KV_BF16 = 0,
  DSV4KV_FP8_E4M3_ROW = 1,
  DSV4KV_FP4_E2M1_G16 = 2,
  DSV4KV_FP8_E4M3_ROW_ROPE_BF16 = 3
} dsv4kv_format;

/* A cache tensor of `batch` sequences x `rows` rows x `dim` channels.
 * `rows` is the per-sequence row capacity (the batch stride in rows). */
typedef struct {
  int32_t fmt;          /* dsv4kv_format */
  int32_t dim;          /* channels per row */
  int64_t rows;         /* rows per sequence */
  const void* codes;    /* device pointer, layout per format, 16-byte aligned */
  const void* scales;   /* device pointer or NULL for bf16, 16-byte aligned   */
} dsv4kv_cache;

/* ---------------------------------------------------------------------------
 * Compressor.  [P1] "c4a (the milder scheme)": each entry is a weighted sum of
 * 8 states with stride 4; "c128a (the aggressive scheme)": 128 states, stride
 * 128.  [P2] Step 4: C4A[1] mixes S0..S7, C4A[2] mixes S4..S11, C128A[0] is
 * S0..S127.
 *
 * For entry i < N = max(0, floor((t - window) / stride)) and channel c:
 *   out[b][i][c] = rope( sum_{j<k_taps} w[j][c] * s_raw[b][stride*i + stride - k_taps + j][c] )
 * where taps at a position < 0 contribute nothing, and rope rotates channel
 * pairs (dim-rope_dim+2m, dim-rope_dim+2m+1) by the angle
 * (pos0 + stride*i) * rope_base^(-2m/rope_dim)  ([P1] "Shared key and value").
 *   s_raw : bf16 [batch][t][dim]   (row 0 is at position pos0)
 *   w     : float [k_taps][dim]
 *   out   : bf16 or (out_fp32 != 0) float, [batch][N][dim]
 * Requirements: dim in {256, 512, 1024}, rope_dim even, 0 <= rope_dim <= dim,
 * 1 <= k_taps, 1 <= stride, window >= 0.  N == 0 launches nothing.
 * ------------------------------------------------------------------------ */
int64_t dsv4kv_compress_entries(int64_t t, int32_t window, int32_t stride);

dsv4kv_status dsv4kv_compress(const void* s_raw, const float* w, int32_t batch, int64_t t,
                              int32_t dim, int32_t k_taps, int32_t stride, int32_t window,
                              int64_t pos0, int32_t rope_dim, double rope_base,
                              int32_t out_fp32, void* out, void* stream);

/* ---------------------------------------------------------------------------
 * Incremental cache maintenance for one decode step ([P1] "compressor-state
 * blocks": the caches are updated as tokens arrive).  Appends the unrotated
 * state of position t of every sequence and keeps, per layer:
 *   raw_ring : bf16 [batch][window + k_taps][dim]; row p % (window + k_taps)
 *              holds S[p] (unrotated) for the last window + k_taps positions;
 *   win_ring : bf16 [batch][window][dim]; row p % window holds
 *              rope(S[p], p) (rotary pairs as in dsv4kv_compress) for the
 *              last `window` positions -- the window cache the decode calls
 *              read (row order does not matter to them; before t + 1 >=
 *              window only rows 0..t are written);
 *   comp     : bf16 [batch][comp_rows][dim]; entry i, the dsv4kv_compress
 *              entry of the history (taps s i + s - K + j, rotated at s i), is
 *              written the step its stride block leaves the window: when
 *              dsv4kv_compress_entries(t + 1, window, stride) grows, entry
 *              dsv4kv_compress_entries(t + 1, window, stride) - 1.
 * Appending positions 0, 1, ..., T-1 one call at a time leaves comp equal to
 * dsv4kv_compress over the whole history (up to fp32 summation order) and
 * the window ring equal to the rotated last `window` states.
 *   s_new : bf16 [batch][dim];  w : float [k_taps][dim]
 * Requirements: dim in {256, 512, 1024}; rope_dim even, <= dim; t >= 0;
 * comp_rows > the entry written (else DSV4KV_ERR_INVALID_ARG); win_ring may
 * be NULL only when window == 0.  Quantised caches are made from these rows
 * with dsv4kv_quantize.
 * ------------------------------------------------------------------------ */
dsv4kv_status dsv4kv_append(const void* s_new, const float* w, int32_t batch, int64_t t, int32_t dim,
                            int32_t k_taps, int32_t stride, int32_t window, int32_t rope_dim, double rope_base,
                            void* raw_ring, void* win_ring, void* comp, int64_t comp_rows, void* stream);

/* ---------------------------------------------------------------------------
 * Quantiser.  [P1] quantisation paragraphs (fp8 attention cache, fp4 indexer
 * cache); [P3] fp4 E2M1 main cache with one E4M3 scale per 16 channels.
 *   DSV4KV_FP8_E4M3_ROW: scale = fp32(amax / 448) (1 if amax == 0),
 *       code = E4M3(fp32(x / scale)), round to nearest even, saturating.
 *   DSV4KV_FP4_E2M1_G16: s = E4M3(fp32(amax16 / 6)) (nearest even,
 *       saturating), code = E2M1(fp32(x / s)) nearest even, saturating;
 *       codes are 0 when s == 0.
 *   DSV4KV_FP8_E4M3_ROW_ROPE_BF16: the fp8 row rule over channels
 *       [0, dim - 64) (amax over those channels only); channels
 *       [dim - 64, dim) rounded to bf16 (nearest even; bf16 input is copied).
 *   in     : bf16 or (in_fp32 != 0) float, [rows][dim]
 *   codes  : u8 [rows][dim] (fp8), [rows][dim/2] (fp4) or [rows][dim + 64]
 *            (fp8 with bf16 rotary channels)
 *   scales : float [rows] (fp8 formats) or u8 [rows][dim/16] (fp4)
 * Requirements: dim in {128, 256, 512, 1024}; fmt != DSV4KV_BF16.
 * ------------------------------------------------------------------------ */
dsv4kv_status dsv4kv_quantize(const void* in, int32_t in_fp32, int64_t rows, int32_t dim,
                              int32_t fmt, void* codes, void* scales, void* stream);

/* ---------------------------------------------------------------------------
 * Lightning indexer + top-k.  [P1] "c4a": DeepSeek Sparse Attention picks the
 * top-k compressed entries per query (k = 512); [P2] Step 5: a learned indexer
 * scores the compressed blocks.
 *   score[b][n] = sum_d qidx[b][d] * key[b][n][d]     (fp32 accumulation)
 * The selected set is the first min(k, n) entries under (score descending,
 * index ascending) — ties go to the lower index.  It is written in ascending
 * index order to idx_out[b][0..count), and idx_out[b][count..k) = -1.
 *   qidx     : bf16 [batch][dim]
 *   keys     : cache of dim channels (BF16 or FP4_E2M1_G16), rows >= n
 *   idx_out  : int32 [batch][k];  count_out : int32 [batch] (may be NULL)
 * Requirements: dim == 128; 1 <= k <= 2048; n >= 0.  Scores are exact (and
 * the selection bit-exact) when every product and partial sum is an integer
 * below 2^24, as for the small-integer indexer inputs of the workloads.
 * ------------------------------------------------------------------------ */
size_t dsv4kv_index_topk_workspace_bytes(int32_t batch, int64_t n, int32_t k);

dsv4kv_status dsv4kv_index_topk(const void* qidx, const dsv4kv_cache* keys, int32_t batch,
                                int64_t n, int32_t k, int32_t* idx_out, int32_t* count_out,
                                void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * dsv4kv_index_topk in its two steps, for callers that time or schedule them
 * apart.  dsv4kv_index_score computes the scores of all n entries ([P2] Step
 * 5: the learned indexer scores the compressed blocks) and a histogram of
 * them into `ws`; dsv4kv_index_select then picks the top-k from that
 * workspace ([P1] "c4a": the top-k entries per query) and leaves it ready for
 * the next dsv4kv_index_score.  The pair, on one workspace with the same
 * batch, n and k and nothing else on that workspace in between, is exactly
 * dsv4kv_index_topk (same arguments, requirements, results and errors).
 * When n <= k dsv4kv_index_score does nothing and dsv4kv_index_select writes
 * 0..n-1.  The workspace contents between the two calls are opaque.
 * ------------------------------------------------------------------------ */
dsv4kv_status dsv4kv_index_score(const void* qidx, const dsv4kv_cache* keys, int32_t batch,
                                 int64_t n, int32_t k, void* ws, size_t ws_bytes, void* stream);

dsv4kv_status dsv4kv_index_select(int32_t batch, int64_t n, int32_t k, int32_t* idx_out,
                                  int32_t* count_out, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Re-index inside a candidate pool.  [P3] "Three mechanisms instead of one
 * trick", CSA2: layers in Reindex mode keep their indexing inside the
 * candidate pool built by the first layer in Full mode, and the layers share
 * the indexer keys.  For sequence b, with pool[b][0..pool_cap) holding entry
 * indices in ascending order (negative = no entry, e.g. the -1 padding of a
 * dsv4kv_index_topk output that built the pool):
 *   idx_out[b] = the first min(k, m) pool entries under (score descending,
 *   entry index ascending), written in ascending entry order, padded with -1
 *   (m = number of pool entries); count_out[b] = min(k, m).
 * score as in dsv4kv_index_topk (this layer's qidx against the shared keys,
 * bf16 or fp4 keys).  The pool size is the caller's choice (the pages give
 * none); pool_cap <= 8192.  A pool entry >= n sets DSV4KV_DEV_BAD_INDEX and is
 * skipped; a pool that is not ascending sets DSV4KV_DEV_BAD_POOL (the set is
 * still the top-k, but ties then follow pool order).  One CTA per sequence;
 * the workspace holds only the status word
 * (dsv4kv_index_topk_pool_workspace_bytes).
 *   qidx  : bf16 [batch][128];  keys: as for dsv4kv_index_topk
 *   pool  : int32 [batch][pool_cap];  idx_out: int32 [batch][k];
 *   count_out: int32 [batch] or NULL
 * ------------------------------------------------------------------------ */
size_t dsv4kv_index_topk_pool_workspace_bytes(int32_t batch, int32_t pool_cap, int32_t k);

dsv4kv_status dsv4kv_index_topk_pool(const void* qidx, const dsv4kv_cache* keys, int32_t batch, int64_t n,
                                     const int32_t* pool, int32_t pool_cap, int32_t k, int32_t* idx_out,
                                     int32_t* count_out, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * dsv4kv_index_topk without a caller workspace.  The pages have no
 * counterpart: this exists for callers that cannot allocate device memory for
 * a workspace — a serving engine whose memory manager has already reserved
 * nearly all of HBM for its KV block pool, a plugin host that forbids device
 * allocations, or a latency-critical path that must not pay for cudaMalloc's
 * implicit synchronisation.  Same inputs, outputs and results as
 * dsv4kv_index_topk.
 *
 * The scratch is a library-owned static device array of
 * dsv4kv_index_topk_noalloc_max_scratch_bytes() bytes (8 MiB) that every GPU
 * which loads the library holds until the process exits.  A call whose
 * scratch need (dsv4kv_index_topk_workspace_bytes) exceeds it returns
 * DSV4KV_ERR_UNSUPPORTED; batch 32 x 32736 entries with k = 512 fits.  The
 * call looks up the array's device address on the current device; the first
 * lookup on a device loads the library's device code there, so make the first
 * call before any stream capture.  Each call clears the scratch counters and
 * histograms on `stream` first.  All calls share the one array, so calls that
 * overlap on the GPU race.  Nothing here allocates memory.
 *
 * The scratch's status word (the DSV4KV_DEV_* flags a workspace would carry)
 * is not cleared by the calls: it accumulates the flags of every call on the
 * device.  dsv4kv_index_topk_noalloc_status copies it into *host_out on
 * `stream` (with pinned host memory the copy is asynchronous: synchronise the
 * stream before reading it) and then, if `clear` != 0, zeroes it on `stream`.
 * A non-zero word means an output since the last clear may be invalid.
 * ------------------------------------------------------------------------ */
size_t dsv4kv_index_topk_noalloc_max_scratch_bytes(void);

dsv4kv_status dsv4kv_index_topk_noalloc(const void* qidx, const dsv4kv_cache* keys, int32_t batch,
                                        int64_t n, int32_t k, int32_t* idx_out, int32_t* count_out,
                                        void* stream);

dsv4kv_status dsv4kv_index_topk_noalloc_status(uint32_t* host_out, int32_t clear, void* stream);

/* ---------------------------------------------------------------------------
 * Decode attention with shared K/V.  [P2] Step 3: one cached vector S_j is
 * both key (score = Q.S_j) and value; [P1] "The sliding window": a 128-token
 * exact window; [P1] "Shared key and value": inverse RoPE on the output.
 *
 * For each sequence b and head h, with rows R = {selected compressed rows}
 * followed by the `window` window rows:
 *   p   = softmax_r( sm_scale * q[b][h] . R[r] )          (one softmax over all rows)
 *   o   = sum_r p[r] * R[r]
 *   out = o with channel pairs (dim-rope_dim+2m, +1) rotated by -t * rope_base^(-2m/rope_dim)
 *   q    : bf16 [batch][heads][dim], already rotated at position t
 *   comp : compressed cache, rows >= n;  win : window cache, rows >= window
 *   idx  : int32 [batch][k], ascending, -1 padded (dsv4kv_index_topk output);
 *          an index outside [0, n) is skipped and flags DSV4KV_DEV_BAD_INDEX
 *   out  : bf16 or (out_fp32 != 0) float, [batch][heads][dim]
 * Requirements: dim == 512; 1 <= heads <= 64; comp and win of the same dim;
 * 0 <= window; k <= 2048.  The dense call reads all n compressed rows
 * ([P1] "c128a": full attention over the compressed entries).
 * ------------------------------------------------------------------------ */
size_t dsv4kv_sparse_decode_workspace_bytes(int32_t batch, int32_t heads, int32_t dim,
                                            int32_t k, int32_t window);

dsv4kv_status dsv4kv_sparse_decode(const void* q, const dsv4kv_cache* comp,
                                   const dsv4kv_cache* win, const int32_t* idx, int32_t batch,
                                   int32_t heads, int64_t n, int32_t window, int32_t k,
                                   int64_t t, float sm_scale, int32_t rope_dim,
                                   double rope_base, int32_t out_fp32, void* out, void* ws,
                                   size_t ws_bytes, void* stream);

size_t dsv4kv_dense_decode_workspace_bytes(int32_t batch, int32_t heads, int32_t dim,
                                           int64_t n, int32_t window);

dsv4kv_status dsv4kv_dense_decode(const void* q, const dsv4kv_cache* comp,
                                  const dsv4kv_cache* win, int32_t batch, int32_t heads,
                                  int64_t n, int32_t window, int64_t t, float sm_scale,
                                  int32_t rope_dim, double rope_base, int32_t out_fp32,
                                  void* out, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Paged and ragged caches.  [P1] hybrid KV cache manager paragraph: the
 * caches are kept in blocks drawn from a shared block pool (window and
 * compressor-state blocks of a constant size per request).
 *
 * A paged cache keeps the rows of every sequence in pages of `page_rows` rows
 * inside one pool that the whole batch shares; row i of sequence b is pool row
 *   table[b * table_stride + i / page_rows] * page_rows + i % page_rows.
 * A ragged batch gives every sequence its own length: t_seq[b] (device int64
 * [batch]) is the position of its decode query, so that it has
 *   n_b = max(0, floor((t_b - window) / stride)) compressed entries and
 *   w_b = min(t_b, window) window rows (logical rows 0 .. w_b - 1 of its
 *   window pages, in any order of positions),
 * its own top-k over its own n_b entries and its own output rotation by -t_b.
 * The calls below are the per-sequence steps of the dense-layout calls above
 * on the rows the tables point to.  t_max (host) must be >= every t_b; it
 * sizes the workspaces and the grids.  A t_b outside [0, t_max] is clamped
 * into it and flags DSV4KV_DEV_BAD_LENGTH; a page number outside
 * [0, pool_pages) flags DSV4KV_DEV_BAD_PAGE and the rows of that page are
 * skipped.  Rows of a page past a sequence's last row are never read.
 * ------------------------------------------------------------------------ */
typedef struct {
  int32_t fmt;            /* dsv4kv_format */
  int32_t dim;            /* channels per row */
  int32_t page_rows;      /* rows per page: a positive multiple of 64 */
  int32_t table_stride;   /* page numbers per sequence in `table` (its row pitch) */
  int64_t pool_pages;     /* pages in the pool */
  const int32_t* table;   /* device int32 [batch][table_stride] page numbers */
  const void* codes;      /* device pool [pool_pages * page_rows][row bytes of fmt], 16-byte aligned */
  const void* scales;     /* device pool of the format's scales per row, or NULL for bf16 */
} dsv4kv_paged_cache;

/* dsv4kv_index_topk over paged indexer keys (bf16 or fp4, dim 128) of a
 * ragged batch: sequence b scores its n_b keys and keeps the first
 * min(k, n_b) under (score descending, index ascending), written ascending
 * to idx_out[b], padded with -1; count_out[b] = min(k, n_b). */
size_t dsv4kv_index_topk_paged_workspace_bytes(int32_t batch, int64_t t_max, int32_t window, int32_t stride,
                                               int32_t k);

dsv4kv_status dsv4kv_index_topk_paged(const void* qidx, const dsv4kv_paged_cache* keys, int32_t batch,
                                      const int64_t* t_seq, int64_t t_max, int32_t window, int32_t stride,
                                      int32_t k, int32_t* idx_out, int32_t* count_out, void* ws,
                                      size_t ws_bytes, void* stream);

/* dsv4kv_sparse_decode over paged compressed and window caches of a ragged
 * batch: sequence b attends to its selected entries (idx[b], indices in
 * [0, n_b), as dsv4kv_index_topk_paged writes them) and its w_b window rows,
 * and its output is rotated by -t_b. */
size_t dsv4kv_sparse_decode_paged_workspace_bytes(int32_t batch, int32_t heads, int32_t dim, int32_t k,
                                                  int32_t window);

dsv4kv_status dsv4kv_sparse_decode_paged(const void* q, const dsv4kv_paged_cache* comp,
                                         const dsv4kv_paged_cache* win, const int32_t* idx, int32_t batch,
                                         int32_t heads, const int64_t* t_seq, int64_t t_max, int32_t window,
                                         int32_t stride, int32_t k, float sm_scale, int32_t rope_dim,
                                         double rope_base, int32_t out_fp32, void* out, void* ws,
                                         size_t ws_bytes, void* stream);

/* dsv4kv_dense_decode over paged caches of a ragged batch: sequence b attends
 * to all its n_b compressed entries and its w_b window rows. */
size_t dsv4kv_dense_decode_paged_workspace_bytes(int32_t batch, int32_t heads, int32_t dim, int64_t t_max,
                                                 int32_t window, int32_t stride);

dsv4kv_status dsv4kv_dense_decode_paged(const void* q, const dsv4kv_paged_cache* comp,
                                        const dsv4kv_paged_cache* win, int32_t batch, int32_t heads,
                                        const int64_t* t_seq, int64_t t_max, int32_t window, int32_t stride,
                                        float sm_scale, int32_t rope_dim, double rope_base, int32_t out_fp32,
                                        void* out, void* ws, size_t ws_bytes, void* stream);

/* Text of the last error on the calling host thread ("" if none). */
const char* dsv4kv_last_error(void);

/* Library version string. */
const char* dsv4kv_version(void);

/* Self-test of the device-side failure path (no passage of the pages: it
 * checks the library's own error reporting).  Launches one thread that waits
 * on a barrier no thread completes, with the same bounded wait as every wait
 * in the library's kernels; after the one-second limit it gives up and ORs
 * DSV4KV_DEV_TIMEOUT into *status.  status: one uint32 in device memory,
 * owned by the caller (not cleared).  Asynchronous on `stream`; the context
 * stays usable.  Errors: DSV4KV_ERR_INVALID_ARG (null status),
 * DSV4KV_ERR_CUDA (launch). */
dsv4kv_status dsv4kv_selftest_wait_timeout(uint32_t* status, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DSV4KV_H_ */
