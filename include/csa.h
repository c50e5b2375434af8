/*
 * csa.h - C ABI of the B200 (sm_100a) kernels for the DeepSeek-V4 hybrid-attention hot
 * path: CSA / HCA sequence compression, lightning-indexer scoring with top-k
 * selection, and shared-KV multi-query attention over compressed entries.
 *
 * Sources (page title, then section / equation):
 *   [P1] "DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch"
 *   [P4] bhhxx.wiki "MHA -> ... -> CSA/HCA" (Chinese), sections 6.1 and 6.2.2
 *
 * Conventions shared by every entry point
 *   - Tensor pointers are DEVICE pointers owned by the caller; the library never
 *     allocates, frees or keeps them.  Scratch comes from a caller workspace whose size
 *     the matching *_workspace_size() call returns.
 *   - Every call is asynchronous on `stream` and returns an int status: CSA_OK (0) or a
 *     negative CSA_ERR_* code.  Argument errors are detected on the host before any
 *     launch and leave every output untouched.  CSA_ERR_CUDA reports a launch failure
 *     (cudaGetLastError after the launch).  No call aborts the process.
 *   - `dtype` (CSA_BF16 or CSA_F32) is the element type of every floating-point tensor
 *     argument of a call except those typed `float*` in the prototype, which are
 *     always fp32.  bf16 data is IEEE bfloat16 bit patterns.
 *   - All arithmetic is fp32 (softmax, accumulation, scores); bf16 outputs are rounded
 *     to nearest even.  Inputs must be finite.
 *   - Row-major layouts, last dimension contiguous.  Pointers must be aligned to their
 *     element size (CSA_ERR_ALIGN otherwise), workspaces to 16 bytes.  The fast paths
 *     use 16-byte vector accesses and are taken when every pointer and row stride of
 *     the call is 16-byte aligned; other layouts run an element-wise path.
 *   - Stateless and thread-safe; calls that share a workspace must not overlap on the
 *     GPU.
 */
#ifndef CSA_B200_H
#define CSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (same ABI); NULL is the legacy default stream. */
typedef struct CUstream_st* csa_stream_t;

enum csa_dtype { CSA_BF16 = 0, CSA_F32 = 1 };

enum csa_status {
    CSA_OK = 0,
    CSA_ERR_ARG = -1,         /* null pointer, negative or inconsistent size */
    CSA_ERR_ALIGN = -2,       /* pointer or stride not 16-byte aligned */
    CSA_ERR_DTYPE = -3,       /* unknown dtype, or out_bf16 with CSA_F32 */
    CSA_ERR_WORKSPACE = -4,   /* workspace NULL or smaller than *_workspace_size() */
    CSA_ERR_CUDA = -5,        /* a CUDA launch or runtime call failed */
    CSA_ERR_UNSUPPORTED = -6, /* shape outside what the kernels implement */
    CSA_ERR_TIMEOUT = -7      /* a bounded device-side wait gave up (see *_status) */
};

/* Human-readable name of a status code (static string, never NULL). */
const char* csa_status_string(int status);

/* Library version as 10000*major + 100*minor + patch. */
int csa_version(void);

/* ---------------------------------------------------------------------------------
 * csa_compress - CSA overlapped compression ([P1] section 4, boxed sum of section 5;
 * [P4] section 6.2.2 compressor path).
 *
 * For every batch b and entry i in [entry_begin, entry_end), and column j < c:
 *   logits  = [ Za[m*i + r][j] + Ba[r][j]      for r < m   (block i, stream a)
 *               Zb[m*(i-1) + r][j] + Bb[r][j]  for r < m ] (block i-1, stream b)
 *   S       = softmax over those 2m logits (one softmax per column)
 *   out[i][j] = sum_r S_a[r] * Ca[m*i + r][j] + sum_r S_b[r] * Cb[m*(i-1) + r][j]
 * For i == 0 the b-rows are absent (logit -inf, value 0: the padding rule of [P1]).
 *
 * Ca, Cb, Za, Zb : token rows of the four projected streams (dtype).  Row r of batch b
 *                  of stream X is at X + b*ld_batch + (r - tok0)*ld_row (elements).
 *                  Rows tok0 .. n-1 must be readable; the call reads rows
 *                  m*(entry_begin-1) (or 0 when entry_begin == 0) .. m*entry_end - 1,
 *                  so tok0 <= that first row and m*entry_end <= n are required.
 *                  One interleaved [n, 4c] projection output works with ld_row = 4c.
 * Ba, Bb         : fp32 [m, c] per-position-in-block biases, or NULL for zero.
 * out            : compressed cache (dtype); entry i of batch b is written at
 *                  out + b*out_ld_batch + i*c.  Entries outside the range are untouched
 *                  (prefill: [0, n/m); incremental decode: [i, i+1)).
 * Constraints    : c >= 1, 1 <= m <= 4096.
 * The indexer keys K^I are produced by the same call with their own streams and c^I
 * ([P1] section 6.4: the indexer compresses its keys with this operation, under its own
 * weights).
 * Kernels        : prefill-sized bf16 calls with m = 4, c a multiple of 256, 16-byte
 *                  aligned streams and row strides a multiple of 8 run a TMA-staged
 *                  kernel (one CTA per SM); all other calls run a per-thread streaming
 *                  kernel.  The staged kernel's waits are bounded: if one ever times out
 *                  (not expected), the entries it did not finish are written as NaN.
 * ------------------------------------------------------------------------------- */
int csa_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                 int64_t ld_row, int64_t ld_batch, int64_t tok0, int64_t n,
                 const float* Ba, const float* Bb,
                 void* out, int64_t out_ld_batch,
                 int B, int c, int m, int64_t entry_begin, int64_t entry_end,
                 int dtype, csa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * hca_compress - HCA compression ([P1] section 10, boxed equations; [P4] section 6.1):
 * non-overlapping blocks of m' tokens, one stream, per-column softmax over the m'
 * logits Z[m'*i + r][j] + Bias[r][j], weighted sum of C[m'*i + r][j].
 *
 * C, Z   : token rows (dtype), row r of batch b at X + b*ld_batch + (r - tok0)*ld_row;
 *          rows m'*entry_begin .. m'*entry_end - 1 are read (tok0 <= m'*entry_begin,
 *          m'*entry_end <= n).
 * Bias   : fp32 [m', c] or NULL.
 * out    : entry i of batch b at out + b*out_ld_batch + i*c (dtype).
 * ------------------------------------------------------------------------------- */
int hca_compress(const void* C, const void* Z,
                 int64_t ld_row, int64_t ld_batch, int64_t tok0, int64_t n,
                 const float* Bias,
                 void* out, int64_t out_ld_batch,
                 int B, int c, int m_prime, int64_t entry_begin, int64_t entry_end,
                 int dtype, csa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * hca_project_compress - hca_compress fused with the projections that produce its
 * inputs ([P1] section 10: C = H W^KV and the pooling logits Z = H W^Z per token, then
 * the boxed softmax pooling over each entry's m' tokens; [P1] section 3 states the
 * projections H W of the CSA streams).  C and Z are computed on the tensor cores in fp32
 * (bf16 products) and never written to memory.  The model width d is not given by the
 * pages; any d that is a multiple of 64 is accepted.
 *
 * H      : bf16 token rows, row r of batch b at H + b*ld_batch + (r - tok0)*ld_row
 *          (ld_row a multiple of 8, ld_batch a multiple of ld_row, 16-byte aligned);
 *          rows m'*entry_begin .. m'*entry_end - 1 are read.
 * Wc, Wz : bf16 [c, d], row j holds output column j's weights (16-byte aligned).
 * Bias   : fp32 [m', c] or NULL.
 * out    : bf16, entry i of batch b at out + b*out_ld_batch + i*c.
 * workspace: >= 256 bytes of zero-filled device memory; csa_workspace_status reports a
 *          bounded-wait timeout.
 * Supported: m' = 128, c a multiple of 128, d a multiple of 64; CSA_ERR_UNSUPPORTED
 * otherwise.
 * ------------------------------------------------------------------------------- */
int hca_project_compress(const void* H, int64_t ld_row, int64_t ld_batch, int64_t tok0,
                         int64_t n, const void* Wc, const void* Wz, int d, const float* Bias,
                         void* out, int64_t out_ld_batch, int B, int c, int m_prime,
                         int64_t entry_begin, int64_t entry_end, void* workspace,
                         size_t ws_bytes, csa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * csa_project_compress - csa_compress fused with the four projections that produce its
 * streams ([P1] section 3: C^a = H W^{aKV}, C^b = H W^{bKV}, Z^a = H W^{aZ},
 * Z^b = H W^{bZ}; sections 4-5: the overlapped 2m-logit softmax and weighted sum, entry 0
 * without a b-part).  The streams are computed on the tensor cores in fp32 and never
 * written to memory.
 *
 * H      : bf16 token rows as for hca_project_compress; rows m*(entry_begin-1) (m*0 for
 *          entry_begin = 0) .. m*entry_end - 1 are read (tok0 <= the first of them).
 * Wa_kv, Wb_kv, Wa_z, Wb_z : bf16 [c, d], row j holds output column j's weights.
 * Ba, Bb : fp32 [m, c] or NULL.
 * out, workspace : as for hca_project_compress.
 * Supported: m = 4, c a multiple of 128, d a multiple of 64; CSA_ERR_UNSUPPORTED
 * otherwise.
 * ------------------------------------------------------------------------------- */
int csa_project_compress(const void* H, int64_t ld_row, int64_t ld_batch, int64_t tok0,
                         int64_t n, const void* Wa_kv, const void* Wb_kv, const void* Wa_z,
                         const void* Wb_z, int d, const float* Ba, const float* Bb, void* out,
                         int64_t out_ld_batch, int B, int c, int m, int64_t entry_begin,
                         int64_t entry_end, void* workspace, size_t ws_bytes,
                         csa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * csa_indexer_topk - lightning-indexer scores and top-k selection ([P1] section 6.4
 * boxed score, section 7 selection and causal rule; [P4] section 6.2.2 indexer).
 *
 * For query g = b*nq + q at position t[g], with visible = min(floor(t[g]/m), N_cap):
 *   I[s] = sum_{h < n_hI} wI[g][h] * max(0, qI[g][h] . KI[b][s])     for s < visible
 *   idx_out[g] = the k indices s of largest I[s].  Ties go to the smaller s.  If
 *   visible <= k, idx_out[g][s] = s for s < visible and -1 after.  Otherwise the k
 *   indices are in unspecified order.
 *
 * qI         : [B, nq, n_hI, cI] (dtype)      wI : fp32 [B, nq, n_hI]
 * KI         : [B, N_cap, cI] (dtype), compressed indexer keys
 * t          : DEVICE int64 [B*nq] query token positions (read on the GPU, so a captured
 *              CUDA graph can advance them between replays)
 * idx_out    : int32 [B, nq, k]
 * scores_out : fp32 [B, nq, k] score of each idx_out entry (-inf for padding), or NULL
 * workspace  : >= csa_indexer_topk_workspace_size(B, nq, N_cap, k) bytes of device
 *              memory, ZERO-FILLED before its first use (csa_workspace_zero).  Each
 *              call leaves its counters zeroed again for the next call.
 * Scores are fp32.  bf16 products are exact in fp32; sums accumulate in fp32 (tensor
 * cores when dtype is bf16, n_hI in {16, 32, 64, 128} and cI in {64, 128, 256}; CUDA
 * cores otherwise).  Requires 1 <= k, N_cap < 2^31 and B*nq <= 65535
 * (CSA_ERR_UNSUPPORTED otherwise).
 * Many queries (chunked prefill): when nq >= 16, dtype is bf16, n_hI is 32, 64 or 128,
 * cI is 64 or 128, N_cap >= 128 and qI and KI are 16-byte aligned, the queries of a
 * batch row are scored together.  Each block of 512/n_hI queries stays on chip while
 * the key tiles stream past it, so a key is read once per block rather than once per
 * query.  The result is the same set of indices.
 * ------------------------------------------------------------------------------- */
size_t csa_indexer_topk_workspace_size(int B, int nq, int64_t N_cap, int k);

int csa_indexer_topk(const void* qI, const float* wI, const void* KI, const int64_t* t,
                     int B, int nq, int64_t N_cap, int n_hI, int cI, int m, int k,
                     int32_t* idx_out, float* scores_out,
                     void* workspace, size_t ws_bytes, int dtype, csa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * csa_indexer_topk_noalloc - csa_indexer_topk for callers that cannot allocate device
 * memory (no counterpart in the pages: it only changes where scratch comes from).
 *
 * Some callers have no way to get a scratch buffer: an engine that reserved all device
 * memory for its own pool and gives kernels no allocator, or a plugin that receives
 * only tensor pointers.  This variant takes the same arguments as csa_indexer_topk
 * minus the workspace and computes the same result, using scratch that lives in the
 * library: a fixed 8 MiB device array per GPU, held from the first use of the library
 * on that GPU until the process exits.  It calls no allocator (no cudaMalloc or
 * cudaFree, nothing that allocates).
 *   - Size limit: csa_indexer_topk_workspace_size(B, nq, N_cap, k) must be at most
 *     8 MiB (about B*nq*(20*N_cap + 33 KB) bytes; e.g. one query over ~400K compressed
 *     entries).  Larger problems return CSA_ERR_WORKSPACE before any launch.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress
 *     with that device current) and caches it; make that first call before any stream
 *     capture.
 *   - Every call shares the one array and clears its counters at the start (an
 *     asynchronous memset on `stream`), so calls whose GPU work overlaps, on any streams
 *     or threads, race with each other: serialise them.
 *   - Argument errors (every code csa_indexer_topk returns before a launch, and
 *     CSA_ERR_WORKSPACE for problems beyond the array) are returned before anything is
 *     enqueued on `stream`.
 *   - A device-side timeout is reported by csa_indexer_topk_noalloc_status, not by the
 *     return value.  The next call clears it, so read it before the next call.
 * ------------------------------------------------------------------------------- */
int csa_indexer_topk_noalloc(const void* qI, const float* wI, const void* KI, const int64_t* t,
                             int B, int nq, int64_t N_cap, int n_hI, int cI, int m, int k,
                             int32_t* idx_out, float* scores_out, int dtype, csa_stream_t stream);

/* csa_indexer_topk_noalloc_status - the status word of the current device's fixed
 * scratch array after the work already enqueued on `stream` (this call waits for it):
 * CSA_ERR_TIMEOUT if a bounded wait of the last csa_indexer_topk_noalloc call gave up
 * (its idx_out is then invalid), CSA_OK otherwise; CSA_ERR_CUDA if the copy fails.  It
 * allocates nothing and leaves the word as it is. */
int csa_indexer_topk_noalloc_status(csa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * csa_sparse_attn - shared-KV multi-query attention over the selected compressed
 * entries ([P1] section 8):
 *   o[g][h] = sum_{s in idx[g]} softmax_s(scale * q[g][h] . C[b][s]) * C[b][s]
 * key = value = the compressed entry.  scale <= 0 selects 1/sqrt(c).
 *
 * q     : [B, nq, n_h, c] (dtype)            cache : [B, N_cap, c] (dtype)
 * idx   : int32 [B, nq, k]; values < 0 or >= N_cap are treated as padding (skipped)
 * out   : [B, nq, n_h, c], fp32, or bf16 when out_bf16 != 0 (dtype must be bf16)
 * lse   : fp32 [B, nq, n_h] natural-log sum of exp(scaled logits), or NULL
 * A query with no valid entry gets out = 0 and lse = -inf.
 * workspace : >= csa_attn_workspace_size(B, nq, n_h, c, k) bytes; zero its first 4 bytes
 *             (the status word) before first use.
 * Constraints: 1 <= c <= 512, n_h >= 1.
 * ------------------------------------------------------------------------------- */
size_t csa_attn_workspace_size(int B, int nq, int n_h, int c, int64_t max_entries);
int csa_sparse_attn(const void* q, const void* cache, const int32_t* idx,
                    int B, int nq, int n_h, int c, int64_t N_cap, int k, float scale,
                    void* out, float* lse, void* workspace, size_t ws_bytes,
                    int dtype, int out_bf16, csa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * hca_dense_attn - dense shared-KV MQA over every visible HCA entry ([P1] section 10:
 * no selection, each query sees all its compressed entries; causal rule s < floor(t/m')).
 * Same arguments as csa_sparse_attn with the index list replaced by the visible range
 * [0, min(floor(t[g]/m_prime), N_cap)) read from the DEVICE int64 array t [B*nq].
 * workspace : >= csa_attn_workspace_size(B, nq, n_h, c, N_cap) bytes.
 * ------------------------------------------------------------------------------- */
int hca_dense_attn(const void* q, const void* cache, const int64_t* t,
                   int B, int nq, int n_h, int c, int64_t N_cap, int m_prime, float scale,
                   void* out, float* lse, void* workspace, size_t ws_bytes,
                   int dtype, int out_bf16, csa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * csa_quantize_e4m3 - per-row E4M3 (FP8) quantisation of indexer keys (or any rows).
 *   Source: [P1] section 6.4 runs the indexer in FP4, which is viable because the scores
 *   are never exponentiated; [P1] section 12 notes FP4 has the peak of FP8 on current
 *   hardware.  The pages give no block-scale format.  The reading used: OCP E4M3 codes
 *   (largest finite 448) with one fp32 scale per row, scale = max|x| / 448 (0 for an
 *   all-zero row); code = E4M3(x * (448 / max|x|)), the factor one fp32 division per row
 *   and the product in fp32, rounded to nearest even and saturated.
 * x      : [rows, cols] (dtype bf16 or fp32) with row stride ld (elements), cols % 4 == 0
 * codes  : [rows, cols] E4M3 bytes, contiguous (4-byte aligned)
 * scales : fp32 [rows]
 * Quantising new compressed entries as they are appended keeps an E4M3 key cache in step.
 * ------------------------------------------------------------------------------- */
int csa_quantize_e4m3(const void* x, int64_t rows, int cols, int64_t ld, void* codes,
                      float* scales, int dtype, csa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * csa_quantize_e2m1 - per-row E2M1 (FP4) quantisation of indexer keys (or any rows).
 *   Source: [P1] section 6.4 runs the indexer in FP4; the element and scale formats are
 *   not given.  The reading used: OCP E2M1 codes (values 0, 0.5, 1, 1.5, 2, 3, 4, 6 and
 *   their negatives) with one fp32 scale per row, scale = max|x| / 6 (0 for an all-zero
 *   row); code = E2M1(x * (6 / max|x|)), the factor one fp32 division per row and the
 *   product in fp32, rounded to nearest even and saturated at +-6.
 * x      : [rows, cols] (dtype bf16 or fp32) with row stride ld (elements), cols % 8 == 0
 * codes  : [rows, cols / 2] bytes, contiguous (4-byte aligned); two codes per byte, the
 *          even column in the low nibble (bits 0-2 magnitude, bit 3 sign)
 * scales : fp32 [rows]
 * ------------------------------------------------------------------------------- */
int csa_quantize_e2m1(const void* x, int64_t rows, int cols, int64_t ld, void* codes,
                      float* scales, int dtype, csa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * csa_indexer_topk_e2m1 - csa_indexer_topk on E2M1 keys: the [P1] section 6.4 scores of
 * the dequantised operands, then the same top-k (section 7).  q^I (bf16) is quantised per
 * head to E4M3 inside the kernel with the csa_quantize_e4m3 rule (the query is 16 KB; the
 * key cache is what the scan streams).  The products run on the tensor cores (E2M1 x
 * E4M3 -> fp32), and the score is
 *   KI_scale[s] * sum_h (w_h * scale_h) * ReLU(q8_h . K4_s),
 * which equals the boxed formula on the dequantised values since the scales are >= 0.
 * KI4      : [B, N_cap, cI / 2] bytes of E2M1 codes as written by csa_quantize_e2m1
 *            (32-byte aligned), KI_scale: fp32 [B, N_cap]
 * qI       : [B, nq, n_hI, cI] bf16 (16-byte aligned); other arguments, the workspace
 *            (csa_indexer_topk_workspace_size) and the outputs as for csa_indexer_topk.
 * Supported: n_hI in {16, 32, 64, 128}, cI in {128, 256}, B*nq <= 65535;
 * CSA_ERR_UNSUPPORTED otherwise.
 * Keys take half a byte: the scan of the 1M-token decode reads 17.8 MB of codes and
 * scales instead of 67.1 MB.
 * ------------------------------------------------------------------------------- */
int csa_indexer_topk_e2m1(const void* qI, const float* wI, const void* KI4,
                          const float* KI_scale, const int64_t* t, int B, int nq,
                          int64_t N_cap, int n_hI, int cI, int m, int k, int32_t* idx_out,
                          float* scores_out, void* workspace, size_t ws_bytes,
                          csa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * csa_indexer_topk_e4m3 - csa_indexer_topk on E4M3 keys: the [P1] section 6.4 scores of
 * the dequantised operands, then the same top-k (section 7).  q^I (bf16) is quantised per
 * head inside the kernel with the csa_quantize_e4m3 rule; the products run on the tensor
 * cores (E4M3 x E4M3 -> fp32), and the score is
 *   KI_scale[s] * sum_h (w_h * scale_h) * ReLU(q8_h . K8_s),
 * which equals the boxed formula on the dequantised values since the scales are >= 0.
 * KI8      : [B, N_cap, cI] E4M3 codes (16-byte aligned), KI_scale: fp32 [B, N_cap]
 * qI       : [B, nq, n_hI, cI] bf16 (16-byte aligned); other arguments, the workspace
 *            (csa_indexer_topk_workspace_size) and the outputs as for csa_indexer_topk.
 * Supported: n_hI in {16, 32, 64, 128}, cI in {128, 256}, B*nq <= 65535;
 * CSA_ERR_UNSUPPORTED otherwise.
 * Keys take 1 byte instead of 2: the scan of the 1M-token decode reads 34.6 MB instead of
 * 67.1 MB.
 * ------------------------------------------------------------------------------- */
int csa_indexer_topk_e4m3(const void* qI, const float* wI, const void* KI8,
                          const float* KI_scale, const int64_t* t, int B, int nq,
                          int64_t N_cap, int n_hI, int cI, int m, int k, int32_t* idx_out,
                          float* scores_out, void* workspace, size_t ws_bytes,
                          csa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * csa_sparse_attn_window, hca_dense_attn_window - csa_sparse_attn / hca_dense_attn with the
 * sliding-window branch.  The query at position t also attends, under the same softmax,
 * to the window key/value entries of the raw tokens max(0, t - n_win + 1) .. t, the
 * current token included.
 *   Source: bhhxx.wiki "MHA -> ... -> CSA/HCA" section 6 gives W_t = {max(1, t - n_window
 *   + 1), ..., t} on 1-based positions and concatenates the window entries with the
 *   compressed entries as one shared key/value set.  dev.to "DSA, CSA, HCA and mHC"
 *   section 4 gives the V4-Pro window: 128 tokens.
 * win     : [B, win_cap, c] (dtype) ring buffer of window entries c_i^window = h_i
 *           W^{window,KV} (projected by the caller); token p of sequence b is row
 *           p % win_cap.  Requires 1 <= n_win <= win_cap < 2^31.  16-byte aligned for the
 *           tensor-core path.
 * t       : DEVICE int64 [B*nq] query positions (hca_dense_attn_window: the same t that
 *           bounds the compressed entries).  t < 0: no window entry.
 * workspace : >= csa_attn_workspace_size(B, nq, n_h, c, k + n_win) bytes (sparse), or
 *             (..., N_cap + n_win) (dense).
 * All other arguments, outputs and errors as for csa_sparse_attn / hca_dense_attn.
 * ------------------------------------------------------------------------------- */
int csa_sparse_attn_window(const void* q, const void* cache, const int32_t* idx,
                           const void* win, const int64_t* t, int B, int nq, int n_h, int c,
                           int64_t N_cap, int k, int n_win, int64_t win_cap, float scale,
                           void* out, float* lse, void* workspace, size_t ws_bytes,
                           int dtype, int out_bf16, csa_stream_t stream);
int hca_dense_attn_window(const void* q, const void* cache, const int64_t* t, const void* win,
                          int B, int nq, int n_h, int c, int64_t N_cap, int m_prime,
                          int n_win, int64_t win_cap, float scale, void* out, float* lse,
                          void* workspace, size_t ws_bytes, int dtype, int out_bf16,
                          csa_stream_t stream);

/* Device status of a workspace of csa_indexer_topk, csa_sparse_attn or hca_dense_attn:
 * synchronises `stream` and returns CSA_OK, or CSA_ERR_TIMEOUT if a tensor-core kernel
 * of an earlier call gave up a bounded wait (its outputs are then invalid).  The status
 * word is the first 4 bytes of the workspace and stays set until it is zeroed. */
int csa_workspace_status(const void* workspace, csa_stream_t stream);

/* Test hook of the failure detection (no counterpart in the pages): sets, on `stream`,
 * the wait budget in SM clock cycles of the one grid-wide wait of csa_indexer_topk and
 * csa_indexer_topk_e4m3 (the meeting of a query's CTAs before the in-place top-k), kept
 * in bytes 8-15 of that call's workspace.  0 (the zero-filled default) keeps the ~1 s
 * budget of every other device wait.  A budget of a few cycles makes the wait run out, so
 * a test can see CSA_ERR_TIMEOUT from csa_workspace_status without faulting or hanging
 * the GPU: after a timeout every CTA skips its remaining selection work and the call's
 * idx_out is invalid.  workspace: 16-byte aligned; cycles >= 0 (CSA_ERR_ARG otherwise). */
int csa_workspace_set_wait_budget(void* workspace, int64_t cycles, csa_stream_t stream);

/* Zero `bytes` of device memory on `stream` (cudaMemsetAsync); for first-use workspaces. */
int csa_workspace_zero(void* workspace, size_t bytes, csa_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* CSA_B200_H */
