/*
 * bifocal.h - C ABI of the B200 (sm_100a) Dynamic Bifocal RoPE attention library.
 *
 * Method: Jet-Long, "Efficient Long-Context Extension with Dynamic Bifocal RoPE"
 * (arXiv 2607.07740), as described by
 *   [VS] the video script "Tom 视频脚本镜像 · arXiv 2607.07740 · Jet-Long"
 *        (section 3 voice-over; section 4 storyboard, scene-2 formula),
 *   [AF] the ai-feeds summary "Jet-Long: 使用动态双焦点RoPE的高效长上下文扩展"
 *        (section 方法: input statement, key modules 1-4, output statement;
 *         section 实验: key findings / ablation),
 *   [KB] the knowledge-base note "Jet-Long：动态双焦点 RoPE 长上下文扩展" (设计原理),
 *   [SN] the seventnews article "L'attention bifocale de Jet-Long tue le compromis
 *        de mise à l'échelle fixe pour les LLM à long contexte".
 *
 * What every attention entry point computes, per query row i and key j <= i
 * (0-based positions, rotate-half RoPE pairing k <-> k + D/2, omega_k = theta^(-2k/D)):
 *   score(i, j) = scale * < R_orig(i) q_i , R_orig(j) k_j >   if i - j <  w0   (local window, [AF] module 1)
 *               = scale * < R_long(i) q_i , R_long(j) k_j >   if i - j >= w0   (long range,   [AF] module 1)
 *   R_orig(p) rotates pair k by p * omega_k. R_long(p) rotates pair k by
 *     p * omega_k / G          (BF_MODE_FREQ_INTERP, frequency interpolation), or
 *     floor(p / G) * omega_k   (BF_MODE_POS_ALIAS, position aliasing);
 *   both named by the ablation in [AF] 实验.  G = max(1, ceil(L / w_pretrained)) ([VS] scene-2).
 *   out_i = softmax_j(score(i, .)) . v ;  lse_i = m_i + ln(sum_j exp(score(i,j) - m_i)).
 * This equals the inclusion-exclusion merge of [AF] module 3 / [SN] (long branch over all keys,
 * minus the long branch on the band, plus the local branch on the band, in log-sum-exp form);
 * the kernels evaluate it as one online softmax that picks the branch per (i, j).
 *
 * Conventions shared by all calls
 *   - Tensor pointers are DEVICE pointers on the current CUDA device, contiguous,
 *     row-major, and owned by the caller. The library never allocates device memory
 *     on a call path: scratch space is a caller-provided workspace whose size the
 *     matching *_workspace_size call returns (256-byte aligned pointer required).
 *   - q and k are RAW (pre-RoPE). RoPE and the correction rotation are applied by the
 *     library. The KV cache holds keys under the ORIGINAL RoPE, in bf16.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - Errors: argument errors return BF_ERR_INVALID / BF_ERR_UNSUPPORTED / BF_ERR_WORKSPACE
 *     before any launch; a failed launch returns BF_ERR_CUDA. No call traps, aborts or prints.
 *     Device-side events the kernels cannot turn into a correct result (a bounded wait that
 *     expires, an fp16 operand out of range) set a device status word, read (and cleared)
 *     by bifocal_last_device_error().
 */
#ifndef BIFOCAL_H_
#define BIFOCAL_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BF_API __attribute__((visibility("default")))
#else
#define BF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BF_OK = 0,
  BF_ERR_INVALID = 1,      /* bad pointer, size, shape or parameter */
  BF_ERR_UNSUPPORTED = 2,  /* valid but not built: head_dim not in {64, 128}, unknown dtype */
  BF_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  BF_ERR_TIMEOUT = 4,      /* a device-side bounded wait expired (reported by bifocal_last_device_error) */
  BF_ERR_WORKSPACE = 5,    /* workspace missing, misaligned or smaller than *_workspace_size */
  BF_ERR_NO_DEVICE = 6,    /* no CUDA device, or the device is not sm_100 */
  BF_ERR_RANGE = 7,        /* an fp16 QK^T operand (a rotated query or key) was not finite once rounded to
                              fp16 (|x| >= 65520, inf or NaN), so the result is not trustworthy (reported by
                              bifocal_last_device_error) */
  BF_ERR_INDEX = 8         /* an index the kernels read from device memory (a sequence length outside
                              [1, max_len], a block-table entry outside [0, pool_pages)) was out of range; the
                              cache rows it would have addressed were neither read nor written (reported by
                              bifocal_last_device_error) */
} bf_status_t;

typedef enum { BF_MODE_FREQ_INTERP = 0, BF_MODE_POS_ALIAS = 1 } bf_mode_t;
typedef enum { BF_DTYPE_BF16 = 0, BF_DTYPE_FP32 = 1 } bf_dtype_t;

/* flags */
#define BF_FLAG_FORCE_BIFOCAL 1 /* run the two-branch kernel even when G == 1 or w0 >= L (results are equal);
                                   taken by every prefill, chunk and decode entry point alike */
#define BF_FLAG_MMA_SYNC 2      /* prefill, D = 128: use the warp-level mma.sync kernel instead of tcgen05
                                   (comparison only; D = 64 always uses it) */
#define BF_FLAG_FUSED_ROPE 8    /* prefill and chunk, bf16 inputs, head_dim 128, even GQA group: apply RoPE and
                                 * the correction rotation inside the attention kernel's tile loads ([AF] module 3,
                                 * on-the-fly rotation): the kernel reads raw q, raw k (prefill) or the cached
                                 * original-RoPE keys (chunk) and forms each fp16 operand tile in shared memory,
                                 * so the workspace is empty (*_workspace_size returns 0) and no rotated copy of
                                 * q or k is written. bifocal_prefill_rope then only writes the cache rows asked
                                 * for, and bifocal_prefill_attention returns BF_ERR_UNSUPPORTED (the kernel needs
                                 * q and k: use bifocal_prefill). Other shapes and fp32 inputs ignore the flag. */
#define BF_FLAG_WINDOW 4        /* sliding-window attention, the local layers of a hybrid model (Jet-Nemotron,
                                 * [AF] 影响): keep only pairs with 0 <= i - j < w0, under the original RoPE;
                                 * the long-range branch is dropped and G plays no part. Taken by
                                 * bifocal_prefill (+ its two steps), bifocal_prefill_chunk and bifocal_decode;
                                 * needs w0 >= 1 (BF_ERR_INVALID otherwise) and, for the prefill forms,
                                 * head_dim 128 with an even GQA group (BF_ERR_UNSUPPORTED otherwise) */

typedef struct {
  int32_t hq;           /* query heads; hq % hkv == 0; query head h reads kv head h / (hq / hkv) */
  int32_t hkv;          /* key/value heads */
  int32_t head_dim;     /* D: 64 or 128 */
  int32_t w0;           /* local window: pairs with i - j < w0 use the original RoPE; w0 >= 0 */
  int32_t w_pretrained; /* pretrained context window, >= 1; sets G */
  int32_t mode;         /* bf_mode_t */
  double rope_theta;    /* RoPE base theta > 1 */
  float softmax_scale;  /* 0 => 1/sqrt(head_dim) */
  int32_t flags;        /* BF_FLAG_* */
} bf_params_t;

/* Dynamic factor G = max(1, ceil(L / w_pretrained)) ([VS] storyboard scene-2; [AF] module 2).
 * Host only, no CUDA call. Returns -1 when L < 0 or w_pretrained < 1. */
BF_API int32_t bifocal_factor(int64_t L, int32_t w_pretrained);

/* Bytes of device workspace bifocal_prefill / rope_causal_prefill need for these sizes and
 * this input dtype: the rotated query and key forms (fp16) and, for fp32 inputs, a bf16
 * copy of v. Host only. Returns 0 on invalid arguments. */
BF_API size_t bifocal_prefill_workspace_size(int32_t dtype, int32_t batch, int32_t L, const bf_params_t* p);

/* Bifocal causal prefill ([AF] 方法: input = sequence length L and the pretrained RoPE
 * configuration; output = the attention output of the current sequence).
 *   q    [batch, L, hq,  D]  raw, dtype (bf16 or fp32)
 *   k, v [batch, L, hkv, D]  raw, dtype
 *   out  [batch, L, hq,  D]  bf16, written
 *   lse  [batch, hq, L]      fp32 natural-log LSE of the scaled scores, written (may be NULL)
 *   kcache_out [batch, L, hkv, D] bf16: keys under the original RoPE (the decode cache); may be NULL
 *   vcache_out [batch, L, hkv, D] bf16: copy of v in bf16; may be NULL
 *   workspace / ws_bytes: >= bifocal_prefill_workspace_size(dtype, batch, L, p), 256-byte aligned.
 * G is taken once from L. When G == 1 or w0 >= L every pair is local and the call runs the
 * plain kernel (identical result) unless BF_FLAG_FORCE_BIFOCAL is set.
 * Errors: BF_ERR_INVALID for NULL q/k/v/out/p, L < 1, batch < 1, hq % hkv != 0, w0 < 0,
 * w_pretrained < 1, theta <= 1, unknown mode; BF_ERR_UNSUPPORTED for head_dim not 64/128 or
 * an unknown dtype; BF_ERR_WORKSPACE for a short/misaligned workspace; BF_ERR_CUDA on launch failure. */
BF_API bf_status_t bifocal_prefill(const void* q, const void* k, const void* v, int32_t dtype, int32_t batch, int32_t L,
                            const bf_params_t* p, void* out, float* lse, void* kcache_out, void* vcache_out,
                            void* workspace, size_t ws_bytes, void* stream);

/* The two steps of bifocal_prefill, for callers that schedule or time them apart.
 * Step 1 (RoPE pass): one HBM pass over the raw q and k that writes, into the workspace, the
 *   QK^T operands under the original and the long-range RoPE (fp16, head-major), a bf16 copy
 *   of fp32 v, and kcache_out / vcache_out when given.
 * Step 2 (attention): the fused two-branch causal attention over those operands and v
 *   (v as passed to step 1), writing out and lse.
 * Both take the arguments of bifocal_prefill; step 2 must see the same q/k/v dtype, batch, L,
 * p and workspace as the step 1 that precedes it on the stream. Errors as bifocal_prefill. */
BF_API bf_status_t bifocal_prefill_rope(const void* q, const void* k, const void* v, int32_t dtype, int32_t batch,
                                        int32_t L, const bf_params_t* p, void* kcache_out, void* vcache_out,
                                        void* workspace, size_t ws_bytes, void* stream);
BF_API bf_status_t bifocal_prefill_attention(const void* v, int32_t dtype, int32_t batch, int32_t L,
                                             const bf_params_t* p, void* out, float* lse, void* workspace,
                                             size_t ws_bytes, void* stream);

/* Step 1 with the step before the path fused in: the per-head RMS norm of the model's attention
 * block (Qwen3's q_norm and k_norm) applied to q and k inside the RoPE pass, so the normalised
 * q and k are never written. Row x of every query head (key head) becomes
 * x * rsqrt(mean_d(x_d^2) + eps) * q_norm_w (k_norm_w), in fp32, before the rotations; kcache_out
 * then holds the normalised keys under the original RoPE. The pages say nothing about norms:
 * this serves the Qwen3 models they evaluate.
 *   q_norm_w, k_norm_w [D] in the input dtype, device pointers (16-byte aligned for bf16, 32 for fp32);
 *   eps >= 0. Follow with bifocal_prefill_attention. Other arguments and errors as bifocal_prefill_rope;
 *   BF_ERR_INVALID also for NULL weights or a negative or non-finite eps. */
BF_API bf_status_t bifocal_prefill_rope_qknorm(const void* q, const void* k, const void* v, int32_t dtype,
                                               int32_t batch, int32_t L, const bf_params_t* p, const void* q_norm_w,
                                               const void* k_norm_w, float eps, void* kcache_out, void* vcache_out,
                                               void* workspace, size_t ws_bytes, void* stream);

/* Plain causal attention under the original RoPE: the same kernels with the long branch
 * compiled out (the comparator for the bifocal overhead). Same arguments as bifocal_prefill;
 * w0, w_pretrained and mode are ignored. */
BF_API bf_status_t rope_causal_prefill(const void* q, const void* k, const void* v, int32_t dtype, int32_t batch, int32_t L,
                                const bf_params_t* p, void* out, float* lse, void* kcache_out, void* vcache_out,
                                void* workspace, size_t ws_bytes, void* stream);

/* Chunked prefill over an existing cache (batch 1): the step between a prefill and decode,
 * for a long prompt processed in chunks or new tokens appended to a conversation.
 *   kcache, vcache [cap, hkv, D] bf16: rows 0..P0-1 hold the cached keys under the ORIGINAL
 *          RoPE and their values (as bifocal_prefill's kcache_out / bifocal_decode write them);
 *          rows P0..P0+C-1 are written with the chunk's keys R_orig(P0+r) k_r and its values.
 *   q    [C, hq,  D] raw, dtype: the chunk's queries at positions P0 .. P0+C-1
 *   k, v [C, hkv, D] raw, dtype
 *   out  [C, hq,  D] bf16, written;  lse [hq, C] fp32, written (may be NULL)
 *   P0 >= 0 cached rows, C >= 1 chunk rows, P0 + C <= cap.
 * G = max(1, ceil((P0 + C) / w_pretrained)), the factor of the length after the chunk, so it
 * may differ from the G the cached rows were prefilled under ([AF] module 2: the factor follows
 * the current length). Chunk row i attends to keys 0..i: pairs with i - j < w0 use the original
 * RoPE, the others the long-range RoPE, a cached key entering the long branch through the
 * correction rotation R_long(j) R_orig(j)^-1 ([AF] module 3). The result is rows P0..P0+C-1 of
 * a bifocal prefill of the whole length whose keys 0..P0-1 are the cached ones.
 *   workspace / ws_bytes: >= bifocal_prefill_chunk_workspace_size(P0, C, p), 256-byte aligned:
 *   the chunk's query forms and the key forms of all P0 + C rows (fp16).
 * Errors: as bifocal_prefill; BF_ERR_INVALID also for NULL caches, P0 < 0, C < 1 or
 * P0 + C > cap; BF_ERR_UNSUPPORTED unless head_dim == 128 and hq / hkv is even (the tcgen05
 * ping-pong kernel is the only one with a query offset). */
BF_API size_t bifocal_prefill_chunk_workspace_size(int32_t P0, int32_t C, const bf_params_t* p);
BF_API bf_status_t bifocal_prefill_chunk(const void* q, const void* k, const void* v, int32_t dtype, int32_t P0,
                                         int32_t C, const bf_params_t* p, void* kcache, void* vcache, int32_t cap,
                                         void* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

/* Chunked prefill for a batch of sequences over a paged cache (vLLM-style block tables), each
 * sequence with its own cached length, chunk length and G = max(1, ceil((P0_b + C_b) / w_pretrained))
 * ([AF] module 2: the factor follows each sequence's current length; [AF] 影响 / [VS] 3: the
 * serving engines this is meant to plug into batch sequences over paged caches). Always the
 * fused kernel: RoPE and the correction rotation of cached keys happen in its tile loads, so
 * there is no workspace and no second key copy.
 *   q [T, hq, D], k / v [T, hkv, D] raw bf16: the chunks packed one after another in batch order
 *          (sequence b's rows start at sum of chunk_lens[0 .. b-1]); T = sum of chunk_lens
 *   chunk_lens, cached_lens [batch] int32, HOST arrays: C_b >= 1 new rows at positions
 *          P0_b .. P0_b + C_b - 1 after P0_b >= 0 cached ones
 *   kpool, vpool [pool_pages * page_size, hkv, D] bf16: keys under the ORIGINAL RoPE; the chunk's
 *          keys R_orig(p) k and values are written at their positions first
 *   block_table [batch, max_pages] int32 (device): key j of sequence b is pool row
 *          block_table[b * max_pages + j / page_size] * page_size + j % page_size
 *   page_size: a multiple of 16 that divides 128 or is a multiple of 128
 *   out [T, hq, D] bf16;  lse [hq, T] fp32 (may be NULL)
 * Sequence b's rows equal bifocal_prefill_chunk on its own cache. Flags: BF_FLAG_WINDOW as for the
 * chunk call; a sequence whose G is 1 or whose w0 >= its length runs the two-branch kernel (as with
 * BF_FLAG_FORCE_BIFOCAL, identical result). Pool rows past a sequence's end are never scored:
 * their key rows are zeroed in shared memory and their value rows too, whatever the pool holds.
 * Every page a sequence's first P0_b + C_b positions use must be a page of the pool. The kernels
 * check each entry they read: one outside [0, pool_pages) is reported as BF_ERR_INDEX by
 * bifocal_last_device_error, its pool rows are not written and its key/value tiles read as zeros
 * (the results of that sequence are then wrong, and nothing outside the pool is touched).
 * Errors: as bifocal_prefill_chunk; BF_ERR_INVALID also for batch < 1, a bad page_size, P0_b < 0,
 * C_b < 1, P0_b + C_b > max_pages * page_size or NULL arrays; BF_ERR_UNSUPPORTED for batch > 64,
 * head_dim != 128 or an odd GQA group. */
BF_API bf_status_t bifocal_prefill_chunk_paged(const void* q, const void* k, const void* v, int32_t batch,
                                               const int32_t* chunk_lens, const int32_t* cached_lens,
                                               const bf_params_t* p, void* kpool, void* vpool, int32_t pool_pages,
                                               int32_t page_size, const int32_t* block_table, int32_t max_pages,
                                               void* out, float* lse, void* stream);

/* Bytes of device workspace bifocal_decode / rope_causal_decode need for a cache of up to
 * L_max rows: the split-KV partial results (fp32). Host only. 0 on invalid arguments. */
BF_API size_t bifocal_decode_workspace_size(int32_t L_max, const bf_params_t* p);

/* One single-batch decode step ([AF] module 3: on-the-fly correction rotation of cached keys;
 * [KB] 设计原理: the near/far boundary slides as tokens are generated).
 *   q      [hq,  D] bf16 raw query of the new token, at position p = L - 1
 *   k_new  [hkv, D] bf16 raw key of the new token;  v_new [hkv, D] bf16
 *   kcache [cap, hkv, D] bf16 keys under the ORIGINAL RoPE; rows 0..L-2 valid on entry.
 *          Row L-1 is written with R_orig(L-1) k_new (the append step).
 *   vcache [cap, hkv, D] bf16; row L-1 is written with v_new.
 *   L      length including the new token, 1 <= L <= cap. G = max(1, ceil(L / w_pretrained)).
 *   out    [hq, D] bf16;  lse [hq] fp32 (may be NULL).
 *   workspace / ws_bytes: >= bifocal_decode_workspace_size(L, p), 256-byte aligned.
 * Cached key j takes part in the long branch through the correction rotation
 * R_long(j) R_orig(j)^-1, applied in registers while it streams from HBM; the cache itself
 * is never rewritten and no second key copy exists.
 * Errors: as bifocal_prefill; BF_ERR_INVALID also for L > cap. */
BF_API bf_status_t bifocal_decode(const void* q, const void* k_new, const void* v_new, void* kcache, void* vcache,
                           int32_t cap, int32_t L, const bf_params_t* p, void* out, float* lse, void* workspace,
                           size_t ws_bytes, void* stream);

/* One decode step for a batch of sequences over a paged cache (vLLM-style block tables), each
 * sequence at its own length, with its own G = max(1, ceil(L_b / w_pretrained)), band edge and
 * correction rotation ([AF] module 2: the factor follows each sequence's current length).
 *   q      [batch, hq, D] bf16 raw queries of the new tokens; k_new, v_new [batch, hkv, D] bf16 raw
 *   kpool, vpool [pool_pages * page_size, hkv, D] bf16: the pages; keys under the ORIGINAL RoPE
 *   block_table [batch, max_pages] int32 (device): sequence b's logical key j is pool row
 *          block_table[b * max_pages + j / page_size] * page_size + j % page_size
 *   seq_lens [batch] int32 (device): L_b, the length with the new token, 1 <= L_b <= max_len;
 *          the new token's key and value are written at logical position L_b - 1
 *   max_len: an upper bound of every L_b (host); it sets the split layout and the workspace
 *   page_size: a multiple of 16 (one 16-key stage never straddles two pages)
 *   out [batch, hq, D] bf16;  lse [batch, hq] fp32 (may be NULL)
 *   workspace / ws_bytes: >= bifocal_decode_paged_workspace_size(batch, max_len, p), 256-byte aligned.
 * Pages past a sequence's length are never read except the tail of its last 16-key stage, whose
 * keys are masked and whose values are zeroed in shared memory before use (an uninitialised
 * slot cannot turn the result into NaN). Each used block_table entry must name a page of the pool
 * and each length lie in [1, max_len]. The kernels check both on the device: a length out of range
 * appends nothing and gives NaN as that sequence's output; a table entry outside [0, pool_pages)
 * is not written and its keys read as zeros; either is reported as BF_ERR_INDEX by
 * bifocal_last_device_error, and nothing outside the pool, the table or the workspace is touched.
 * Errors: as bifocal_decode; BF_ERR_INVALID also for batch, pool_pages, max_pages or max_len < 1, a
 * page_size that is not a positive multiple of 16, max_pages * page_size < max_len or a NULL
 * table; BF_ERR_UNSUPPORTED for BF_FLAG_WINDOW. */
BF_API size_t bifocal_decode_paged_workspace_size(int32_t batch, int32_t max_len, const bf_params_t* p);
BF_API bf_status_t bifocal_decode_paged(const void* q, const void* k_new, const void* v_new, void* kpool,
                                        void* vpool, int32_t pool_pages, int32_t page_size,
                                        const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens,
                                        int32_t max_len, int32_t batch, const bf_params_t* p, void* out,
                                        float* lse, void* workspace, size_t ws_bytes, void* stream);

/* bifocal_decode without a caller workspace, for callers that cannot allocate device memory
 * themselves: for example a plug-in hosted by a runtime that owns and pre-plans all device
 * memory, or a latency-critical loop that may not call cudaMalloc (which synchronises the
 * device). There is no counterpart in the paper; this is a deployment convenience.
 * The split-KV partials live in a static device array of BIFOCAL_NOALLOC_SCRATCH_BYTES
 * (16 MiB) that every GPU loading the library holds until the process exits. A call needs
 * bifocal_decode_workspace_size(L, p) bytes of it (5.3 MB for 32 query heads of 128);
 * larger problems are rejected with BF_ERR_WORKSPACE before any launch.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 * with that device current; make that first call before any stream capture. The address is
 * kept per device together with the id of the context it was read in; after a device reset
 * (a new primary context) the next call looks it up again.
 * All calls share the one array and it keeps the last call's contents: nothing in it needs
 * to start at zero, but calls that overlap on the GPU (other streams, other threads) race
 * on it and must be serialised by the caller. Arguments and errors as bifocal_decode. */
#define BIFOCAL_NOALLOC_SCRATCH_BYTES (16u << 20)
BF_API bf_status_t bifocal_decode_noalloc(const void* q, const void* k_new, const void* v_new, void* kcache,
                                          void* vcache, int32_t cap, int32_t L, const bf_params_t* p, void* out,
                                          float* lse, void* stream);

/* Plain-RoPE decode step (comparator): same arguments; every cached key is used as stored. */
BF_API bf_status_t rope_causal_decode(const void* q, const void* k_new, const void* v_new, void* kcache, void* vcache,
                               int32_t cap, int32_t L, const bf_params_t* p, void* out, float* lse,
                               void* workspace, size_t ws_bytes, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
BF_API const char* bifocal_status_string(int32_t status);

/* Reads and clears the device status word of the current device. The kernels set it, without
 * trapping, for the first of these events since it was last cleared:
 *   - a bounded wait expired (a producer never delivered, or a wait ran past the limit): BF_ERR_TIMEOUT;
 *   - an fp16 QK^T operand (a query or key after RoPE or the correction rotation, or a cached
 *     bf16 key converted to fp16) was not finite once rounded to fp16 (|x| >= 65520, inf or
 *     NaN): BF_ERR_RANGE. The decode kernel detects it as a non-finite running max or sum;
 *   - a sequence length or block-table entry read from device memory by the paged entry points
 *     was out of range: BF_ERR_INDEX. The kernels skip every cache row it would address (no
 *     append, no pool write, its key tiles read as zeros) and a paged decode writes NaN as the
 *     output of a sequence whose length is out of range.
 * Synchronises `stream` first. Returns BF_OK, BF_ERR_TIMEOUT, BF_ERR_RANGE, BF_ERR_INDEX or
 * BF_ERR_CUDA. */
BF_API bf_status_t bifocal_last_device_error(void* stream);

/* The raw device status word (not cleared): 0, or code | (site << 8) for the first event, where
 * code is 1 (a bounded wait expired), 2 (an fp16 operand out of range) or 3 (a device-side index
 * out of range) and `site` numbers the wait or the check in the kernel source. Synchronises the
 * device. Returns -1 on a CUDA error. */
BF_API int32_t bifocal_device_status_word(void);

/* Test-only fault injection for the failure-detection tests. Not needed by any caller of the
 * attention entry points; everything is off unless a test turns it on.
 *   kind BF_FAULT_NONE: every injection off.
 *   kind BF_FAULT_PREFILL_SKIP_FILL: in the tcgen05 ping-pong prefill kernel, the producer of CTA 0
 *        never issues K/V fill number `arg` (no expect_tx, no copy), so the MMA issuer's wait for
 *        it can only expire: the CTA gives up, every role leaves through the normal teardown
 *        (no copy in flight, tensor memory freed) and the status word reports the wait's site.
 *   kind BF_FAULT_DECODE_SKIP_STAGE: in the split-KV decode kernel, the producer of CTA 0 issues
 *        no stage from stage `arg` on; the consumer warps' wait for stage `arg` expires likewise.
 *   wait_limit_ns: the limit of every bounded wait in ns; 0 restores the default of 2 s. A wait
 *        consults it only after 20 ms, so a smaller limit acts as 20 ms.
 * Synchronises the device before and after setting the controls. Returns BF_ERR_INVALID for an
 * unknown kind, a negative arg (with a fault kind) or a negative limit; BF_ERR_CUDA on a CUDA error. */
#define BF_FAULT_NONE 0
#define BF_FAULT_PREFILL_SKIP_FILL 1
#define BF_FAULT_DECODE_SKIP_STAGE 2
BF_API bf_status_t bifocal_test_set_fault(int32_t kind, int32_t arg, int64_t wait_limit_ns);

/* Library build identification (static string): kernels compiled in and their target. */
BF_API const char* bifocal_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* BIFOCAL_H_ */
