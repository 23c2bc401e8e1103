/*
 * exact-attention for B200 (sm_100a): C ABI.
 *
 * Exact scaled-dot-product attention O = softmax(scale * Q K^T) V computed
 * tile by tile with an online softmax, so the n x n score matrix never reaches
 * device memory ("FlashAttention 实战指南:如何把训练内存省 20 倍、速度提 4 倍",
 * §长序列注意力为什么会爆内存: tiling into on-chip memory, a running row max
 * and row sum, recomputation in the backward pass; the result equals the
 * plain three-step definition, "AI模型推理优化 Flash Attention原理",
 * §先搞清楚原理).
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor arguments are DEVICE pointers owned by the caller, contiguous
 *   with the last dimension at stride 1, 16-byte aligned. The library never
 *   allocates or frees device memory; scratch space is passed in through a
 *   caller-owned workspace sized by the matching *_workspace_size() query.
 * - Layout (guide §上手…三步走): q (B, S, Hq, D); k, v (B, S, Hkv, D);
 *   out like q; lse float32 (B, Hq, S).
 *   Varlen (cu_seqlens != NULL): sequences are packed along the token axis,
 *   q (total, Hq, D), k, v (total, Hkv, D), lse (Hq, total); cu_seqlens is a
 *   DEVICE int32 array of B + 1 non-decreasing prefix sums with
 *   cu_seqlens[0] = 0 and cu_seqlens[B] = total; S is then the maximum
 *   sequence length (an upper bound is fine).
 * - dtype applies to q, k, v, out, dout, dq, dk, dv, k_new, v_new and the
 *   caches alike; arithmetic accumulates in float32.
 * - Options (guide §进阶参数): causal; a sliding window
 *   (window_left, window_right), -1 meaning unbounded, bounds inclusive,
 *   causal forcing window_right = 0; softcap > 0 replaces every logit x by
 *   softcap * tanh(x / softcap) after scaling (0 disables it); GQA: Hq must be
 *   an integer multiple of Hkv and query head h reads kv head h / (Hq / Hkv).
 *   When the query and key lengths differ (decode) the causal diagonal is
 *   aligned to the bottom-right corner.
 * - ALiBi (guide §进阶参数 alibi_slopes: a position bias that decays the
 *   scores of distant keys): alibi_slopes is NULL or a DEVICE float32 array;
 *   query head h of sequence b uses slope s = alibi_slopes[b *
 *   alibi_batch_stride + h] (batch stride 0: one (Hq) vector for every
 *   sequence; Hq: a (B, Hq) array), and every logit of query i and key j gets
 *   -s * |i + Sk - Sq - j| added after scaling and softcap, before masking.
 * - LSE is the natural-log log-sum-exp of each row's scaled (and softcapped,
 *   biased) logits; a row with no visible key gets O = 0 and LSE = -inf.
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *   default stream) and returns after the launch. Errors never abort: the
 *   call returns a status and fa_last_error() describes it. Invalid
 *   arguments are rejected on the host before anything is launched.
 * - Head dimension D must be 64 or 128; the forward calls (fa_fwd,
 *   fa_fwd_qkvpacked) also take 256 ("FlashAttention 实战指南" §版本怎么选:
 *   head dims up to 256), the backward and kv-cache calls do not
 *   (FA_ERR_UNSUPPORTED). The device must be compute capability 10.0 (B200).
 */
#ifndef EXACT_ATTENTION_FA_H_
#define EXACT_ATTENTION_FA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null pointer, bad shape, bad option, misaligned */
  FA_ERR_UNSUPPORTED = 2, /* head dim or device not supported */
  FA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
  FA_ERR_TIMEOUT = 4      /* a kernel gave up on a bounded wait (see fa_get_device_status) */
} fa_status;

typedef enum { FA_BF16 = 0, FA_FP16 = 1 } fa_dtype;

/*
 * Forward pass: out = softmax(scale * q k^T [softcap, mask]) v and lse.
 * Guide §长序列注意力为什么会爆内存 (tiling + online softmax), §进阶参数
 * (causal, window, softcap, GQA), §上手…三步走 (varlen via cu_seqlens).
 *   total_tokens: number of packed tokens when cu_seqlens != NULL, else ignored.
 * Errors: FA_ERR_INVALID_ARG for null q/k/v/out/lse, B/Hq/Hkv/S < 1,
 *   Hq % Hkv != 0, window < -1, softcap < 0 or not finite, scale not finite,
 *   misaligned pointers, alibi_batch_stride neither 0 nor >= Hq;
 *   FA_ERR_UNSUPPORTED for D not in {64, 128} or a
 *   device other than compute capability 10.0; FA_ERR_CUDA on launch failure.
 */
FA_API fa_status fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                 int Hq, int Hkv, int S, int D, float scale, int causal, int window_left,
                 int window_right, float softcap, const float* alibi_slopes,
                 int alibi_batch_stride, const int32_t* cu_seqlens, int total_tokens,
                 fa_dtype dtype, void* stream);

/*
 * fa_fwd on a qkv-packed input (guide §上手…三步走: when Q, K and V are
 * already one tensor, the packed entry avoids splitting it): qkv is
 * (B, S, 3, H, D) (varlen: (total, 3, H, D)), i.e. token t holds its q heads,
 * then its k heads, then its v heads; Hq = Hkv = H. out (B, S, H, D) and lse
 * as in fa_fwd. The kernels read the three tensors in place through strided
 * tensor maps: no copy. Arguments and errors otherwise as fa_fwd.
 */
FA_API fa_status fa_fwd_qkvpacked(const void* qkv, void* out, float* lse, int B, int H, int S,
                                  int D, float scale, int causal, int window_left,
                                  int window_right, float softcap, const float* alibi_slopes,
                                  int alibi_batch_stride, const int32_t* cu_seqlens,
                                  int total_tokens, fa_dtype dtype, void* stream);

/*
 * FP8 forward ("FlashAttention 实战指南" §版本怎么选: FlashAttention-3 runs
 * the forward pass in FP8; the page gives no format, and this one is the
 * common reading): q, k, v are FP8 E4M3 codes (one byte each: sign, 4
 * exponent bits with bias 7, 3 mantissa bits; exponent 0 subnormal; 0x7F and
 * 0xFF NaN; largest finite 448) in the layouts of fa_fwd, and element x of
 * q stands for value(x) * q_descale (likewise k, v). The result is fa_fwd's
 * on those values: out = softmax(scale * Q K^T [softcap, bias, mask]) V in
 * out_dtype (bf16 or fp16), lse float32 as in fa_fwd. Q K^T runs on the
 * tensor cores in E4M3 with float32 accumulation (exact products); the
 * probabilities are rounded to E4M3 for the P V product (relative error at
 * most 2^-4 each, the largest of a row kept in [16, 256] so that none leaves
 * the format's normal range above 2^-10 of it) and the row sums and LSE are
 * taken from the unrounded values.
 *   q_descale, k_descale, v_descale: finite and > 0.
 * D must be 128 or 256 (FA_ERR_UNSUPPORTED otherwise). Every other option
 * (causal, window, softcap, ALiBi, GQA, varlen) as in fa_fwd.
 * Errors: as fa_fwd, plus FA_ERR_INVALID_ARG for a descale that is not
 *   finite and positive.
 */
FA_API fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, void* out, float* lse,
                            int B, int Hq, int Hkv, int S, int D, float scale, float q_descale,
                            float k_descale, float v_descale, int causal, int window_left,
                            int window_right, float softcap, const float* alibi_slopes,
                            int alibi_batch_stride, const int32_t* cu_seqlens, int total_tokens,
                            fa_dtype out_dtype, void* stream);

/*
 * Workspace bytes needed by fa_bwd for these sizes: two float32 values per
 * token and query head (the row's dot(dO, O) and its LSE in the exp2
 * domain), each sequence's rows padded to a multiple of 128, i.e.
 * 2 * Hq * 128 * (T / 128 + B + 1) * 4 bytes with T = B * S or total_tokens;
 * total_tokens as in fa_fwd (ignored if <= 0).
 */
FA_API size_t fa_bwd_workspace_size(int B, int Hq, int S, int D, int total_tokens);

/*
 * Backward pass: gradients of sum(out * dout) with respect to q, k, v, by
 * recomputing the attention probabilities from q, k and the saved lse
 * instead of storing them (guide §长序列注意力为什么会爆内存: the backward
 * pass does not keep the attention matrix and recomputes it when needed).
 *   out, lse: the results of fa_fwd with the same arguments.
 *   dq like q; dk, dv like k, v (for GQA the contributions of every query
 *   head of a group are summed into the shared kv head).
 *   workspace: device memory of at least fa_bwd_workspace_size() bytes,
 *   256-byte aligned; its contents on entry do not matter.
 *   The result is deterministic: no atomics; dK, dV come from one CTA per key
 *   tile and dQ from one CTA per query tile.
 * Errors: as fa_fwd, plus FA_ERR_INVALID_ARG for null dout/dq/dk/dv or a
 *   workspace that is null or too small, and FA_ERR_UNSUPPORTED for more than
 *   8192 query heads.
 */
FA_API fa_status fa_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int S,
                 int D, float scale, int causal, int window_left, int window_right, float softcap,
                 const float* alibi_slopes, int alibi_batch_stride, const int32_t* cu_seqlens,
                 int total_tokens, fa_dtype dtype, void* workspace, size_t workspace_bytes,
                 void* stream);

/*
 * fa_bwd for fa_fwd_qkvpacked: qkv (B, S, 3, H, D) as in the forward, out,
 * lse, dout unpacked; the gradients are written packed into dqkv, the same
 * layout as qkv. Workspace as fa_bwd_workspace_size(B, H, S, D, ...).
 * Arguments and errors otherwise as fa_bwd.
 */
FA_API fa_status fa_bwd_qkvpacked(const void* qkv, const void* out, const float* lse,
                                  const void* dout, void* dqkv, int B, int H, int S, int D,
                                  float scale, int causal, int window_left, int window_right,
                                  float softcap, const float* alibi_slopes, int alibi_batch_stride,
                                  const int32_t* cu_seqlens, int total_tokens, fa_dtype dtype,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes needed by fa_fwd_kvcache: the float32 per-split partial
 * results (num_splits > 1; 0 bytes for them otherwise) and, with rotary
 * tables (rotary_dim > 0), the rotated queries in the input dtype. */
FA_API size_t fa_kvcache_workspace_size(int B, int Sq, int Hq, int D, int num_splits,
                                        int rotary_dim);

/*
 * One decode step against a paged (or contiguous) KV cache (guide §增量解码场景
 * flash_attn_with_kvcache): the Sq new keys/values of each sequence are
 * appended IN PLACE at logical positions L .. L + Sq - 1 (L =
 * cache_seqlens[b]), then the Sq new queries attend over the Lk = L + Sq
 * keys with bottom-right alignment: query t sits at position Lk - Sq + t and,
 * when causal, sees the keys up to its own position; the window bounds are
 * taken from that position (the convention of fa_fwd). The KV range is split
 * into num_splits parts whose partial results are merged by a log-sum-exp
 * combine.
 *   q (B, Sq, Hq, D); k_new, v_new (B, Sq, Hkv, D), or both NULL for no append
 *     (then Lk = L and the queries sit at L - Sq .. L - 1).
 *   k_cache, v_cache (num_pages, page_size, Hkv, D): the page pool; logical
 *     position p of sequence b lives in page block_table[b, p / page_size],
 *     slot p % page_size ("FlashAttention技术深度解析" §动态缓存架构: a page
 *     table maps logical blocks to physical ones).
 *   block_table: DEVICE int32 (B, max_pages_per_seq), every referenced entry
 *     in [0, num_pages). NULL selects a contiguous (non-paged) cache:
 *     k_cache, v_cache (B, capacity, Hkv, D) with page_size = capacity (any
 *     value >= 1), max_pages_per_seq = 1 and num_pages = B, so that sequence
 *     b is page b.
 *   cache_seqlens: DEVICE int32 (B), valid length BEFORE the append; the
 *     library does not increment it (the caller advances its own position).
 *   rotary_cos, rotary_sin: DEVICE float32 (rotary_rows, rotary_dim / 2)
 *     angle tables, or NULL with rotary_dim = 0 for no rotary encoding (the
 *     guide names rotary_cos / rotary_sin as the in-call rotary position
 *     encoding). With them, q and the new keys of token t are rotated at
 *     position Lk - Sq + t before the attention and the append: each pair
 *     (a, b) of the first rotary_dim dimensions becomes
 *     (a cos - b sin, a sin + b cos), pairs (i, i + rotary_dim/2), or
 *     (2i, 2i + 1) when rotary_interleaved is nonzero; the rotated values are
 *     rounded to the input dtype (the cache holds rotated keys). rotary_dim is
 *     a multiple of 16 up to D; every rotated position must lie in
 *     [0, rotary_rows).
 *   out (B, Sq, Hq, D); lse float32 (B, Hq, Sq).
 *   page_size: a multiple of 64 (paged cache). Cache slots at positions
 *     >= Lk are never read into a result, whatever they hold (NaN included).
 *   workspace: at least fa_kvcache_workspace_size(B, Sq, Hq, D, num_splits,
 *     rotary_dim) bytes of device memory (may be NULL when that is 0).
 * Errors: as fa_fwd, plus FA_ERR_INVALID_ARG for null cache/lengths, Sq < 1,
 *   num_splits < 1, page_size not a positive multiple of 64 (or a
 *   contiguous cache described otherwise than above), a bad
 *   rotary_dim or missing tables, or a workspace that is too small. Lengths
 *   and table entries live on the device and are not read by the host;
 *   cache_seqlens[b] (+ Sq with an append) must not exceed
 *   max_pages_per_seq * page_size. A device-side violation (length, page
 *   index or rotary position out of range) is skipped and reported by
 *   fa_get_device_status as FA_ERR_INVALID_ARG; the outputs are then invalid.
 */
FA_API fa_status fa_fwd_kvcache(const void* q, const void* k_new, const void* v_new, void* k_cache,
                                void* v_cache, const int32_t* block_table,
                                const int32_t* cache_seqlens, const float* rotary_cos,
                                const float* rotary_sin, void* out, float* lse, int B, int Sq,
                                int Hq, int Hkv, int D, int page_size, int max_pages_per_seq,
                                int num_pages, int rotary_rows, int rotary_dim,
                                int rotary_interleaved, float scale, int causal, int window_left,
                                int window_right, float softcap, const float* alibi_slopes,
                                int alibi_batch_stride, int num_splits, fa_dtype dtype,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_fwd_kvcache against an int8 KV cache ("FlashAttention技术深度解析：重塑LLM
 * 推理性能的新范式" §发展趋势 / 量化技术融合 names an INT8/INT4 quantised KV
 * cache; the pages give no format, and this one is the plainest reading):
 * every cached (token, kv head) row of D values is stored as int8 codes with
 * one float32 scale and stands for code * scale. A row x is quantised as
 * scale = max|x| / 127 and code = round-half-even(x / scale), both in
 * float32 with IEEE division (a zero row: scale 0, codes 0); the new rows of
 * an append are quantised that way on the device (keys after the rotary
 * rotation and the rounding to the input dtype, i.e. what fa_fwd_kvcache
 * would store). The attention is then fa_fwd_kvcache's on the values the
 * codes stand for, with the same arguments, results, options and errors,
 * and these differences:
 *   k_cache, v_cache: DEVICE int8 (num_pages, page_size, Hkv, D) codes.
 *   k_scale, v_scale: DEVICE float32 (num_pages, Hkv, page_size), the row
 *     scales (per page, head-major so that a page's scales of one head are
 *     contiguous); 16-byte aligned; written for the appended rows.
 *   q, k_new, v_new, out stay in dtype (bf16 or fp16).
 *   A contiguous cache (block_table NULL) needs a capacity (page_size) that
 *     is a multiple of 64.
 * Slots at positions >= Lk are never read into a result, whatever codes and
 * scales (NaN included) they hold. Errors: as fa_fwd_kvcache, plus
 * FA_ERR_INVALID_ARG for a NULL or misaligned k_scale / v_scale.
 */
FA_API fa_status fa_fwd_kvcache_int8(const void* q, const void* k_new, const void* v_new,
                                     int8_t* k_cache, int8_t* v_cache, float* k_scale,
                                     float* v_scale, const int32_t* block_table,
                                     const int32_t* cache_seqlens, const float* rotary_cos,
                                     const float* rotary_sin, void* out, float* lse, int B, int Sq,
                                     int Hq, int Hkv, int D, int page_size, int max_pages_per_seq,
                                     int num_pages, int rotary_rows, int rotary_dim,
                                     int rotary_interleaved, float scale, int causal,
                                     int window_left, int window_right, float softcap,
                                     const float* alibi_slopes, int alibi_batch_stride,
                                     int num_splits, fa_dtype dtype, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * Quantise a 16-bit KV cache into the int8 format of fa_fwd_kvcache_int8
 * (e.g. a cache filled by a prefill): src (num_pages, page_size, Hkv, D) in
 * dtype -> codes int8 of the same shape and scales float32 (num_pages, Hkv,
 * page_size), every row by the rule above. All pointers are DEVICE memory;
 * src 16-byte aligned, codes 8-byte aligned. Errors: FA_ERR_INVALID_ARG for
 * NULL or misaligned pointers, sizes < 1 or a bad dtype; FA_ERR_UNSUPPORTED
 * for D other than 64 or 128; FA_ERR_CUDA for launch failures.
 */
FA_API fa_status fa_kv_quantize_int8(const void* src, int8_t* codes, float* scales, int num_pages,
                                     int page_size, int Hkv, int D, fa_dtype dtype, void* stream);

/*
 * fa_fwd_kvcache_int8 with an int4 cache (the same page; the other reading
 * of its INT8/INT4 sentence): every cached row is int4 codes with one
 * float32 scale, scale = max|x| / 7 and code = round-half-even(x / scale) in
 * [-7, 7] (float32, IEEE division; a zero row: scale 0, codes 0), stored two
 * per byte biased by 8, the code of even d in the low nibble.
 *   k_cache, v_cache: DEVICE uint8 (num_pages, page_size, Hkv, D / 2).
 *   k_scale, v_scale: as fa_fwd_kvcache_int8.
 * Everything else as fa_fwd_kvcache_int8; D must be 64 or 128
 * (FA_ERR_UNSUPPORTED otherwise).
 */
FA_API fa_status fa_fwd_kvcache_int4(const void* q, const void* k_new, const void* v_new,
                                     uint8_t* k_cache, uint8_t* v_cache, float* k_scale,
                                     float* v_scale, const int32_t* block_table,
                                     const int32_t* cache_seqlens, const float* rotary_cos,
                                     const float* rotary_sin, void* out, float* lse, int B, int Sq,
                                     int Hq, int Hkv, int D, int page_size, int max_pages_per_seq,
                                     int num_pages, int rotary_rows, int rotary_dim,
                                     int rotary_interleaved, float scale, int causal,
                                     int window_left, int window_right, float softcap,
                                     const float* alibi_slopes, int alibi_batch_stride,
                                     int num_splits, fa_dtype dtype, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * fa_kv_quantize_int8 into the int4 format: codes uint8 (num_pages,
 * page_size, Hkv, D / 2), 8-byte aligned; D 64 or 128.
 */
FA_API fa_status fa_kv_quantize_int4(const void* src, uint8_t* codes, float* scales, int num_pages,
                                     int page_size, int Hkv, int D, fa_dtype dtype, void* stream);

/*
 * fa_fwd_kvcache without a workspace argument, for callers that cannot
 * allocate device memory on their decode path: a serving loop that has
 * handed all free device memory to its KV-cache pool up front (so a late
 * cudaMalloc would fail), code embedded in a host runtime that owns the
 * allocator and passes in only input and output buffers, or a latency-bound
 * loop that must not call cudaMalloc/cudaFree because those calls can
 * synchronise the device. The source pages have no counterpart to this
 * call; it exists only for such callers.
 *
 * Arguments, results and errors are those of fa_fwd_kvcache. The split
 * partials and rotated queries that fa_fwd_kvcache keeps in the caller's
 * workspace live instead in one statically sized device array inside this
 * library,
 * FA_NOALLOC_SCRATCH_BYTES (24 MiB) large, which every GPU that loads the
 * library holds until the process exits. A call whose partials need more
 * (fa_kvcache_workspace_size(B, Sq, Hq, D, num_splits, rotary_dim) >
 * FA_NOALLOC_SCRATCH_BYTES)
 * is rejected with FA_ERR_INVALID_ARG before anything is launched. The call
 * itself allocates nothing: no cudaMalloc, cudaFree or allocating library
 * routine.
 *
 * - The first call on a device looks up the array's device address on that
 *   device (cudaGetSymbolAddress, with that device current) and caches it
 *   with the device's current context; make that first call outside any
 *   stream capture. After a cudaDeviceReset the context, and with it the
 *   array's address, is new: the next call looks the address up again (so
 *   it too belongs outside a capture).
 * - Every call on a device shares the one array and leaves its contents
 *   behind. Nothing in it needs to start at zero: each call writes every
 *   partial it later reads. Calls whose kernels overlap on the GPU (other
 *   streams, other host threads) race on the array and must be serialised
 *   by the caller, e.g. by issuing them on one stream.
 */
#define FA_NOALLOC_SCRATCH_BYTES (24u * 1024u * 1024u)
FA_API fa_status fa_fwd_kvcache_noalloc(const void* q, const void* k_new, const void* v_new,
                                        void* k_cache, void* v_cache, const int32_t* block_table,
                                        const int32_t* cache_seqlens, const float* rotary_cos,
                                        const float* rotary_sin, void* out, float* lse, int B,
                                        int Sq, int Hq, int Hkv, int D, int page_size,
                                        int max_pages_per_seq, int num_pages, int rotary_rows,
                                        int rotary_dim, int rotary_interleaved, float scale,
                                        int causal, int window_left, int window_right,
                                        float softcap, const float* alibi_slopes,
                                        int alibi_batch_stride, int num_splits, fa_dtype dtype,
                                        void* stream);

/*
 * Per-kernel timing, for profiling (off by default). While enabled, every
 * call records a pair of CUDA events around each kernel it launches, on the
 * caller's stream, so the durations are those of the kernels themselves as
 * they ran in the caller's stream order.
 *   fa_kernel_timing_enable(1/0) switches recording on or off (host-wide).
 *   fa_kernel_timing_read(name, &total_ms, &launches) waits for the recorded
 *     events and returns the summed duration and count of the launches of
 *     the kernel `name` ("fwd", "fwd_fp8", "bwd_pre", "bwd_dkdv", "bwd_dq", "kv_append",
 *     "decode_split", "lse_combine", "fwd_fp8") since the last reset.
 *   fa_kernel_timing_reset() drops all records.
 * Errors: FA_ERR_INVALID_ARG for null arguments, FA_ERR_CUDA if an event
 * call fails.
 */
FA_API fa_status fa_kernel_timing_enable(int enable);
FA_API fa_status fa_kernel_timing_read(const char* name, float* total_ms, int* launches);
FA_API fa_status fa_kernel_timing_reset(void);

/*
 * Self-test of the approximations the kernels evaluate on the FMA pipe
 * instead of the special-function unit (the pages have no counterpart; this
 * exists so that their error can be checked against CUDA's own functions on
 * the device): for the n DEVICE floats x, out_poly receives the library's
 * approximation and out_ref the CUDA math function on the same input, with
 *   which = 0: 2^x by the cubic of the forward's softmax (x >= -125;
 *              relative error 7.5e-5 plus float32 rounding), reference exp2f;
 *   which = 1: tanh(x) by the degree-4 odd polynomial (|x| <= 0.5; about
 *              4e-8 absolute plus float32 rounding), reference tanhf;
 *   which = 2: tanh(x) by the degree-2 polynomial with folded scales
 *              (|x| <= 0.25; about 1e-7 absolute plus float32 rounding),
 *              reference tanhf.
 * Asynchronous on `stream`. Errors: FA_ERR_INVALID_ARG for another `which`,
 * n < 0 or null pointers with n > 0; FA_ERR_CUDA on launch failure.
 */
FA_API fa_status fa_selftest_poly(int which, const float* x, float* out_poly, float* out_ref, int n,
                                  void* stream);

/*
 * Self-test of the failure path (the pages have no counterpart): runs the
 * forward kernel (non-causal, D = 128, Hq = Hkv = H, layouts of fa_fwd) in
 * a test build of it whose producer never issues the first K tile's load,
 * with every bounded wait limited to wait_limit_ns (1 ms .. 4 s; the
 * library's own calls use 4 s). Each CTA's waits on that tile run out; the
 * CTA then records FA_ERR_TIMEOUT in the device status word, lets the copies
 * and tensor-core operations it did issue finish, releases its tensor memory
 * and returns, so the context stays usable and fa_get_device_status reports
 * FA_ERR_TIMEOUT. out and lse are not valid afterwards. Asynchronous on
 * `stream`. Errors: FA_ERR_INVALID_ARG for null or misaligned pointers, bad
 * sizes or a limit outside the range; FA_ERR_CUDA on launch failure.
 */
FA_API fa_status fa_selftest_fwd_timeout(const void* q, const void* k, const void* v, void* out,
                                         float* lse, int B, int H, int S, float scale,
                                         unsigned long long wait_limit_ns, fa_dtype dtype,
                                         void* stream);

/*
 * Reads and clears the library's device status word on the current device
 * (synchronous). *status_out = 0 if no kernel reported a problem since the
 * last call, FA_ERR_TIMEOUT if one gave up on a bounded wait, and
 * FA_ERR_INVALID_ARG if a decode kernel met a cache length or page-table
 * entry out of range (it then skipped the out-of-range access and its output
 * is not valid). With FA_ERR_TIMEOUT, fa_last_error() names the wait that
 * gave up when the kernel recorded it. Returns FA_ERR_CUDA if the word cannot
 * be read.
 */
FA_API fa_status fa_get_device_status(int* status_out);

/* Message describing the last error returned on the calling thread. */
FA_API const char* fa_last_error(void);

/* Library version string. */
FA_API const char* fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTENTION_FA_H_ */
