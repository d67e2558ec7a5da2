/*
 * qk4v8 — block-scaled low-bit FlashAttention (QK4V8) for NVIDIA B200 (sm_100a).
 *
 * C ABI of libqk4v8.so. Every pointer argument is a DEVICE pointer unless stated otherwise;
 * the caller allocates and owns every buffer (inputs, outputs and workspaces). The library
 * never allocates, frees or synchronises, except qk4v8_check_status(), which synchronises the
 * given stream. All launches are asynchronous on `stream` and deterministic for a fixed shape.
 *
 * Errors: arguments are validated on the host before any launch and a bad argument returns
 * QK4V8_ERR_INVALID_ARG (or QK4V8_ERR_UNSUPPORTED for a valid but unimplemented shape) with
 * nothing launched. A failed launch returns QK4V8_ERR_CUDA. Problems found on the device (a
 * pipeline wait that ran past its time limit, a page id out of range) set a device status
 * word that qk4v8_check_status() reports and clears.
 *
 * Formats (tqpw.cn "块缩放数值格式" article §2.1-2.2; zdszero quantization primer, format
 * table):
 *   NVFP4  E2M1 elements packed two per byte (element 2i in the low nibble), one E4M3 scale
 *          per 16 consecutive elements, one FP32 tensor scale.
 *   MXFP8  E4M3 elements, one E8M0 scale (value 2^(code-127)) per 32 consecutive elements.
 * Conversions round to nearest even and saturate (E2M1 to +-6, E4M3 to +-448); the sign bit
 * of a code is the sign of its input.
 */
#ifndef QK4V8_H
#define QK4V8_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QK4V8_OK = 0,
  QK4V8_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned buffer, ... */
  QK4V8_ERR_UNSUPPORTED = 2,  /* valid request outside what the kernels implement */
  QK4V8_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  QK4V8_ERR_TIMEOUT = 4,      /* a device-side pipeline wait passed its time limit */
  QK4V8_ERR_BOUNDS = 5        /* a device-side index check failed (e.g. page id) */
} qk4v8_status;

/* Element types. Inputs of the quantizers are F16 or BF16; attention outputs may also be F32. */
typedef enum { QK4V8_F16 = 0, QK4V8_BF16 = 1, QK4V8_F32 = 2 } qk4v8_dtype;

/* Library version (major * 100 + minor). */
int qk4v8_version(void);

/* sizeof the parameter structs, for bindings that mirror them: which = 0 gives
 * sizeof(qk4v8_fwd_params), 1 sizeof(qk4v8_decode_params), 2 sizeof(qk4v8_append_params),
 * 3 sizeof(qk4v8_qkv_params), anything else 0. */
size_t qk4v8_struct_size(int32_t which);

/* Human-readable name of a status code (static string). */
const char* qk4v8_status_string(qk4v8_status status);

/*
 * Synchronise `stream`, then report and clear the device status word: QK4V8_ERR_TIMEOUT or
 * QK4V8_ERR_BOUNDS when a kernel flagged one, QK4V8_ERR_CUDA when the stream reported an
 * error, else QK4V8_OK.
 */
qk4v8_status qk4v8_check_status(cudaStream_t stream);

/*
 * Where the first device wait that timed out since the last call sat, then cleared (0 when
 * none): kernel << 56 (1 prefill, 2 decode) | role << 48 (0 producer warp, 1 MMA issuer,
 * 2 softmax warps) | barrier index << 40 | (key tile & 0xFFFFF) << 20 | (block & 0xFFFFF).
 * Synchronous; call it after qk4v8_check_status() reported QK4V8_ERR_TIMEOUT.
 */
uint64_t qk4v8_timeout_site(void);

/*
 * Host-side self-test (no GPU needed) of the once-per-device latch that guards each kernel's
 * one-time set-up, its opt-in to more than 48 KB of dynamic shared memory, which CUDA keeps
 * per device: a process driving several GPUs opts every kernel in on each device it uses.
 * Runs a counting set-up step through a test instance of that latch for device `dev` and
 * returns how many times the step has run for `dev` so far (1 after any number of calls), or
 * -1 when dev is outside [0, 64).
 */
int32_t qk4v8_selftest_device_once(int32_t dev);

/*
 * Failure-path self-test: launches one warp that waits on a barrier nothing arrives at. Its
 * bounded wait gives up after about a second and the kernel returns; the following
 * qk4v8_check_status() reports QK4V8_ERR_TIMEOUT and qk4v8_timeout_site() names kernel 3.
 * Nothing faults or hangs; the context stays usable.
 */
qk4v8_status qk4v8_selftest_wait_timeout(cudaStream_t stream);

/*
 * quantize_nvfp4 — NVFP4 quantization of Q or K (tqpw.cn article §2.2: E2M1 elements, E4M3
 * scale per 16 elements, FP32 tensor scale). Per call:
 *   s_t = fl32(amax / 2688) over all of x (2688 = 6 * 448; s_t = 1 when amax is 0), or
 *         s_t = tensor_scale_in when tensor_scale_in > 0 (e.g. a KV cache's fixed scale);
 *   per 16-element block: s_b = E4M3(fl32(fl32(amax_b / 6) / s_t));
 *         code_i = E2M1(fl32(x_i / fl32(s_b * s_t))), every code 0 when s_b is 0.
 * x       [rows, cols] fp16/bf16, row i at x + i*row_stride elements; 16-byte aligned,
 *         cols % 16 == 0, row_stride % 8 == 0, row_stride >= cols.
 * codes   [rows, cols/2] bytes out (8-byte aligned); scales [rows, cols/16] E4M3 codes out.
 * tensor_scale  one float out (s_t).
 * x16     optional [rows, cols] fp16 copy of x out (16-byte aligned), for FP16 tiles; or NULL.
 * workspace     >= quantize_nvfp4_workspace_size() bytes, 4-byte aligned: the per-CTA
 *               maxima of the amax pass (unused, may be NULL, when tensor_scale_in > 0).
 */
size_t quantize_nvfp4_workspace_size(void);
qk4v8_status quantize_nvfp4(const void* x, qk4v8_dtype dtype, int64_t rows, int32_t cols,
                            int64_t row_stride, float tensor_scale_in, uint8_t* codes,
                            uint8_t* scales, float* tensor_scale, void* x16, void* workspace,
                            size_t workspace_bytes, cudaStream_t stream);

/*
 * Outlier-aware key quantization (sns.style BitDecoding-FP4 summary, third algorithm item:
 * static smoothing, Hadamard rotation and scale search against outlier key channels).
 *
 * qk_smooth_rotate — rows of 128 (x [rows, 128] fp16/bf16, 8-byte aligned) -> out, same shape
 * and type: per channel x * lam[c] (role 0, queries) or x / lam[c] (role 1, keys; lam [128]
 * float, a fixed calibration vector, or NULL for none), then x H with H the 128-point Sylvester
 * Walsh-Hadamard matrix (seven float32 butterfly stages, stage s turning each pair
 * (i, i + 2^s) into (a + b, a - b)), then 2^-3 (queries) or 2^-4 (keys), rounded once to the
 * type. Since H H^T = 128 I, a query and a key treated this way have the same dot product.
 *
 * quantize_nvfp4_searched — quantize_nvfp4 with a per-block scale search: the E4M3 scale codes
 * c0, c0 - 1, c0 - 2, c0 + 1 (c0 quantize_nvfp4's choice; codes outside 1..126 skipped) each
 * encode the block and the one with the smallest squared error (float32, accumulated over the
 * 16 elements in order) is kept, ties to the earlier candidate. Arguments as quantize_nvfp4.
 */
qk4v8_status qk_smooth_rotate(const void* x, qk4v8_dtype dtype, int64_t rows, int32_t head_dim,
                              const float* lam, int32_t role, void* out, cudaStream_t stream);
qk4v8_status quantize_nvfp4_searched(const void* x, qk4v8_dtype dtype, int64_t rows, int32_t cols,
                                     int64_t row_stride, float tensor_scale_in, uint8_t* codes,
                                     uint8_t* scales, float* tensor_scale, void* x16,
                                     void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * quantize_nvfp4_residual — the second tensor of dual-residual query quantization
 * (sns.style BitDecoding-FP4 summary, first algorithm item: the query as two FP4 tensors, the
 * second compensating the residual the first leaves). Given x and its NVFP4 encoding (codes,
 * scales, *tensor_scale) from quantize_nvfp4, per element in FP32 steps
 *   den = fl32(s_b * s_t),  d = fl32(value(code) * den),  r = fl32(x - d),
 * and r is NVFP4-encoded with the SAME tensor scale s_t (so Q1 K^T and Q2 K^T share one
 * accumulator): codes2 [rows, cols/2], scales2 [rows, cols/16]. Shapes and alignment as for
 * quantize_nvfp4 (codes2 8-byte aligned). attn_qk4v8_fwd and attn_qk4v8_decode_paged take the
 * result as q2_codes / q2_scales.
 */
qk4v8_status quantize_nvfp4_residual(const void* x, qk4v8_dtype dtype, int64_t rows,
                                     int32_t cols, int64_t row_stride, const uint8_t* codes,
                                     const uint8_t* scales, const float* tensor_scale,
                                     uint8_t* codes2, uint8_t* scales2, cudaStream_t stream);

/*
 * quantize_mxfp8_v — MXFP8 quantization of V along the token axis (tqpw.cn article §2.1:
 * E8M0 scale per 32 elements; here the 32 elements are consecutive tokens of one channel,
 * the contraction axis of P V). Shared exponent e = floor(log2 amax) - 8 clamped to
 * [-127, 127] (scale code e + 127; 127 for an all-zero group); code_i = E4M3(v_i * 2^-e).
 * v       [batch_heads, n_tokens, head_dim] fp16/bf16, contiguous, 16-byte aligned.
 * codes   [batch_heads, head_dim, n_pad] out, n_pad = n_tokens rounded up to 128; token-
 *         contiguous per channel; padding tokens encode 0. 16-byte aligned.
 * scales  [batch_heads, head_dim, n_pad/32] E8M0 codes out.
 * v16     optional [batch_heads, head_dim, n_pad] fp16 copy out (same transposed layout,
 *         padding 0), for FP16 tiles; or NULL. 16-byte aligned.
 * head_dim is 64 or 128.
 */
qk4v8_status quantize_mxfp8_v(const void* v, qk4v8_dtype dtype, int32_t batch_heads,
                              int32_t n_tokens, int32_t head_dim, uint8_t* codes,
                              uint8_t* scales, void* v16, cudaStream_t stream);

/*
 * quantize_qkv — Q and K to NVFP4 (each with its own dynamic tensor scale, exactly as
 * quantize_nvfp4 with tensor_scale_in <= 0) and V to MXFP8 (exactly as quantize_mxfp8_v), for
 * one attention call, in two launches: the amax pass of Q and K (per-CTA maxima, no grid-wide
 * wait) together with V's MXFP8 encode (V needs no tensor scale), then one launch that encodes
 * Q and K. The encode launch takes Q and K from their last 16-element blocks to their first,
 * so the parts the amax pass read last, still cached in L2, are read again first. Same formats and arithmetic as the per-tensor calls (the tqpw.cn
 * article §2.2 for NVFP4, §2.1 for MXFP8); outputs are bit-identical to theirs.
 * q [q_rows, head_dim], k [k_rows, head_dim], v [v_bh, v_tokens, head_dim]: dense fp16/bf16
 * (one dtype), 16-byte aligned; head_dim 64 or 128.
 * q_codes/q_scales/q_tensor_scale, k_...: as quantize_nvfp4's outputs (codes 8-byte aligned).
 * v_codes/v_scales: as quantize_mxfp8_v's outputs (codes 16-byte aligned).
 * q16/k16: optional fp16 copies of Q and K (both or neither), as quantize_nvfp4's x16.
 * v16: optional fp16 copy of V, as quantize_mxfp8_v's v16, independent of q16/k16 (the
 * FP16-tile attention needs only this one: it reads the caller's Q and K as they are).
 * workspace >= quantize_qkv_workspace_size() bytes, 4-byte aligned (the amax partials).
 * Errors: QK4V8_ERR_INVALID_ARG for null pointers, bad sizes or alignment, a short workspace;
 * QK4V8_ERR_UNSUPPORTED for another head_dim.
 */
typedef struct {
  const void* q;
  const void* k;
  const void* v;
  qk4v8_dtype dtype;
  int32_t head_dim;
  int64_t q_rows, k_rows;
  int32_t v_bh, v_tokens;
  uint8_t* q_codes;
  uint8_t* q_scales;
  float* q_tensor_scale;
  uint8_t* k_codes;
  uint8_t* k_scales;
  float* k_tensor_scale;
  uint8_t* v_codes;
  uint8_t* v_scales;
  void* q16;
  void* k16;
  void* v16;
} qk4v8_qkv_params;

size_t quantize_qkv_workspace_size(void);
qk4v8_status quantize_qkv(const qk4v8_qkv_params* params, void* workspace, size_t workspace_bytes,
                          cudaStream_t stream);

/*
 * tile_score_select — ThriftAttention-style tile importance (ai-feeds.com ThriftAttention
 * summary, method step 2 and limitations: a cheap L2-norm bound on each 128x128 query-key
 * tile's largest weight; the top ~5 % of tiles get FP16). Score of tile (qt, kt) =
 * max_{i in qt} N_i(q) * max_{j in kt} N_j(k), N = |x_hat|^2 * 2^20 / s_t^2 computed exactly
 * in integers from the NVFP4 codes; exact 128-bit products, so the selection is exact.
 * Per (batch, query head) it keeps k = ceil(n_candidates * frac_bp / 10000) tiles, where the
 * candidates are all tiles (causal: kt <= qt), ranked by score descending then by the lower
 * linear index qt * T + kt (T = ceil(n_tokens / 128)).
 * q_codes/q_scales  [batch, q_heads, n_tokens, head_dim/2 | head_dim/16] (quantize_nvfp4
 *                   output); k_codes/k_scales likewise with kv_heads. Query head h uses KV
 *                   head h / (q_heads / kv_heads).
 * idx     [batch*q_heads, k_max] out: linear indices in rank order (first n_sel[bh] valid).
 * n_sel   [batch*q_heads] out.  bitmap  optional [batch*q_heads, T, T] out (1 = selected).
 * k_max   capacity of idx per head; must be >= k; at most 4096.
 * workspace >= tile_score_select_workspace_size(...) bytes, 8-byte aligned.
 */
size_t tile_score_select_workspace_size(int32_t batch, int32_t q_heads, int32_t kv_heads,
                                        int32_t n_tokens);
qk4v8_status tile_score_select(const uint8_t* q_codes, const uint8_t* q_scales,
                               const uint8_t* k_codes, const uint8_t* k_scales, int32_t batch,
                               int32_t q_heads, int32_t kv_heads, int32_t n_tokens,
                               int32_t head_dim, int32_t causal, int32_t frac_bp, int32_t k_max,
                               int32_t* idx, int32_t* n_sel, uint8_t* bitmap, void* workspace,
                               size_t workspace_bytes, cudaStream_t stream);

/*
 * attn_qk4v8_fwd — QK4V8 FlashAttention forward (hotelren.com MpFA article §1, §3.3-3.4;
 * the pages' mpfa_flash_attn(q, k, v, q_scale, k_scale, v_scale, block_size, num_warps,
 * causal) call, §4.3). S = Q K^T on block-scaled FP4 tensor cores, FP32 online softmax over
 * 128-key tiles, P quantized to E4M3 as P*448 against the running max after each tile,
 * O += P V on block-scaled FP8 tensor cores, O / l with l the sum of the quantized weights.
 * With fp16_bitmap set, a marked tile (ThriftAttention, method step 3) instead computes
 * S = q k from the caller's 16-bit Q and K (fp16 or bf16, multiplied exactly by the 16-bit
 * tensor cores), P = fp16(448 exp(s - m)), O += P fp16(v) on FP16 tensor cores, merged into
 * the same (m, l, O).
 * Causal masking keeps key j <= query i and needs n_q == n_k.
 */
typedef struct {
  const uint8_t* q_codes;      /* [B, Hq, Nq, D/2]   NVFP4 (16-byte aligned) */
  const uint8_t* q_scales;     /* [B, Hq, Nq, D/16]  E4M3 (8-byte aligned for D = 128) */
  const float* q_tensor_scale; /* device scalar */
  const uint8_t* k_codes;      /* [B, Hkv, Nk, D/2] */
  const uint8_t* k_scales;     /* [B, Hkv, Nk, D/16] */
  const float* k_tensor_scale; /* device scalar */
  const uint8_t* v_codes;      /* [B, Hkv, D, Nk_pad] MXFP8 (quantize_mxfp8_v layout) */
  const uint8_t* v_scales;     /* [B, Hkv, D, Nk_pad/32] E8M0 */
  int32_t batch, q_heads, kv_heads, n_q, n_k, head_dim; /* head_dim 64 or 128 */
  int32_t causal;
  float softmax_scale;         /* e.g. 1/sqrt(head_dim) */
  const uint8_t* fp16_bitmap;  /* optional [B*Hq, ceil(Nq/128), ceil(Nk/128)]; or NULL */
  const void* q16;             /* when fp16_bitmap is set: the 16-bit Q [B, Hq, Nq, D] (the
                                  tensor q_codes was quantized from; type qk16_dtype) */
  const void* k16;             /* the 16-bit K [B, Hkv, Nk, D] (type qk16_dtype) */
  const void* v16;             /* fp16 [B, Hkv, D, Nk_pad] (quantize_mxfp8_v's v16) */
  qk4v8_dtype out_dtype;
  void* out;                   /* [B, Hq, Nq, D] out (out_dtype), 16-byte aligned */
  float* lse;                  /* optional [B, Hq, Nq] natural-log sum-exp out; or NULL */
  int32_t p_underflow_aware;   /* 0 or 1 as in qk4v8_decode_params (each 32-key block of a
                                  tile row scaled by its own power of two before the E4M3
                                  encode); not with fp16_bitmap */
  const uint8_t* q2_codes;     /* optional second Q tensor (quantize_nvfp4_residual, same
                                  layout and tensor scale as q): S = (Q1 + Q2) K^T, two FP4
                                  MMAs into one accumulator; NULL for one Q tensor; not with
                                  fp16_bitmap */
  const uint8_t* q2_scales;
  qk4v8_dtype qk16_dtype;      /* QK4V8_F16 or QK4V8_BF16: the type of q16 and k16 (read
                                  only when fp16_bitmap is set) */
} qk4v8_fwd_params;

qk4v8_status attn_qk4v8_fwd(const qk4v8_fwd_params* params, cudaStream_t stream);

/*
 * attn_qk4v8_decode_paged — one decoding step over a paged NVFP4-K / MXFP8-V KV cache
 * (sns.style BitDecoding-FP4 summary: the cache is read once per step; GQA queries share one
 * tensor-core MMA; P quantization fused). Split-K: the keys of a sequence are cut into
 * splits of split_tokens keys (a multiple of 128); each split runs the QK4V8 online softmax
 * from its own running max, and the splits merge exactly (M = max m_s,
 * O = sum e^(m_s - M) O_s / sum e^(m_s - M) l_s). With split_tokens at least the longest
 * context every sequence is one split: the sequential method with one running max.
 * Page layout (64 tokens per page, per page and KV head):
 *   K codes [64, D/2], K scales [64, D/16] (NVFP4, one FP32 scale for the whole cache),
 *   V codes [D, 64] (token-contiguous), V scales [D, 2] (E8M0 per 32 tokens).
 * Tokens of a sequence's last page at or beyond its context length must hold finite codes
 * (zero is the usual padding).
 */
typedef struct {
  const uint8_t* q_codes;      /* [S, Hq, D/2] NVFP4 of the step's queries */
  const uint8_t* q_scales;     /* [S, Hq, D/16] */
  const float* q_tensor_scale;
  const uint8_t* k_pages;      /* [num_pages, Hkv, 64, D/2] */
  const uint8_t* k_page_scales;/* [num_pages, Hkv, 64, D/16] */
  const float* k_tensor_scale;
  const uint8_t* v_pages;      /* [num_pages, Hkv, D, 64] */
  const uint8_t* v_page_scales;/* [num_pages, Hkv, D, 2] */
  const int32_t* page_table;   /* [S, max_pages] physical page of each logical page */
  const int32_t* context_lens; /* [S], 1 <= len <= min(max_context, 64 * max_pages); a
                                  length outside that range sets QK4V8_ERR_BOUNDS (reported by
                                  qk4v8_check_status) and that sequence's rows get O = 0 and
                                  lse = -inf */
  int32_t num_seqs, num_pages, max_pages, q_heads, kv_heads, head_dim; /* head_dim 128;
                                  num_pages * kv_heads * head_dim < 2^31 (32-bit tensor-map
                                  row coordinates), else QK4V8_ERR_UNSUPPORTED */
  int32_t max_context;         /* host-side bound on context_lens (sizes grid and workspace) */
  int32_t split_tokens;        /* keys per split, a positive multiple of 128, at most 16384 */
  float softmax_scale;
  qk4v8_dtype out_dtype;
  void* out;                   /* [S, Hq, D] out (out_dtype) */
  float* lse;                  /* optional [S, Hq] out; or NULL */
  int32_t p_underflow_aware;   /* 0: P encoded as E4M3(448 p~) per 128-key block; 1: each
                                  32-key block of a query row as E4M3(448 p~ 2^-e) with
                                  e = ceil(log2 max p~) clipped to [-127, 0] and the MMA's E8M0
                                  scale 2^e (sns.style BitDecoding-FP4 summary, underflow-aware
                                  probability scaling: long-context P must not round to zero) */
  const uint8_t* q2_codes;     /* optional second Q tensor [S, Hq, D/2] from
                                  quantize_nvfp4_residual (same tensor scale as q): S^T = K
                                  (Q1 + Q2)^T, two FP4 MMAs into one accumulator; or NULL */
  const uint8_t* q2_scales;    /* [S, Hq, D/16] with q2_codes */
} qk4v8_decode_params;

size_t attn_qk4v8_decode_workspace_size(const qk4v8_decode_params* params);
qk4v8_status attn_qk4v8_decode_paged(const qk4v8_decode_params* params, void* workspace,
                                     size_t workspace_bytes, cudaStream_t stream);

/*
 * attn_qk4v8_decode_paged_noalloc — the same decode step for callers that cannot hand the
 * library device memory for its scratch: an engine that fixed every buffer at start-up and
 * allows no allocation inside its step loop, a plugin whose host framework owns all device
 * memory and passes no workspace, or a host program that links only this library and has no
 * allocator of its own. (The pages have no counterpart; this is an integration variant.)
 * The split partials go to one file-scope device buffer of
 * QK4V8_NOALLOC_DECODE_SCRATCH_BYTES (16 MiB), present on every GPU that loads the library
 * until the process exits; attn_qk4v8_decode_workspace_size(params) must not exceed it,
 * otherwise QK4V8_ERR_UNSUPPORTED is returned and nothing is launched. Nothing is allocated
 * or freed. The first call on a device looks up that buffer's device address with the device
 * current (set-up, once per device); make that first call before any stream capture. All
 * calls share the one buffer and it keeps the last call's contents (every entry a call reads
 * it writes first, so nothing needs clearing); calls that overlap on the GPU (other streams,
 * other host threads) race on it and must be serialised by the caller.
 */
#define QK4V8_NOALLOC_DECODE_SCRATCH_BYTES (16u * 1024u * 1024u)
qk4v8_status attn_qk4v8_decode_paged_noalloc(const qk4v8_decode_params* params,
                                             cudaStream_t stream);

/*
 * kv_append_paged — quantize new tokens' K and V into the paged NVFP4-K / MXFP8-V cache that
 * attn_qk4v8_decode_paged reads (hotelren.com MpFA article §6: QK4V8 combined with paged KV
 * management; sns.style BitDecoding-FP4 summary: a native FP4 paged KV cache, filled as the
 * sequence grows). For sequence s the new tokens are rows cu_new[s] .. cu_new[s+1]-1 of
 * k_new / v_new and take positions lens[s] .. lens[s] + n_s - 1 (n_s = cu_new[s+1] -
 * cu_new[s] >= 0); position t lives in physical page page_table[s][t / 64], slot t % 64.
 *   K: NVFP4 per 16 channels with the cache's fixed tensor scale (the quantize_nvfp4
 *      arithmetic with tensor_scale_in = *k_tensor_scale), per token.
 *   V: MXFP8 per channel and 32-token group (groups aligned at position 0). Every group the
 *      new tokens fall in is encoded again from all of its tokens so far, the earlier ones
 *      taken from v_tail, so after the call the sequence's pages hold exactly what
 *      quantize_mxfp8_v gives for the whole prefix (codes past the new length are 0).
 * k_new, v_new  [total_new, Hkv, D] fp16/bf16 (dtype), token-major, 16-byte aligned.
 * cu_new        [S + 1] int32, cu_new[0] = 0, nondecreasing, cu_new[S] = total_new.
 * lens          [S] int32 lengths before the call (not modified; the caller adds n_s).
 * v_tail        [S, Hkv, D, 32] of dtype, 16-byte aligned, caller-owned state: for each
 *               sequence the tokens of its last, incomplete V group in the input precision
 *               (position 32*(len/32) + i at index i; later entries are don't-care). Read and
 *               rewritten by every call that appends to the sequence; zero it for a new one.
 * max_new       host-side bound on n_s (sizes nothing on the device; n_s above it is an
 *               error). head_dim must be 128.
 * Device checks: a page id outside [0, num_pages) or a position at or past 64 * max_pages
 * sets QK4V8_ERR_BOUNDS (reported by qk4v8_check_status) and that token is not written.
 */
typedef struct {
  const void* k_new;           /* [total_new, Hkv, D] */
  const void* v_new;           /* [total_new, Hkv, D] */
  qk4v8_dtype dtype;
  const int32_t* cu_new;       /* [S + 1] */
  const int32_t* lens;         /* [S] */
  const int32_t* page_table;   /* [S, max_pages] */
  uint8_t* k_pages;            /* [num_pages, Hkv, 64, D/2] */
  uint8_t* k_page_scales;      /* [num_pages, Hkv, 64, D/16] */
  const float* k_tensor_scale;
  uint8_t* v_pages;            /* [num_pages, Hkv, D, 64] */
  uint8_t* v_page_scales;      /* [num_pages, Hkv, D, 2] */
  void* v_tail;                /* [S, Hkv, D, 32] of dtype */
  int32_t num_seqs, num_pages, max_pages, kv_heads, head_dim, max_new;
} qk4v8_append_params;

qk4v8_status kv_append_paged(const qk4v8_append_params* params, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QK4V8_H */
