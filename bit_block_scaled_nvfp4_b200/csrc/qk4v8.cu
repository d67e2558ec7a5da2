// C-ABI entry points of libqk4v8.so: argument validation, TMA descriptor set-up and kernel
// launches. The arithmetic lives in the kernels (quantize.cuh, tilescore.cuh, attn_fwd.cuh,
// decode.cuh); this file only checks, describes memory and launches.
#include <cudaTypedefs.h>
#include <cstring>
#include <mutex>

#include "qk4v8.h"
#include "ptx.cuh"
#include "quantize.cuh"
#include "tilescore.cuh"
#include "attn_fwd.cuh"
#include "attn_pp.cuh"
#include "decode.cuh"
#include "append.cuh"

using namespace qk4v8;

namespace {

constexpr int kNumSMs = 148;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

qk4v8_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? QK4V8_OK : QK4V8_ERR_CUDA;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Tiled tensor map; dims/box innermost first, strides in bytes for dims 1.. .
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
              const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
              CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t gd[3];
  cuuint64_t gs[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) { gd[i] = dims[i]; bx[i] = box[i]; }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides[i];
  return fn(m, dt, rank, const_cast<void*>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Number of SMs of the current device (queried once per device).
int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

int grid_for(int64_t work, int threads) {
  int64_t g = (work + threads - 1) / threads;
  if (g > kNumSMs * 16) g = kNumSMs * 16;
  return static_cast<int>(g < 1 ? 1 : g);
}

template <typename K>
bool set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
         cudaSuccess;
}

// A set-up step that must run once per device: CUDA keeps a kernel's shared-memory opt-in
// (cudaFuncAttributeMaxDynamicSharedMemorySize) per device context, so a process that drives
// several GPUs opts each kernel in on each of them. Thread-safe; a failed step is retried on
// the next call. Devices beyond kMaxDevices run the step on every call.
constexpr int kMaxDevices = 64;
class PerDeviceOnce {
 public:
  template <typename F>
  bool run(int dev, F&& step) {
    if (dev < 0 || dev >= kMaxDevices) return step();
    std::lock_guard<std::mutex> lock(mu_);
    if (done_[dev]) return true;
    if (!step()) return false;
    done_[dev] = true;
    return true;
  }

 private:
  std::mutex mu_;
  bool done_[kMaxDevices] = {};
};

int current_device() {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
}

}  // namespace

extern "C" {

int qk4v8_version(void) { return 100; }

size_t qk4v8_struct_size(int32_t which) {
  return which == 0   ? sizeof(qk4v8_fwd_params)
         : which == 1 ? sizeof(qk4v8_decode_params)
         : which == 2 ? sizeof(qk4v8_append_params)
         : which == 3 ? sizeof(qk4v8_qkv_params)
                      : 0;
}

const char* qk4v8_status_string(qk4v8_status s) {
  switch (s) {
    case QK4V8_OK: return "ok";
    case QK4V8_ERR_INVALID_ARG: return "invalid argument";
    case QK4V8_ERR_UNSUPPORTED: return "unsupported shape or option";
    case QK4V8_ERR_CUDA: return "CUDA error";
    case QK4V8_ERR_TIMEOUT: return "device wait timed out";
    case QK4V8_ERR_BOUNDS: return "device index out of range";
  }
  return "unknown status";
}

qk4v8_status qk4v8_check_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return QK4V8_ERR_CUDA;
  unsigned int st = 0;
  if (cudaMemcpyFromSymbol(&st, g_status, sizeof(st)) != cudaSuccess) return QK4V8_ERR_CUDA;
  if (st != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return QK4V8_ERR_CUDA;
    return (st & kStatusTimeout) ? QK4V8_ERR_TIMEOUT : QK4V8_ERR_BOUNDS;
  }
  return QK4V8_OK;
}

uint64_t qk4v8_timeout_site(void) {
  unsigned long long site = 0;
  if (cudaMemcpyFromSymbol(&site, g_timeout_site, sizeof(site)) != cudaSuccess) return 0;
  if (site != 0) {
    const unsigned long long zero = 0;
    cudaMemcpyToSymbol(g_timeout_site, &zero, sizeof(zero));
  }
  return site;
}

int32_t qk4v8_selftest_device_once(int32_t dev) {
  static PerDeviceOnce latch;
  static int32_t runs[kMaxDevices] = {};
  if (dev < 0 || dev >= kMaxDevices) return -1;
  latch.run(dev, [dev] { ++runs[dev]; return true; });
  return runs[dev];
}

qk4v8_status qk4v8_selftest_wait_timeout(cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>();
  return launch_status();
}

// ------------------------------------------------------------------------------------------
// the amax pass's per-CTA maxima (at most kAmaxPartials)
constexpr int kAmaxPartials = 1024;
size_t quantize_nvfp4_workspace_size(void) { return 4 * kAmaxPartials; }

}  // extern "C"

// NVFP4 quantize; kSearch: per-block scale search (outlier-aware keys).
template <bool kSearch>
static qk4v8_status quantize_nvfp4_impl(const void* x, qk4v8_dtype dtype, int64_t rows, int32_t cols,
                                        int64_t row_stride, float tensor_scale_in, uint8_t* codes,
                                        uint8_t* scales, float* tensor_scale, void* x16, void* workspace,
                                        size_t workspace_bytes, cudaStream_t stream) {
  if (x == nullptr || codes == nullptr || scales == nullptr || tensor_scale == nullptr)
    return QK4V8_ERR_INVALID_ARG;
  if (dtype != QK4V8_F16 && dtype != QK4V8_BF16) return QK4V8_ERR_INVALID_ARG;
  if (rows < 0 || cols <= 0 || cols % 16 != 0 || row_stride < cols || row_stride % 8 != 0)
    return QK4V8_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(codes, 8) || (x16 != nullptr && !aligned(x16, 16)))
    return QK4V8_ERR_INVALID_ARG;
  if (!(tensor_scale_in > 0.f) &&
      (workspace == nullptr || workspace_bytes < quantize_nvfp4_workspace_size() || !aligned(workspace, 4)))
    return QK4V8_ERR_INVALID_ARG;
  const int64_t blocks = rows * (cols / 16);
  const int grid = grid_for(blocks, 256);
  // amax pass: four CTAs per SM (at most kAmaxPartials), each writing one partial maximum
  int64_t ag = (blocks + 255) / 256;
  if (ag > 4 * kNumSMs) ag = 4 * kNumSMs;
  const int agrid = static_cast<int>(ag < 1 ? 1 : ag);
  static_assert(4 * kNumSMs <= kAmaxPartials, "amax partials");
  float* amax = static_cast<float*>(workspace);
  if (!(tensor_scale_in > 0.f)) {
    if (dtype == QK4V8_BF16)
      nvfp4_amax_kernel<__nv_bfloat16><<<agrid, 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(x), rows, cols, row_stride, amax);
    else
      nvfp4_amax_kernel<__half><<<agrid, 256, 0, stream>>>(static_cast<const __half*>(x), rows,
                                                           cols, row_stride, amax);
    if (launch_status() != QK4V8_OK) return QK4V8_ERR_CUDA;
  }
  __half* h = static_cast<__half*>(x16);
  if (dtype == QK4V8_BF16) {
    auto xb = static_cast<const __nv_bfloat16*>(x);
    if (h) nvfp4_encode_kernel<__nv_bfloat16, true, kSearch><<<grid, 256, 0, stream>>>(xb, rows, cols, row_stride, amax, agrid, tensor_scale_in, codes, scales, tensor_scale, h);
    else nvfp4_encode_kernel<__nv_bfloat16, false, kSearch><<<grid, 256, 0, stream>>>(xb, rows, cols, row_stride, amax, agrid, tensor_scale_in, codes, scales, tensor_scale, h);
  } else {
    auto xh = static_cast<const __half*>(x);
    if (h) nvfp4_encode_kernel<__half, true, kSearch><<<grid, 256, 0, stream>>>(xh, rows, cols, row_stride, amax, agrid, tensor_scale_in, codes, scales, tensor_scale, h);
    else nvfp4_encode_kernel<__half, false, kSearch><<<grid, 256, 0, stream>>>(xh, rows, cols, row_stride, amax, agrid, tensor_scale_in, codes, scales, tensor_scale, h);
  }
  return launch_status();
}

extern "C" {
qk4v8_status quantize_nvfp4(const void* x, qk4v8_dtype dtype, int64_t rows, int32_t cols,
                            int64_t row_stride, float tensor_scale_in, uint8_t* codes,
                            uint8_t* scales, float* tensor_scale, void* x16, void* workspace,
                            size_t workspace_bytes, cudaStream_t stream) {
  return quantize_nvfp4_impl<false>(x, dtype, rows, cols, row_stride, tensor_scale_in, codes,
                                    scales, tensor_scale, x16, workspace, workspace_bytes, stream);
}

qk4v8_status quantize_nvfp4_searched(const void* x, qk4v8_dtype dtype, int64_t rows, int32_t cols,
                                     int64_t row_stride, float tensor_scale_in, uint8_t* codes,
                                     uint8_t* scales, float* tensor_scale, void* x16,
                                     void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return quantize_nvfp4_impl<true>(x, dtype, rows, cols, row_stride, tensor_scale_in, codes,
                                   scales, tensor_scale, x16, workspace, workspace_bytes, stream);
}

qk4v8_status qk_smooth_rotate(const void* x, qk4v8_dtype dtype, int64_t rows, int32_t head_dim,
                              const float* lam, int32_t role, void* out, cudaStream_t stream) {
  if (x == nullptr || out == nullptr || rows < 0) return QK4V8_ERR_INVALID_ARG;
  if (dtype != QK4V8_F16 && dtype != QK4V8_BF16) return QK4V8_ERR_INVALID_ARG;
  if (role != 0 && role != 1) return QK4V8_ERR_INVALID_ARG;
  if (head_dim != 128) return QK4V8_ERR_UNSUPPORTED;
  if (!aligned(x, 8) || !aligned(out, 8) || (lam != nullptr && !aligned(lam, 4)))
    return QK4V8_ERR_INVALID_ARG;
  if (rows == 0) return QK4V8_OK;
  const int64_t grid = (rows + 7) / 8;                 // 8 rows (warps) per CTA
  if (grid > 0x7fffffffLL) return QK4V8_ERR_UNSUPPORTED;
  if (dtype == QK4V8_BF16)
    smooth_rotate_kernel<__nv_bfloat16><<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), rows, lam, role, static_cast<__nv_bfloat16*>(out));
  else
    smooth_rotate_kernel<__half><<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        static_cast<const __half*>(x), rows, lam, role, static_cast<__half*>(out));
  return launch_status();
}

// ------------------------------------------------------------------------------------------
}  // extern "C"
static qk4v8_status quantize_nvfp4_residual_impl(const void* x, qk4v8_dtype dtype, int64_t rows,
                                          int32_t cols, int64_t row_stride, const uint8_t* codes,
                                          const uint8_t* scales, const float* tensor_scale,
                                          uint8_t* codes2, uint8_t* scales2, cudaStream_t stream) {
  if (x == nullptr || codes == nullptr || scales == nullptr || tensor_scale == nullptr ||
      codes2 == nullptr || scales2 == nullptr)
    return QK4V8_ERR_INVALID_ARG;
  if (dtype != QK4V8_F16 && dtype != QK4V8_BF16) return QK4V8_ERR_INVALID_ARG;
  if (rows < 0 || cols <= 0 || cols % 16 != 0 || row_stride < cols || row_stride % 8 != 0)
    return QK4V8_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(codes, 8) || !aligned(codes2, 8)) return QK4V8_ERR_INVALID_ARG;
  const int64_t blocks = rows * (cols / 16);
  const int grid = grid_for(blocks, 256);
  if (dtype == QK4V8_BF16)
    nvfp4_residual_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), rows, cols, row_stride, codes, scales, tensor_scale,
        codes2, scales2);
  else
    nvfp4_residual_kernel<__half><<<grid, 256, 0, stream>>>(
        static_cast<const __half*>(x), rows, cols, row_stride, codes, scales, tensor_scale,
        codes2, scales2);
  return launch_status();
}

template <typename T, int D>
static void launch_mxfp8(const void* v, int32_t bh, int32_t n, int32_t npad, uint8_t* codes,
                         uint8_t* scales, void* v16, cudaStream_t stream) {
  dim3 grid(npad / 128, bh);
  if (v16) mxfp8_v_kernel<T, D, true><<<grid, 256, 0, stream>>>(static_cast<const T*>(v), n, npad, codes, scales, static_cast<__half*>(v16));
  else mxfp8_v_kernel<T, D, false><<<grid, 256, 0, stream>>>(static_cast<const T*>(v), n, npad, codes, scales, nullptr);
}

extern "C" {
qk4v8_status quantize_mxfp8_v(const void* v, qk4v8_dtype dtype, int32_t batch_heads,
                              int32_t n_tokens, int32_t head_dim, uint8_t* codes,
                              uint8_t* scales, void* v16, cudaStream_t stream) {
  if (v == nullptr || codes == nullptr || scales == nullptr) return QK4V8_ERR_INVALID_ARG;
  if (dtype != QK4V8_F16 && dtype != QK4V8_BF16) return QK4V8_ERR_INVALID_ARG;
  if (batch_heads <= 0 || n_tokens <= 0) return QK4V8_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return QK4V8_ERR_UNSUPPORTED;
  if (!aligned(v, 16) || !aligned(codes, 16) || (v16 != nullptr && !aligned(v16, 16)))
    return QK4V8_ERR_INVALID_ARG;
  if (batch_heads > 65535) return QK4V8_ERR_UNSUPPORTED;
  const int32_t npad = (n_tokens + 127) / 128 * 128;
  if (dtype == QK4V8_BF16) {
    if (head_dim == 128) launch_mxfp8<__nv_bfloat16, 128>(v, batch_heads, n_tokens, npad, codes, scales, v16, stream);
    else launch_mxfp8<__nv_bfloat16, 64>(v, batch_heads, n_tokens, npad, codes, scales, v16, stream);
  } else {
    if (head_dim == 128) launch_mxfp8<__half, 128>(v, batch_heads, n_tokens, npad, codes, scales, v16, stream);
    else launch_mxfp8<__half, 64>(v, batch_heads, n_tokens, npad, codes, scales, v16, stream);
  }
  return launch_status();
}

// ------------------------------------------------------------------------------------------
size_t quantize_qkv_workspace_size(void) { return 2 * 4 * kAmaxPartials; }
}  // extern "C"

template <typename T, int D>
static qk4v8_status launch_qkv(const qk4v8_qkv_params* p, float* q_part, float* k_part,
                               cudaStream_t stream) {
  // first launch: the amax pass (four CTAs per SM, split between Q and K in proportion to their
  // sizes) and V's MXFP8 encode; second launch: the NVFP4 encode of Q and K
  const int64_t qb = p->q_rows * (D / 16), kb = p->k_rows * (D / 16);
  const int total = 4 * kNumSMs;
  int gq = static_cast<int>((static_cast<double>(total) * qb) / static_cast<double>(qb + kb) + 0.5);
  gq = gq < 1 ? 1 : (gq > total - 1 ? total - 1 : gq);
  const int gk = total - gq;
  static_assert(4 * kNumSMs <= kAmaxPartials, "amax partials");
  QkvEncodeArgs a;
  a.q = p->q; a.k = p->k; a.v = p->v;
  a.q_blocks = qb; a.k_blocks = kb;
  a.q_partial = q_part; a.k_partial = k_part; a.q_nparts = gq; a.k_nparts = gk;
  a.q_codes = p->q_codes; a.q_scales = p->q_scales; a.q_ts = p->q_tensor_scale;
  a.k_codes = p->k_codes; a.k_scales = p->k_scales; a.k_ts = p->k_tensor_scale;
  a.v_codes = p->v_codes; a.v_scales = p->v_scales;
  a.q16 = static_cast<__half*>(p->q16); a.k16 = static_cast<__half*>(p->k16);
  a.v16 = static_cast<__half*>(p->v16);
  a.q_chunks = static_cast<int32_t>((qb + kChunkBlocks - 1) / kChunkBlocks);
  a.k_chunks = static_cast<int32_t>((kb + kChunkBlocks - 1) / kChunkBlocks);
  a.nv_ctas = (a.q_chunks + a.k_chunks + kChunksPerCta - 1) / kChunksPerCta;
  a.v_npad = (p->v_tokens + 127) / 128 * 128;
  a.v_tiles = a.v_npad / 128;
  a.v_n = p->v_tokens;
  const int64_t grid1 = total + static_cast<int64_t>(a.v_tiles) * p->v_bh;
  if (grid1 > 0x7fffffffLL) return QK4V8_ERR_UNSUPPORTED;
  if (p->v16 != nullptr)
    qk_amax_v_kernel<T, D, true><<<static_cast<unsigned>(grid1), 256, 0, stream>>>(a, p->q_rows, p->k_rows, gq, gk);
  else
    qk_amax_v_kernel<T, D, false><<<static_cast<unsigned>(grid1), 256, 0, stream>>>(a, p->q_rows, p->k_rows, gq, gk);
  if (launch_status() != QK4V8_OK) return QK4V8_ERR_CUDA;
  if (p->q16 != nullptr)
    qk_encode_kernel<T, true><<<static_cast<unsigned>(a.nv_ctas), 256, 0, stream>>>(a);
  else
    qk_encode_kernel<T, false><<<static_cast<unsigned>(a.nv_ctas), 256, 0, stream>>>(a);
  return launch_status();
}

extern "C" {
qk4v8_status quantize_qkv(const qk4v8_qkv_params* p, void* workspace, size_t workspace_bytes,
                          cudaStream_t stream) {
  if (p == nullptr || !p->q || !p->k || !p->v || !p->q_codes || !p->q_scales ||
      !p->q_tensor_scale || !p->k_codes || !p->k_scales || !p->k_tensor_scale || !p->v_codes ||
      !p->v_scales || workspace == nullptr)
    return QK4V8_ERR_INVALID_ARG;
  if (p->dtype != QK4V8_F16 && p->dtype != QK4V8_BF16) return QK4V8_ERR_INVALID_ARG;
  if (p->q_rows <= 0 || p->k_rows <= 0 || p->v_bh <= 0 || p->v_tokens <= 0)
    return QK4V8_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128) return QK4V8_ERR_UNSUPPORTED;
  const bool qk16 = p->q16 != nullptr;
  if ((p->k16 != nullptr) != qk16) return QK4V8_ERR_INVALID_ARG;
  if (!aligned(p->q, 16) || !aligned(p->k, 16) || !aligned(p->v, 16) || !aligned(p->q_codes, 8) ||
      !aligned(p->k_codes, 8) || !aligned(p->v_codes, 16) || !aligned(workspace, 4) ||
      (qk16 && (!aligned(p->q16, 16) || !aligned(p->k16, 16))) || !aligned(p->v16, 16))
    return QK4V8_ERR_INVALID_ARG;
  if (workspace_bytes < quantize_qkv_workspace_size()) return QK4V8_ERR_INVALID_ARG;
  if (p->v_bh > 0x7fffffff / ((p->v_tokens + 127) / 128)) return QK4V8_ERR_UNSUPPORTED;
  if ((p->q_rows + p->k_rows) * (p->head_dim / 16) / kChunkBlocks > 0x3fffffffLL) return QK4V8_ERR_UNSUPPORTED;
  float* q_part = static_cast<float*>(workspace);
  float* k_part = q_part + kAmaxPartials;
  if (p->dtype == QK4V8_BF16)
    return p->head_dim == 128 ? launch_qkv<__nv_bfloat16, 128>(p, q_part, k_part, stream)
                              : launch_qkv<__nv_bfloat16, 64>(p, q_part, k_part, stream);
  return p->head_dim == 128 ? launch_qkv<__half, 128>(p, q_part, k_part, stream)
                            : launch_qkv<__half, 64>(p, q_part, k_part, stream);
}

// ------------------------------------------------------------------------------------------
size_t tile_score_select_workspace_size(int32_t batch, int32_t q_heads, int32_t kv_heads,
                                        int32_t n_tokens) {
  const int64_t t = (n_tokens + 127) / 128;
  return static_cast<size_t>((static_cast<int64_t>(batch) * q_heads * t +
                              static_cast<int64_t>(batch) * kv_heads * t) * 8);
}

qk4v8_status tile_score_select(const uint8_t* q_codes, const uint8_t* q_scales,
                               const uint8_t* k_codes, const uint8_t* k_scales, int32_t batch,
                               int32_t q_heads, int32_t kv_heads, int32_t n_tokens,
                               int32_t head_dim, int32_t causal, int32_t frac_bp, int32_t k_max,
                               int32_t* idx, int32_t* n_sel, uint8_t* bitmap, void* workspace,
                               size_t workspace_bytes, cudaStream_t stream) {
  if (!q_codes || !q_scales || !k_codes || !k_scales || !idx || !n_sel || !workspace)
    return QK4V8_ERR_INVALID_ARG;
  if (batch <= 0 || q_heads <= 0 || kv_heads <= 0 || n_tokens <= 0 || q_heads % kv_heads)
    return QK4V8_ERR_INVALID_ARG;
  if (frac_bp < 0 || frac_bp > 10000 || k_max < 0) return QK4V8_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return QK4V8_ERR_UNSUPPORTED;
  if (!aligned(q_codes, 16) || !aligned(k_codes, 16) || !aligned(workspace, 8))
    return QK4V8_ERR_INVALID_ARG;
  if (workspace_bytes < tile_score_select_workspace_size(batch, q_heads, kv_heads, n_tokens))
    return QK4V8_ERR_INVALID_ARG;
  const int32_t T = (n_tokens + 127) / 128;
  int64_t n_cand = 0;
  if (causal) for (int qt = 0; qt < T; ++qt) n_cand += qt + 1;
  else n_cand = static_cast<int64_t>(T) * T;
  const int64_t k = (n_cand * frac_bp + 9999) / 10000;
  if (k > k_max) return QK4V8_ERR_INVALID_ARG;
  if (k_max > kSelectMax || T > 4096) return QK4V8_ERR_UNSUPPORTED;
  auto* qmax = static_cast<unsigned long long*>(workspace);
  auto* kmax = qmax + static_cast<int64_t>(batch) * q_heads * T;
  if (cudaMemsetAsync(workspace, 0, tile_score_select_workspace_size(batch, q_heads, kv_heads, n_tokens), stream) != cudaSuccess)
    return QK4V8_ERR_CUDA;
  const int64_t qrows = static_cast<int64_t>(batch) * q_heads * n_tokens;
  const int64_t krows = static_cast<int64_t>(batch) * kv_heads * n_tokens;
  if (head_dim == 128) {
    row_norm_tile_max_kernel<128><<<(qrows * 4 + 255) / 256, 256, 0, stream>>>(q_codes, q_scales, static_cast<int64_t>(batch) * q_heads, n_tokens, T, qmax);
    row_norm_tile_max_kernel<128><<<(krows * 4 + 255) / 256, 256, 0, stream>>>(k_codes, k_scales, static_cast<int64_t>(batch) * kv_heads, n_tokens, T, kmax);
  } else {
    row_norm_tile_max_kernel<64><<<(qrows * 2 + 255) / 256, 256, 0, stream>>>(q_codes, q_scales, static_cast<int64_t>(batch) * q_heads, n_tokens, T, qmax);
    row_norm_tile_max_kernel<64><<<(krows * 2 + 255) / 256, 256, 0, stream>>>(k_codes, k_scales, static_cast<int64_t>(batch) * kv_heads, n_tokens, T, kmax);
  }
  if (launch_status() != QK4V8_OK) return QK4V8_ERR_CUDA;
  const int smem = (2 * T + 2) * 8 + kSelectMax * (16 + 4);
  static PerDeviceOnce opt_in;
  if (!opt_in.run(current_device(), [] {
        return set_smem(tile_select_kernel, (2 * 4096 + 2) * 8 + kSelectMax * 20);
      }))
    return QK4V8_ERR_CUDA;
  tile_select_kernel<<<batch * q_heads, kSelectThreads, smem, stream>>>(
      qmax, kmax, q_heads, kv_heads, T, T, causal, frac_bp, k_max, idx, n_sel, bitmap);
  return launch_status();
}

// ------------------------------------------------------------------------------------------
}  // extern "C"
template <int D, bool kMixed, bool kUA = false, bool kDQ = false>
static qk4v8_status launch_fwd(const qk4v8_fwd_params* p, cudaStream_t stream) {
  using L = FwdLayout<D, kMixed, kDQ>;
  const int32_t B = p->batch, Hq = p->q_heads, Hkv = p->kv_heads;
  const int32_t Nq = p->n_q, Nk = p->n_k;
  const int32_t npad = (Nk + 127) / 128 * 128;
  const CUtensorMapSwizzle qk_sw = (D == 128) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  CUtensorMap tq, tk, tv, tq16, tk16, tv16;
  {
    const uint64_t dq[3] = {D / 2, static_cast<uint64_t>(Nq), static_cast<uint64_t>(B) * Hq};
    const uint64_t sq[2] = {D / 2, static_cast<uint64_t>(Nq) * (D / 2)};
    const uint32_t bq[3] = {D / 2, 128, 1};
    if (!make_map(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, p->q_codes, dq, sq, bq, qk_sw)) return QK4V8_ERR_CUDA;
    const uint64_t dk[3] = {D / 2, static_cast<uint64_t>(Nk), static_cast<uint64_t>(B) * Hkv};
    const uint64_t sk[2] = {D / 2, static_cast<uint64_t>(Nk) * (D / 2)};
    if (!make_map(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, p->k_codes, dk, sk, bq, qk_sw)) return QK4V8_ERR_CUDA;
    const uint64_t dv[2] = {static_cast<uint64_t>(npad), static_cast<uint64_t>(B) * Hkv * D};
    const uint64_t sv[1] = {static_cast<uint64_t>(npad)};
    const uint32_t bv[2] = {128, D};
    if (!make_map(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, p->v_codes, dv, sv, bv, CU_TENSOR_MAP_SWIZZLE_128B)) return QK4V8_ERR_CUDA;
  }
  constexpr bool dual = kDQ;
  if (dual) {                                   // the FP16-Q map slot carries the second Q
    tk16 = tk; tv16 = tv;
    const uint64_t dq[3] = {D / 2, static_cast<uint64_t>(Nq), static_cast<uint64_t>(B) * Hq};
    const uint64_t sq[2] = {D / 2, static_cast<uint64_t>(Nq) * (D / 2)};
    const uint32_t bq[3] = {D / 2, 128, 1};
    if (!make_map(&tq16, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, p->q2_codes, dq, sq, bq, qk_sw)) return QK4V8_ERR_CUDA;
  } else if (kMixed) {
    const uint64_t dq[3] = {D, static_cast<uint64_t>(Nq), static_cast<uint64_t>(B) * Hq};
    const uint64_t sq[2] = {D * 2, static_cast<uint64_t>(Nq) * D * 2};
    const uint32_t bq[3] = {64, 128, 1};
    // the caller's 16-bit Q and K, in their own type
    const CUtensorMapDataType t16 = (p->qk16_dtype == QK4V8_BF16) ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                                 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (!make_map(&tq16, t16, 3, p->q16, dq, sq, bq, CU_TENSOR_MAP_SWIZZLE_128B)) return QK4V8_ERR_CUDA;
    const uint64_t dk[3] = {D, static_cast<uint64_t>(Nk), static_cast<uint64_t>(B) * Hkv};
    const uint64_t sk[2] = {D * 2, static_cast<uint64_t>(Nk) * D * 2};
    if (!make_map(&tk16, t16, 3, p->k16, dk, sk, bq, CU_TENSOR_MAP_SWIZZLE_128B)) return QK4V8_ERR_CUDA;
    const uint64_t dv[2] = {static_cast<uint64_t>(npad), static_cast<uint64_t>(B) * Hkv * D};
    const uint64_t sv[1] = {static_cast<uint64_t>(npad) * 2};
    const uint32_t bv[2] = {64, D};
    if (!make_map(&tv16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, p->v16, dv, sv, bv, CU_TENSOR_MAP_SWIZZLE_128B)) return QK4V8_ERR_CUDA;
  } else {
    tq16 = tq; tk16 = tk; tv16 = tv;
  }
  static PerDeviceOnce opt_in;                  // one per kernel instance
  if (!opt_in.run(current_device(), [] { return set_smem(attn_fwd_kernel<D, kMixed, kUA, kDQ>, L::SMEM_ALLOC); }))
    return QK4V8_ERR_CUDA;
  FwdArgs a;
  a.q_scales = p->q_scales; a.k_scales = p->k_scales; a.v_scales = p->v_scales;
  a.q2_scales = dual ? p->q2_scales : nullptr;
  a.q_ts = p->q_tensor_scale; a.k_ts = p->k_tensor_scale;
  a.bitmap = p->fp16_bitmap; a.out = p->out; a.lse = p->lse;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.Npad = npad;
  a.Tq = (Nq + 127) / 128; a.Tk = (Nk + 127) / 128;
  a.causal = p->causal ? 1 : 0;
  a.softmax_scale = p->softmax_scale;
  a.out_kind = static_cast<int32_t>(p->out_dtype);
  a.qk16_bf16 = (kMixed && p->qk16_dtype == QK4V8_BF16) ? 1 : 0;
  // Persistent: one CTA per SM (or per work item when there are fewer items).
  const int64_t items = static_cast<int64_t>(a.Tq) * B * Hq;
  if (items > INT32_MAX / 2) return QK4V8_ERR_UNSUPPORTED;
  const int64_t grid = items < sm_count() ? items : sm_count();
  attn_fwd_kernel<D, kMixed, kUA, kDQ><<<static_cast<unsigned>(grid), L::THREADS, L::SMEM_ALLOC, stream>>>(tq, tk, tv, tq16, tk16, tv16, a);
  return launch_status();
}

// The FP4-only path: two query tiles per CTA, one softmax warpgroup each (attn_pp.cuh).
template <int D>
static qk4v8_status launch_pp(const qk4v8_fwd_params* p, cudaStream_t stream) {
  using L = PPLayout<D>;
  const int32_t B = p->batch, Hq = p->q_heads, Hkv = p->kv_heads;
  const int32_t Nq = p->n_q, Nk = p->n_k;
  const int32_t npad = (Nk + 127) / 128 * 128;
  const CUtensorMapSwizzle qk_sw = (D == 128) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  CUtensorMap tq, tk, tv;
  const uint64_t dq[3] = {D / 2, static_cast<uint64_t>(Nq), static_cast<uint64_t>(B) * Hq};
  const uint64_t sq[2] = {D / 2, static_cast<uint64_t>(Nq) * (D / 2)};
  const uint32_t bq[3] = {D / 2, 128, 1};
  if (!make_map(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, p->q_codes, dq, sq, bq, qk_sw)) return QK4V8_ERR_CUDA;
  const uint64_t dk[3] = {D / 2, static_cast<uint64_t>(Nk), static_cast<uint64_t>(B) * Hkv};
  const uint64_t sk[2] = {D / 2, static_cast<uint64_t>(Nk) * (D / 2)};
  if (!make_map(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, p->k_codes, dk, sk, bq, qk_sw)) return QK4V8_ERR_CUDA;
  const uint64_t dv[2] = {static_cast<uint64_t>(npad), static_cast<uint64_t>(B) * Hkv * D};
  const uint64_t sv[1] = {static_cast<uint64_t>(npad)};
  const uint32_t bv[2] = {128, D};
  if (!make_map(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, p->v_codes, dv, sv, bv, CU_TENSOR_MAP_SWIZZLE_128B)) return QK4V8_ERR_CUDA;
  // One-time set-up per device: the shared-memory opt-in, and a check that the kernel launches
  // with the register count its setmaxnreg split is computed from (a split above the launch's
  // registers would leave the softmax warps waiting for registers that never free).
  static PerDeviceOnce opt_in;
  if (!opt_in.run(current_device(), [] {
        cudaFuncAttributes fa;
        return set_smem(attn_pp_kernel<D>, L::SMEM_ALLOC) &&
               cudaFuncGetAttributes(&fa, attn_pp_kernel<D>) == cudaSuccess &&
               fa.numRegs == L::REGS_LAUNCH;
      }))
    return QK4V8_ERR_CUDA;
  FwdArgs a;
  a.q_scales = p->q_scales; a.k_scales = p->k_scales; a.v_scales = p->v_scales;
  a.q2_scales = nullptr;
  a.q_ts = p->q_tensor_scale; a.k_ts = p->k_tensor_scale;
  a.bitmap = nullptr; a.out = p->out; a.lse = p->lse;
  a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.Nq = Nq; a.Nk = Nk; a.Npad = npad;
  a.Tq = (Nq + 127) / 128; a.Tk = (Nk + 127) / 128;
  a.causal = p->causal ? 1 : 0;
  a.softmax_scale = p->softmax_scale;
  a.out_kind = static_cast<int32_t>(p->out_dtype);
  a.qk16_bf16 = 0;
  const int64_t items = static_cast<int64_t>(a.Tq) * B * Hq;     // an upper bound of the pairs
  if (items > INT32_MAX / 2) return QK4V8_ERR_UNSUPPORTED;
  const int64_t n_pairs = pp_items(B, Hq, Hkv, a.Tq);
  const int64_t grid = n_pairs < sm_count() ? n_pairs : sm_count();
  attn_pp_kernel<D><<<static_cast<unsigned>(grid), L::THREADS, L::SMEM_ALLOC, stream>>>(tq, tk, tv, a);
  return launch_status();
}

extern "C" {
qk4v8_status attn_qk4v8_fwd(const qk4v8_fwd_params* p, cudaStream_t stream) {
  if (p == nullptr) return QK4V8_ERR_INVALID_ARG;
  if (!p->q_codes || !p->q_scales || !p->q_tensor_scale || !p->k_codes || !p->k_scales ||
      !p->k_tensor_scale || !p->v_codes || !p->v_scales || !p->out)
    return QK4V8_ERR_INVALID_ARG;
  if (p->batch <= 0 || p->q_heads <= 0 || p->kv_heads <= 0 || p->n_q <= 0 || p->n_k <= 0)
    return QK4V8_ERR_INVALID_ARG;
  if (p->q_heads % p->kv_heads) return QK4V8_ERR_INVALID_ARG;
  if (p->causal && p->n_q != p->n_k) return QK4V8_ERR_INVALID_ARG;
  if (p->out_dtype != QK4V8_F16 && p->out_dtype != QK4V8_BF16 && p->out_dtype != QK4V8_F32)
    return QK4V8_ERR_INVALID_ARG;
  if (!(p->softmax_scale > 0.f)) return QK4V8_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128) return QK4V8_ERR_UNSUPPORTED;
  const size_t sa = p->head_dim == 128 ? 8 : 4;
  if (!aligned(p->q_codes, 16) || !aligned(p->k_codes, 16) || !aligned(p->v_codes, 16) ||
      !aligned(p->q_scales, sa) || !aligned(p->k_scales, sa) || !aligned(p->v_scales, 4) ||
      !aligned(p->out, 16))
    return QK4V8_ERR_INVALID_ARG;
  const bool mixed = p->fp16_bitmap != nullptr;
  if (mixed && (!p->q16 || !p->k16 || !p->v16 || !aligned(p->q16, 16) || !aligned(p->k16, 16) ||
                !aligned(p->v16, 16) || (p->qk16_dtype != QK4V8_F16 && p->qk16_dtype != QK4V8_BF16)))
    return QK4V8_ERR_INVALID_ARG;
  const int64_t tiles = static_cast<int64_t>((p->n_q + 127) / 128) * p->batch * p->q_heads;
  if (tiles > 0x7fffffffLL) return QK4V8_ERR_UNSUPPORTED;
  if (p->p_underflow_aware != 0 && p->p_underflow_aware != 1) return QK4V8_ERR_INVALID_ARG;
  if ((p->q2_codes == nullptr) != (p->q2_scales == nullptr)) return QK4V8_ERR_INVALID_ARG;
  if (p->q2_codes != nullptr && (!aligned(p->q2_codes, 16) || !aligned(p->q2_scales, sa)))
    return QK4V8_ERR_INVALID_ARG;
  if (p->q2_codes != nullptr && mixed) return QK4V8_ERR_UNSUPPORTED;
  const bool dq = p->q2_codes != nullptr;
  if (p->p_underflow_aware || dq) {
    if (mixed) return QK4V8_ERR_UNSUPPORTED;
    if (p->head_dim == 128) {
      if (p->p_underflow_aware) return dq ? launch_fwd<128, false, true, true>(p, stream) : launch_fwd<128, false, true>(p, stream);
      return launch_fwd<128, false, false, true>(p, stream);
    }
    if (p->p_underflow_aware) return dq ? launch_fwd<64, false, true, true>(p, stream) : launch_fwd<64, false, true>(p, stream);
    return launch_fwd<64, false, false, true>(p, stream);
  }
  if (p->head_dim == 128) return mixed ? launch_fwd<128, true>(p, stream) : launch_pp<128>(p, stream);
  return mixed ? launch_fwd<64, true>(p, stream) : launch_pp<64>(p, stream);
}

// ------------------------------------------------------------------------------------------
static int32_t decode_splits(const qk4v8_decode_params* p) {
  return (p->max_context + p->split_tokens - 1) / p->split_tokens;
}

size_t attn_qk4v8_decode_workspace_size(const qk4v8_decode_params* p) {
  if (p == nullptr || p->split_tokens <= 0 || p->max_context <= 0) return 0;
  return static_cast<size_t>(p->num_seqs) * p->q_heads * decode_splits(p) * (p->head_dim + 2) * 4;
}

qk4v8_status attn_qk4v8_decode_paged(const qk4v8_decode_params* p, void* workspace,
                                     size_t workspace_bytes, cudaStream_t stream) {
  if (p == nullptr) return QK4V8_ERR_INVALID_ARG;
  if (!p->q_codes || !p->q_scales || !p->q_tensor_scale || !p->k_pages || !p->k_page_scales ||
      !p->k_tensor_scale || !p->v_pages || !p->v_page_scales || !p->page_table ||
      !p->context_lens || !p->out || !workspace)
    return QK4V8_ERR_INVALID_ARG;
  if (p->num_seqs <= 0 || p->num_pages <= 0 || p->max_pages <= 0 || p->q_heads <= 0 ||
      p->kv_heads <= 0 || p->q_heads % p->kv_heads || p->max_context <= 0)
    return QK4V8_ERR_INVALID_ARG;
  if (p->split_tokens <= 0 || p->split_tokens % 128) return QK4V8_ERR_INVALID_ARG;
  if (p->split_tokens > 64 * DecLayout<4>::MAX_SPLIT_PAGES) return QK4V8_ERR_UNSUPPORTED;
  if (p->max_context > 64 * p->max_pages) return QK4V8_ERR_INVALID_ARG;
  if (p->out_dtype != QK4V8_F16 && p->out_dtype != QK4V8_BF16 && p->out_dtype != QK4V8_F32)
    return QK4V8_ERR_INVALID_ARG;
  if (!(p->softmax_scale > 0.f)) return QK4V8_ERR_INVALID_ARG;
  if (p->p_underflow_aware != 0 && p->p_underflow_aware != 1) return QK4V8_ERR_INVALID_ARG;
  if ((p->q2_codes == nullptr) != (p->q2_scales == nullptr)) return QK4V8_ERR_INVALID_ARG;
  if (p->q2_codes != nullptr && (!aligned(p->q2_codes, 16) || !aligned(p->q2_scales, 8)))
    return QK4V8_ERR_INVALID_ARG;
  if (p->head_dim != 128 || p->q_heads / p->kv_heads > 16) return QK4V8_ERR_UNSUPPORTED;
  if (!aligned(p->q_codes, 16) || !aligned(p->k_pages, 16) || !aligned(p->v_pages, 16) ||
      !aligned(p->q_scales, 8) || !aligned(p->k_page_scales, 8) || !aligned(p->v_page_scales, 4) ||
      !aligned(workspace, 16))
    return QK4V8_ERR_INVALID_ARG;
  if (workspace_bytes < attn_qk4v8_decode_workspace_size(p)) return QK4V8_ERR_INVALID_ARG;
  const int32_t n_splits = decode_splits(p);
  if (n_splits > 65535 || p->num_seqs > 65535 || p->kv_heads > 65535) return QK4V8_ERR_UNSUPPORTED;
  // the page maps' rows (page, KV head, channel) are addressed by 32-bit TMA coordinates
  if (static_cast<int64_t>(p->num_pages) * p->kv_heads * 128 > 0x7fffffffLL) return QK4V8_ERR_UNSUPPORTED;
  constexpr int D = 128;
  CUtensorMap tq, tq2, tkp, tvp;
  {
    const uint64_t dq[2] = {D / 2, static_cast<uint64_t>(p->num_seqs) * p->q_heads};
    const uint64_t sq[1] = {D / 2};
    const uint32_t bq[2] = {D / 2, 16};
    if (!make_map(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, p->q_codes, dq, sq, bq, CU_TENSOR_MAP_SWIZZLE_64B)) return QK4V8_ERR_CUDA;
    tq2 = tq;                                    // the second Q tensor's map (dual-residual Q)
    if (p->q2_codes != nullptr &&
        !make_map(&tq2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, p->q2_codes, dq, sq, bq, CU_TENSOR_MAP_SWIZZLE_64B))
      return QK4V8_ERR_CUDA;
    const uint64_t dk[2] = {D / 2, static_cast<uint64_t>(p->num_pages) * p->kv_heads * 64};
    const uint32_t bk[2] = {D / 2, 64};
    if (!make_map(&tkp, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, p->k_pages, dk, sq, bk, CU_TENSOR_MAP_SWIZZLE_64B)) return QK4V8_ERR_CUDA;
    const uint64_t dv[2] = {64, static_cast<uint64_t>(p->num_pages) * p->kv_heads * D};
    const uint64_t sv[1] = {64};
    const uint32_t bv[2] = {64, D};
    if (!make_map(&tvp, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, p->v_pages, dv, sv, bv, CU_TENSOR_MAP_SWIZZLE_64B)) return QK4V8_ERR_CUDA;
  }
  static PerDeviceOnce opt_in;
  if (!opt_in.run(current_device(), [] {
        return set_smem(decode_kernel<4, false>, DecLayout<4>::SMEM_ALLOC) &&
               set_smem(decode_kernel<8, false>, DecLayout<8>::SMEM_ALLOC) &&
               set_smem(decode_kernel<16, false>, DecLayout<16>::SMEM_ALLOC) &&
               set_smem(decode_kernel<4, true>, DecLayout<4>::SMEM_ALLOC) &&
               set_smem(decode_kernel<8, true>, DecLayout<8>::SMEM_ALLOC) &&
               set_smem(decode_kernel<16, true>, DecLayout<16>::SMEM_ALLOC) &&
               set_smem(decode_kernel<4, false, true>, DecLayout<4, true>::SMEM_ALLOC) &&
               set_smem(decode_kernel<8, false, true>, DecLayout<8, true>::SMEM_ALLOC) &&
               set_smem(decode_kernel<16, false, true>, DecLayout<16, true>::SMEM_ALLOC) &&
               set_smem(decode_kernel<4, true, true>, DecLayout<4, true>::SMEM_ALLOC) &&
               set_smem(decode_kernel<8, true, true>, DecLayout<8, true>::SMEM_ALLOC) &&
               set_smem(decode_kernel<16, true, true>, DecLayout<16, true>::SMEM_ALLOC);
      }))
    return QK4V8_ERR_CUDA;
  DecArgs a;
  a.q_scales = p->q_scales; a.q2_scales = p->q2_scales; a.q_ts = p->q_tensor_scale;
  a.k_page_scales = p->k_page_scales; a.k_ts = p->k_tensor_scale;
  a.v_page_scales = p->v_page_scales; a.page_table = p->page_table; a.lens = p->context_lens;
  a.ws = static_cast<float*>(workspace);
  a.S = p->num_seqs; a.Hq = p->q_heads; a.Hkv = p->kv_heads; a.max_pages = p->max_pages;
  a.n_splits = n_splits; a.split_tokens = p->split_tokens; a.num_pages = p->num_pages;
  a.softmax_scale = p->softmax_scale;
  dim3 grid(n_splits, p->kv_heads, p->num_seqs);
  // the softmax handles the g = Hq / Hkv real query columns: an instance per bound on g
  const int g = p->q_heads / p->kv_heads;
  const bool ua = p->p_underflow_aware != 0;
  const bool dq = p->q2_codes != nullptr;
#define QK4V8_DEC1(GM, UA, DQ) \
  decode_kernel<GM, UA, DQ><<<grid, DecLayout<GM, DQ>::THREADS, DecLayout<GM, DQ>::SMEM_ALLOC, stream>>>(tq, tkp, tvp, tq2, a)
#define QK4V8_DEC(GM)                                                                              \
  (ua ? (dq ? QK4V8_DEC1(GM, true, true) : QK4V8_DEC1(GM, true, false))                            \
      : (dq ? QK4V8_DEC1(GM, false, true) : QK4V8_DEC1(GM, false, false)))
  if (g <= 4) QK4V8_DEC(4);
  else if (g <= 8) QK4V8_DEC(8);
  else QK4V8_DEC(16);
#undef QK4V8_DEC1
#undef QK4V8_DEC
  if (launch_status() != QK4V8_OK) return QK4V8_ERR_CUDA;
  decode_merge_kernel<<<p->num_seqs * p->q_heads, 128, 0, stream>>>(
      a.ws, n_splits, static_cast<int32_t>(p->out_dtype), p->out, p->lse);
  return launch_status();
}

}  // extern "C"

// ------------------------------------------------------------------------------------------
// Allocation-free decode: the split partials live in one fixed file-scope device buffer.
// Host code must not use the array's name as a pointer (on the host it is only a stand-in);
// its device address is looked up once per device with the device current.
// ------------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_decode_scratch[QK4V8_NOALLOC_DECODE_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
}  // namespace

extern "C" qk4v8_status attn_qk4v8_decode_paged_noalloc(const qk4v8_decode_params* p,
                                                        cudaStream_t stream) {
  if (p == nullptr) return QK4V8_ERR_INVALID_ARG;
  const size_t need = attn_qk4v8_decode_workspace_size(p);
  if (need == 0) return QK4V8_ERR_INVALID_ARG;
  if (need > QK4V8_NOALLOC_DECODE_SCRATCH_BYTES) return QK4V8_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QK4V8_ERR_CUDA;
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_noalloc_decode_scratch) != cudaSuccess || addr == nullptr)
        return QK4V8_ERR_CUDA;
      g_noalloc_ptr[dev] = addr;
    }
    ptr = g_noalloc_ptr[dev];
  }
  return attn_qk4v8_decode_paged(p, ptr, QK4V8_NOALLOC_DECODE_SCRATCH_BYTES, stream);
}

// ------------------------------------------------------------------------------------------
extern "C" qk4v8_status kv_append_paged(const qk4v8_append_params* p, cudaStream_t stream) {
  if (p == nullptr || p->k_new == nullptr || p->v_new == nullptr || p->cu_new == nullptr ||
      p->lens == nullptr || p->page_table == nullptr || p->k_pages == nullptr ||
      p->k_page_scales == nullptr || p->k_tensor_scale == nullptr || p->v_pages == nullptr ||
      p->v_page_scales == nullptr || p->v_tail == nullptr)
    return QK4V8_ERR_INVALID_ARG;
  if (p->dtype != QK4V8_F16 && p->dtype != QK4V8_BF16) return QK4V8_ERR_INVALID_ARG;
  if (p->num_seqs <= 0 || p->kv_heads <= 0 || p->num_pages <= 0 || p->max_pages <= 0 ||
      p->max_new < 0)
    return QK4V8_ERR_INVALID_ARG;
  if (p->head_dim != 128) return QK4V8_ERR_UNSUPPORTED;
  if (p->num_seqs > 65535 || p->kv_heads > 65535) return QK4V8_ERR_UNSUPPORTED;
  if (!aligned(p->k_new, 16) || !aligned(p->v_new, 16) || !aligned(p->k_pages, 8) ||
      !aligned(p->v_pages, 16) || !aligned(p->v_tail, 16))
    return QK4V8_ERR_INVALID_ARG;
  AppendArgs a;
  a.k_new = p->k_new; a.v_new = p->v_new; a.cu_new = p->cu_new; a.lens = p->lens;
  a.page_table = p->page_table;
  a.k_pages = p->k_pages; a.k_scales = p->k_page_scales; a.k_ts = p->k_tensor_scale;
  a.v_pages = p->v_pages; a.v_scales = p->v_page_scales; a.v_tail = p->v_tail;
  a.S = p->num_seqs; a.num_pages = p->num_pages; a.max_pages = p->max_pages;
  a.Hkv = p->kv_heads; a.max_new = p->max_new;
  // one CTA per (32-token group the new tokens touch, KV head, sequence)
  const dim3 grid((p->max_new + 31) / 32 + 1, p->kv_heads, p->num_seqs);
  if (p->dtype == QK4V8_BF16) kv_append_kernel<__nv_bfloat16><<<grid, 128, 0, stream>>>(a);
  else kv_append_kernel<__half><<<grid, 128, 0, stream>>>(a);
  return launch_status();
}

extern "C" qk4v8_status quantize_nvfp4_residual(const void* x, qk4v8_dtype dtype, int64_t rows,
                                                int32_t cols, int64_t row_stride,
                                                const uint8_t* codes, const uint8_t* scales,
                                                const float* tensor_scale, uint8_t* codes2,
                                                uint8_t* scales2, cudaStream_t stream) {
  return quantize_nvfp4_residual_impl(x, dtype, rows, cols, row_stride, codes, scales,
                                      tensor_scale, codes2, scales2, stream);
}
