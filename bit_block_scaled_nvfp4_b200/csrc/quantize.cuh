// Quantize kernels: NVFP4 for Q and K (tqpw.cn "块缩放数值格式" article §2.2: E2M1
// elements, E4M3 scale per 16 elements, FP32 tensor scale) and MXFP8 for V (§2.1: E8M0 scale
// per 32 elements; here along the token axis, per channel).
//
// NVFP4 arithmetic (every step a single IEEE FP32 operation rounded to nearest, subnormals
// kept):  s_t = amax / 2688 (1 when amax == 0);  s_b = E4M3(amax_b / 6 / s_t);
// den = s_b * s_t;  code = E2M1(x / den), all codes 0 when s_b == 0.  E2M1 pairs are packed
// low nibble first. Conversions round to nearest even and saturate; the sign bit of every
// code is the sign of its input, so a negative value that rounds to zero is negative zero.
#pragma once
#include "ptx.cuh"

namespace qk4v8 {

template <typename T> __device__ __forceinline__ float to_float(T v);
template <> __device__ __forceinline__ float to_float<__half>(__half v) { return __half2float(v); }
template <> __device__ __forceinline__ float to_float<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// Eight 16-bit values from one 16-byte load.
template <typename T>
__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const T* h = reinterpret_cast<const T*>(&u);
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = to_float<T>(h[i]);
}

__device__ __forceinline__ float e4m3_code_to_float(uint32_t code) {
  return __low2float(e4m3x2_to_half2(code & 0xFFu));
}

// Element offset of 16-element block i (row i / bpr, block i % bpr of that row); a dense
// tensor needs no division.
__device__ __forceinline__ int64_t block_offset(int64_t i, uint32_t bpr, int64_t row_stride,
                                                bool contiguous) {
  if (contiguous) return i * 16;
  const int64_t r = i / bpr;
  return r * row_stride + static_cast<int64_t>(i - r * bpr) * 16;
}

// ---------------------------------------------------------------------------------------
// Pass 1: tensor amax. A grid of four CTAs per SM; CTA c writes the maximum of |x| over its
// share to partial[c] (no atomics, nothing to clear), and the encode pass reduces the
// partials. Four blocks of 16 per thread are loaded before any is reduced.
// ---------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const T* __restrict__ x, int64_t rows,
                                                         int32_t cols, int64_t row_stride,
                                                         float* __restrict__ partial) {
  const uint32_t blocks_per_row = static_cast<uint32_t>(cols / 16);
  const int64_t total = rows * blocks_per_row;
  const bool contiguous = (row_stride == cols);
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
  float m = 0.f;
  for (int64_t i0 = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i0 < total;
       i0 += 4 * step) {
    uint4 u[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t i = i0 + k * step;
      u[2 * k] = u[2 * k + 1] = make_uint4(0, 0, 0, 0);
      if (i < total) {
        const uint4* p = reinterpret_cast<const uint4*>(x + block_offset(i, blocks_per_row, row_stride, contiguous));
        u[2 * k] = __ldg(p);
        u[2 * k + 1] = __ldg(p + 1);
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float f[8];
      unpack8<T>(u[k], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t = fmaxf(t, wm[w]);
    partial[blockIdx.x] = t;
  }
}

// Maximum of n (<= 1024) partial maxima, by every thread of a 256-thread CTA.
__device__ __forceinline__ float reduce_partials(const float* __restrict__ partial, int n) {
  float m = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, partial[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) t = fmaxf(t, wm[w]);
  return t;
}

// One 16-element NVFP4 block with tensor scale s_t: returns the E4M3 scale code and writes
// the 8 code bytes (element 2i in the low nibble of byte i) to w[0..1].
__device__ __forceinline__ void e2m1_encode16(const float* f, float den, uint32_t* w);
__device__ __forceinline__ uint32_t nvfp4_encode16(const float* f, float s_t, uint32_t* w) {
  float amax_b = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) amax_b = fmaxf(amax_b, fabsf(f[k]));
  const float sbf = __fdiv_rn(__fdiv_rn(amax_b, 6.f), s_t);
  const uint32_t sc = cvt_e4m3x2(sbf, 0.f) & 0xFFu;
  const float sbv = e4m3_code_to_float(sc);
  w[0] = w[1] = 0u;
  if (sbv != 0.f) e2m1_encode16(f, __fmul_rn(sbv, s_t), w);
  return sc;
}

// The 16 E2M1 codes of a block under divisor den (> 0): code_i = E2M1(fl32(x_i / den)), the
// quotient correctly rounded (Markstein's division inside its safe range, else IEEE).
__device__ __forceinline__ void e2m1_encode16(const float* f, float den, uint32_t* w) {
  w[0] = w[1] = 0u;
  const bool fast = (den >= 0x1p-90f && den <= 0x1p90f);
  const float y = __frcp_rn(den);
#pragma unroll
  for (int k = 0; k < 16; k += 2) {
    const float q0 = fast ? div_markstein(f[k], den, y) : __fdiv_rn(f[k], den);
    const float q1 = fast ? div_markstein(f[k + 1], den, y) : __fdiv_rn(f[k + 1], den);
    uint32_t byte = cvt_e2m1x2(q0, q1) & 0x77u;
    byte |= (__float_as_uint(f[k]) >> 31) << 3;
    byte |= (__float_as_uint(f[k + 1]) >> 31) << 7;
    w[k >> 3] |= byte << ((k & 7) * 4);
  }
}

// E2M1 code (magnitude in bits 0-2, sign in bit 3) -> its value, exactly.
__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const uint32_t m = c & 7u;
  const float v = (m < 2u) ? 0.5f * static_cast<float>(m)
                           : __uint_as_float((((m >> 1) + 126u) << 23) | ((m & 1u) << 22));
  return (c & 8u) ? -v : v;
}

// NVFP4 block with a scale search (outlier-aware keys): the E4M3 scale codes c0, c0 - 1,
// c0 - 2, c0 + 1 (c0 the usual choice; codes outside 1..126 skipped) each encode the block, and
// the one with the smallest squared error sum_i fl32(d_i^2), d_i = fl32(x_i - fl32(v_i den)),
// accumulated in order with float32 adds, wins (ties to the earlier candidate).
__device__ __forceinline__ uint32_t nvfp4_encode16_searched(const float* f, float s_t, uint32_t* w) {
  float amax_b = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) amax_b = fmaxf(amax_b, fabsf(f[k]));
  const int c0 = static_cast<int>(cvt_e4m3x2(__fdiv_rn(__fdiv_rn(amax_b, 6.f), s_t), 0.f) & 0xFFu);
  w[0] = w[1] = 0u;
  if (c0 == 0) return 0u;
  float best = INFINITY;
  int best_c = c0;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int c = c0 + (t == 3 ? 1 : -t);
    if (c < 1 || c > 126) continue;
    const float den = __fmul_rn(e4m3_code_to_float(static_cast<uint32_t>(c)), s_t);
    uint32_t wc[2];
    e2m1_encode16(f, den, wc);
    float err = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float d = __fsub_rn(f[i], __fmul_rn(e2m1_value((wc[i >> 3] >> (4 * (i & 7))) & 0xFu), den));
      err = __fadd_rn(err, __fmul_rn(d, d));
    }
    if (err < best) {
      best = err;
      best_c = c;
      w[0] = wc[0];
      w[1] = wc[1];
    }
  }
  return static_cast<uint32_t>(best_c);
}

// ---------------------------------------------------------------------------------------
// Pass 2: encode. One thread per 16-element block.
// ---------------------------------------------------------------------------------------
template <typename T, bool kWrite16, bool kSearch = false>
__global__ void __launch_bounds__(256) nvfp4_encode_kernel(
    const T* __restrict__ x, int64_t rows, int32_t cols, int64_t row_stride,
    const float* __restrict__ amax_partial, int32_t n_partial, float tensor_scale_in,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, float* __restrict__ ts_out,
    __half* __restrict__ x16) {
  float s_t;
  if (tensor_scale_in > 0.f) {
    s_t = tensor_scale_in;
  } else {
    const float amax = reduce_partials(amax_partial, n_partial);
    s_t = (amax == 0.f) ? 1.f : __fdiv_rn(amax, 2688.f);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *ts_out = s_t;
  const uint32_t blocks_per_row = static_cast<uint32_t>(cols / 16);
  const int64_t total = rows * blocks_per_row;
  const bool contiguous = (row_stride == cols);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4* p = reinterpret_cast<const uint4*>(x + block_offset(i, blocks_per_row, row_stride, contiguous));
    const uint4 a = __ldg(p), b = __ldg(p + 1);
    float f[16];
    unpack8<T>(a, f);
    unpack8<T>(b, f + 8);
    uint32_t w[2];
    const uint32_t sc = kSearch ? nvfp4_encode16_searched(f, s_t, w) : nvfp4_encode16(f, s_t, w);
    const int64_t blk = i;                        // outputs are dense: block i of row i / bpr
    *reinterpret_cast<uint2*>(codes + blk * 8) = make_uint2(w[0], w[1]);
    scales[blk] = static_cast<uint8_t>(sc);
    if constexpr (kWrite16) {
      __align__(16) __half h[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) h[k] = __float2half_rn(f[k]);
      uint4* o = reinterpret_cast<uint4*>(x16 + blk * 16);
      o[0] = *reinterpret_cast<uint4*>(h);
      o[1] = *reinterpret_cast<uint4*>(h + 8);
    }
  }
}

// ---------------------------------------------------------------------------------------
// Residual of an NVFP4 encoding, encoded again with the same tensor scale (dual-residual
// quantization: x ~ x_hat1 + x_hat2). Per element, in FP32 steps: den = fl32(s_b * s_t),
// d = fl32(value(code) * den), r = fl32(x - d); then r is NVFP4-encoded with s_t.
// ---------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) nvfp4_residual_kernel(
    const T* __restrict__ x, int64_t rows, int32_t cols, int64_t row_stride,
    const uint8_t* __restrict__ codes1, const uint8_t* __restrict__ scales1,
    const float* __restrict__ ts, uint8_t* __restrict__ codes2, uint8_t* __restrict__ scales2) {
  const float s_t = *ts;
  const uint32_t blocks_per_row = static_cast<uint32_t>(cols / 16);
  const int64_t total = rows * blocks_per_row;
  const bool contiguous = (row_stride == cols);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4* p = reinterpret_cast<const uint4*>(x + block_offset(i, blocks_per_row, row_stride, contiguous));
    const uint4 a = __ldg(p), b = __ldg(p + 1);
    const uint2 c1 = __ldg(reinterpret_cast<const uint2*>(codes1 + i * 8));
    const float den = __fmul_rn(e4m3_code_to_float(scales1[i]), s_t);
    float f[16];
    unpack8<T>(a, f);
    unpack8<T>(b, f + 8);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const uint32_t code = ((k < 8 ? c1.x : c1.y) >> (4 * (k & 7))) & 0xFu;
      f[k] = __fsub_rn(f[k], __fmul_rn(e2m1_value(code), den));
    }
    uint32_t w[2];
    const uint32_t sc = nvfp4_encode16(f, s_t, w);
    *reinterpret_cast<uint2*>(codes2 + i * 8) = make_uint2(w[0], w[1]);
    scales2[i] = static_cast<uint8_t>(sc);
  }
}

// ---------------------------------------------------------------------------------------
// Smoothing and Hadamard rotation of 128-wide rows (outlier-aware key quantization): per
// channel x * lam (queries, role 0) or x / lam (keys, role 1), then x H by seven butterfly
// stages — stage s replaces the pair (i, i + 2^s) by (a + b, a - b) — then 2^-3 (queries) or
// 2^-4 (keys), so that logits are unchanged, and one rounding to the 16-bit type. One warp per
// row; lane l holds elements 4l .. 4l+3, so stages 0-1 stay in the lane and stages 2-6 pair
// lanes l and l ^ 2^(s-2).
// ---------------------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ T from_float(float v);
template <> __device__ __forceinline__ __half from_float<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

template <typename T>
__global__ void __launch_bounds__(256) smooth_rotate_kernel(const T* __restrict__ x, int64_t rows,
                                                            const float* __restrict__ lam,
                                                            int32_t role, T* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const T* src = x + row * 128 + lane * 4;
  float v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) v[k] = to_float<T>(src[k]);
  if (lam != nullptr) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      v[k] = role == 0 ? __fmul_rn(v[k], lam[lane * 4 + k]) : __fdiv_rn(v[k], lam[lane * 4 + k]);
  }
#pragma unroll
  for (int s = 0; s < 2; ++s) {                        // pairs inside the lane
    const int h = 1 << s;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (i & h) continue;
      const float a = v[i], b = v[i + h];
      v[i] = __fadd_rn(a, b);
      v[i + h] = __fsub_rn(a, b);
    }
  }
#pragma unroll
  for (int s = 2; s < 7; ++s) {                        // pairs across lanes
    const int h = 1 << (s - 2);
    const bool upper = (lane & h) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float p = __shfl_xor_sync(0xffffffffu, v[i], h);
      v[i] = upper ? __fsub_rn(p, v[i]) : __fadd_rn(v[i], p);
    }
  }
  const float post = role == 0 ? 0.125f : 0.0625f;
  T* dst = out + row * 128 + lane * 4;
#pragma unroll
  for (int k = 0; k < 4; ++k) dst[k] = from_float<T>(__fmul_rn(v[k], post));
}

// ---------------------------------------------------------------------------------------
// MXFP8 for V. v: [BH, N, D] token-major. codes: [BH, D, Npad] token-contiguous; scales:
// [BH, D, Npad/32] E8M0. Npad = N rounded up to 128; padding tokens read as 0.
// Shared exponent (OCP MX rule): e = floor(log2 amax) - 8 clamped to [-127, 127]; code
// e + 127; all-zero group -> 127. Elements E4M3(v * 2^-e) (exact power-of-two scaling).
// Optional fp16 copy written transposed like the codes: [BH, D, Npad].
// Grid (Npad/128, BH); 256 threads; one 128-token x D tile per CTA.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ int floor_log2_pos(float a) {   // a > 0, finite
  const uint32_t bits = __float_as_uint(a);
  const int ef = static_cast<int>(bits >> 23);
  if (ef > 0) return ef - 127;
  return (31 - __clz(bits & 0x7FFFFFu)) - 149;              // subnormal
}

// One MXFP8 group of 32 values: returns the shared exponent e (scale code e + 127) and writes
// the 32 E4M3 codes of v * 2^-e to cb.
__device__ __forceinline__ int mxfp8_encode32(const float* f, uint8_t* cb) {
  float amax = 0.f;
#pragma unroll
  for (int t = 0; t < 32; ++t) amax = fmaxf(amax, fabsf(f[t]));
  int e = 0;
  if (amax > 0.f) e = max(-127, min(127, floor_log2_pos(amax) - 8));
  const float mul = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);   // 2^-e
#pragma unroll
  for (int t = 0; t < 32; t += 2) {
    uint32_t two = cvt_e4m3x2(__fmul_rn(f[t], mul), __fmul_rn(f[t + 1], mul)) & 0x7F7Fu;
    two |= (__float_as_uint(f[t]) >> 31) << 7;
    two |= (__float_as_uint(f[t + 1]) >> 31) << 15;
    cb[t] = static_cast<uint8_t>(two & 0xFF);
    cb[t + 1] = static_cast<uint8_t>(two >> 8);
  }
  return e;
}

template <typename T, int D, bool kWrite16>
__global__ void __launch_bounds__(256) mxfp8_v_kernel(const T* __restrict__ v, int32_t N,
                                                      int32_t Npad, uint8_t* __restrict__ codes,
                                                      uint8_t* __restrict__ scales,
                                                      __half* __restrict__ v16t) {
  constexpr int LD = D + 8;                       // padded row (elements)
  __shared__ __align__(16) T tile[128 * LD];
  const int tile_id = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int tok0 = tile_id * 128;
  // Load 128 tokens x D (16-byte chunks), zero past N.
  // (256 threads: every load of the tile is in flight before the first shared store)
  constexpr int CH = D / 8;                       // chunks per token
  constexpr int ITER = 128 * CH / 256;
  uint4 u[ITER];
#pragma unroll
  for (int k = 0; k < ITER; ++k) {
    const int i = threadIdx.x + k * 256, t = i / CH, c = i % CH;
    u[k] = make_uint4(0, 0, 0, 0);
    if (tok0 + t < N) u[k] = __ldg(reinterpret_cast<const uint4*>(v + (bh * N + tok0 + t) * D + c * 8));
  }
#pragma unroll
  for (int k = 0; k < ITER; ++k) {
    const int i = threadIdx.x + k * 256, t = i / CH, c = i % CH;
    *reinterpret_cast<uint4*>(&tile[t * LD + c * 8]) = u[k];
  }
  __syncthreads();
  for (int task = threadIdx.x; task < D * 4; task += blockDim.x) {
    const int c = task % D, g = task / D;
    float f[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) f[t] = to_float<T>(tile[(g * 32 + t) * LD + c]);
    __align__(16) uint8_t cb[32];
    const int e = mxfp8_encode32(f, cb);
    const int64_t rowc = bh * D + c;
    uint4* dst = reinterpret_cast<uint4*>(codes + rowc * Npad + tok0 + g * 32);
    dst[0] = *reinterpret_cast<uint4*>(cb);
    dst[1] = *reinterpret_cast<uint4*>(cb + 16);
    scales[rowc * (Npad / 32) + tile_id * 4 + g] = static_cast<uint8_t>(e + 127);
    if constexpr (kWrite16) {
      __align__(16) __half h[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) h[t] = __float2half_rn(f[t]);
      uint4* o = reinterpret_cast<uint4*>(v16t + rowc * Npad + tok0 + g * 32);
#pragma unroll
      for (int k = 0; k < 4; ++k) o[k] = reinterpret_cast<uint4*>(h)[k];
    }
  }
}

}  // namespace qk4v8
