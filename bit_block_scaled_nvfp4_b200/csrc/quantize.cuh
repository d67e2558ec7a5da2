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
// The maximum of |x| over CTA `cta`'s share (of `nctas`) of a tensor's 16-element blocks,
// valid in thread 0 of the CTA (256 threads).
template <typename T>
__device__ __forceinline__ float amax_share(const T* __restrict__ x, int64_t rows, int32_t cols,
                                            int64_t row_stride, int cta, int nctas) {
  const uint32_t blocks_per_row = static_cast<uint32_t>(cols / 16);
  const int64_t total = rows * blocks_per_row;
  const bool contiguous = (row_stride == cols);
  const int64_t step = static_cast<int64_t>(nctas) * blockDim.x;
  float m = 0.f;
  for (int64_t i0 = cta * static_cast<int64_t>(blockDim.x) + threadIdx.x; i0 < total;
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
  float t = 0.f;
  if (threadIdx.x == 0)
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t = fmaxf(t, wm[w]);
  return t;
}

template <typename T>
__global__ void __launch_bounds__(256) nvfp4_amax_kernel(const T* __restrict__ x, int64_t rows,
                                                         int32_t cols, int64_t row_stride,
                                                         float* __restrict__ partial) {
  const float t = amax_share(x, rows, cols, row_stride, blockIdx.x, gridDim.x);
  if (threadIdx.x == 0) partial[blockIdx.x] = t;
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

// ---------------------------------------------------------------------------------------
// The same block encoding on sixteen 16-bit inputs held packed (u[0], u[1]: element 2j in the
// low half of 32-bit word j), with the same FP32 results step for step:
//   amax_b  max of the magnitudes, taken in the 16-bit format (exact);
//   s_b     E4M3(fl32(fl32(amax_b / 6) / s_t)), each quotient correctly rounded: Markstein's
//           correction q' = RN(q + (a - b q) y) with q = RN(a y), y = RN(1/b) (RN(1/6) a
//           constant, y_t = RN(1/s_t) from the caller), which is RN(a / b) while nothing
//           under- or overflows; IEEE division outside [2^-60, 2^60];
//   codes   E2M1(fl32(x / den)) as in e2m1_encode16, two elements per packed FP32 operation;
//           each code's sign bit taken from its input's sign bit.
// ---------------------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float2 to_float2(uint32_t w);
template <> __device__ __forceinline__ float2 to_float2<__nv_bfloat16>(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
template <> __device__ __forceinline__ float2 to_float2<__half>(uint32_t w) {
  return __half22float2(*reinterpret_cast<const __half2*>(&w));
}
template <typename T> __device__ __forceinline__ float amax16_packed(const uint4* u);
template <> __device__ __forceinline__ float amax16_packed<__nv_bfloat16>(const uint4* u) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(u);
  __nv_bfloat162 m;
  *reinterpret_cast<uint32_t*>(&m) = w[0] & 0x7FFF7FFFu;
#pragma unroll
  for (int j = 1; j < 8; ++j) {
    const uint32_t a = w[j] & 0x7FFF7FFFu;
    m = __hmax2(m, *reinterpret_cast<const __nv_bfloat162*>(&a));
  }
  return fmaxf(__low2float(m), __high2float(m));
}
template <> __device__ __forceinline__ float amax16_packed<__half>(const uint4* u) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(u);
  __half2 m;
  *reinterpret_cast<uint32_t*>(&m) = w[0] & 0x7FFF7FFFu;
#pragma unroll
  for (int j = 1; j < 8; ++j) {
    const uint32_t a = w[j] & 0x7FFF7FFFu;
    m = __hmax2(m, *reinterpret_cast<const __half2*>(&a));
  }
  return fmaxf(__low2float(m), __high2float(m));
}
// RN(a / b) with y = RN(1 / b): Markstein's correction inside [2^-60, 2^60] for a and b (a > 0
// or 0), IEEE division outside it.
__device__ __forceinline__ float div_rn_with(float a, float b, float y) {
  const bool fast = (a >= 0x1p-60f && a <= 0x1p60f && b >= 0x1p-60f && b <= 0x1p60f) || a == 0.f;
  return fast ? div_markstein(a, b, y) : __fdiv_rn(a, b);
}
// Per tensor scale s_t, for every E4M3 block-scale code c: den = fl32(decode(c) * s_t) and
// y = RN(1 / den) (0 when den is 0 or outside Markstein's safe range [2^-90, 2^90]), built by
// a CTA's threads into shared memory once, so a block looks both up instead of computing them.
__device__ __forceinline__ void nvfp4_den_table(float s_t, float2* tab) {
  for (int c = threadIdx.x; c < 128; c += blockDim.x) {
    const float den = __fmul_rn(e4m3_code_to_float(static_cast<uint32_t>(c)), s_t);
    const bool fast = den >= 0x1p-90f && den <= 0x1p90f;
    tab[c] = make_float2(den, fast ? __frcp_rn(den) : 0.f);
  }
}
// Four E2M1 pair bytes (each in the low byte of c[0..3]) and the input words they came from ->
// one code word: magnitudes from the conversion, each sign bit from its input's sign bit.
__device__ __forceinline__ uint32_t e2m1_word(const uint32_t* c, const uint32_t* w) {
  const uint32_t codes = __byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x0040), 0x5410);
  const uint32_t a = __byte_perm(w[0], w[1], 0x7531), b = __byte_perm(w[2], w[3], 0x7531);
  const uint32_t lo = __byte_perm(a, b, 0x6420), hi = __byte_perm(a, b, 0x7531);   // sign bytes
  return (codes & 0x77777777u) | ((lo >> 4) & 0x08080808u) | (hi & 0x80808080u);
}
template <typename T, bool kWrite16>
__device__ __forceinline__ uint32_t nvfp4_encode16_packed(const uint4* u, float s_t, float y_t,
                                                          const float2* tab, uint32_t* out,
                                                          uint4* h16) {
  constexpr float kInv6 = 0x1.555556p-3f;             // RN(1/6)
  const float amax_b = amax16_packed<T>(u);
  const float sbf = div_rn_with(div_rn_with(amax_b, 6.f, kInv6), s_t, y_t);
  const uint32_t sc = cvt_e4m3x2(sbf, 0.f) & 0xFFu;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(u);
  out[0] = out[1] = 0u;
  if constexpr (kWrite16) {
    uint32_t hw[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const __half2 h = __float22half2_rn(to_float2<T>(w[j]));
      hw[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    h16[0] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    h16[1] = make_uint4(hw[4], hw[5], hw[6], hw[7]);
  }
  if (sc == 0u) return sc;                            // s_b = 0: every code 0
  const float2 dy = tab[sc];
  const float den = dy.x;
  uint32_t cb[8];
  if (dy.y != 0.f) {
    const float2 y2 = make_float2(dy.y, dy.y), nd2 = make_float2(-den, -den);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 x = to_float2<T>(w[j]);
      const float2 q = __fmul2_rn(x, y2);
      const float2 r = __ffma2_rn(nd2, q, x);
      const float2 qq = __ffma2_rn(r, y2, q);
      cb[j] = cvt_e2m1x2(qq.x, qq.y);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 x = to_float2<T>(w[j]);
      cb[j] = cvt_e2m1x2(__fdiv_rn(x.x, den), __fdiv_rn(x.y, den));
    }
  }
  out[0] = e2m1_word(cb, w);
  out[1] = e2m1_word(cb + 4, w + 4);
  return sc;
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
  const float y_t = __frcp_rn(s_t);
  __shared__ float2 tab[128];
  if constexpr (!kSearch) {
    nvfp4_den_table(s_t, tab);
    __syncthreads();
  }
  const uint32_t blocks_per_row = static_cast<uint32_t>(cols / 16);
  const int64_t total = rows * blocks_per_row;
  const bool contiguous = (row_stride == cols);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4* p = reinterpret_cast<const uint4*>(x + block_offset(i, blocks_per_row, row_stride, contiguous));
    uint4 u[2] = {__ldg(p), __ldg(p + 1)};
    const int64_t blk = i;                        // outputs are dense: block i of row i / bpr
    uint32_t w[2];
    uint32_t sc;
    if constexpr (kSearch) {
      float f[16];
      unpack8<T>(u[0], f);
      unpack8<T>(u[1], f + 8);
      sc = nvfp4_encode16_searched(f, s_t, w);
      if constexpr (kWrite16) {
        __align__(16) __half h[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) h[k] = __float2half_rn(f[k]);
        uint4* o = reinterpret_cast<uint4*>(x16 + blk * 16);
        o[0] = *reinterpret_cast<uint4*>(h);
        o[1] = *reinterpret_cast<uint4*>(h + 8);
      }
    } else {
      uint4 h[2];
      sc = nvfp4_encode16_packed<T, kWrite16>(u, s_t, y_t, tab, w, h);
      if constexpr (kWrite16) {
        uint4* o = reinterpret_cast<uint4*>(x16 + blk * 16);
        o[0] = h[0];
        o[1] = h[1];
      }
    }
    *reinterpret_cast<uint2*>(codes + blk * 8) = make_uint2(w[0], w[1]);
    scales[blk] = static_cast<uint8_t>(sc);
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

// One 128-token x D tile (tile_id) of batch-head bh, staged through `tile` (128 x (D + 8)).
template <typename T, int D, bool kWrite16>
__device__ __forceinline__ void mxfp8_v_tile(const T* __restrict__ v, int32_t N, int32_t Npad,
                                             uint8_t* __restrict__ codes,
                                             uint8_t* __restrict__ scales,
                                             __half* __restrict__ v16t, int tile_id, int64_t bh,
                                             T* tile) {
  constexpr int LD = D + 8;                       // padded row (elements)
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

template <typename T, int D, bool kWrite16>
__global__ void __launch_bounds__(256) mxfp8_v_kernel(const T* __restrict__ v, int32_t N,
                                                      int32_t Npad, uint8_t* __restrict__ codes,
                                                      uint8_t* __restrict__ scales,
                                                      __half* __restrict__ v16t) {
  __shared__ __align__(16) T tile[128 * (D + 8)];
  mxfp8_v_tile<T, D, kWrite16>(v, N, Npad, codes, scales, v16t, blockIdx.x, blockIdx.y, tile);
}

// ---------------------------------------------------------------------------------------
// Q, K and V of one attention call: after qk_amax_kernel, one launch encodes everything.
// ---------------------------------------------------------------------------------------
constexpr int kChunkBlocks = 1024;                // 16-element blocks per chunk (4 per thread)
constexpr int kChunksPerCta = 4;                  // chunks one NVFP4 CTA of the fused encode takes

// The eight 16-byte loads of a thread's four blocks t, t + 256, t + 512, t + 768 of chunk
// `chunk` of a dense tensor of `total` blocks (zero past the end).
template <typename T>
__device__ __forceinline__ void nvfp4_chunk_load(const T* __restrict__ x, int64_t total,
                                                 int64_t chunk, uint4* u) {
  const int64_t b0 = chunk * kChunkBlocks + threadIdx.x;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int64_t i = b0 + k * 256;
    u[2 * k] = u[2 * k + 1] = make_uint4(0, 0, 0, 0);
    if (i < total) {
      const uint4* p = reinterpret_cast<const uint4*>(x + i * 16);
      u[2 * k] = __ldg(p);
      u[2 * k + 1] = __ldg(p + 1);
    }
  }
}

// NVFP4 encode of a thread's four blocks of chunk `chunk` (loaded by nvfp4_chunk_load);
// consecutive threads write consecutive code words and scale bytes.
template <typename T, bool kWrite16>
__device__ __forceinline__ void nvfp4_chunk_encode(const uint4* u, int64_t total, int64_t chunk,
                                                   float s_t, float y_t, const float2* tab,
                                                   uint8_t* __restrict__ codes,
                                                   uint8_t* __restrict__ scales,
                                                   __half* __restrict__ x16) {
  const int64_t b0 = chunk * kChunkBlocks + threadIdx.x;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int64_t i = b0 + k * 256;
    if (i >= total) break;
    uint32_t w[2];
    uint4 h[2];
    const uint32_t sc = nvfp4_encode16_packed<T, kWrite16>(u + 2 * k, s_t, y_t, tab, w, h);
    *reinterpret_cast<uint2*>(codes + i * 8) = make_uint2(w[0], w[1]);
    scales[i] = static_cast<uint8_t>(sc);
    if constexpr (kWrite16) {
      uint4* o = reinterpret_cast<uint4*>(x16 + i * 16);
      o[0] = h[0];
      o[1] = h[1];
    }
  }
}

struct QkvEncodeArgs {
  const void* q;
  const void* k;
  const void* v;
  int64_t q_blocks, k_blocks;                     // 16-element blocks of Q and K
  const float* q_partial;
  const float* k_partial;
  int32_t q_nparts, k_nparts;                     // per-CTA maxima of the amax pass
  uint8_t* q_codes;
  uint8_t* q_scales;
  float* q_ts;
  uint8_t* k_codes;
  uint8_t* k_scales;
  float* k_ts;
  uint8_t* v_codes;
  uint8_t* v_scales;
  __half* q16;
  __half* k16;
  __half* v16;
  int32_t q_chunks, k_chunks;                     // chunks of kChunkBlocks blocks per tensor
  int32_t nv_ctas;                                // NVFP4 CTAs (kChunksPerCta positions each)
  int32_t v_tiles, v_n, v_npad;                   // 128-token V tiles per batch-head, tokens
};

// Position p of the Q/K chunk order: the K chunks spread among the Q chunks in proportion to
// the sizes (p is a K chunk when the count of K chunks before it, floor(p k / n), steps at p),
// each tensor from its last chunk to its first.
__device__ __forceinline__ void qk_position(const QkvEncodeArgs& a, int64_t p, bool& k_role,
                                            int64_t& chunk) {
  const int64_t n = static_cast<int64_t>(a.q_chunks) + a.k_chunks;
  const int64_t kc0 = p * a.k_chunks / n, kc1 = (p + 1) * a.k_chunks / n;
  k_role = kc1 > kc0;
  chunk = k_role ? (a.k_chunks - 1 - kc0) : (a.q_chunks - 1 - (p - kc0));
}

// First launch: the amax pass of Q and K and the whole MXFP8 encode of V (which needs no
// tensor scale, so its traffic overlaps the read-only amax pass). CTAs [0, gq) take Q's
// share of the amax pass and [gq, gq + gk) K's, each writing its maximum to its tensor's
// partials; the rest encode V tiles.
template <typename T, int D, bool kWrite16>
__global__ void __launch_bounds__(256) qk_amax_v_kernel(QkvEncodeArgs a, int64_t q_rows,
                                                        int64_t k_rows, int32_t gq, int32_t gk) {
  __shared__ __align__(16) T tile[128 * (D + 8)];
  const int c = blockIdx.x;
  if (c < gq) {
    const float t = amax_share(static_cast<const T*>(a.q), q_rows, D, D, c, gq);
    if (threadIdx.x == 0) const_cast<float*>(a.q_partial)[c] = t;
  } else if (c < gq + gk) {
    const float t = amax_share(static_cast<const T*>(a.k), k_rows, D, D, c - gq, gk);
    if (threadIdx.x == 0) const_cast<float*>(a.k_partial)[c - gq] = t;
  } else {
    const int t = c - gq - gk;
    mxfp8_v_tile<T, D, kWrite16>(static_cast<const T*>(a.v), a.v_n, a.v_npad, a.v_codes, a.v_scales,
                                 a.v16, t % a.v_tiles, t / a.v_tiles, tile);
  }
}

// Second launch: the NVFP4 encode of Q and K. Each CTA encodes kChunksPerCta consecutive
// positions of the Q/K chunk order, so the tails the amax pass read last, still in L2, are
// encoded first. A CTA issues its first chunk's loads before it reduces the amax partials and
// builds the two tensors' scale tables. Four CTAs per SM (at most 64 registers a thread): the
// per-block arithmetic is long, and other warps hide its latency better than a second register
// buffer would.
template <typename T, bool kWrite16>
__global__ void __launch_bounds__(256, 4) qk_encode_kernel(QkvEncodeArgs a) {
  __shared__ float2 tabq[128], tabk[128];
  const int c = blockIdx.x;
  const int64_t n = static_cast<int64_t>(a.q_chunks) + a.k_chunks;
  const int64_t p0 = static_cast<int64_t>(c) * kChunksPerCta;
  const int np = static_cast<int>(min(static_cast<int64_t>(kChunksPerCta), n - p0));
  bool kr;
  int64_t ch;
  qk_position(a, p0, kr, ch);
  uint4 u[8];
  nvfp4_chunk_load<T>(static_cast<const T*>(kr ? a.k : a.q), kr ? a.k_blocks : a.q_blocks, ch, u);
  const float amq = reduce_partials(a.q_partial, a.q_nparts);
  __syncthreads();                                 // the reduction's scratch is reused
  const float amk = reduce_partials(a.k_partial, a.k_nparts);
  const float stq = (amq == 0.f) ? 1.f : __fdiv_rn(amq, 2688.f);
  const float stk = (amk == 0.f) ? 1.f : __fdiv_rn(amk, 2688.f);
  const float ytq = __frcp_rn(stq), ytk = __frcp_rn(stk);
  nvfp4_den_table(stq, tabq);
  nvfp4_den_table(stk, tabk);
  __syncthreads();
  for (int i = 0; i < np; ++i) {
    if (i > 0) {
      qk_position(a, p0 + i, kr, ch);
      nvfp4_chunk_load<T>(static_cast<const T*>(kr ? a.k : a.q), kr ? a.k_blocks : a.q_blocks, ch, u);
    }
    if (ch == 0 && threadIdx.x == 0) *(kr ? a.k_ts : a.q_ts) = kr ? stk : stq;
    if (kr)
      nvfp4_chunk_encode<T, kWrite16>(u, a.k_blocks, ch, stk, ytk, tabk, a.k_codes, a.k_scales, a.k16);
    else
      nvfp4_chunk_encode<T, kWrite16>(u, a.q_blocks, ch, stq, ytq, tabq, a.q_codes, a.q_scales, a.q16);
  }
}

}  // namespace qk4v8
