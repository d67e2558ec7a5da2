// Quantize-on-append into the paged NVFP4-K / MXFP8-V cache (hotelren.com MpFA article §6:
// QK4V8 with paged KV management; sns.style BitDecoding-FP4 summary: a native FP4 paged KV
// cache). One CTA per (32-token group the new tokens fall in, KV head, sequence), 128 threads:
//   K: the group's new tokens, each 16-element block NVFP4 with the cache's fixed tensor scale
//      (the quantize_nvfp4 arithmetic), written to the token's page slot;
//   V: the group encoded again (MXFP8, one E8M0 scale per channel) from all of its tokens so
//      far — earlier ones from the caller's tail, which keeps each sequence's last incomplete
//      group in the input precision — so the pages always equal the encoding of the whole
//      prefix; codes past the new length are 0.
// Only the CTA of the first touched group reads the tail, and it also writes the new tail
// (from its own tile, or from the new tokens of the last group), so no two CTAs race on it.
#pragma once
#include "quantize.cuh"

namespace qk4v8 {

struct AppendArgs {
  const void* k_new;
  const void* v_new;
  const int32_t* cu_new;
  const int32_t* lens;
  const int32_t* page_table;
  uint8_t* k_pages;
  uint8_t* k_scales;
  const float* k_ts;
  uint8_t* v_pages;
  uint8_t* v_scales;
  void* v_tail;
  int32_t S, num_pages, max_pages, Hkv, max_new;
};

template <typename T>
__global__ void __launch_bounds__(128) kv_append_kernel(AppendArgs a) {
  constexpr int D = 128;
  constexpr int LD = D + 8;                            // padded smem row (elements)
  __shared__ __align__(16) T tile[32 * LD];            // [token in group][channel]
  const int gi = blockIdx.x, h = blockIdx.y, s = blockIdx.z, tid = threadIdx.x;
  const int c0 = a.cu_new[s];
  const int n = a.cu_new[s + 1] - c0;
  const int len0 = a.lens[s];
  if (n == 0) return;                                  // nothing new: pages and tail unchanged
  if (n < 0 || n > a.max_new || len0 < 0 ||
      static_cast<int64_t>(len0) + n > static_cast<int64_t>(a.max_pages) * 64) {
    if (tid == 0 && gi == 0 && h == 0) flag_error(kStatusBounds);
    return;
  }
  const int len1 = len0 + n;
  const int g_first = len0 >> 5, g_last = (len1 - 1) >> 5;
  const int grp = g_first + gi;
  if (grp > g_last) return;
  const int pos0 = grp * 32;
  const int32_t* table = a.page_table + static_cast<int64_t>(s) * a.max_pages;
  const int page = table[pos0 >> 6];
  if (page < 0 || page >= a.num_pages) {
    if (tid == 0) flag_error(kStatusBounds);
    return;
  }
  const T* kn = static_cast<const T*>(a.k_new);
  const T* vn = static_cast<const T*>(a.v_new);
  const int64_t tok_stride = static_cast<int64_t>(a.Hkv) * D;    // elements per new token
  T* tail = static_cast<T*>(a.v_tail) + (static_cast<int64_t>(s) * a.Hkv + h) * D * 32;
  const int lo = max(len0, pos0), hi = min(len1, pos0 + 32);       // new tokens of this group

  // ---- V tile: new tokens by 16-byte rows (all loads in flight), older ones from the tail ----
  {
    uint4 u[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {                      // 32 tokens x 16 chunks of 8 channels
      const int i = tid + k * 128, t = i >> 4, ch = i & 15, pos = pos0 + t;
      u[k] = make_uint4(0, 0, 0, 0);
      if (pos >= lo && pos < hi)
        u[k] = __ldg(reinterpret_cast<const uint4*>(vn + (c0 + pos - len0) * tok_stride + h * D + ch * 8));
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = tid + k * 128, t = i >> 4, ch = i & 15, pos = pos0 + t;
      if (pos < lo) continue;                          // filled from the tail below
      *reinterpret_cast<uint4*>(&tile[t * LD + ch * 8]) = u[k];
    }
    if (pos0 < len0) {                                 // first group: tokens before the call
      const uint4* tc = reinterpret_cast<const uint4*>(tail + tid * 32);   // channel tid, 64 B
      uint4 tv[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) tv[k] = tc[k];
      const T* tt = reinterpret_cast<const T*>(tv);
#pragma unroll
      for (int t = 0; t < 32; ++t)
        if (t < len0 - pos0) tile[t * LD + tid] = tt[t];
    }
  }
  // ---- K of the group's new tokens: (token, 16-element block) jobs, loads first ----
  const float s_t = *a.k_ts;
  const int n_jobs = (hi - lo) * (D / 16);
  uint4 kv[2][2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int job = tid + r * 128;
    if (job < n_jobs) {
      const int i = lo + (job >> 3) - len0, b = job & 7;
      const uint4* src = reinterpret_cast<const uint4*>(kn + (c0 + i) * tok_stride + h * D + b * 16);
      kv[r][0] = __ldg(src);
      kv[r][1] = __ldg(src + 1);
    }
  }
  __syncthreads();
  // ---- V: channel tid of the group ----
  {
    float f[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) f[t] = (pos0 + t < len1) ? to_float<T>(tile[t * LD + tid]) : 0.f;
    __align__(16) uint8_t cb[32];
    const int e = mxfp8_encode32(f, cb);
    const int64_t crow = (static_cast<int64_t>(page) * a.Hkv + h) * D + tid;
    uint4* dst = reinterpret_cast<uint4*>(a.v_pages + crow * 64 + (pos0 & 63));
    dst[0] = reinterpret_cast<const uint4*>(cb)[0];
    dst[1] = reinterpret_cast<const uint4*>(cb)[1];
    a.v_scales[crow * 2 + ((pos0 >> 5) & 1)] = static_cast<uint8_t>(e + 127);
  }
  // ---- K encode and store ----
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int job = tid + r * 128;
    if (job < n_jobs) {
      const int pos = lo + (job >> 3), b = job & 7;
      float f[16];
      unpack8<T>(kv[r][0], f);
      unpack8<T>(kv[r][1], f + 8);
      uint32_t w[2];
      const uint32_t sc = nvfp4_encode16(f, s_t, w);
      const int64_t row = (static_cast<int64_t>(page) * a.Hkv + h) * 64 + (pos & 63);
      *reinterpret_cast<uint2*>(a.k_pages + row * (D / 2) + b * 8) = make_uint2(w[0], w[1]);
      a.k_scales[row * (D / 16) + b] = static_cast<uint8_t>(sc);
    }
  }
  // ---- new tail (first group's CTA only): the last group's tokens, if it is incomplete ----
  // (entries past the group's new length are don't-care; they are written as 0)
  if (gi == 0 && (len1 & 31) != 0) {
    const int pl = g_last * 32;
    __align__(16) T tv[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      T v = static_cast<T>(0.f);
      if (t < len1 - pl)
        v = (g_last == grp) ? tile[t * LD + tid] : vn[(c0 + pl + t - len0) * tok_stride + h * D + tid];
      tv[t] = v;
    }
    uint4* tc = reinterpret_cast<uint4*>(tail + tid * 32);
#pragma unroll
    for (int k = 0; k < 4; ++k) tc[k] = reinterpret_cast<const uint4*>(tv)[k];
  }
}

}  // namespace qk4v8
