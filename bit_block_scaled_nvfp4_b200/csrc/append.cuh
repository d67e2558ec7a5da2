// Quantize-on-append into the paged NVFP4-K / MXFP8-V cache (hotelren.com MpFA article §6:
// QK4V8 with paged KV management; sns.style BitDecoding-FP4 summary: a native FP4 paged KV
// cache). One CTA per (KV head, sequence), one thread per channel (D = 128):
//   K: every new token's 16-element blocks, NVFP4 with the cache's fixed tensor scale (the
//      quantize_nvfp4 arithmetic), written to the token's page slot;
//   V: every 32-token group the new tokens fall in, encoded again (MXFP8, one E8M0 scale per
//      channel and group) from all of its tokens so far — the earlier ones from the caller's
//      tail buffer, which keeps the last incomplete group in the input precision — so the
//      pages always equal the encoding of the whole prefix; codes past the new length are 0.
// The tail is read and rewritten by the one thread that owns its channel, so a call whose new
// tokens span several groups has no race on it.
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
  const int h = blockIdx.x, s = blockIdx.y, c = threadIdx.x;
  const int c0 = a.cu_new[s];
  const int n = a.cu_new[s + 1] - c0;
  const int len0 = a.lens[s];
  if (n == 0) return;                                // nothing new: pages and tail unchanged
  if (n < 0 || n > a.max_new || len0 < 0 ||
      static_cast<int64_t>(len0) + n > static_cast<int64_t>(a.max_pages) * 64) {
    if (c == 0 && h == 0) flag_error(kStatusBounds);
    return;
  }
  const int32_t* table = a.page_table + static_cast<int64_t>(s) * a.max_pages;
  auto page_of = [&](int pos) -> int {                 // -1: out of range (flagged)
    const int p = table[pos >> 6];
    if (p < 0 || p >= a.num_pages) { flag_error(kStatusBounds); return -1; }
    return p;
  };
  const T* kn = static_cast<const T*>(a.k_new);
  const T* vn = static_cast<const T*>(a.v_new);
  const int64_t tok_stride = static_cast<int64_t>(a.Hkv) * D;    // elements per new token

  // ---- K: (new token, 16-element block) jobs over the CTA ----
  const float s_t = *a.k_ts;
  for (int job = c; job < n * (D / 16); job += blockDim.x) {
    const int i = job >> 3, b = job & 7;
    const int pos = len0 + i;
    const int p = page_of(pos);
    if (p < 0) continue;
    const uint4* src = reinterpret_cast<const uint4*>(kn + (c0 + i) * tok_stride + h * D + b * 16);
    float f[16];
    unpack8<T>(src[0], f);
    unpack8<T>(src[1], f + 8);
    uint32_t w[2];
    const uint32_t sc = nvfp4_encode16(f, s_t, w);
    const int64_t row = (static_cast<int64_t>(p) * a.Hkv + h) * 64 + (pos & 63);
    *reinterpret_cast<uint2*>(a.k_pages + row * (D / 2) + b * 8) = make_uint2(w[0], w[1]);
    a.k_scales[row * (D / 16) + b] = static_cast<uint8_t>(sc);
  }

  // ---- V: channel c of every touched 32-token group, in order ----
  T* tail = static_cast<T*>(a.v_tail) + ((static_cast<int64_t>(s) * a.Hkv + h) * D + c) * 32;
  const int len1 = len0 + n;
  const int g_first = len0 >> 5, g_end = (len1 + 31) >> 5;
  T prev[32];                                          // the group's tokens before this call
#pragma unroll
  for (int t = 0; t < 32; ++t) prev[t] = tail[t];
  for (int grp = g_first; grp < g_end; ++grp) {
    const int pos0 = grp * 32;
    float f[32];
    T keep[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const int pos = pos0 + t;
      T v = static_cast<T>(0.f);
      if (pos < len0) v = prev[t];                     // only in the first group
      else if (pos < len1) v = vn[(c0 + pos - len0) * tok_stride + h * D + c];
      keep[t] = v;
      f[t] = to_float<T>(v);
    }
    __align__(16) uint8_t cb[32];
    const int e = mxfp8_encode32(f, cb);
    const int p = page_of(pos0);
    if (p >= 0) {
      const int64_t crow = (static_cast<int64_t>(p) * a.Hkv + h) * D + c;
      uint4* dst = reinterpret_cast<uint4*>(a.v_pages + crow * 64 + (pos0 & 63));
      dst[0] = reinterpret_cast<const uint4*>(cb)[0];
      dst[1] = reinterpret_cast<const uint4*>(cb)[1];
      a.v_scales[crow * 2 + ((pos0 >> 5) & 1)] = static_cast<uint8_t>(e + 127);
    }
    if (grp == g_end - 1 && (len1 & 31) != 0) {       // the new last group is incomplete
#pragma unroll
      for (int t = 0; t < 32; ++t) tail[t] = keep[t];
    }
  }
}

}  // namespace qk4v8
