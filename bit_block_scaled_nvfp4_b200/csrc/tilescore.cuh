// Tile importance scores and top-fraction selection (ai-feeds.com ThriftAttention summary,
// "方法" step 2: score each 128x128 query-key tile by a cheap bound on its largest attention
// weight and keep about the top 5 %; "局限": the bound is an L2 norm of the query-key
// product).
//
// Score of tile (qt, kt): max_{i in qt} N_i(q) * max_{j in kt} N_j(k), where for a row of
// NVFP4 codes N = sum_blocks (2^9 s_b)^2 * sum_e (2 e)^2 is |x_hat|^2 * 2^20 / s_t^2 as an
// exact integer (< 2^51). Scores are exact 128-bit integers, so the ranking is bit-exact.
// Kept per (batch, query head): ceil(n_candidates * frac_bp / 10000), ranked by score
// descending, ties by the lower linear index qt * T + kt.
#pragma once
#include "ptx.cuh"

namespace qk4v8 {

// (2^9 * E4M3 value) of a non-negative finite E4M3 code, as an integer.
__device__ __forceinline__ uint64_t e4m3_times512(uint32_t c) {
  const uint32_t e = (c >> 3) & 0xF, m = c & 7;
  return e == 0 ? m : static_cast<uint64_t>(8 + m) << (e - 1);
}

// Sum over the 8 E2M1 codes of a 32-bit word of (2 * magnitude)^2: the squares
// 0,1,4,9,16,36,64,144 of the 8 magnitude codes as a byte table, looked up four codes at a time
// with a byte permute (the sign bit of each code masked off) and summed with dp4a.
__device__ __forceinline__ uint32_t e2m1_sq2_sum(uint32_t w) {
  constexpr uint32_t kLo = 0x09040100u, kHi = 0x90402410u;
  const uint32_t a = __byte_perm(kLo, kHi, w & 0x7777u);
  const uint32_t b = __byte_perm(kLo, kHi, (w >> 16) & 0x7777u);
  return __dp4a(b, 0x01010101u, __dp4a(a, 0x01010101u, 0u));
}

// Per-row exact norm and per-tile maximum. rows of one tensor [BH, N, D] in NVFP4.
// tile_max: [BH, T] u64, zeroed by the caller. D/32 consecutive threads share a row, each
// taking 16 bytes of codes (two 16-element blocks), so the loads are coalesced.
template <int D>
__global__ void __launch_bounds__(256) row_norm_tile_max_kernel(
    const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, int64_t BH, int32_t N,
    int32_t T, unsigned long long* __restrict__ tile_max) {
  constexpr int TPR = D / 32;                    // threads per row
  const int64_t gtid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int64_t row = gtid / TPR;
  const int part = static_cast<int>(gtid % TPR);
  const bool live = row < BH * N;
  uint64_t nr = 0;
  int64_t bh = 0;
  int tile = 0;
  if (live) {
    bh = row / N;
    const int n = static_cast<int>(row - bh * N);
    tile = n / 128;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(codes + row * (D / 2)) + part);
    const uint8_t* sc = scales + row * (D / 16) + part * 2;
    const uint32_t s0 = e2m1_sq2_sum(u.x) + e2m1_sq2_sum(u.y);
    const uint32_t s1 = e2m1_sq2_sum(u.z) + e2m1_sq2_sum(u.w);
    const uint64_t f0 = e4m3_times512(sc[0]), f1 = e4m3_times512(sc[1]);
    nr = f0 * f0 * s0 + f1 * f1 * s1;
  }
  // whole-row sums in every lane of the row's group
#pragma unroll
  for (int o = 1; o < TPR; o <<= 1) nr += __shfl_xor_sync(0xffffffffu, nr, o);
  // One atomic per warp when all its rows fall in the same (bh, tile); else one per row.
  const int64_t key = live ? bh * T + tile : -1;
  const int64_t key0 = __shfl_sync(0xffffffffu, key, 0);
  if (__all_sync(0xffffffffu, key == key0)) {
    unsigned long long m = nr;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, m, o);
      m = other > m ? other : m;
    }
    if ((threadIdx.x & 31) == 0 && key0 >= 0) atomicMax(tile_max + key0, m);
  } else if (live && part == 0) {
    atomicMax(tile_max + key, static_cast<unsigned long long>(nr));
  }
}

struct U128 {
  uint64_t hi, lo;
};
__device__ __forceinline__ U128 mul_u64(uint64_t a, uint64_t b) {
  return U128{__umul64hi(a, b), a * b};
}
__device__ __forceinline__ uint32_t byte_of(const U128& v, int p) {     // p = 0..15, 15 = MSB
  return p >= 8 ? static_cast<uint32_t>(v.hi >> (8 * (p - 8))) & 0xFF
                : static_cast<uint32_t>(v.lo >> (8 * p)) & 0xFF;
}
// true when v's bytes above position p equal prefix's
__device__ __forceinline__ bool prefix_match(const U128& v, const U128& pre, int p) {
  if (p >= 15) return true;
  if (p >= 7) {     // compare hi bytes (p+1-8 .. 7)
    const int sh = 8 * (p + 1 - 8);
    return (v.hi >> sh) == (pre.hi >> sh);
  }
  const int sh = 8 * (p + 1);
  return v.hi == pre.hi && (v.lo >> sh) == (pre.lo >> sh);
}
__device__ __forceinline__ bool u128_gt(const U128& a, const U128& b) {
  return a.hi > b.hi || (a.hi == b.hi && a.lo > b.lo);
}
__device__ __forceinline__ bool u128_eq(const U128& a, const U128& b) {
  return a.hi == b.hi && a.lo == b.lo;
}

constexpr int kSelectThreads = 1024;
constexpr int kSelectMax = 4096;

// One CTA per (b, hq). Tile maxima come from row_norm_tile_max_kernel.
// Dynamic shared memory: mq[T] + mk[T] (u64) + sort arrays (kSelectMax entries).
__global__ void __launch_bounds__(kSelectThreads) tile_select_kernel(
    const unsigned long long* __restrict__ q_tile_max, const unsigned long long* __restrict__ k_tile_max,
    int32_t Hq, int32_t Hkv, int32_t Tq, int32_t Tk, int32_t causal, int32_t frac_bp,
    int32_t k_max, int32_t* __restrict__ idx_out, int32_t* __restrict__ n_sel_out,
    uint8_t* __restrict__ bitmap) {
  extern __shared__ __align__(16) unsigned char sm[];
  const int bhq = blockIdx.x;
  const int b = bhq / Hq, hq = bhq % Hq;
  const int hk = hq / (Hq / Hkv);
  uint64_t* mq = reinterpret_cast<uint64_t*>(sm);
  uint64_t* mk = mq + Tq;
  U128* s_key = reinterpret_cast<U128*>(mk + Tk + (Tk & 1));
  int32_t* s_idx = reinterpret_cast<int32_t*>(s_key + kSelectMax);
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_bin, s_above, s_cnt_gt, s_cnt_eq;
  __shared__ uint32_t warp_tot[kSelectThreads / 32];
  const int tid = threadIdx.x;
  for (int i = tid; i < Tq; i += blockDim.x) mq[i] = q_tile_max[(int64_t)bhq * Tq + i];
  for (int i = tid; i < Tk; i += blockDim.x) mk[i] = k_tile_max[((int64_t)b * Hkv + hk) * Tk + i];
  __syncthreads();
  const int64_t total = static_cast<int64_t>(Tq) * Tk;
  int64_t n_cand = 0;
  if (causal) {
    for (int qt = 0; qt < Tq; ++qt) n_cand += min(qt + 1, Tk);
  } else {
    n_cand = total;
  }
  const int kk = static_cast<int>((n_cand * frac_bp + 9999) / 10000);
  const int k = min(kk, k_max);
  // --- radix select the k-th largest score (tau) -------------------------------------
  U128 pre{0, 0};
  uint32_t k_rem = static_cast<uint32_t>(k);
  const int lane = tid & 31;
  // Row norms are below 2^51, so scores are below 2^102: bytes 13-15 are always zero.
  if (k > 0) {
    for (int p = 12; p >= 0; --p) {
      for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
      __syncthreads();
      // Warp per query-tile row, lanes over key tiles (no index division). Lanes with the
      // same digit add once per warp (most scores share their high bytes, and one shared-
      // memory atomic per candidate would serialise on a few bins).
      for (int qt = tid >> 5; qt < Tq; qt += kSelectThreads / 32) {
        const uint64_t a = mq[qt];
        const int kt_end = causal ? min(qt + 1, Tk) : Tk;
        for (int kb = 0; kb < kt_end; kb += 32) {
          const int kt = kb + lane;
          int bin = -1;
          if (kt < kt_end) {
            const U128 v = mul_u64(a, mk[kt]);
            if (prefix_match(v, pre, p)) bin = static_cast<int>(byte_of(v, p));
          }
          const unsigned same = __match_any_sync(0xffffffffu, bin);
          if (bin >= 0 && lane == __ffs(same) - 1) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(same)));
        }
      }
      __syncthreads();
      // The digit of the k_rem-th largest: the first bin from the top whose running count
      // reaches k_rem (bin 0 if none does). Thread t holds bin 255 - t; an inclusive scan over
      // the 256 bins in that order gives each bin its count from the top.
      if (tid < 256) {
        const uint32_t h = hist[255 - tid];
        uint32_t incl = h;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t up = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += up;
        }
        if (lane == 31) warp_tot[tid >> 5] = incl;
        named_bar_sync(1, 256);
        for (int w2 = 0; w2 < (tid >> 5); ++w2) incl += warp_tot[w2];
        const uint32_t before = incl - h;
        if ((incl >= k_rem || tid == 255) && before < k_rem) {
          s_bin = static_cast<uint32_t>(255 - tid);
          s_above = before;
        }
      }
      __syncthreads();
      const uint32_t bin = s_bin;
      k_rem -= s_above;
      if (p >= 8) pre.hi |= static_cast<uint64_t>(bin) << (8 * (p - 8));
      else pre.lo |= static_cast<uint64_t>(bin) << (8 * p);
      __syncthreads();
    }
  }
  // pre = tau; take every score > tau and the k_rem lowest-index scores == tau.
  if (tid == 0) { s_cnt_gt = 0; s_cnt_eq = 0; }
  __syncthreads();
  const uint32_t n_gt = static_cast<uint32_t>(k) - k_rem;
  if (k > 0) {
    for (int64_t base = 0; base < total; base += blockDim.x) {
      const int64_t c = base + tid;
      bool gt = false, eq = false;
      U128 v{0, 0};
      if (c < total) {
        const int qt = static_cast<int>(static_cast<uint32_t>(c) / static_cast<uint32_t>(Tk));
        const int kt = static_cast<int>(c) - qt * Tk;
        if (!(causal && kt > qt)) {
          v = mul_u64(mq[qt], mk[kt]);
          gt = u128_gt(v, pre);
          eq = u128_eq(v, pre);
        }
      }
      // ordered compaction of the ties (block-wide exclusive scan)
      const unsigned bal = __ballot_sync(0xffffffffu, eq);
      const int w = tid >> 5;
      if (lane == 0) warp_tot[w] = __popc(bal);
      __syncthreads();
      if (w == 0) {                    // exclusive scan of the 32 warp counts
        const uint32_t t = warp_tot[lane];
        uint32_t incl = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t up = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += up;
        }
        warp_tot[lane] = incl - t;
      }
      __syncthreads();
      const uint32_t eq_rank = s_cnt_eq + warp_tot[w] + __popc(bal & ((1u << lane) - 1u));
      if (gt) {
        const uint32_t slot = atomicAdd(&s_cnt_gt, 1u);
        s_key[slot] = v;
        s_idx[slot] = static_cast<int32_t>(c);
      }
      if (eq && eq_rank < k_rem) {
        const uint32_t slot = n_gt + eq_rank;
        s_key[slot] = v;
        s_idx[slot] = static_cast<int32_t>(c);
      }
      __syncthreads();
      if (tid == kSelectThreads - 1) s_cnt_eq = eq_rank + (eq ? 1u : 0u);
      __syncthreads();
    }
  }
  // --- sort the k selected by (score desc, index asc): bitonic over a power of two -------
  int np2 = 1;
  while (np2 < k) np2 <<= 1;
  for (int i = k + tid; i < np2; i += blockDim.x) { s_key[i] = U128{0, 0}; s_idx[i] = 0x7fffffff; }
  __syncthreads();
  for (int size = 2; size <= np2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < np2; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool up = (i & size) == 0;   // "up" = rank order (best first)
          const U128 a = s_key[i], bk = s_key[j];
          const int ia = s_idx[i], ib = s_idx[j];
          // a before b in rank order?
          const bool a_first = u128_gt(a, bk) || (u128_eq(a, bk) && ia < ib);
          if (a_first != up) {
            s_key[i] = bk; s_key[j] = a; s_idx[i] = ib; s_idx[j] = ia;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < k; i += blockDim.x) idx_out[(int64_t)bhq * k_max + i] = s_idx[i];
  if (tid == 0) n_sel_out[bhq] = k;
  if (bitmap != nullptr) {
    uint8_t* bm = bitmap + (int64_t)bhq * total;
    for (int64_t c = tid; c < total; c += blockDim.x) bm[c] = 0;
    __syncthreads();
    for (int i = tid; i < k; i += blockDim.x) bm[s_idx[i]] = 1;
  }
}

}  // namespace qk4v8
