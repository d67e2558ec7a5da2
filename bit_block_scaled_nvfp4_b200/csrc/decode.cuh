// Split-K paged decode over an NVFP4-K / MXFP8-V KV cache, and the split merge.
//
// Method: sns.style BitDecoding-FP4 summary (the whole KV cache is read once per decoding
// step; GQA query heads stacked into one tensor-core MMA on a paged cache; probability
// quantization fused into the kernel), with the QK4V8 arithmetic of the prefill kernel.
//
// Grid (split, kv head, sequence). Each CTA walks its split's pages two at a time (128 keys)
// and keeps (m, l, O) for the g query heads of its KV head. tcgen05 block-scaled MMAs need
// M = 128, so the g <= 16 query heads form the N dimension (N = 16) and keys / channels form
// M: S^T = K Q^T (M = 128 keys) and O^T += V^T P^T (M = 128 channels); each softmax thread
// owns one key; the block max per query is one warp reduction (redux.sync) and an exchange
// of the four warps' maxima through shared memory. l comes from the tensor core: a second MMA
// with an all-ones A operand (L^T += 1 P^T) sums the quantized P per query, rescaled with O.
// Partials (O unnormalised, m, l) go to the workspace; the merge kernel combines the splits:
// M = max m_s, O = sum e^(m_s - M) O_s / sum e^(m_s - M) l_s.
//
// Warp roles (two or three CTAs per SM): warp 0 K producer (TMA of the two pages' K codes,
// K scale factors by 4-byte asynchronous copies into the tcgen05 layout), warp 7 V producer
// (TMA of V codes, bulk copy of the pages' V scales), warp 1 QK^T issuer, warp 6 PV issuer (and
// the V scale rearrangement), warps 2-5 softmax. K and V stages form separate rings.
//
// Instances: GM (a bound on g: 4, 8 or 16 query columns reduced and exponentiated), kUA
// (underflow-aware P scaling: each warp's 32 keys are one block of P^T, encoded against its own
// power of two, which the PV MMA applies back as the block's E8M0 scale) and kDQ (a second Q
// tensor from dual-residual query quantization, two more FP4 MMAs into S^T).
#pragma once
#include "ptx.cuh"
#include "attn_fwd.cuh"

namespace qk4v8 {

struct DecArgs {
  const uint8_t* q_scales;       // [S*Hq, D/16]
  const uint8_t* q2_scales;      // the second Q tensor's, or null
  const float* q_ts;
  const uint8_t* k_page_scales;  // [P, Hkv, 64, D/16]
  const float* k_ts;
  const uint8_t* v_page_scales;  // [P, Hkv, D, 2]
  const int32_t* page_table;     // [S, max_pages]
  const int32_t* lens;           // [S]
  float* ws;                     // [S*Hq, n_splits, D + 2]
  int32_t S, Hq, Hkv, max_pages, n_splits, split_tokens, num_pages;
  float softmax_scale;
};

// GM: a compile-time bound on g (4, 8 or 16); the softmax reduces and exponentiates only
// the first GM query columns of the N = 16 MMA operand (rows >= g of Q^T and P^T are zero).
// With GM = 4 the kernel fits three CTAs per SM (80 registers, two stages per ring); the
// wider instances keep two CTAs per SM and three stages.
template <int GM, bool kDQ = false>
struct DecLayout {
  static constexpr int CTAS_PER_SM = GM <= 4 ? 3 : 2;
  static constexpr int D = 128;
  // Separate K and V rings: a K stage is free after QK^T of its block, a V stage only after
  // PV, so the next blocks' K loads do not wait for the softmax.
  static constexpr int NK = GM <= 4 ? 2 : 3, NVS = NK;
  static constexpr int OFF_Q = 0;                 // 16 rows x 64 B (SW64)
  static constexpr int OFF_QSF = 1024;            // 2 chunks
  // P^T scale factors: two chunks by block parity (query row n, 32-key block b at byte
  // n*16 + b; E8M0 127 = 1.0 unless underflow-aware scaling lowers it), then a constant chunk of
  // 1.0 for the ones operand
  static constexpr int OFF_PSF = 2048;
  // second Q tensor of dual-residual query quantization (its own instance): operand + scales
  static constexpr int OFF_Q2 = 4096, OFF_Q2SF = 5120;
  static constexpr int OFF_P = kDQ ? 6144 : 4096; // 2 x [16 rows x 128 B] (SW128), 1024-aligned
  static constexpr int OFF_ONES = OFF_P + 2 * 2048;       // 128 x 32 B of E4M3 1.0 (SW32)
  static constexpr int OFF_KST = OFF_ONES + 4096;         // 12288, 1024-aligned
  static constexpr int ST_K = 0;                  // 128 keys x 64 B (SW64)
  static constexpr int ST_KSF = 8192;             // 2 chunks
  static constexpr int KST_BYTES = 9216;
  static constexpr int OFF_VST = OFF_KST + NK * KST_BYTES;
  static constexpr int ST_V0 = 0;                 // 128 channels x 64 B (page 0 tokens)
  static constexpr int ST_V1 = 8192;              // page 1 tokens
  static constexpr int ST_VSF = 16384;            // 1 chunk (tcgen05 layout)
  static constexpr int ST_VRAW = 16896;           // the two pages' V scales as stored (2 x 256 B)
  static constexpr int VST_BYTES = 17408;
  static constexpr int OFF_BAR = OFF_VST + NVS * VST_BYTES;
  static constexpr int OFF_RED = OFF_BAR + 256;   // block max exchange [2 parities][4 warps][16]
  static constexpr int OFF_PID = OFF_RED + 2 * 4 * 16 * 4;   // page ids of the split
  static constexpr int MAX_SPLIT_PAGES = 256;                // split_tokens <= 16384
  static constexpr int SMEM_BYTES = OFF_PID + MAX_SPLIT_PAGES * 4;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
  // S^T x2 [0,32), O^T [32,48), L^T [48,64) (every row: l), Q / P scales, K and V scales by
  // stage
  static constexpr uint32_t T_S = 0, T_O = 32, T_L = 48, T_QSF = 64, T_PSF = 72, T_ONESF = 80,
                            T_KSF = 84,
                            T_VSF = T_KSF + 8 * NK;
  static constexpr uint32_t T_Q2SF = T_VSF + 4 * NVS;          // 2 chunks (kDQ only)
  static_assert(T_Q2SF + (kDQ ? 8 : 0) <= 128, "TMEM columns");
  static constexpr int NQ = 16;                   // MMA N (query heads, padded)
  static constexpr int PV_WARP = 6;
  static constexpr int VLOAD_WARP = 7;
  static constexpr int THREADS = 256;
};

// kUA: underflow-aware P scaling (a separate instance, so that the default path carries none
// of its work).
// kDQ: a second Q tensor (dual-residual query quantization, same tensor scale) whose QK^T
// MMAs accumulate into the same S^T; tm_q2 maps it (unused otherwise).
template <int GM, bool kUA, bool kDQ = false>
__global__ void __launch_bounds__(256, DecLayout<GM>::CTAS_PER_SM)
decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kp,
              const __grid_constant__ CUtensorMap tm_vp, const __grid_constant__ CUtensorMap tm_q2,
              DecArgs a) {
  using L = DecLayout<GM, kDQ>;
  constexpr int D = L::D;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + L::NK;
  uint64_t* v_full = k_empty + L::NK;
  uint64_t* v_empty = v_full + L::NVS;
  uint64_t* s_full = v_empty + L::NVS;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_full + 4;
  uint64_t* pv_done = s_full + 6;
  uint64_t* mma_final = s_full + 8;        // [2]: QK^T issuer, PV issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red_max = reinterpret_cast<float*>(sm + L::OFF_RED);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int g = a.Hq / a.Hkv;
  int len = a.lens[s];
  if (len < 1 || len > a.n_splits * a.split_tokens || len > a.max_pages * 64) {
    if (split == 0 && h == 0 && threadIdx.x == 0) flag_error(kStatusBounds);
    len = 0;                               // every split empty; the merge yields no value
  }
  const int k_begin = split * a.split_tokens;
  const int k_end = min(len, k_begin + a.split_tokens);
  const int nblk = k_end > k_begin ? (k_end - k_begin + 127) / 128 : 0;
  const int64_t qrow0 = static_cast<int64_t>(s) * a.Hq + h * g;
  float* part = a.ws + (qrow0 * a.n_splits + split) * (D + 2);   // + q * n_splits * (D+2)
  const int64_t q_stride = static_cast<int64_t>(a.n_splits) * (D + 2);

  if (nblk == 0) {                         // empty split: weight zero in the merge
    for (int q = 0; q < g; ++q)
      for (int c = threadIdx.x; c < D + 2; c += blockDim.x)
        part[q * q_stride + c] = (c == D) ? -INFINITY : 0.f;
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    // k_full: the producer's expect-tx arrival plus one cp.async arrival per producer lane
    for (int i = 0; i < L::NK; ++i) { mbar_init(k_full + i, 33); mbar_init(k_empty + i, 1); }
    for (int i = 0; i < L::NVS; ++i) { mbar_init(v_full + i, 1); mbar_init(v_empty + i, 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1); mbar_init(s_free + i, 4);
      mbar_init(p_full + i, 4); mbar_init(pv_done + i, 1);
    }
    mbar_init(mma_final, 1);
    mbar_init(mma_final + 1, 1);
    abort_flag[0] = 0;
    abort_flag[1] = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < 128; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sm + L::OFF_PSF)[i] = 0x7F7F7F7Fu;
  for (int i = threadIdx.x; i < 128; i += blockDim.x) {
    reinterpret_cast<uint32_t*>(sm + L::OFF_PSF + 512)[i] = 0x7F7F7F7Fu;
    reinterpret_cast<uint32_t*>(sm + L::OFF_PSF + 1024)[i] = 0x7F7F7F7Fu;
  }
  for (int i = threadIdx.x; i < 2 * 16 * 128 / 16; i += blockDim.x)   // zero both P^T buffers
    reinterpret_cast<uint4*>(sm + L::OFF_P)[i] = make_uint4(0, 0, 0, 0);
  for (int i = threadIdx.x; i < 4096 / 16; i += blockDim.x)            // the ones operand
    reinterpret_cast<uint4*>(sm + L::OFF_ONES)[i] = make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
  // Page ids of this split, checked once, into shared memory (read by both producers).
  int32_t* pid = reinterpret_cast<int32_t*>(sm + L::OFF_PID);
  {
    const int n_split_pages = (k_end - k_begin + 63) / 64;
    for (int i = threadIdx.x; i < n_split_pages; i += blockDim.x) {
      int p = a.page_table[static_cast<int64_t>(s) * a.max_pages + k_begin / 64 + i];
      if (p < 0 || p >= a.num_pages) { flag_error(kStatusBounds); p = 0; }
      pid[i] = p;
    }
  }
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  // Producer: warp-uniform waits; MMA issuer: single-thread waits (both on abort_flag).
  // Softmax: warp-uniform waits on its own flag, which it only reads after a barrier of all
  // four softmax warps, so that the four always leave the loop together.
  volatile int* soft_flag = abort_flag + 1;
  const uint32_t role = (warp == 0 || warp == L::VLOAD_WARP) ? kRoleProducer
                        : (warp == 1 || warp == L::PV_WARP) ? kRoleMma : kRoleSoftmax;
  auto site = [&](uint64_t* bar, int blk) {
    return wait_site(kKernelDecode, role, static_cast<uint32_t>(bar - bars), blk);
  };
  auto waitw = [&](uint64_t* bar, uint32_t parity, int blk) -> bool {
    return bounded_wait_warp(bar, parity, abort_flag, site(bar, blk));
  };
  auto wait1 = [&](uint64_t* bar, uint32_t parity, int blk) -> bool {
    return bounded_wait(bar, parity, abort_flag, site(bar, blk));
  };
  auto waits = [&](uint64_t* bar, uint32_t parity, int blk) -> bool {
    int ok = 0;
    if (lane == 0) {
      ok = mbar_wait(bar, parity) ? 1 : 0;
      if (!ok) record_timeout(site(bar, blk));
    }
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
  };

  if (warp == 0) {
    // ================================ producer ================================
    {
      // Q scale factors of the g heads (rows 0..15 of the N = 16 operand; rows >= g are 0).
      uint32_t w0 = 0, w1 = 0;
      if (lane < g) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(a.q_scales + (qrow0 + lane) * (D / 16)));
        w0 = v.x; w1 = v.y;
      }
      *reinterpret_cast<uint4*>(sm + L::OFF_QSF + lane * 16) = make_uint4(w0, 0, 0, 0);
      *reinterpret_cast<uint4*>(sm + L::OFF_QSF + 512 + lane * 16) = make_uint4(w1, 0, 0, 0);
      if constexpr (kDQ) {                             // the second Q tensor's scales
        uint32_t u0 = 0, u1 = 0;
        if (lane < g) {
          const uint2 v = __ldg(reinterpret_cast<const uint2*>(a.q2_scales + (qrow0 + lane) * (D / 16)));
          u0 = v.x; u1 = v.y;
        }
        *reinterpret_cast<uint4*>(sm + L::OFF_Q2SF + lane * 16) = make_uint4(u0, 0, 0, 0);
        *reinterpret_cast<uint4*>(sm + L::OFF_Q2SF + 512 + lane * 16) = make_uint4(u1, 0, 0, 0);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full, 16 * 64 * (kDQ ? 2 : 1));
        tma_load_2d(sm + L::OFF_Q, &tm_q, q_full, 0, static_cast<int>(qrow0));
        if constexpr (kDQ) tma_load_2d(sm + L::OFF_Q2, &tm_q2, q_full, 0, static_cast<int>(qrow0));
      }
    }
    int issued = 0;
    for (int blk = 0; blk < nblk; ++blk) {
      const int st_i = blk % L::NK;
      if (blk >= L::NK && !waitw(k_empty + st_i, ((blk / L::NK) - 1) & 1, blk)) break;
      unsigned char* st = sm + L::OFF_KST + st_i * L::KST_BYTES;
      const int k0 = k_begin + blk * 128;
      const int p0 = pid[2 * blk];
      const int p1 = (k0 + 64 < len) ? pid[2 * blk + 1] : p0;
      // K scale factors straight into the tcgen05 layout with 4-byte asynchronous copies: key
      // row r = r0 + 32 r1 (rows 0..63 from page p0, 64..127 from p1) -> byte r0*16 + r1*4 of
      // the chunk of its 64-element MMA step. This warp does not wait for them.
#pragma unroll
      for (int r1 = 0; r1 < 4; ++r1) {
        const int r = r1 * 32 + lane;
        const int pp = r < 64 ? p0 : p1;
        const uint8_t* src = a.k_page_scales + ((static_cast<int64_t>(pp) * a.Hkv + h) * 64 + (r & 63)) * (D / 16);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) cp_async4(st + L::ST_KSF + kk * 512 + lane * 16 + r1 * 4, src + kk * 4, true);
      }
      cp_async_arrive_noinc(k_full + st_i);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(k_full + st_i, 128 * 64);
        tma_load_2d(st + L::ST_K, &tm_kp, k_full + st_i, 0, (p0 * a.Hkv + h) * 64);
        tma_load_2d(st + L::ST_K + 4096, &tm_kp, k_full + st_i, 0, (p1 * a.Hkv + h) * 64);
      }
      issued = blk + 1;
    }
    // Drain: never leave a copy in flight into this CTA's shared memory.
    for (int i = 0; i < L::NK && i < issued; ++i) {
      const int last = i + ((issued - 1 - i) / L::NK) * L::NK;
      mbar_wait(k_full + i, (last / L::NK) & 1);
    }
    mbar_wait(q_full, 0);
  } else if (warp == L::VLOAD_WARP) {
    // ============================== V producer ==============================
    // V codes of the block's two pages by TMA; their V scales (256 B each, as stored) by bulk
    // copy, to be rearranged into the tcgen05 layout by the PV warp.
    if (lane == 0) {
      int issued = 0;
      for (int blk = 0; blk < nblk; ++blk) {
        const int st_i = blk % L::NVS;
        if (blk >= L::NVS && !wait1(v_empty + st_i, ((blk / L::NVS) - 1) & 1, blk)) break;
        unsigned char* st = sm + L::OFF_VST + st_i * L::VST_BYTES;
        const int k0 = k_begin + blk * 128;
        const int p0 = pid[2 * blk];
        const int p1 = (k0 + 64 < len) ? pid[2 * blk + 1] : p0;
        mbar_arrive_expect_tx(v_full + st_i, 2 * D * 64 + 2 * D * 2);
        tma_load_2d(st + L::ST_V0, &tm_vp, v_full + st_i, 0, (p0 * a.Hkv + h) * D);
        tma_load_2d(st + L::ST_V1, &tm_vp, v_full + st_i, 0, (p1 * a.Hkv + h) * D);
        bulk_load(st + L::ST_VRAW, a.v_page_scales + (static_cast<int64_t>(p0) * a.Hkv + h) * D * 2, D * 2, v_full + st_i);
        bulk_load(st + L::ST_VRAW + D * 2, a.v_page_scales + (static_cast<int64_t>(p1) * a.Hkv + h) * D * 2, D * 2, v_full + st_i);
        issued = blk + 1;
      }
      for (int i = 0; i < L::NVS && i < issued; ++i) {
        const int last = i + ((issued - 1 - i) / L::NVS) * L::NVS;
        mbar_wait(v_full + i, (last / L::NVS) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================ QK^T issuer (one thread) ============================
    const uint32_t idesc_qk = idesc_block_scaled(kFmtE2M1_mxf4, kFmtE2M1_mxf4, 0, 128, L::NQ);
    const uint32_t sQ = smem_u32(sm + L::OFF_Q);
    if (lane == 0) {
      bool ok = wait1(q_full, 0, -1);
      if (ok) {
        tc_fence_after();
        tmem_cp_sf(tbase + L::T_QSF, sm + L::OFF_QSF);
        tmem_cp_sf(tbase + L::T_QSF + 4, sm + L::OFF_QSF + 512);
        if constexpr (kDQ) {
          tmem_cp_sf(tbase + L::T_Q2SF, sm + L::OFF_Q2SF);
          tmem_cp_sf(tbase + L::T_Q2SF + 4, sm + L::OFF_Q2SF + 512);
        }
      }
      for (int blk = 0; ok && blk < nblk; ++blk) {
        const int st_i = blk % L::NK, b2 = blk & 1;
        if (!wait1(k_full + st_i, (blk / L::NK) & 1, blk)) { ok = false; break; }
        // the K scale factors arrived by cp.async (generic proxy); the tensor core reads them
        // through the async proxy
        fence_proxy_async_smem();
        if (blk >= 2 && !wait1(s_free + b2, ((blk - 2) >> 1) & 1, blk)) { ok = false; break; }
        tc_fence_after();
        unsigned char* st = sm + L::OFF_KST + st_i * L::KST_BYTES;
        const uint32_t tk = tbase + L::T_KSF + 8 * st_i;
        tmem_cp_sf(tk, st + L::ST_KSF);
        tmem_cp_sf(tk + 4, st + L::ST_KSF + 512);
        const uint32_t sK = smem_u32(st + L::ST_K);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const uint64_t da = make_sdesc(sK + kk * 32, 16, 512, kSw64);
          const uint64_t db = make_sdesc(sQ + kk * 32, 16, 512, kSw64);
          mma_nvf4(tbase + L::T_S + b2 * 16, da, db, idesc_qk, tk + 4 * kk,
                   tbase + L::T_QSF + 4 * kk, kk > 0 ? 1u : 0u);
        }
        if constexpr (kDQ) {                           // S^T += K Q2^T
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint64_t da = make_sdesc(sK + kk * 32, 16, 512, kSw64);
            const uint64_t db = make_sdesc(smem_u32(sm + L::OFF_Q2) + kk * 32, 16, 512, kSw64);
            mma_nvf4(tbase + L::T_S + b2 * 16, da, db, idesc_qk, tk + 4 * kk,
                     tbase + L::T_Q2SF + 4 * kk, 1u);
          }
        }
        mma_commit(s_full + b2);
        mma_commit(k_empty + st_i);
      }
      mma_commit(mma_final);
      mbar_wait(mma_final, 0);
    }
    __syncwarp();
  } else if (warp == L::PV_WARP) {
    // ============================== PV issuer ==============================
    // The whole warp rearranges the V scales of each block into the tcgen05 layout; lane 0
    // issues the tcgen05 copies and MMAs and their commits. PV(blk) goes out as soon as P(blk)
    // is ready, independently of the QK^T stream (which waits for the next block's loads).
    const uint32_t idesc_pv = idesc_block_scaled(kFmtE4M3, kFmtE4M3, 1, 128, L::NQ);
    const uint32_t sP = smem_u32(sm + L::OFF_P);
    if (lane == 0) {
      tc_fence_after();
      tmem_cp_sf(tbase + L::T_ONESF, sm + L::OFF_PSF + 1024);
    }
    bool ok = true;
    for (int bb = 0; ok && bb < nblk; ++bb) {
      const int st_i = bb % L::NVS, b2 = bb & 1;
      if (!waitw(p_full + b2, (bb >> 1) & 1, bb)) { ok = false; break; }
      if (!waitw(v_full + st_i, (bb / L::NVS) & 1, bb)) { ok = false; break; }
      unsigned char* st = sm + L::OFF_VST + st_i * L::VST_BYTES;
      {
        // channel c = r0 + 32 r1: word [page0 g0, page0 g1, page1 g0, page1 g1] at r0*16 + r1*4
        const uint16_t* raw = reinterpret_cast<const uint16_t*>(st + L::ST_VRAW);
        uint32_t vw[4];
#pragma unroll
        for (int r1 = 0; r1 < 4; ++r1) {
          const int c = r1 * 32 + lane;
          vw[r1] = static_cast<uint32_t>(raw[c]) | (static_cast<uint32_t>(raw[D + c]) << 16);
        }
        *reinterpret_cast<uint4*>(st + L::ST_VSF + lane * 16) = make_uint4(vw[0], vw[1], vw[2], vw[3]);
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (lane == 0) {
        tc_fence_after();
        const uint32_t tv = tbase + L::T_VSF + 4 * st_i;
        // P^T scales: this block's (slot b2) with underflow-aware scaling, else the 1.0 chunk
        const uint32_t tp = kUA ? tbase + L::T_PSF + 4 * b2 : tbase + L::T_ONESF;
        tmem_cp_sf(tv, st + L::ST_VSF);
        if (kUA) tmem_cp_sf(tp, sm + L::OFF_PSF + 512 * b2);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t sV = smem_u32(st + ((kk >> 1) ? L::ST_V1 : L::ST_V0));
          const uint64_t da = make_sdesc(sV + (kk & 1) * 32, 16, 512, kSw64);
          const uint64_t db = make_sdesc(sP + b2 * 2048 + kk * 32, 16, 1024, kSw128);
          mma_mxf8(tbase + L::T_O, da, db, idesc_with_sf_ids(idesc_pv, kk, kk),
                   tv | (static_cast<uint32_t>(kk) << 30),
                   tp | (static_cast<uint32_t>(kk) << 30),
                   (bb > 0 || kk > 0) ? 1u : 0u);
        }
        // l on the tensor core: L^T += 1 P^T (A = 128 rows of E4M3 1.0, the same 32-key slice
        // for every step, scale 1.0; B with the P^T scales), so every row of L^T holds the row
        // sums of the quantized P, rescaled with O^T.
        const uint64_t d1 = make_sdesc(smem_u32(sm + L::OFF_ONES), 16, 256, kSw32);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t db = make_sdesc(sP + b2 * 2048 + kk * 32, 16, 1024, kSw128);
          mma_mxf8(tbase + L::T_L, d1, db, idesc_with_sf_ids(idesc_pv, kk, kk),
                   (tbase + L::T_ONESF) | (static_cast<uint32_t>(kk) << 30),
                   tp | (static_cast<uint32_t>(kk) << 30),
                   (bb > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(pv_done + b2);
        mma_commit(v_empty + st_i);
      }
      __syncwarp();
    }
    if (lane == 0) {
      mma_commit(mma_final + 1);
      mbar_wait(mma_final + 1, 0);
    }
    __syncwarp();
  } else {
    // ============================ softmax (one key per thread) ============================
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const float C = (*a.q_ts) * (*a.k_ts) * a.softmax_scale * kLog2e;
    float m_run[GM];
#pragma unroll
    for (int q = 0; q < GM; ++q) m_run[q] = -INFINITY;
    unsigned char* sP = sm + L::OFF_P;
    bool failed = false;
    for (int blk = 0; blk < nblk; ++blk) {
      const int b2 = blk & 1;
      // On a timeout the body still runs (on whatever TMEM holds) so that the four warps
      // meet at the named barrier; the shared flag, set before it, then ends the loop for all.
      if (!waits(s_full + b2, (blk >> 1) & 1, blk)) failed = true;
      tc_fence_after();
      float x[16];
      tmem_ld16(tbase + L::T_S + b2 * 16 + lane_addr, reinterpret_cast<uint32_t*>(x));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free + b2);
      const bool valid = k_begin + blk * 128 + r < k_end;
      // Block max per query: over this warp's 32 keys in one warp reduction, then over the
      // four warps through shared memory (slots alternate by block parity, so a fast warp's
      // next write cannot land before the others have read).
      float* rm = red_max + b2 * 64;
      float own[GM];                                       // this warp's 32-key block max
#pragma unroll
      for (int q = 0; q < GM; ++q) {
        x[q] = (valid && q < g) ? x[q] : -INFINITY;        // raw MMA units
        asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(own[q]) : "f"(x[q]));
        if (lane == 0) rm[wq * 16 + q] = own[q];
      }
      if (failed && lane == 0) *soft_flag = 1;
      named_bar_sync(1, 128);
      if (*soft_flag) break;
      float alpha[GM], moff[GM];
      bool all_one = true;
#pragma unroll
      for (int q = 0; q < GM; ++q) {
        const float mb = fmaxf(fmaxf(rm[q], rm[16 + q]), fmaxf(rm[32 + q], rm[48 + q]));
        const float m_new = fmaxf(m_run[q], mb);
        const bool dead = (m_new == -INFINITY);
        moff[q] = dead ? 0.f : m_new;
        alpha[q] = dead ? 1.f : ex2_approx((m_run[q] - m_new) * C);
        all_one = all_one && (alpha[q] == 1.f);
        m_run[q] = m_new;
      }
      // Underflow-aware P scaling: this warp's 32 keys are one block of the P^T operand; with
      // mu = log2 of the block's largest p~ (<= 0), P is encoded as 448 p~ 2^-e, e = ceil(mu)
      // clipped to [-127, 0], and the MMA's E8M0 scale of that block is 2^e.
      float pe[GM];
#pragma unroll
      for (int q = 0; q < GM; ++q) {
        const float mu = (own[q] - moff[q]) * C;
        pe[q] = (kUA && mu > -1.0e30f) ? fminf(fmaxf(ceilf(mu), -127.f), 0.f) : 0.f;
      }
      uint32_t codes[GM / 4];
#pragma unroll
      for (int q = 0; q < GM; q += 4) {
        float p[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) p[i] = ex2_approx((x[q + i] - moff[q + i]) * C - pe[q + i]) * 448.f;
        codes[q >> 2] = cvt_e4m3x2(p[0], p[1]) | (cvt_e4m3x2(p[2], p[3]) << 16);
      }
      // P^T buffer b2 was read by PV(blk-2); O^T and L^T are rescaled below after PV(blk-1).
      if (blk >= 1) {
        if (!waits(pv_done + ((blk - 1) & 1), ((blk - 1) >> 1) & 1, blk)) failed = true;
        tc_fence_after();
      }
      // P^T scales of this warp's block (row q, byte wq of the block-parity chunk)
      if (kUA && lane == 0) {
#pragma unroll
        for (int q = 0; q < GM; ++q)
          if (q < g) sm[L::OFF_PSF + 512 * b2 + q * 16 + wq] = static_cast<unsigned char>(127 + static_cast<int>(pe[q]));
      }
      // P^T row q (query), column r (key), 128-byte swizzle.
      unsigned char* pb = sP + b2 * 2048;
#pragma unroll
      for (int q = 0; q < GM; ++q) {
        if (q < g)
          pb[q * 128 + ((((r >> 4) ^ (q & 7))) << 4) + (r & 15)] =
              static_cast<unsigned char>(codes[q >> 2] >> (8 * (q & 3)));
      }
      fence_proxy_async_smem();
      if (blk >= 1 && !__all_sync(0xffffffffu, all_one)) {
        float o[16], l[16];
        tmem_ld16(tbase + L::T_O + lane_addr, reinterpret_cast<uint32_t*>(o));
        tmem_ld16(tbase + L::T_L + lane_addr, reinterpret_cast<uint32_t*>(l));
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < GM; ++q) { o[q] *= alpha[q]; l[q] *= alpha[q]; }
        tmem_st16(tbase + L::T_O + lane_addr, reinterpret_cast<uint32_t*>(o));
        tmem_st16(tbase + L::T_L + lane_addr, reinterpret_cast<uint32_t*>(l));
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + b2);
    }
    if (!*soft_flag && !failed && waits(pv_done + ((nblk - 1) & 1), ((nblk - 1) >> 1) & 1, nblk)) {
      tc_fence_after();
      float o[16], l[16];
      tmem_ld16(tbase + L::T_O + lane_addr, reinterpret_cast<uint32_t*>(o));
      tmem_ld16(tbase + L::T_L + lane_addr, reinterpret_cast<uint32_t*>(l));
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < GM; ++q) {
        if (q < g) {
          part[q * q_stride + r] = o[q];
          // the merge works in log2 units: store m * C
          if (r == 0) { part[q * q_stride + D] = m_run[q] * C; part[q * q_stride + D + 1] = l[q]; }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 128);
  }
}

// Merge the splits: one CTA per (sequence, query head), one thread per channel.
__global__ void __launch_bounds__(128) decode_merge_kernel(const float* __restrict__ ws,
                                                           int32_t n_splits, int32_t out_kind,
                                                           void* __restrict__ out,
                                                           float* __restrict__ lse) {
  constexpr int D = 128;
  const int64_t row = blockIdx.x;
  const float* p = ws + row * n_splits * (D + 2);
  float M = -INFINITY;
  for (int i = 0; i < n_splits; ++i) M = fmaxf(M, p[i * (D + 2) + D]);
  float Lsum = 0.f, acc = 0.f;
  for (int i = 0; i < n_splits; ++i) {
    const float m = p[i * (D + 2) + D];
    const float w = (m == -INFINITY) ? 0.f : ex2_approx(m - M);
    Lsum += w * p[i * (D + 2) + D + 1];
    acc += w * p[i * (D + 2) + threadIdx.x];
  }
  // A row with no key (its context length failed the bounds check, so every split is empty)
  // gets O = 0 and lse = -inf rather than 0/0; the status word reports the error.
  const bool empty = !(Lsum > 0.f);
  const float v = empty ? 0.f : acc / Lsum;
  if (out_kind == 2) static_cast<float*>(out)[row * D + threadIdx.x] = v;
  else if (out_kind == 1) static_cast<__nv_bfloat16*>(out)[row * D + threadIdx.x] = __float2bfloat16_rn(v);
  else static_cast<__half*>(out)[row * D + threadIdx.x] = __float2half_rn(v);
  if (lse != nullptr && threadIdx.x == 0) lse[row] = empty ? -INFINITY : M * kLn2 + logf(Lsum * (1.f / 448.f));
}

}  // namespace qk4v8
