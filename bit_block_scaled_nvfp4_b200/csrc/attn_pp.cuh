// QK4V8 prefill attention, FP4 tiles: two query tiles per CTA, one softmax warpgroup each.
//
// Same method and arithmetic as attn_fwd.cuh (hotelren.com MpFA article §1, §3.3-3.4: NVFP4 Q
// and K, MXFP8 V, FP32 online softmax over 128-key tiles, P = E4M3(448 p~) against the running
// max after the tile, l = the sum of the quantized weights through 16 ones rows after every V
// tile, O / l at the end); what differs is the work split.
//
// A work item is two query tiles ("units") that read the same K and V tiles: two query heads of
// one GQA group at the same query tile when a group has an even number of heads, else two
// consecutive query tiles of one head (the second may be absent at the end; under causal
// masking the first skips the second's diagonal key tile). Warpgroup u (warps 4 + 4u .. 7 + 4u)
// owns unit u for the whole item: its rows' running max stays in registers, so no max is handed
// between warpgroups, and the two warpgroups run their own chains, alternating on the
// exponential unit. Per key tile one K/V stage (a ring of four) serves both units.
//
// TMEM (512 columns): one S buffer [0, 128) shared by the units in turn (the QK^T issuer writes
// S for unit 0, waits for warpgroup 0 to have read it, then writes S for unit 1, ...); O_0 and
// O_1 (D + 16 columns each: the ones rows give l in column D); scale factors after them. Two S
// buffers and two O accumulators with their ones columns would need 544 columns.
//
// Warp roles: warp 0 producer (TMA of both units' Q per item and of the K/V stage per key
// tile; scale factors by 4-byte cp.async straight into the tcgen05 scale layout), warp 1 TMEM
// owner and QK^T issuer, warp 2 PV issuer, warp 3 idle, warps 4-11 the two softmax
// warpgroups (warp w reaches TMEM lane quadrant w % 4).
#pragma once
#include "attn_fwd.cuh"

namespace qk4v8 {

struct PPItem {
  int qt[2], bhq[2], nt[2];   // nt = 0: unit absent
  int bhk;
};

// Items of the pair schedule, heaviest first.
__device__ __forceinline__ PPItem pp_item(const FwdArgs& a, int idx, bool head_pairs) {
  PPItem w;
  if (head_pairs) {
    const int npairs = a.B * (a.Hq / 2);
    const int qt = a.Tq - 1 - idx / npairs;
    const int pair = idx % npairs;
    const int b = pair / (a.Hq / 2), hq0 = 2 * (pair % (a.Hq / 2));
    w.qt[0] = w.qt[1] = qt;
    w.bhq[0] = b * a.Hq + hq0;
    w.bhq[1] = w.bhq[0] + 1;
    w.bhk = b * a.Hkv + hq0 / (a.Hq / a.Hkv);
  } else {
    const int BH = a.B * a.Hq;
    const int i = (a.Tq + 1) / 2 - 1 - idx / BH;
    const int bhq = idx % BH;
    const int b = bhq / a.Hq, hq = bhq % a.Hq;
    w.qt[0] = 2 * i;
    w.qt[1] = 2 * i + 1;
    w.bhq[0] = w.bhq[1] = bhq;
    w.bhk = b * a.Hkv + hq / (a.Hq / a.Hkv);
  }
#pragma unroll
  for (int u = 0; u < 2; ++u)
    w.nt[u] = (w.qt[u] >= a.Tq) ? 0 : (a.causal ? min(w.qt[u] + 1, a.Tk) : a.Tk);
  return w;
}
__host__ __device__ constexpr bool pp_head_pairs(int Hq, int Hkv) { return (Hq / Hkv) % 2 == 0; }
__host__ __device__ constexpr int pp_items(int B, int Hq, int Hkv, int Tq) {
  return pp_head_pairs(Hq, Hkv) ? Tq * B * (Hq / 2) : ((Tq + 1) / 2) * B * Hq;
}

template <int D>
struct PPLayout {
  static constexpr int NK = 4;                          // K/V ring stages
  static constexpr int KSTEPS = D / 64;
  static constexpr int NV = D + 16;
  static constexpr int Q_BYTES = 128 * D / 2;
  static constexpr int K_BYTES = 128 * D / 2;
  static constexpr int V_TMA_BYTES = D * 128;
  static constexpr int V_BYTES = NV * 128;
  static constexpr int STG_BYTES = K_BYTES + V_BYTES + 2048;
  static constexpr int OFF_Q = 0;                                   // [item parity][unit]
  static constexpr int OFF_QSF = OFF_Q + 4 * Q_BYTES;               // [item parity][unit] 1 KB
  static constexpr int OFF_PSF = OFF_QSF + 4096;                    // all 1.0 (E8M0 127)
  static constexpr int OFF_STG = OFF_PSF + 1024;
  __host__ __device__ static constexpr int k_off(int s) { return OFF_STG + s * STG_BYTES; }
  __host__ __device__ static constexpr int v_off(int s) { return k_off(s) + K_BYTES; }
  __host__ __device__ static constexpr int k_sf_off(int s) { return k_off(s) + K_BYTES + V_BYTES; }
  __host__ __device__ static constexpr int v_sf_off(int s) { return k_sf_off(s) + 1024; }
  static constexpr int OFF_P = OFF_STG + NK * STG_BYTES;            // [unit] 16 KB
  static constexpr int OFF_BAR = OFF_P + 2 * 16384;
  static constexpr int N_BARS = 4 + 2 * NK + 11;
  static constexpr int SMEM_BYTES = OFF_BAR + N_BARS * 8 + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory");
  static_assert(OFF_STG % 1024 == 0 && STG_BYTES % 1024 == 0 && OFF_P % 1024 == 0, "alignment");
  // TMEM columns: S, O_0, O_1 (32-column aligned), Q scale factors [item parity][unit], P scale
  // factors, K and V scale factors in two slots by key-tile parity.
  static constexpr uint32_t T_S = 0, T_O0 = 128;
  static constexpr uint32_t T_O1 = (T_O0 + NV + 31) / 32 * 32;
  static constexpr uint32_t T_QSF = T_O1 + NV;
  static constexpr uint32_t T_PSF = T_QSF + 32, T_KSF = T_PSF + 4, T_VSF = T_KSF + 16;
  static_assert(T_VSF + 16 <= 512, "TMEM columns");
  static constexpr uint32_t QK_SW = (D == 128) ? kSw64 : kSw32;
  static constexpr uint32_t QK_SBO = 8 * D / 2;
  static constexpr int THREADS = 384;
  // Registers: 168 a thread at launch (384 threads); warpgroup 0 (producer, issuers) gives
  // some to the two softmax warpgroups: 4*32*96 + 8*32*200 <= 384*168.
  static constexpr int REGS_LAUNCH = 168, REGS_WG0 = 96, REGS_SOFTMAX = 200;
  static_assert(4 * 32 * REGS_WG0 + 8 * 32 * REGS_SOFTMAX <= THREADS * REGS_LAUNCH, "register split");
};

template <int D>
__global__ void __launch_bounds__(384, 1)
attn_pp_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, FwdArgs a) {
  using L = PPLayout<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  // A waiter never runs two phases behind a barrier: per-unit barriers count that unit's key
  // tiles; the shared S buffer's s_free counts QK^Ts in issue order.
  uint64_t* q_full = bars + 0;             // [2], by item parity (both units' Q)
  uint64_t* q_empty = bars + 2;            // [2], by item parity
  uint64_t* k_full = bars + 4;             // [NK]
  uint64_t* k_empty = k_full + L::NK;      // [NK]
  uint64_t* s_full = k_empty + L::NK;      // [2], by unit: S holds this unit's scores
  uint64_t* s_free = s_full + 2;           // S has been read (phase per QK^T)
  uint64_t* p_full = s_free + 1;           // [2], by unit
  uint64_t* pv_done = p_full + 2;          // [2], by unit
  uint64_t* mma_final = pv_done + 2;       // [2]: QK issuer, PV issuer
  uint64_t* pv_tile = mma_final + 2;       // [2], by key-tile parity: the tile's PVs are done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = static_cast<int>(gridDim.x), cta = static_cast<int>(blockIdx.x);
  const bool head_pairs = pp_head_pairs(a.Hq, a.Hkv);
  const int n_items = pp_items(a.B, a.Hq, a.Hkv, a.Tq);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) { mbar_init(q_full + i, 33); mbar_init(q_empty + i, 1); }
    for (int s = 0; s < L::NK; ++s) { mbar_init(k_full + s, 33); mbar_init(k_empty + s, 2); }
    for (int u = 0; u < 2; ++u) {
      mbar_init(s_full + u, 1);
      mbar_init(p_full + u, 4);
      mbar_init(pv_done + u, 1);
    }
    mbar_init(s_free, 4);
    mbar_init(mma_final, 1); mbar_init(mma_final + 1, 1);
    mbar_init(pv_tile, 1); mbar_init(pv_tile + 1, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // P scale factors (E8M0 127 = 1.0, also the second V scale chunk), the 16 rows of 1.0 after
  // each V tile (E4M3 0x38), and at D < 128 the unused V scale rows.
  for (int i = threadIdx.x; i < 128; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sm + L::OFF_PSF)[i] = 0x7F7F7F7Fu;
  for (int s = 0; s < L::NK; ++s)
    for (int i = threadIdx.x; i < 16 * 128 / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(sm + L::v_off(s) + L::V_TMA_BYTES)[i] =
          make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
  if constexpr (D < 128) {
    for (int s = 0; s < L::NK; ++s)
      for (int i = threadIdx.x; i < 128; i += blockDim.x)
        if (((i >> 2) & 31) + 32 * (i & 3) >= D)
          reinterpret_cast<uint32_t*>(sm + L::v_sf_off(s))[i] = 0x7F7F7F7Fu;
  }
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  const uint32_t role = (warp == 0 || warp == 3) ? kRoleProducer
                        : (warp == 1 || warp == 2) ? kRoleMma : kRoleSoftmax;
  auto site = [&](uint64_t* bar, int tile) {
    return wait_site(kKernelFwd, role, static_cast<uint32_t>(bar - bars), tile);
  };
  auto waitw = [&](uint64_t* bar, uint32_t parity, int tile) -> bool {
    return bounded_wait_warp(bar, parity, abort_flag, site(bar, tile));
  };
  auto wait1 = [&](uint64_t* bar, uint32_t parity, int tile) -> bool {
    return bounded_wait(bar, parity, abort_flag, site(bar, tile));
  };

  if (warp < 4) {
  setmaxnreg_to<L::REGS_WG0, L::REGS_LAUNCH>();
  if (warp == 0) {
    // ================================ producer ================================
    if (lane == 0) { prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v); }
    const uint64_t once = kL2EvictFirst;           // Q is read once per item
    int g = 0, q_issued = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int idx = fwd_item_index(it, G, cta);
      if (idx >= n_items) break;
      const PPItem w = pp_item(a, idx, head_pairs);
      const int qb = it & 1;
      if (it >= 2 && !waitw(q_empty + qb, ((it - 2) >> 1) & 1, g)) { ok = false; break; }
      int qbytes = 0;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (w.nt[u] == 0) continue;
        qbytes += L::Q_BYTES;
        const int64_t row0 = static_cast<int64_t>(w.bhq[u]) * a.Nq + w.qt[u] * 128;
#pragma unroll
        for (int r1 = 0; r1 < 4; ++r1) {
          const int r = r1 * 32 + lane;
          const bool valid = w.qt[u] * 128 + r < a.Nq;
          const uint8_t* src = a.q_scales + (valid ? (row0 + r) * (D / 16) : 0);
#pragma unroll
          for (int kk = 0; kk < L::KSTEPS; ++kk)
            cp_async4(sm + L::OFF_QSF + (qb * 2 + u) * 1024 + kk * 512 + lane * 16 + r1 * 4, src + kk * 4, valid);
        }
      }
      cp_async_arrive_noinc(q_full + qb);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full + qb, qbytes);
        for (int u = 0; u < 2; ++u)
          if (w.nt[u] > 0)
            tma_load_3d_hint(sm + L::OFF_Q + (qb * 2 + u) * L::Q_BYTES, &tm_q, q_full + qb, 0,
                             w.qt[u] * 128, w.bhq[u], once);
      }
      q_issued = it + 1;
      const int NT = max(w.nt[0], w.nt[1]);
      for (int j = 0; j < NT; ++j, ++g) {
        const int s = g % L::NK;
        if (g >= L::NK && !waitw(k_empty + s, ((g / L::NK) - 1) & 1, g)) { ok = false; break; }
        unsigned char* ksf = sm + L::k_sf_off(s);
        unsigned char* vsf = sm + L::v_sf_off(s);
        const int64_t krow0 = static_cast<int64_t>(w.bhk) * a.Nk + j * 128;
#pragma unroll
        for (int r1 = 0; r1 < 4; ++r1) {
          const int r = r1 * 32 + lane;
          const bool valid = j * 128 + r < a.Nk;
          const uint8_t* src = a.k_scales + (valid ? (krow0 + r) * (D / 16) : 0);
#pragma unroll
          for (int kk = 0; kk < L::KSTEPS; ++kk)
            cp_async4(ksf + kk * 512 + lane * 16 + r1 * 4, src + kk * 4, valid);
          if (r < D)
            cp_async4(vsf + lane * 16 + r1 * 4,
                      a.v_scales + (static_cast<int64_t>(w.bhk) * D + r) * (a.Npad / 32) + j * 4, true);
        }
        cp_async_arrive_noinc(k_full + s);
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_expect_tx(k_full + s, L::K_BYTES + L::V_TMA_BYTES);
          tma_load_3d(sm + L::k_off(s), &tm_k, k_full + s, 0, j * 128, w.bhk);
          tma_load_2d(sm + L::v_off(s), &tm_v, k_full + s, j * 128, w.bhk * D);
        }
      }
    }
    // Drain: never leave a copy in flight into this CTA's shared memory.
    for (int s = 0; s < L::NK && s < g; ++s) {
      const int last = s + ((g - 1 - s) / L::NK) * L::NK;
      mbar_wait(k_full + s, (last / L::NK) & 1);
    }
    for (int qb = 0; qb < 2 && qb < q_issued; ++qb) {
      const int last = qb + ((q_issued - 1 - qb) / 2) * 2;
      mbar_wait(q_full + qb, (last >> 1) & 1);
    }
  } else if (warp == 1) {
    // ============================ QK^T issuer (one thread) ============================
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_block_scaled(kFmtE2M1_mxf4, kFmtE2M1_mxf4, 0, 128, 128);
      const uint32_t tS = tbase + L::T_S;
      bool ok = true;
      int g = 0, nq = 0;                         // key tiles, QK^Ts issued
      for (int it = 0; ok; ++it) {
        const int idx = fwd_item_index(it, G, cta);
        if (idx >= n_items) break;
        const PPItem w = pp_item(a, idx, head_pairs);
        const int qb = it & 1;
        if (!wait1(q_full + qb, (it >> 1) & 1, g)) { ok = false; break; }
        // The Q scale slots qb were last read by item it - 2's QK^Ts, each of which had its S
        // read out (s_free) before the next QK^T was issued.
        fence_proxy_async_smem();
        tc_fence_after();
#pragma unroll
        for (int u = 0; u < 2; ++u)
          if (w.nt[u] > 0)
            for (int kk = 0; kk < L::KSTEPS; ++kk)
              tmem_cp_sf(tbase + L::T_QSF + 8 * (qb * 2 + u) + 4 * kk,
                         sm + L::OFF_QSF + (qb * 2 + u) * 1024 + kk * 512);
        const int NT = max(w.nt[0], w.nt[1]);
        for (int j = 0; j < NT && ok; ++j, ++g) {
          const int s = g % L::NK;
          if (!wait1(k_full + s, (g / L::NK) & 1, g)) { ok = false; break; }
          fence_proxy_async_smem();
          tc_fence_after();
          // K scale slot g & 1 was last read by tile g - 2's QK^Ts (done: their S were read)
          const uint32_t tk = tbase + L::T_KSF + 8 * (g & 1);
          for (int kk = 0; kk < L::KSTEPS; ++kk) tmem_cp_sf(tk + 4 * kk, sm + L::k_sf_off(s) + kk * 512);
          const uint32_t sK = smem_u32(sm + L::k_off(s));
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            if (j >= w.nt[u]) continue;
            // S was last written by QK^T nq - 1: its unit must have read it out
            if (nq >= 1 && !wait1(s_free, (nq - 1) & 1, g)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sQ = smem_u32(sm + L::OFF_Q + (qb * 2 + u) * L::Q_BYTES);
            const uint32_t tq = tbase + L::T_QSF + 8 * (qb * 2 + u);
            for (int kk = 0; kk < L::KSTEPS; ++kk) {
              const uint64_t da = make_sdesc(sQ + kk * 32, 16, L::QK_SBO, L::QK_SW);
              const uint64_t db = make_sdesc(sK + kk * 32, 16, L::QK_SBO, L::QK_SW);
              mma_nvf4(tS, da, db, idesc_qk, tq + 4 * kk, tk + 4 * kk, kk > 0 ? 1u : 0u);
            }
            mma_commit(s_full + u);
            ++nq;
          }
          if (!ok) break;
          mma_commit(k_empty + s);
        }
        if (!ok) break;
        mma_commit(q_empty + qb);
      }
      mma_commit(mma_final);
      mbar_wait(mma_final, 0);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ============================== PV issuer (one thread) ==============================
    if (lane == 0) {
      const uint32_t idesc_pv = idesc_block_scaled(kFmtE4M3, kFmtE4M3, 1, 128, L::NV);
      const uint32_t sP = smem_u32(sm + L::OFF_P);
      tc_fence_after();
      tmem_cp_sf(tbase + L::T_PSF, sm + L::OFF_PSF);
      for (int b2 = 0; b2 < 2; ++b2)               // second V scale chunk (rows 128..): 1.0
        tmem_cp_sf(tbase + L::T_VSF + 8 * b2 + 4, sm + L::OFF_PSF);
      bool ok = true;
      int g = 0, n[2] = {0, 0};                   // key tiles; per unit, its tiles so far
      for (int it = 0; ok; ++it) {
        const int idx = fwd_item_index(it, G, cta);
        if (idx >= n_items) break;
        const PPItem w = pp_item(a, idx, head_pairs);
        const int NT = max(w.nt[0], w.nt[1]);
        for (int j = 0; j < NT && ok; ++j, ++g) {
          const int s = g % L::NK, b2 = g & 1;
          if (!wait1(k_full + s, (g / L::NK) & 1, g)) { ok = false; break; }
          bool sf_copied = false;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            if (j >= w.nt[u]) continue;
            // unit u's P of this tile; its softmax wrote it after PV_u of the unit's previous
            // tile was done, and its epilogue (if this is an item's first tile) has read O_u
            if (!wait1(p_full + u, n[u] & 1, g)) { ok = false; break; }
            fence_proxy_async_smem();
            tc_fence_after();
            const uint32_t tv = tbase + L::T_VSF + 8 * b2;
            if (!sf_copied) {
              // V scale slot b2 was last read by tile g - 2's PVs
              if (g >= 2 && !wait1(pv_tile + b2, ((g - 2) >> 1) & 1, g)) { ok = false; break; }
              tmem_cp_sf(tv, sm + L::v_sf_off(s));
              sf_copied = true;
            }
            const uint32_t sV = smem_u32(sm + L::v_off(s));
            const uint32_t tO = tbase + (u == 0 ? L::T_O0 : L::T_O1);
            const uint32_t tp = tbase + L::T_PSF;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t da = make_sdesc(sP + u * 16384 + kk * 32, 16, 1024, kSw128);
              const uint64_t db = make_sdesc(sV + kk * 32, 16, 1024, kSw128);
              mma_mxf8(tO, da, db, idesc_with_sf_ids(idesc_pv, kk, kk),
                       tp | (static_cast<uint32_t>(kk) << 30),
                       tv | (static_cast<uint32_t>(kk) << 30), (j > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(pv_done + u);
            ++n[u];
          }
          if (!ok) break;
          mma_commit(pv_tile + b2);
          mma_commit(k_empty + s);
        }
      }
      mma_commit(mma_final + 1);
      mbar_wait(mma_final + 1, 0);
    }
    __syncwarp();
  }
  } else {
    setmaxnreg_to<L::REGS_SOFTMAX, L::REGS_LAUNCH>();
    // ================================ softmax ================================
    const int wq = warp & 3;                 // TMEM lane quadrant
    const int unit = (warp - 4) >> 2;        // the query tile this warpgroup owns
    const int row = wq * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    // 448 p = 2^(s C + (log2 448 - m C)) with scores in the FP4 MMA's raw units and
    // C = s_tQ s_tK softmax_scale log2(e).
    const float C = (*a.q_ts) * (*a.k_ts) * a.softmax_scale * kLog2e;
    const float2 Ct = make_float2(C, C);
    unsigned char* sP = sm + L::OFF_P + unit * 16384;
    const uint32_t tO = tbase + (unit == 0 ? L::T_O0 : L::T_O1) + lane_addr;
    const uint32_t tS = tbase + L::T_S + lane_addr;
    bool ok = true;
    int n = 0;                               // this unit's key tiles so far
    for (int it = 0; ok; ++it) {
      const int idx = fwd_item_index(it, G, cta);
      if (idx >= n_items) break;
      const PPItem w = pp_item(a, idx, head_pairs);
      const int nt = w.nt[unit];
      if (nt == 0) continue;
      const int qi = w.qt[unit] * 128 + row;
      float m_run = -INFINITY;
      for (int j = 0; j < nt; ++j, ++n) {
        float x[128];
        if (!waitw(s_full + unit, n & 1, n)) { ok = false; break; }
        tc_fence_after();
        {
          uint32_t* xr = reinterpret_cast<uint32_t*>(x);
#pragma unroll
          for (int c = 0; c < 128; c += 32) tmem_ld32(tS + c, xr + c);
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        const int kbase = j * 128;
        if ((a.causal && kbase + 127 > qi) || (kbase + 128 > a.Nk)) {
          const int lim = min(a.Nk - 1, a.causal ? qi : a.Nk - 1) - kbase;   // last valid column
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] = (c <= lim) ? x[c] : -INFINITY;
        }
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
#pragma unroll
          for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], x[c + 2 * q], x[c + 2 * q + 1]);
        }
        const float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        const float m_prev = m_run;
        const float m_new = fmaxf(m_prev, mt);
        m_run = m_new;
        const bool dead = (m_new == -INFINITY);
        const float bias = kLog2_448 - (dead ? 0.f : m_new) * C;
        const float2 B2 = make_float2(bias, bias);
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          const float2 t = __ffma2_rn(make_float2(x[c], x[c + 1]), Ct, B2);
          x[c] = ex2_approx(t.x);
          x[c + 1] = ex2_approx(t.y);
        }
        // The P buffer and O were last used by PV of this unit's previous tile (all lanes poll:
        // the scores are live here).
        if (n >= 1 && !bounded_wait_warp_all(pv_done + unit, (n - 1) & 1, abort_flag, site(pv_done + unit, n))) {
          ok = false;
          break;
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {               // 16 keys per 16-byte chunk
          uint32_t w4[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int c = ch * 16 + q * 4;
            w4[q] = cvt_e4m3x2(x[c], x[c + 1]) | (cvt_e4m3x2(x[c + 2], x[c + 3]) << 16);
          }
          *reinterpret_cast<uint4*>(sP + row * 128 + ((ch ^ (row & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async_smem();
        // O holds the item's tiles before j relative to m_prev. Rows whose max rose are brought
        // to m_new; a warp whose rows all kept their max skips it. Of the 16 ones columns only
        // column D (l) is read, so only it is rescaled.
        const float alpha = (m_prev == -INFINITY || dead) ? 1.f : ex2_approx((m_prev - m_new) * C);
        if (j >= 1 && !__all_sync(0xffffffffu, alpha == 1.f)) {
          tc_fence_after();
          const float2 A2 = make_float2(alpha, alpha);
          uint32_t o[D], ol;
#pragma unroll
          for (int cc = 0; cc < D; cc += 32) tmem_ld32(tO + cc, o + cc);
          tmem_ld1(tO + D, &ol);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < D; k += 2) {
            const float2 v = __fmul2_rn(make_float2(__uint_as_float(o[k]), __uint_as_float(o[k + 1])), A2);
            o[k] = __float_as_uint(v.x);
            o[k + 1] = __float_as_uint(v.y);
          }
          ol = __float_as_uint(__uint_as_float(ol) * alpha);
#pragma unroll
          for (int cc = 0; cc < D; cc += 32) tmem_st32(tO + cc, o + cc);
          tmem_st1(tO + D, &ol);
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + unit);
      }
      if (!ok) break;
      // ---- epilogue of this unit: O / l (O and l relative to the final max) ----
      if (!waitw(pv_done + unit, (n - 1) & 1, n)) { ok = false; break; }
      tc_fence_after();
      uint32_t lr[16];
      tmem_ld16(tO + D, lr);
      tmem_wait_ld();
      const float l_run = __uint_as_float(lr[0]);
      const float inv_l = __frcp_rn(l_run);     // O / l by Markstein's division (ptx.cuh)
      const bool store = qi < a.Nq;
      const int64_t orow = static_cast<int64_t>(w.bhq[unit]) * a.Nq + qi;
      // O is written once: streaming (evict-first) stores keep K and V in L2
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        tmem_ld32(tO + c, o);
        tmem_wait_ld();
        if (store) {
          float v[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = div_markstein(__uint_as_float(o[k]), l_run, inv_l);
          if (a.out_kind == 2) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow * D + c);
#pragma unroll
            for (int k = 0; k < 8; ++k) __stcs(dst + k, make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]));
          } else {
            __align__(16) uint32_t packed[16];
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
              if (a.out_kind == 1) {
                __nv_bfloat162 t = __floats2bfloat162_rn(v[k], v[k + 1]);
                packed[k >> 1] = *reinterpret_cast<uint32_t*>(&t);
              } else {
                __half2 t = __floats2half2_rn(v[k], v[k + 1]);
                packed[k >> 1] = *reinterpret_cast<uint32_t*>(&t);
              }
            }
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + orow * D + c);
#pragma unroll
            for (int k = 0; k < 4; ++k) __stcs(dst + k, reinterpret_cast<uint4*>(packed)[k]);
          }
        }
      }
      if (store && a.lse != nullptr)
        a.lse[orow] = m_run * C * kLn2 + logf(l_run * (1.f / 448.f));
      // The reads of O above have completed (each tcgen05.ld waited); this warpgroup's next
      // p_full arrival, which lets the next item's first PV overwrite O, follows them.
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

}  // namespace qk4v8
