// QK4V8 prefill attention on sm_100a tensor cores.
//
// Method (hotelren.com MpFA article §1, §3.3-3.4; problem statement): Q and K in NVFP4, V in
// MXFP8; S = Q K^T on block-scaled FP4 tensor cores (tcgen05 kind::mxf4nvf4, E4M3 scale per
// 16 elements) accumulated in FP32; online softmax in FP32 over 128-key tiles; P quantized to
// E4M3 as P*448 against the running max after the tile; O += P V on block-scaled FP8 tensor
// cores (kind::mxf8f6f4, E8M0 scale per 32 tokens; P's scale is 1); O / l at the end, where
// l sums the quantized weights. Optional FP16 tiles (ai-feeds.com ThriftAttention summary,
// "方法" step 3): a tile marked in the selection bitmap runs QK^T and PV with kind::f16 on
// FP16 copies of Q, K, V, with P = fp16(448 exp(s - m)), into the same (m, l, O).
//
// l comes from the tensor core: every V tile in shared memory carries 16 extra rows of 1.0
// after its D channel rows, so the PV MMA (N = D + 16) accumulates sum_j P_j into O column D,
// with the same rescaling as O.
//
// Softmax in two groups by key-tile parity. Group 0 (warps 4-7) takes the even key tiles and
// group 1 (warps 8-11) the odd ones; each thread owns one query row and all 128 keys of the
// tile. The groups exchange the running max per tile through shared memory right after the
// tile max (long before the exponentials), so one group's exponentials run while the other
// loads, reduces and stores: the exp unit, the bound of this kernel, stays busy.
//
// S is double-buffered by tile parity, so QK^T of tile j+1 runs while tile j is in the
// softmax. O is a single accumulator kept relative to the running max of the last tile whose
// PV went in. Tile j's P is computed against m(j); before PV(j) the rows whose max rose at
// tile j are rescaled (after PV(j-1) is done). Late in a row the max rarely rises, so most
// warps skip the rescale and PV(j) follows PV(j-1) without a round trip.
//
// Two MMA issuers: one thread issues QK^T, another PV, each waiting only on its own inputs,
// so neither stream of tensor-core work stalls behind the other's waits (an issuing thread
// blocks while the tensor core drains what it issued).
//
// One CTA per (128-query tile, batch, query head), heaviest causal tiles first. Warp roles:
//   warp 0     producer: TMA of Q/K/V code tiles (swizzled), scale factors gathered into the
//              tcgen05 scale layout with 4-byte asynchronous copies, FP16 tiles when selected
//   warp 1     TMEM owner and QK^T issuer (one thread)
//   warp 2     PV issuer (one thread)
//   warps 4-11 softmax (two groups of four; warp w reaches TMEM lane quadrant w % 4)
// TMEM (512 columns): S_0, S_1 [0,256), O (D + 16 columns) from 256, scale factors from 400.
#pragma once
#include "ptx.cuh"

namespace qk4v8 {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2_448 = 8.807354922057604f;   // log2(448)
// Share of the exponentials taken on the FMA pipe, in eighths. 0: all on the special-function
// unit, the fastest setting measured on B200 for this kernel's instruction mix (2/8 ran 2%
// slower: the extra FMA-pipe instructions cost more issue slots than the exp unit saved).
constexpr int kPolyOf8 = 0;

struct FwdArgs {
  const uint8_t* q_scales;
  const uint8_t* k_scales;
  const uint8_t* v_scales;
  const float* q_ts;
  const float* k_ts;
  const uint8_t* bitmap;      // [B*Hq, Tq, Tk] or null
  void* out;
  float* lse;
  int32_t B, Hq, Hkv, Nq, Nk, Npad, Tq, Tk;
  int32_t causal;
  float softmax_scale;
  int32_t out_kind;          // 0 fp16, 1 bf16, 2 fp32
};

template <int D, bool kMixed>
struct FwdLayout {
  static constexpr int NS = kMixed ? 2 : 4;   // the FP16 operand stage needs the room
  static constexpr int KSTEPS = D / 64;                 // FP4 MMAs per QK (K = 64 each)
  static constexpr int NV = D + 16;                     // PV MMA N: D channels + ones rows
  static constexpr int Q_BYTES = 128 * D / 2;
  static constexpr int K_BYTES = 128 * D / 2;
  static constexpr int V_TMA_BYTES = D * 128;
  static constexpr int V_BYTES = NV * 128;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_QSF = OFF_Q + Q_BYTES;                         // KSTEPS chunks
  static constexpr int OFF_PSF = OFF_QSF + 1024;                          // all 1.0 (E8M0 127)
  static constexpr int OFF_STAGE = OFF_PSF + 1024;
  static constexpr int ST_K = 0;
  static constexpr int ST_V = K_BYTES;
  static constexpr int ST_KSF = ST_V + V_BYTES;
  static constexpr int ST_VSF = ST_KSF + 1024;
  static constexpr int STAGE_BYTES = ST_VSF + 1024;
  static constexpr int OFF_P = OFF_STAGE + NS * STAGE_BYTES;               // 2 x 16 KB
  static constexpr int OFF_RED = OFF_P + 2 * 16384;   // running max hand-off [2][128]
  static constexpr int OFF_Q16 = OFF_RED + 2048;
  static constexpr int F16_TILE = 128 * D * 2;
  static constexpr int V16_ATOM = NV * 128;                                // 64 keys x NV rows
  static constexpr int OFF_K16 = OFF_Q16 + (kMixed ? F16_TILE : 0);
  static constexpr int OFF_V16 = OFF_K16 + (kMixed ? F16_TILE : 0);
  static constexpr int OFF_BAR = OFF_V16 + (kMixed ? 2 * V16_ATOM : 0);
  static constexpr int N_BARS = 1 + 2 * NS + 15;
  static constexpr int SMEM_BYTES = OFF_BAR + N_BARS * 8 + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;                     // alignment slack
  // TMEM columns
  // S_b at T_S + 128 b; K and V scale factors in two slots by tile parity (8 columns each: a
  // slot is rewritten only after the MMA two tiles back that read it has completed).
  static constexpr uint32_t T_S = 0, T_O = 256, T_QSF = 400, T_PSF = 408, T_KSF = 412,
                            T_VSF = 428;
  static_assert(T_O + NV <= T_QSF && T_VSF + 16 <= 512, "TMEM columns");
  static constexpr uint32_t QK_SW = (D == 128) ? kSw64 : kSw32;
  static constexpr uint32_t QK_SBO = 8 * D / 2;
  // Warpgroup 0: producer (warp 0), QK^T issuer (1), PV issuer (2), spare (3); warpgroups 1
  // and 2: the two softmax groups.
  static constexpr int PV_WARP = 2;
  static constexpr int THREADS = 384;
};

template <int D, bool kMixed>
__global__ void __launch_bounds__(384, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q16,
                const __grid_constant__ CUtensorMap tm_k16, const __grid_constant__ CUtensorMap tm_v16,
                FwdArgs a) {
  using L = FwdLayout<D, kMixed>;
  extern __shared__ unsigned char smem_raw[];
  // 1024-byte aligned base, kept as an offset from the shared array so that the compiler
  // still sees shared-memory accesses (not generic ones)
  unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = bars + 1 + L::NS;
  // Barriers a group waits on come in pairs by key-tile parity: a waiter must never run more
  // than one phase ahead of a barrier (a parity wait cannot tell phase k from phase k - 2).
  uint64_t* s_full = bars + 1 + 2 * L::NS; // [2], by tile parity
  uint64_t* s_free = s_full + 2;           // [2], by tile parity
  uint64_t* p_full = s_full + 4;           // [2], by tile parity
  uint64_t* pv_done = s_full + 6;          // [2], by tile parity
  uint64_t* m_ready = s_full + 8;          // [2], by tile parity: running max handed on
  uint64_t* kv16_full = s_full + 10;
  uint64_t* kv16_empty = s_full + 11;
  uint64_t* q16_full = s_full + 12;
  uint64_t* mma_final = s_full + 13;      // [2]: QK issuer, PV issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BHq = a.B * a.Hq;
  const int qt = a.Tq - 1 - static_cast<int>(blockIdx.x / BHq);
  const int bhq = static_cast<int>(blockIdx.x % BHq);
  const int b = bhq / a.Hq, hq = bhq % a.Hq;
  const int hk = hq / (a.Hq / a.Hkv);
  const int bhk = b * a.Hkv + hk;
  const int nt = a.causal ? min(qt + 1, a.Tk) : a.Tk;
  const uint8_t* bm_row = kMixed ? a.bitmap + (static_cast<int64_t>(bhq) * a.Tq + qt) * a.Tk : nullptr;

  if (threadIdx.x == 0) {
    // full barriers: the TMA's expect-tx arrival plus one cp.async arrival per producer lane
    mbar_init(q_full, 33);
    // a stage is free once both the QK^T (K) and the PV (V) issuers are done with it
    for (int s = 0; s < L::NS; ++s) { mbar_init(kv_full + s, 33); mbar_init(kv_empty + s, 2); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_free + i, 4);
      mbar_init(s_full + i, 1);
      mbar_init(p_full + i, 4);
      mbar_init(pv_done + i, 1);
      mbar_init(m_ready + i, 4);
    }
    mbar_init(kv16_full, 1); mbar_init(kv16_empty, 1); mbar_init(q16_full, 1);
    mbar_init(mma_final, 1); mbar_init(mma_final + 1, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Constants in shared memory: the P scale factors (E8M0 127 = 1.0, also the second V scale
  // chunk) and the 16 rows of 1.0 after each V tile (E4M3 0x38; FP16 0x3C00 in the FP16 V).
  // Every byte of a ones row is equal, so the 128-byte swizzle leaves them unchanged.
  for (int i = threadIdx.x; i < 128; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sm + L::OFF_PSF)[i] = 0x7F7F7F7Fu;
  for (int s = 0; s < L::NS; ++s)
    for (int i = threadIdx.x; i < 16 * 128 / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(sm + L::OFF_STAGE + s * L::STAGE_BYTES + L::ST_V + L::V_TMA_BYTES)[i] =
          make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
  if constexpr (D < 128) {
    for (int s = 0; s < L::NS; ++s)
      for (int i = threadIdx.x; i < 128; i += blockDim.x)
        if (((i >> 2) & 31) + 32 * (i & 3) >= D)       // word i: row (i/4)%32 + 32 (i%4)
          reinterpret_cast<uint32_t*>(sm + L::OFF_STAGE + s * L::STAGE_BYTES + L::ST_VSF)[i] = 0x7F7F7F7Fu;
  }
  if constexpr (kMixed) {
    for (int h = 0; h < 2; ++h)
      for (int i = threadIdx.x; i < 16 * 128 / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(sm + L::OFF_V16 + h * L::V16_ATOM + D * 128)[i] =
            make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);
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

  // Barrier ids in timeout reports are their index in the barrier block.
  const uint32_t role = warp == 0 ? kRoleProducer : (warp == 1 || warp == L::PV_WARP) ? kRoleMma : kRoleSoftmax;
  auto site = [&](uint64_t* bar, int tile) {
    return wait_site(kKernelFwd, role, static_cast<uint32_t>(bar - bars), tile);
  };
  auto waitw = [&](uint64_t* bar, uint32_t parity, int tile) -> bool {
    return bounded_wait_warp(bar, parity, abort_flag, site(bar, tile));
  };
  auto wait1 = [&](uint64_t* bar, uint32_t parity, int tile) -> bool {
    return bounded_wait(bar, parity, abort_flag, site(bar, tile));
  };

  if (warp == 0) {
    // ================================ producer ================================
    if (lane == 0) { prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v); }
    // Scale factors go straight from global memory into the tcgen05 scale layout with 4-byte
    // asynchronous copies (row r = r0 + 32 r1 of a 128-row chunk -> byte r0*16 + r1*4; one
    // 4-byte word holds the 4 scales of one 64-element MMA step), completing on the same
    // barrier as the TMA of the codes, so this warp never waits on their latency.
    {
      const int64_t row0 = static_cast<int64_t>(bhq) * a.Nq + qt * 128;
#pragma unroll
      for (int r1 = 0; r1 < 4; ++r1) {
        const int r = r1 * 32 + lane;
        const bool ok = qt * 128 + r < a.Nq;
        const uint8_t* src = a.q_scales + (ok ? (row0 + r) * (D / 16) : 0);
#pragma unroll
        for (int kk = 0; kk < L::KSTEPS; ++kk)
          cp_async4(sm + L::OFF_QSF + kk * 512 + lane * 16 + r1 * 4, src + kk * 4, ok);
      }
      cp_async_arrive_noinc(q_full);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full, L::Q_BYTES);
        tma_load_3d(sm + L::OFF_Q, &tm_q, q_full, 0, qt * 128, bhq);
      }
    }
    bool q16_loaded = false;
    int n16 = 0, issued = 0;
    for (int j = 0; j < nt; ++j) {
      const int s = j % L::NS;
      if (j >= L::NS && !waitw(kv_empty + s, ((j / L::NS) - 1) & 1, j)) break;
      unsigned char* st = sm + L::OFF_STAGE + s * L::STAGE_BYTES;
      // K scale factors of keys j*128 .. j*128+127; V scale factors of this key tile (channel
      // row c, 4 E8M0 codes of 32 tokens each). Rows past Nk read as zero; V rows from D on
      // (the ones rows) hold 1.0 set once at start.
      const int64_t krow0 = static_cast<int64_t>(bhk) * a.Nk + j * 128;
#pragma unroll
      for (int r1 = 0; r1 < 4; ++r1) {
        const int r = r1 * 32 + lane;
        const bool ok = j * 128 + r < a.Nk;
        const uint8_t* src = a.k_scales + (ok ? (krow0 + r) * (D / 16) : 0);
#pragma unroll
        for (int kk = 0; kk < L::KSTEPS; ++kk)
          cp_async4(st + L::ST_KSF + kk * 512 + lane * 16 + r1 * 4, src + kk * 4, ok);
        if (r < D)
          cp_async4(st + L::ST_VSF + lane * 16 + r1 * 4,
                    a.v_scales + (static_cast<int64_t>(bhk) * D + r) * (a.Npad / 32) + j * 4, true);
      }
      cp_async_arrive_noinc(kv_full + s);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(kv_full + s, L::K_BYTES + L::V_TMA_BYTES);
        tma_load_3d(st + L::ST_K, &tm_k, kv_full + s, 0, j * 128, bhk);
        tma_load_2d(st + L::ST_V, &tm_v, kv_full + s, j * 128, bhk * D);
      }
      issued = j + 1;
      if constexpr (kMixed) {
        if (bm_row[j]) {
          if (!q16_loaded) {
            if (lane == 0) {
              mbar_arrive_expect_tx(q16_full, L::F16_TILE);
              for (int h = 0; h < D / 64; ++h)
                tma_load_3d(sm + L::OFF_Q16 + h * 16384, &tm_q16, q16_full, h * 64, qt * 128, bhq);
            }
            q16_loaded = true;
          }
          if (n16 >= 1 && !waitw(kv16_empty, (n16 - 1) & 1, j)) break;
          if (lane == 0) {
            mbar_arrive_expect_tx(kv16_full, L::F16_TILE + 2 * D * 128);
            for (int h = 0; h < D / 64; ++h)
              tma_load_3d(sm + L::OFF_K16 + h * 16384, &tm_k16, kv16_full, h * 64, j * 128, bhk);
            for (int h = 0; h < 2; ++h)
              tma_load_2d(sm + L::OFF_V16 + h * L::V16_ATOM, &tm_v16, kv16_full, j * 128 + h * 64, bhk * D);
          }
          ++n16;
        }
      }
    }
    // Drain: never leave a copy in flight into this CTA's shared memory.
    for (int s = 0; s < L::NS && s < issued; ++s) {
      const int last = s + ((issued - 1 - s) / L::NS) * L::NS;
      mbar_wait(kv_full + s, (last / L::NS) & 1);
    }
    mbar_wait(q_full, 0);
    if (kMixed && n16 > 0) { mbar_wait(kv16_full, (n16 - 1) & 1); mbar_wait(q16_full, 0); }
  } else if (warp == 1) {
    // ============================ QK^T issuer (one thread) ============================
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_block_scaled(kFmtE2M1_mxf4, kFmtE2M1_mxf4, 0, 128, 128);
      const uint32_t idesc_qk16 = idesc_f16(128, 128);
      const uint32_t sQ = smem_u32(sm + L::OFF_Q);
      bool ok = wait1(q_full, 0, -1);
      if (ok) {
        // the scale factors arrived by cp.async (generic proxy); the tensor core reads them
        // through the async proxy
        fence_proxy_async_smem();
        tc_fence_after();
        for (int kk = 0; kk < L::KSTEPS; ++kk)
          tmem_cp_sf(tbase + L::T_QSF + 4 * kk, sm + L::OFF_QSF + kk * 512);
      }
      int n16 = 0;
      bool q16_ready = false;
      for (int j = 0; ok && j < nt; ++j) {
        const int s = j % L::NS;
        const bool f16 = kMixed && bm_row[j];
        if (!wait1(kv_full + s, (j / L::NS) & 1, j)) { ok = false; break; }
        fence_proxy_async_smem();
        tc_fence_after();
        // S_{j&1} (and K scale slot j&1) were last used by tile j-2
        if (j >= 2 && !wait1(s_free + (j & 1), ((j - 2) >> 1) & 1, j)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tS = tbase + L::T_S + (j & 1) * 128;
        if (!f16) {
          unsigned char* st = sm + L::OFF_STAGE + s * L::STAGE_BYTES;
          const uint32_t tk = tbase + L::T_KSF + 8 * (j & 1);
          for (int kk = 0; kk < L::KSTEPS; ++kk) tmem_cp_sf(tk + 4 * kk, st + L::ST_KSF + kk * 512);
          const uint32_t sK = smem_u32(st + L::ST_K);
          for (int kk = 0; kk < L::KSTEPS; ++kk) {
            const uint64_t da = make_sdesc(sQ + kk * 32, 16, L::QK_SBO, L::QK_SW);
            const uint64_t db = make_sdesc(sK + kk * 32, 16, L::QK_SBO, L::QK_SW);
            mma_nvf4(tS, da, db, idesc_qk, tbase + L::T_QSF + 4 * kk, tk + 4 * kk, kk > 0 ? 1u : 0u);
          }
        } else {
          if (!q16_ready) {
            if (!wait1(q16_full, 0, j)) { ok = false; break; }
            q16_ready = true;
          }
          if (!wait1(kv16_full, n16 & 1, j)) { ok = false; break; }
          tc_fence_after();
          ++n16;
          const uint32_t sQ16 = smem_u32(sm + L::OFF_Q16), sK16 = smem_u32(sm + L::OFF_K16);
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t da = make_sdesc(sQ16 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kSw128);
            const uint64_t db = make_sdesc(sK16 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kSw128);
            mma_f16(tS, da, db, idesc_qk16, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(s_full + (j & 1));
        mma_commit(kv_empty + s);                  // K half of the stage is free
      }
      // Everything this thread issued has completed before TMEM is released.
      mma_commit(mma_final);
      mbar_wait(mma_final, 0);
    }
    __syncwarp();
  } else if (warp == L::PV_WARP) {
    // ============================== PV issuer (one thread) ==============================
    if (lane == 0) {
      const uint32_t idesc_pv = idesc_block_scaled(kFmtE4M3, kFmtE4M3, 1, 128, L::NV);
      const uint32_t idesc_pv16 = idesc_f16(128, L::NV);
      const uint32_t sP = smem_u32(sm + L::OFF_P);
      tc_fence_after();
      tmem_cp_sf(tbase + L::T_PSF, sm + L::OFF_PSF);
      for (int b2 = 0; b2 < 2; ++b2)               // second V scale chunk (rows 128..): 1.0
        tmem_cp_sf(tbase + L::T_VSF + 8 * b2 + 4, sm + L::OFF_PSF);
      bool ok = true;
      int n16 = 0;
      for (int jj = 0; ok && jj < nt; ++jj) {
        const int s = jj % L::NS, b2 = jj & 1;
        const bool f16 = kMixed && bm_row[jj];
        if (!wait1(p_full + b2, (jj >> 1) & 1, jj)) { ok = false; break; }
        if (!wait1(kv_full + s, (jj / L::NS) & 1, jj)) { ok = false; break; }
        if (f16 && !wait1(kv16_full, n16 & 1, jj)) { ok = false; break; }
        fence_proxy_async_smem();
        tc_fence_after();
        const uint32_t tO = tbase + L::T_O;
        if (!f16) {
          unsigned char* st = sm + L::OFF_STAGE + s * L::STAGE_BYTES;
          const uint32_t tv = tbase + L::T_VSF + 8 * b2;   // PV(jj-2), its last reader, is done
          tmem_cp_sf(tv, st + L::ST_VSF);
          const uint32_t sV = smem_u32(st + L::ST_V);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t da = make_sdesc(sP + b2 * 16384 + kk * 32, 16, 1024, kSw128);
            const uint64_t db = make_sdesc(sV + kk * 32, 16, 1024, kSw128);
            mma_mxf8(tO, da, db, idesc_with_sf_ids(idesc_pv, kk, kk),
                     (tbase + L::T_PSF) | (static_cast<uint32_t>(kk) << 30),
                     tv | (static_cast<uint32_t>(kk) << 30), (jj > 0 || kk > 0) ? 1u : 0u);
          }
        } else {
          ++n16;
          const uint32_t sV16 = smem_u32(sm + L::OFF_V16);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t da = make_sdesc(sP + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kSw128);
            const uint64_t db = make_sdesc(sV16 + (kk >> 2) * L::V16_ATOM + (kk & 3) * 32, 16, 1024, kSw128);
            mma_f16(tO, da, db, idesc_pv16, (jj > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(kv16_empty);
        }
        mma_commit(pv_done + b2);
        mma_commit(kv_empty + s);                  // V half of the stage is free
      }
      mma_commit(mma_final + 1);
      mbar_wait(mma_final + 1, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ================================ softmax ================================
    const int wq = warp & 3;                 // TMEM lane quadrant
    const int grp = (warp - 4) >> 2;         // key-tile parity this group handles
    const int row = wq * 32 + lane;
    const int qi = qt * 128 + row;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    float* red_m = reinterpret_cast<float*>(sm + L::OFF_RED);         // [2 parities][128]
    // Scores stay in the FP4 MMA's raw units (S = sum codes*scales); the running max m is
    // kept in those units and 448 p = 2^(s C + (log2 448 - m C)) with
    // C = s_tQ s_tK softmax_scale log2(e). FP16 tiles produce true dot products and are
    // brought into raw units by 1 / (s_tQ s_tK).
    const float C = (*a.q_ts) * (*a.k_ts) * a.softmax_scale * kLog2e;
    const float R16 = 1.f / ((*a.q_ts) * (*a.k_ts));
    const float2 C2 = make_float2(C, C);
    unsigned char* sP = sm + L::OFF_P;
    const uint32_t tO = tbase + L::T_O + lane_addr;
    bool ok = true;
    for (int j = grp; j < nt; j += 2) {
      const int b2 = j & 1;                  // == grp
      const bool f16 = kMixed && bm_row[j];
      const bool prev_f16 = kMixed && j >= 1 && bm_row[j - 1];
      float x[128];
      if (!waitw(s_full + b2, (j >> 1) & 1, j)) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t* xr = reinterpret_cast<uint32_t*>(x);
        const uint32_t tS = tbase + L::T_S + b2 * 128 + lane_addr;
#pragma unroll
        for (int c = 0; c < 128; c += 32) tmem_ld32(tS + c, xr + c);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free + b2);
      if (f16) {
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] *= R16;
      }
      const int kbase = j * 128;
      if ((a.causal && kbase + 127 > qi) || (kbase + 128 > a.Nk)) {
        const int lim = min(a.Nk - 1, a.causal ? qi : a.Nk - 1) - kbase;   // last valid column
#pragma unroll
        for (int c = 0; c < 128; ++c) x[c] = (c <= lim) ? x[c] : -INFINITY;
      }
      float mt;
      {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
#pragma unroll
          for (int u = 0; u < 4; ++u) m4[u] = fmax3(m4[u], x[c + 2 * u], x[c + 2 * u + 1]);
        }
        mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      }
      // Running max before this tile: handed on by the group that processed tile j - 1.
      float m_prev = -INFINITY;
      if (j >= 1) {
        if (!waitw(m_ready + ((j - 1) & 1), ((j - 1) >> 1) & 1, j)) { ok = false; break; }
        __syncwarp();
        m_prev = red_m[((j - 1) & 1) * 128 + row];
      }
      const float m_new = fmaxf(m_prev, mt);
      red_m[b2 * 128 + row] = m_new;
      __syncwarp();
      if (lane == 0) mbar_arrive(m_ready + b2);
      const bool dead = (m_new == -INFINITY);
      const float bias = kLog2_448 - (dead ? 0.f : m_new) * C;
      const float2 B2 = make_float2(bias, bias);
      uint32_t pw[kMixed ? 64 : 32];      // e4m3: 32 words; fp16: 64 words
      if (!f16) {
        // kPolyOf8 of every 8 groups of 4 scores take the FMA-pipe exponential, the rest the
        // special-function unit, so both pipes work on the tile.
#pragma unroll
        for (int c = 0; c < 128; c += 4) {
          const float2 t0 = __ffma2_rn(make_float2(x[c], x[c + 1]), C2, B2);
          const float2 t1 = __ffma2_rn(make_float2(x[c + 2], x[c + 3]), C2, B2);
          float2 e0, e1;
          if (((c >> 2) & 7) < kPolyOf8) {
            e0 = exp2_poly2(t0);
            e1 = exp2_poly2(t1);
          } else {
            e0 = make_float2(ex2_approx(t0.x), ex2_approx(t0.y));
            e1 = make_float2(ex2_approx(t1.x), ex2_approx(t1.y));
          }
          pw[c >> 2] = cvt_e4m3x2(e0.x, e0.y) | (cvt_e4m3x2(e1.x, e1.y) << 16);
        }
      } else if constexpr (kMixed) {
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          const float2 t = __ffma2_rn(make_float2(x[c], x[c + 1]), C2, B2);
          const __half2 h = __floats2half2_rn(ex2_approx(t.x), ex2_approx(t.y));
          pw[c >> 1] = *reinterpret_cast<const uint32_t*>(&h);
        }
      }
      // P buffer b2 was last used by PV(j-2). An FP16 tile's P fills both buffers:
      // writing one needs PV(j-1) done as well, and the tile after an FP16 tile too. PV(j-2)'s
      // completion implies PV(j-3)'s, so the wait on the other parity's barrier is for its
      // next phase.
      if (j >= 2 && !waitw(pv_done + b2, ((j - 2) >> 1) & 1, j)) { ok = false; break; }
      if ((f16 || prev_f16) && j >= 1 &&
          !waitw(pv_done + ((j - 1) & 1), ((j - 1) >> 1) & 1, j)) { ok = false; break; }
      if (!f16) {
        unsigned char* prow = sP + b2 * 16384 + row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) =
              make_uint4(pw[4 * c], pw[4 * c + 1], pw[4 * c + 2], pw[4 * c + 3]);
      } else if constexpr (kMixed) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          unsigned char* prow = sP + h * 16384 + row * 128;     // atom h = keys 64h .. 64h+63
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) =
                make_uint4(pw[32 * h + 4 * c], pw[32 * h + 4 * c + 1], pw[32 * h + 4 * c + 2],
                           pw[32 * h + 4 * c + 3]);
        }
      }
      fence_proxy_async_smem();
      // O holds the tiles before j relative to m(j-1) = m_prev. Rows whose max rose at this
      // tile are brought to m_new once PV(j-1) is done (the next phase of that parity's
      // barrier: PV(j-2), waited above, implies PV(j-3)); a warp whose rows all kept their
      // max hands P(j) on at once.
      const float alpha = (m_prev == -INFINITY || dead) ? 1.f : ex2_approx((m_prev - m_new) * C);
      if (j >= 1 && !__all_sync(0xffffffffu, alpha == 1.f)) {
        if (!waitw(pv_done + ((j - 1) & 1), ((j - 1) >> 1) & 1, j)) { ok = false; break; }
        tc_fence_after();
        const float2 A2 = make_float2(alpha, alpha);
#pragma unroll
        for (int cc = 0; cc < D; cc += 32) {
          uint32_t o[32];
          tmem_ld32(tO + cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float2 u = __fmul2_rn(make_float2(__uint_as_float(o[k]), __uint_as_float(o[k + 1])), A2);
            o[k] = __float_as_uint(u.x);
            o[k + 1] = __float_as_uint(u.y);
          }
          tmem_st32(tO + cc, o);
        }
        {
          uint32_t o[16];
          tmem_ld16(tO + D, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st16(tO + D, o);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + b2);
    }
    // ---- epilogue: O / l (O and l already relative to the final max) ----
    // PV(nt-1)'s completion covers every earlier MMA of the issuing thread; the group that
    // owns tile nt-1 waits for it (the next phase of its own barrier) and the named barrier
    // passes that on to the other group.
    if (ok && grp == ((nt - 1) & 1)) ok = waitw(pv_done + grp, ((nt - 1) >> 1) & 1, nt);
    tc_fence_before();
    named_bar_sync(1, 256);
    if (ok && !*abort_flag) {
      tc_fence_after();
      const float m_run = red_m[((nt - 1) & 1) * 128 + row];   // m(nt-1), published last
      uint32_t lr[16];
      tmem_ld16(tO + D, lr);
      tmem_wait_ld();
      const float l_run = __uint_as_float(lr[0]);
      const bool store = qi < a.Nq;
      const int64_t orow = static_cast<int64_t>(bhq) * a.Nq + qi;
#pragma unroll
      for (int cc = 0; cc < D / 2; cc += 32) {
        const int c = grp * (D / 2) + cc;
        uint32_t o[32];
        tmem_ld32(tO + c, o);
        tmem_wait_ld();
        if (store) {
          float v[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = __fdiv_rn(__uint_as_float(o[k]), l_run);
          if (a.out_kind == 2) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow * D + c);
#pragma unroll
            for (int k = 0; k < 8; ++k) dst[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
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
            for (int k = 0; k < 4; ++k) dst[k] = reinterpret_cast<uint4*>(packed)[k];
          }
        }
      }
      if (store && grp == 0 && a.lse != nullptr)
        a.lse[orow] = m_run * C * kLn2 + logf(l_run * (1.f / 448.f));
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
