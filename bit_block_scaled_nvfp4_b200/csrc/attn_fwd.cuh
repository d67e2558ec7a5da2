// QK4V8 prefill attention on sm_100a tensor cores.
//
// Method (hotelren.com MpFA article §1, §3.3-3.4; problem statement): Q and K in NVFP4, V in
// MXFP8; S = Q K^T on block-scaled FP4 tensor cores (tcgen05 kind::mxf4nvf4, E4M3 scale per
// 16 elements) accumulated in FP32; online softmax in FP32 over 128-key tiles; P quantized to
// E4M3 as P*448 against the running max after the tile; O += P V on block-scaled FP8 tensor
// cores (kind::mxf8f6f4, E8M0 scale per 32 tokens; P's scale is 1); O / l at the end, where
// l sums the quantized weights. Optional FP16 tiles (ai-feeds.com ThriftAttention summary,
// "方法" step 3): a tile marked in the selection bitmap runs QK^T with kind::f16 on the caller's
// 16-bit Q and K (fp16 or bf16: both products are exact) and PV on an FP16 copy of V, with
// P = fp16(448 exp(s - m)), into the same (m, l, O).
//
// l comes from the tensor core: every V tile in shared memory carries 16 extra rows of 1.0
// after its D channel rows, so the PV MMA (N = D + 16) accumulates sum_j P_j into O column D,
// with the same rescaling as O (an FP16 tile's PV adds a second MMA of N = 16 over a constant
// block of FP16 ones).
//
// Persistent: one CTA per SM walks a list of work items (128-query tile, batch, query head),
// heaviest causal items first, dealt to the CTAs in a zigzag so their loads even out. All
// pipelines run on across items (a CTA-wide key-tile counter g numbers the S, P and scale
// buffers, and a stage counter the K/V ring, where a selected FP16 tile takes two stages), so
// the next item's Q, K and V loads and its first QK^T overlap the current item's last tiles
// and epilogue; Q has two buffers.
//
// Softmax in two groups by the parity of g. Group 0 (warps 4-7) and group 1 (warps 8-11);
// each thread owns one query row and all 128 keys of its tile. The groups hand the running max
// on per tile through shared memory right after the tile max (long before the exponentials),
// so one group's exponentials run while the other loads, reduces and stores.
//
// S is double-buffered by tile parity, so QK^T of the next tile runs while a tile is in the
// softmax. O is a single accumulator kept relative to the running max of the last tile whose
// PV went in; before PV(j) the rows whose max rose at tile j are rescaled (after PV(j-1) is
// done); late in a row the max rarely rises, so most warps skip the rescale. Two MMA issuer
// threads (QK^T and PV) each wait only on their own inputs (an issuing thread blocks while the
// tensor core drains what it issued).
//
// Warp roles:
//   warp 0     producer: TMA of Q/K/V code tiles (swizzled), scale factors gathered into the
//              tcgen05 scale layout with 4-byte asynchronous copies; a selected tile's FP16 K
//              and V into two ring stages
//   warp 1     TMEM owner and QK^T issuer (one thread)
//   warp 2     PV issuer (one thread)
//   warp 3     FP16 Q producer (FP16-tile kernel only)
//   warps 4-11 softmax (two groups of four; warp w reaches TMEM lane quadrant w % 4)
// TMEM (512 columns): S_0, S_1 [0,256), O (D + 16 columns) from 256, scale factors from 400.
//
// Variants, each its own instance so the default one carries none of their work: kUA,
// underflow-aware P scaling (sns.style BitDecoding-FP4 summary: each 32-key block of a row
// encoded against its own power of two, applied back as the P operand's E8M0 block scale), and
// kDQ, a second Q tensor (the same summary's dual-residual query quantization: its QK^T MMAs
// accumulate into the same S).
#pragma once
#include "ptx.cuh"

namespace qk4v8 {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2_448 = 8.807354922057604f;   // log2(448)
// The exponentials all run on the special-function unit. Evaluating a share of them as
// 2^n p(t - n) on the FMA pipe measured slower on B200 for every share from 1/4 to 1/2 of
// them (3 to 13 %): the extra FMA-pipe and ALU instructions cost more issue slots than the
// unit saves, and a degree-3 p (7.5e-5) flips enough E4M3 codes to fail parity on short
// causal rows. ex2.approx.f16x2 gives no more results per cycle than the f32 form.

struct FwdArgs {
  const uint8_t* q_scales;
  const uint8_t* q2_scales;   // dual-residual second Q tensor's scales, or null (no second Q)
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
  int32_t qk16_bf16;         // FP16 tiles: Q and K are the caller's bf16 (else fp16) tensors
};

// A work item of the persistent prefill kernel: the 128-query tile, batch and query head it
// covers, heaviest causal items first (item = (Tq - 1 - qt) * B*Hq + b*Hq + hq).
struct FwdItem {
  int qt, bhq, bhk, nt;
};
__device__ __forceinline__ FwdItem fwd_item(const FwdArgs& a, int idx) {
  const int BHq = a.B * a.Hq;
  FwdItem w;
  w.qt = a.Tq - 1 - idx / BHq;
  w.bhq = idx % BHq;
  const int b = w.bhq / a.Hq, hq = w.bhq % a.Hq;
  w.bhk = b * a.Hkv + hq / (a.Hq / a.Hkv);
  w.nt = a.causal ? min(w.qt + 1, a.Tk) : a.Tk;
  return w;
}
// Item of round `it` for CTA c of G: c, 2G-1-c, 2G+c, 4G-1-c, ... (zigzag over the heaviest-
// first order, so the CTAs' total work evens out).
__device__ __forceinline__ int fwd_item_index(int it, int G, int c) {
  return it * G + ((it & 1) ? (G - 1 - c) : c);
}

template <int D, bool kMixed, bool kDQ = false>
struct FwdLayout {
  // K and V stages: one ring of four, stage s holding key tile g's K and V (one full and one
  // empty barrier). Separate K and V rings, which let K run ahead, measured slower: the two
  // softmax groups fall into step and contend for the exponential unit at the same time. In
  // the FP16-tile kernel a selected tile takes two consecutive stages, its FP16 K in the first
  // and its FP16 V in the second, so a stage is large enough for either.
  static constexpr int NK = 4;
  static constexpr int NVS = NK;                        // V shares each K stage
  // P buffers, one per tile parity: the exponentials of tile g wait for PV(g - 2).
  static constexpr int NP = 2;
  static constexpr int KSTEPS = D / 64;                 // FP4 MMAs per QK (K = 64 each)
  static constexpr int NV = D + 16;                     // PV MMA N: D channels + ones rows
  static constexpr int Q_BYTES = 128 * D / 2;
  static constexpr int K_BYTES = 128 * D / 2;
  static constexpr int V_TMA_BYTES = D * 128;
  static constexpr int V_BYTES = NV * 128;
  static constexpr int OFF_Q = 0;                                         // 2 buffers
  static constexpr int OFF_QSF = OFF_Q + 2 * Q_BYTES;                     // 2 x KSTEPS chunks
  static constexpr int OFF_PSF = OFF_QSF + 2048;                          // all 1.0 (E8M0 127)
  // Stage s: one block [K | V (+ ones rows) | K scales | V scales] (measured faster than
  // separate K and V arrays).
  // P scale factors of the underflow-aware variant, two chunks by tile parity (row r's four
  // 32-key block scales in the word at (r % 32) * 16 + (r / 32) * 4)
  static constexpr int OFF_PSFU = OFF_PSF + 1024;
  static constexpr int OFF_STG = OFF_PSFU + 1024;
  static constexpr int F16_TILE = 128 * D * 2;     // FP16 Q, K or V (no ones rows) of a tile
  static constexpr int STG_FP4 = K_BYTES + V_BYTES + 2048;
  static constexpr int STG_BYTES = (kMixed && F16_TILE > STG_FP4) ? F16_TILE : STG_FP4;
  __device__ static constexpr int k_off(int s) { return OFF_STG + s * STG_BYTES; }
  __device__ static constexpr int k_sf_off(int s) { return k_off(s) + K_BYTES + V_BYTES; }
  __device__ static constexpr int v_off(int s) { return k_off(s) + K_BYTES; }
  __device__ static constexpr int v_sf_off(int s) { return k_off(s) + K_BYTES + V_BYTES + 1024; }
  static constexpr int OFF_P = OFF_STG + NK * STG_BYTES;                   // NP x 16 KB
  static constexpr int OFF_RED = OFF_P + NP * 16384;   // running max hand-off [2][128], final [128]
  static constexpr int OFF_Q16 = OFF_RED + 2048;
  // The FP16 PV's ones rows (the row sum l in column D of O): 16 rows of 1.0 for each 64-key
  // atom, read by a second MMA of N = 16 (an FP16 V in a ring stage has no ones rows).
  static constexpr int OFF_ONES16 = OFF_Q16 + (kMixed ? F16_TILE : 0);
  static constexpr int V16_ATOM = D * 128;                                 // 64 keys x D rows
  // second Q tensor of dual-residual query quantization (its own instance): two buffers by
  // item parity and their scale factors
  static constexpr int OFF_Q2 = OFF_ONES16 + (kMixed ? 2 * 2048 : 0);
  static constexpr int OFF_Q2SF = OFF_Q2 + (kDQ ? 2 * Q_BYTES : 0);
  static constexpr int OFF_BAR = OFF_Q2SF + (kDQ ? 2048 : 0);
  // barriers: 4 for Q, a full/empty pair per stage, 2 NK spare words (kept so the layout
  // is unchanged), 2 NP for P and 17 singles and pairs (kernel head)
  static constexpr int N_BARS = 2 * NK + 2 * NVS + 2 * NP + 17;
  static constexpr int SMEM_BYTES = OFF_BAR + N_BARS * 8 + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;                     // alignment slack
  static_assert(SMEM_ALLOC <= 227 * 1024, "shared memory");
  static_assert(STG_BYTES % 1024 == 0 && OFF_STG % 1024 == 0 && OFF_Q16 % 1024 == 0 &&
                OFF_ONES16 % 1024 == 0, "1024-byte aligned operand atoms");
  // TMEM columns. S_b at T_S + 128 b; Q scale factors in two slots by item parity, K and V
  // scale factors in two slots by tile parity (8 columns each: a slot is rewritten only after
  // the MMA two items / tiles back that read it has completed).
  static constexpr uint32_t T_S = 0, T_O = 256, T_QSF = 400, T_PSF = 416, T_KSF = 420,
                            T_VSF = 436, T_PSFU = 452,    // T_PSFU: 2 slots by tile parity
                            T_Q2SF = 460;                 // 2 slots by item parity
  static_assert(T_O + NV <= T_QSF && T_Q2SF + 16 <= 512, "TMEM columns");
  static constexpr uint32_t QK_SW = (D == 128) ? kSw64 : kSw32;
  static constexpr uint32_t QK_SBO = 8 * D / 2;
  static constexpr int PV_WARP = 2;
  static constexpr int THREADS = 384;
};

// kUA: underflow-aware P scaling — each 32-key block of a tile row encoded as
// E4M3(448 p~ 2^-e), e = ceil(log2 of the block's largest p~) clipped to [-127, 0], with the
// block's E8M0 P scale 2^e in the PV MMA (FP4 tiles only).
// kDQ: dual-residual query quantization — a second Q tensor (same layout and tensor scale)
// whose QK^T MMAs accumulate into the same S (FP4 tiles only).
template <int D, bool kMixed, bool kUA = false, bool kDQ = false>
__global__ void __launch_bounds__(384, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q16,
                const __grid_constant__ CUtensorMap tm_k16, const __grid_constant__ CUtensorMap tm_v16,
                FwdArgs a) {
  using L = FwdLayout<D, kMixed, kDQ>;
  static_assert(!(kMixed && kDQ), "no second Q tensor with FP16 tiles");
  extern __shared__ unsigned char smem_raw[];
  // 1024-byte aligned base, kept as an offset from the shared array so that the compiler
  // still sees shared-memory accesses (not generic ones)
  unsigned char* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  // Barriers a waiter uses come in pairs by parity where needed: a waiter must never run more
  // than one phase ahead of a barrier (a parity wait cannot tell phase k from phase k - 2).
  uint64_t* q_full = bars + 0;             // [2], by item parity
  uint64_t* q_empty = bars + 2;            // [2], by item parity
  uint64_t* k_full = bars + 4;             // [NK]
  uint64_t* k_empty = k_full + L::NK;
  uint64_t* v_full = k_full;               // V lands on its stage's full barrier with K
  uint64_t* v_empty = k_empty;             // ... and frees it with K (two commits)
  uint64_t* s_full = bars + 4 + 2 * L::NK + 2 * L::NVS;          // [2], by tile parity
  uint64_t* s_free = s_full + 2;           // [2], by tile parity
  uint64_t* m_ready = s_full + 4;          // [2], by tile parity: running max handed on
  uint64_t* o_free = s_full + 6;           // the epilogue has read O
  uint64_t* q16_full = s_full + 9;
  uint64_t* q16_empty = s_full + 10;
  uint64_t* mma_final = s_full + 11;       // [2]: QK issuer, PV issuer
  uint64_t* p_full = s_full + 13;          // [NP], by tile number mod NP
  uint64_t* pv_done = p_full + L::NP;      // [NP], by tile number mod NP
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::N_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = static_cast<int>(gridDim.x), cta = static_cast<int>(blockIdx.x);
  const int n_items = a.Tq * a.B * a.Hq;

  if (threadIdx.x == 0) {
    // full barriers: the TMA's expect-tx arrival plus one cp.async arrival per producer lane
    for (int i = 0; i < 2; ++i) { mbar_init(q_full + i, 33); mbar_init(q_empty + i, 1); }
    // full: the TMA's expect-tx arrival plus one cp.async arrival per producer lane (a single
    // ring: K and V on one barrier; its empty barrier takes both issuers' commits)
    for (int s = 0; s < L::NK; ++s) { mbar_init(k_full + s, 33); mbar_init(k_empty + s, 2); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_free + i, 4);
      mbar_init(s_full + i, 1);
      mbar_init(m_ready + i, 4);
    }
    for (int i = 0; i < L::NP; ++i) { mbar_init(p_full + i, 4); mbar_init(pv_done + i, 1); }
    mbar_init(o_free, 8);
    mbar_init(q16_full, 1); mbar_init(q16_empty, 1);
    mbar_init(mma_final, 1); mbar_init(mma_final + 1, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Constants in shared memory: the P scale factors (E8M0 127 = 1.0, also the second V scale
  // chunk) and the 16 rows of 1.0 after each V tile (E4M3 0x38; FP16 0x3C00 in the FP16 V).
  // Every byte of a ones row is equal, so the 128-byte swizzle leaves them unchanged.
  for (int i = threadIdx.x; i < 128; i += blockDim.x)
    reinterpret_cast<uint32_t*>(sm + L::OFF_PSF)[i] = 0x7F7F7F7Fu;
  for (int s = 0; s < L::NVS; ++s)
    for (int i = threadIdx.x; i < 16 * 128 / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(sm + L::v_off(s) + L::V_TMA_BYTES)[i] =
          make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
  if constexpr (D < 128) {
    for (int s = 0; s < L::NVS; ++s)
      for (int i = threadIdx.x; i < 128; i += blockDim.x)
        if (((i >> 2) & 31) + 32 * (i & 3) >= D)       // word i: row (i/4)%32 + 32 (i%4)
          reinterpret_cast<uint32_t*>(sm + L::v_sf_off(s))[i] = 0x7F7F7F7Fu;
  }
  if constexpr (kMixed) {
    for (int i = threadIdx.x; i < 2 * 2048 / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(sm + L::OFF_ONES16)[i] =
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

  // Barrier ids in timeout reports are their index in the barrier block; the tile number is
  // the CTA's running key-tile counter.
  const uint32_t role = (warp == 0 || warp == 3) ? kRoleProducer
                        : (warp == 1 || warp == L::PV_WARP) ? kRoleMma : kRoleSoftmax;
  auto site = [&](uint64_t* bar, int tile) {
    return wait_site(kKernelFwd, role, static_cast<uint32_t>(bar - bars), tile);
  };
  auto waitw = [&](uint64_t* bar, uint32_t parity, int tile) -> bool {
    return bounded_wait_warp(bar, parity, abort_flag, site(bar, tile));
  };
  auto wait1 = [&](uint64_t* bar, uint32_t parity, int tile) -> bool {
    return bounded_wait(bar, parity, abort_flag, site(bar, tile));
  };
  // Producer steps (one warp): key tile j (the CTA's g-th) of an item into K stage g % NK /
  // V stage g % NVS. Scale factors go straight from global memory into the tcgen05 scale
  // layout with 4-byte asynchronous copies (row r = r0 + 32 r1 of a 128-row chunk -> byte
  // r0*16 + r1*4; one 4-byte word holds the 4 scales of one 64-element MMA step, or the 4
  // E8M0 scales of a V channel row), completing on the same barrier as the TMA of the codes,
  // so the producer never waits on their latency.
  // Both halves of a single-ring stage with one arrival per lane and one TMA transaction count
  // (measured faster than two arrivals on the same barrier).
  // r is the stage counter (ring position), g the tile counter (for timeout reports).
  // dirty: stages whose constant rows an FP16 tile's K or V overwrote.
  uint32_t dirty = 0;
  auto load_kv = [&](int r, int g, int j, const FwdItem& w) -> bool {
    const int s = r % L::NK;
    if (r >= L::NK && !waitw(k_empty + s, ((r / L::NK) - 1) & 1, g)) return false;
    if (kMixed && ((dirty >> s) & 1u)) {
      // the ones rows after V (E4M3 1.0) and, at D < 128, the unused V scale rows (1.0)
      uint4* ones = reinterpret_cast<uint4*>(sm + L::v_off(s) + L::V_TMA_BYTES);
      for (int i = lane; i < 16 * 128 / 16; i += 32)
        ones[i] = make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
      if constexpr (D < 128)
        for (int i = lane; i < 128; i += 32)
          if (((i >> 2) & 31) + 32 * (i & 3) >= D)
            reinterpret_cast<uint32_t*>(sm + L::v_sf_off(s))[i] = 0x7F7F7F7Fu;
      fence_proxy_async_smem();
      dirty &= ~(1u << s);
    }
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
    return true;
  };
  // Half of a selected tile in the FP16-tile kernel: its FP16 K (two 64-channel atoms) or its
  // FP16 V (two 64-key atoms of D rows) into stage r. Only one issuer reads each half, so the
  // producer arrives on the stage's empty barrier for the other (after it saw the stage's
  // previous use released, so the arrival counts toward this use).
  auto load_f16 = [&](int r, int g, int j, const FwdItem& w, bool v) -> bool {
    const int s = r % L::NK;
    if (r >= L::NK && !waitw(k_empty + s, ((r / L::NK) - 1) & 1, g)) return false;
    dirty |= 1u << s;
    mbar_arrive(k_full + s);                     // the 32 lane arrivals of the full barrier
    __syncwarp();
    if (lane == 0) {
      mbar_arrive_expect_tx(k_full + s, L::F16_TILE);
      unsigned char* st = sm + L::k_off(s);
      if (!v) {
        for (int h = 0; h < D / 64; ++h)
          tma_load_3d(st + h * 16384, &tm_k16, k_full + s, h * 64, j * 128, w.bhk);
      } else {
        for (int h = 0; h < 2; ++h)
          tma_load_2d(st + h * L::V16_ATOM, &tm_v16, k_full + s, j * 128 + h * 64, w.bhk * D);
      }
      mbar_arrive(k_empty + s);
    }
    return true;
  };
  // Drain of a ring: wait for the last copy issued into each stage (n = stages issued).
  auto drain = [&](uint64_t* full, int n_stages, int n) {
    for (int s = 0; s < n_stages && s < n; ++s) {
      const int last = s + ((n - 1 - s) / n_stages) * n_stages;
      mbar_wait(full + s, (last / n_stages) & 1);
    }
  };

  if (warp == 0) {
    // ================================ producer ================================
    if (lane == 0) { prefetch_tmap(&tm_q); prefetch_tmap(&tm_k); prefetch_tmap(&tm_v); }
    // Q is read once per item: its codes load evict-first, so that L2 keeps K and V, which
    // every query tile of the head reads again.
    const uint64_t once = kL2EvictFirst;
    int g = 0, r = 0, q_issued = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int idx = fwd_item_index(it, G, cta);
      if (idx >= n_items) break;
      const FwdItem w = fwd_item(a, idx);
      const uint8_t* bm_row = kMixed ? a.bitmap + (static_cast<int64_t>(w.bhq) * a.Tq + w.qt) * a.Tk : nullptr;
      const int qb = it & 1;
      // Q buffer qb was last read by the QK^T MMAs of item it - 2.
      if (it >= 2 && !waitw(q_empty + qb, ((it - 2) >> 1) & 1, g)) { ok = false; break; }
      {
        const int64_t row0 = static_cast<int64_t>(w.bhq) * a.Nq + w.qt * 128;
#pragma unroll
        for (int r1 = 0; r1 < 4; ++r1) {
          const int r = r1 * 32 + lane;
          const bool valid = w.qt * 128 + r < a.Nq;
          const uint8_t* src = a.q_scales + (valid ? (row0 + r) * (D / 16) : 0);
#pragma unroll
          for (int kk = 0; kk < L::KSTEPS; ++kk)
            cp_async4(sm + L::OFF_QSF + qb * 1024 + kk * 512 + lane * 16 + r1 * 4, src + kk * 4, valid);
          if constexpr (kDQ) {                           // the second Q tensor's scales
            const uint8_t* src2 = a.q2_scales + (valid ? (row0 + r) * (D / 16) : 0);
#pragma unroll
            for (int kk = 0; kk < L::KSTEPS; ++kk)
              cp_async4(sm + L::OFF_Q2SF + qb * 1024 + kk * 512 + lane * 16 + r1 * 4, src2 + kk * 4, valid);
          }
        }
        cp_async_arrive_noinc(q_full + qb);
        __syncwarp();
        if (lane == 0) {
          constexpr bool dual = kDQ;
          mbar_arrive_expect_tx(q_full + qb, L::Q_BYTES * (dual ? 2 : 1));
          tma_load_3d_hint(sm + L::OFF_Q + qb * L::Q_BYTES, &tm_q, q_full + qb, 0, w.qt * 128, w.bhq, once);
          // (without FP16 tiles the FP16-Q map slot carries the second Q tensor's map)
          if (dual) tma_load_3d_hint(sm + L::OFF_Q2 + qb * L::Q_BYTES, &tm_q16, q_full + qb, 0, w.qt * 128, w.bhq, once);
        }
        q_issued = it + 1;
      }
      for (int j = 0; j < w.nt; ++j, ++g) {
        if (kMixed && bm_row[j]) {
          if (!load_f16(r, g, j, w, false)) { ok = false; break; }
          ++r;
          if (!load_f16(r, g, j, w, true)) { ok = false; break; }
          ++r;
        } else {
          if (!load_kv(r, g, j, w)) { ok = false; break; }
          ++r;
        }
      }
    }
    // Drain: never leave a copy in flight into this CTA's shared memory.
    drain(k_full, L::NK, r);
    for (int qb = 0; qb < 2 && qb < q_issued; ++qb) {
      const int last = qb + ((q_issued - 1 - qb) / 2) * 2;
      mbar_wait(q_full + qb, (last >> 1) & 1);
    }
  } else if (kMixed && warp == 3) {
    // ============================== FP16 Q producer ==============================
    // The FP16 Q of each item with a selected tile, on a warp of its own so that the producer
    // never waits for the single FP16 Q buffer to drain (the selected tiles' FP16 K and V come
    // through the ring).
    if (lane == 0) { prefetch_tmap(&tm_q16); prefetch_tmap(&tm_k16); prefetch_tmap(&tm_v16); }
    const uint64_t once = kL2EvictFirst;             // FP16 Q: read once per item
    int g = 0, nq16 = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int idx = fwd_item_index(it, G, cta);
      if (idx >= n_items) break;
      const FwdItem w = fwd_item(a, idx);
      const uint8_t* bm_row = a.bitmap + (static_cast<int64_t>(w.bhq) * a.Tq + w.qt) * a.Tk;
      bool q16_loaded = false;
      for (int j = 0; j < w.nt && !q16_loaded; ++j) {
        if (!bm_row[j]) continue;
        // the single FP16 Q buffer was last read by the FP16 QK^Ts of an earlier item
        if (nq16 >= 1 && !waitw(q16_empty, (nq16 - 1) & 1, g + j)) { ok = false; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(q16_full, L::F16_TILE);
          for (int h = 0; h < D / 64; ++h)
            tma_load_3d_hint(sm + L::OFF_Q16 + h * 16384, &tm_q16, q16_full, h * 64, w.qt * 128, w.bhq, once);
        }
        q16_loaded = true;
        ++nq16;
      }
      g += w.nt;
    }
    // Drain: never leave a copy in flight into this CTA's shared memory.
    if (nq16 > 0) mbar_wait(q16_full, (nq16 - 1) & 1);
  } else if (warp == 1) {
    // ============================ QK^T issuer (one thread) ============================
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_block_scaled(kFmtE2M1_mxf4, kFmtE2M1_mxf4, 0, 128, 128);
      const uint32_t idesc_qk16 = idesc_f16(128, 128, a.qk16_bf16 != 0);
      bool ok = true;
      int g = 0, r = 0, nq16 = 0;
      for (int it = 0; ok; ++it) {
        const int idx = fwd_item_index(it, G, cta);
        if (idx >= n_items) break;
        const FwdItem w = fwd_item(a, idx);
        const uint8_t* bm_row = kMixed ? a.bitmap + (static_cast<int64_t>(w.bhq) * a.Tq + w.qt) * a.Tk : nullptr;
        const int qb = it & 1;
        if (!wait1(q_full + qb, (it >> 1) & 1, g)) { ok = false; break; }
        // Q scale slot qb was last read by item it - 2, whose QK^Ts are done once tile g - 2
        // (the latest tile it can own) has been read out of S.
        if (g >= 2 && !wait1(s_free + (g & 1), ((g - 2) >> 1) & 1, g)) { ok = false; break; }
        // the scale factors arrived by cp.async (generic proxy); the tensor core reads them
        // through the async proxy
        fence_proxy_async_smem();
        tc_fence_after();
        const uint32_t tq = tbase + L::T_QSF + 8 * qb;
        for (int kk = 0; kk < L::KSTEPS; ++kk)
          tmem_cp_sf(tq + 4 * kk, sm + L::OFF_QSF + qb * 1024 + kk * 512);
        const uint32_t sQ = smem_u32(sm + L::OFF_Q + qb * L::Q_BYTES);
        constexpr bool dual = kDQ;
        const uint32_t tq2 = tbase + L::T_Q2SF + 8 * qb;
        if (dual)
          for (int kk = 0; kk < L::KSTEPS; ++kk)
            tmem_cp_sf(tq2 + 4 * kk, sm + L::OFF_Q2SF + qb * 1024 + kk * 512);
        const uint32_t sQ2 = smem_u32(sm + L::OFF_Q2 + qb * L::Q_BYTES);
        bool q16_ready = false, had16 = false;
        for (int j = 0; j < w.nt; ++j, ++g) {
          // tile j's stage: its K and V, or (selected tile) its FP16 K; the FP16 V in the next
          const int s = r % L::NK;
          const bool f16 = kMixed && bm_row[j];
          if (!wait1(k_full + s, (r / L::NK) & 1, g)) { ok = false; break; }
          r += f16 ? 2 : 1;
          fence_proxy_async_smem();
          // S_{g&1} (and K scale slot g&1) were last used by tile g - 2
          if (g >= 2 && !wait1(s_free + (g & 1), ((g - 2) >> 1) & 1, g)) { ok = false; break; }
          tc_fence_after();
          const uint32_t tS = tbase + L::T_S + (g & 1) * 128;
          if (!f16) {
            const uint32_t tk = tbase + L::T_KSF + 8 * (g & 1);
            for (int kk = 0; kk < L::KSTEPS; ++kk) tmem_cp_sf(tk + 4 * kk, sm + L::k_sf_off(s) + kk * 512);
            const uint32_t sK = smem_u32(sm + L::k_off(s));
            for (int kk = 0; kk < L::KSTEPS; ++kk) {
              const uint64_t da = make_sdesc(sQ + kk * 32, 16, L::QK_SBO, L::QK_SW);
              const uint64_t db = make_sdesc(sK + kk * 32, 16, L::QK_SBO, L::QK_SW);
              mma_nvf4(tS, da, db, idesc_qk, tq + 4 * kk, tk + 4 * kk, kk > 0 ? 1u : 0u);
            }
            if (dual) {                              // S += Q2 K^T (same tensor scales)
              for (int kk = 0; kk < L::KSTEPS; ++kk) {
                const uint64_t da = make_sdesc(sQ2 + kk * 32, 16, L::QK_SBO, L::QK_SW);
                const uint64_t db = make_sdesc(sK + kk * 32, 16, L::QK_SBO, L::QK_SW);
                mma_nvf4(tS, da, db, idesc_qk, tq2 + 4 * kk, tk + 4 * kk, 1u);
              }
            }
          } else {
            if (!q16_ready) {
              if (!wait1(q16_full, nq16 & 1, g)) { ok = false; break; }
              ++nq16;
              q16_ready = true;
            }
            tc_fence_after();
            had16 = true;
            const uint32_t sQ16 = smem_u32(sm + L::OFF_Q16), sK16 = smem_u32(sm + L::k_off(s));
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t da = make_sdesc(sQ16 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kSw128);
              const uint64_t db = make_sdesc(sK16 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kSw128);
              mma_f16(tS, da, db, idesc_qk16, kk > 0 ? 1u : 0u);
            }
          }
          mma_commit(s_full + (g & 1));
          mma_commit(k_empty + s);
          if (f16) {
            // The FP16 V went into the next stage, which this thread does not read. Waiting for
            // it to land keeps this thread's next wait on that stage one phase after it (a parity
            // wait cannot tell a phase from the one two later). The PV issuer, which skips the
            // FP16 K's stage, needs no such wait: it reaches a later tile only after this tile's
            // P, which follows the FP16 K's arrival.
            const int rv = r - 1;
            if (!wait1(k_full + rv % L::NK, (rv / L::NK) & 1, g)) { ok = false; break; }
          }
        }
        if (!ok) break;
        mma_commit(q_empty + qb);                    // Q buffer qb is free
        if (kMixed && had16) mma_commit(q16_empty);
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
      const uint32_t idesc_pv16 = idesc_f16(128, D);
      const uint32_t idesc_l16 = idesc_f16(128, 16);
      const uint32_t sOnes16 = smem_u32(sm + L::OFF_ONES16);
      const uint32_t sP = smem_u32(sm + L::OFF_P);
      const uint32_t tO = tbase + L::T_O;
      tc_fence_after();
      tmem_cp_sf(tbase + L::T_PSF, sm + L::OFF_PSF);
      for (int b2 = 0; b2 < 2; ++b2)               // second V scale chunk (rows 128..): 1.0
        tmem_cp_sf(tbase + L::T_VSF + 8 * b2 + 4, sm + L::OFF_PSF);
      bool ok = true;
      int g = 0, r = 0;
      for (int it = 0; ok; ++it) {
        const int idx = fwd_item_index(it, G, cta);
        if (idx >= n_items) break;
        const FwdItem w = fwd_item(a, idx);
        const uint8_t* bm_row = kMixed ? a.bitmap + (static_cast<int64_t>(w.bhq) * a.Tq + w.qt) * a.Tk : nullptr;
        // the first PV of an item overwrites O: the previous item's epilogue must have read it
        if (it >= 1 && !wait1(o_free, (it - 1) & 1, g)) { ok = false; break; }
        for (int j = 0; j < w.nt; ++j, ++g) {
          const bool f16 = kMixed && bm_row[j];
          const int rv = f16 ? r + 1 : r;            // the stage holding this tile's V
          r += f16 ? 2 : 1;
          const int s = rv % L::NVS, b2 = g & 1, pb = g % L::NP;
          if (!wait1(p_full + pb, (g / L::NP) & 1, g)) { ok = false; break; }
          if (!wait1(v_full + s, (rv / L::NVS) & 1, g)) { ok = false; break; }
          fence_proxy_async_smem();
          tc_fence_after();
          if (!f16) {
            const uint32_t tv = tbase + L::T_VSF + 8 * b2;   // PV(g-2), its last reader, is done
            tmem_cp_sf(tv, sm + L::v_sf_off(s));
            // P scales: the tile's own (slot b2, written by the softmax) in the underflow-aware
            // variant, else the constant 1.0 chunk
            const uint32_t tp = kUA ? tbase + L::T_PSFU + 4 * b2 : tbase + L::T_PSF;
            if constexpr (kUA) tmem_cp_sf(tp, sm + L::OFF_PSFU + 512 * b2);
            const uint32_t sV = smem_u32(sm + L::v_off(s));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t da = make_sdesc(sP + pb * 16384 + kk * 32, 16, 1024, kSw128);
              const uint64_t db = make_sdesc(sV + kk * 32, 16, 1024, kSw128);
              mma_mxf8(tO, da, db, idesc_with_sf_ids(idesc_pv, kk, kk),
                       tp | (static_cast<uint32_t>(kk) << 30),
                       tv | (static_cast<uint32_t>(kk) << 30), (j > 0 || kk > 0) ? 1u : 0u);
            }
          } else {
            // O[:, 0:D) += P V over the FP16 V in the stage; O[:, D:D+16) += P 1 (l in column D)
            const uint32_t sV16 = smem_u32(sm + L::k_off(s));
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t da = make_sdesc(sP + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kSw128);
              const uint64_t db = make_sdesc(sV16 + (kk >> 2) * L::V16_ATOM + (kk & 3) * 32, 16, 1024, kSw128);
              mma_f16(tO, da, db, idesc_pv16, (j > 0 || kk > 0) ? 1u : 0u);
              const uint64_t d1 = make_sdesc(sOnes16 + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024, kSw128);
              mma_f16(tO + D, da, d1, idesc_l16, (j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          mma_commit(pv_done + pb);
          mma_commit(v_empty + s);
        }
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
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    float* red_m = reinterpret_cast<float*>(sm + L::OFF_RED);         // [2 parities][128]
    float* red_fin = red_m + 256;                                     // [2 items][128]
    // Scores stay in the FP4 MMA's raw units (S = sum codes*scales); the running max m is
    // kept in those units and 448 p = 2^(s C + (log2 448 - m C)) with
    // C = s_tQ s_tK softmax_scale log2(e). FP16 tiles produce true dot products: their max is
    // brought into raw units by R16 = 1 / (s_tQ s_tK) and their exponent multiplier is C R16.
    const float C = (*a.q_ts) * (*a.k_ts) * a.softmax_scale * kLog2e;
    const float R16 = 1.f / ((*a.q_ts) * (*a.k_ts));
    const float2 C2 = make_float2(C, C);
    unsigned char* sP = sm + L::OFF_P;
    const uint32_t tO = tbase + L::T_O + lane_addr;
    // A warp whose wait fails keeps walking the items without doing work (ok == false), so
    // that the two groups always meet at every item's named barrier.
    bool ok = true;
    bool prev_last_f16 = false;              // the previous item's last tile ran in FP16
    int g = 0;
    for (int it = 0;; ++it) {
      const int idx = fwd_item_index(it, G, cta);
      if (idx >= n_items) break;
      const FwdItem w = fwd_item(a, idx);
      const uint8_t* bm_row = kMixed ? a.bitmap + (static_cast<int64_t>(w.bhq) * a.Tq + w.qt) * a.Tk : nullptr;
      const int qi = w.qt * 128 + row;
      const int g0 = g;
      float m_last = -INFINITY;              // running max after this group's latest tile
      for (int j = (grp - g0) & 1; j < w.nt; j += 2) {
        if (!ok) continue;
        const int gg = g0 + j;
        const int b2 = gg & 1;               // == grp
        const int pb = gg % L::NP;           // P buffer
        const bool f16 = kMixed && bm_row[j];
        const bool prev_f16 = kMixed && (j >= 1 ? bm_row[j - 1] != 0 : prev_last_f16);
        float x[128];
        if (!waitw(s_full + b2, (gg >> 1) & 1, gg)) { ok = false; continue; }
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
        const int kbase = j * 128;
        if ((a.causal && kbase + 127 > qi) || (kbase + 128 > a.Nk)) {
          const int lim = min(a.Nk - 1, a.causal ? qi : a.Nk - 1) - kbase;   // last valid column
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] = (c <= lim) ? x[c] : -INFINITY;
        }
        float mt;
        float bm[4];                         // 32-key block maxima (underflow-aware variant)
        if constexpr (kUA) {
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            bm[b] = -INFINITY;
#pragma unroll
            for (int c = 0; c < 32; c += 2) bm[b] = fmax3(bm[b], x[32 * b + c], x[32 * b + c + 1]);
          }
          mt = fmaxf(fmaxf(bm[0], bm[1]), fmaxf(bm[2], bm[3]));
        } else {
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < 128; c += 8) {
#pragma unroll
            for (int u = 0; u < 4; ++u) m4[u] = fmax3(m4[u], x[c + 2 * u], x[c + 2 * u + 1]);
          }
          mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        }
        // An FP16 tile's scores are true dot products: its max is brought into raw units here
        // (exact: a positive factor commutes with the max) and its exponent takes the factor
        // in its multiplier, so both kinds of tile share one exponential loop.
        if (kMixed && f16) mt *= R16;
        // Running max before this tile: handed on by the group that processed tile gg - 1 of
        // the same item (the first tile of an item starts from -inf).
        float m_prev = -INFINITY;
        if (j >= 1) {
          if (!waitw(m_ready + ((gg - 1) & 1), ((gg - 1) >> 1) & 1, gg)) { ok = false; continue; }
          __syncwarp();
          m_prev = red_m[((gg - 1) & 1) * 128 + row];
        }
        const float m_new = fmaxf(m_prev, mt);
        m_last = m_new;
        red_m[b2 * 128 + row] = m_new;
        __syncwarp();
        if (lane == 0) mbar_arrive(m_ready + b2);
        const bool dead = (m_new == -INFINITY);
        const float bias = kLog2_448 - (dead ? 0.f : m_new) * C;
        const float2 B2 = make_float2(bias, bias);
        float2 Bb[4];                        // per-block bias (underflow-aware variant)
        uint32_t psf_word = 0u;
        if constexpr (kUA) {
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const float mu = (bm[b] - m_new) * C;       // log2 of the block's largest p~ (<= 0)
            const float e = (!dead && mu > -1.0e30f) ? fminf(fmaxf(ceilf(mu), -127.f), 0.f) : 0.f;
            Bb[b] = make_float2(bias - e, bias - e);
            psf_word |= static_cast<uint32_t>(127 + static_cast<int>(e)) << (8 * b);
          }
        }
        // P buffer pb was last used by PV(gg-NP), the last phase of its barrier that can have
        // completed. An FP16 tile's P fills both buffers (NP = 2 in that kernel): writing one
        // needs PV(gg-1) done as well, and the tile after an FP16 tile too. The waits come
        // before the exponentials so that P can be stored 16 bytes at a time as it is produced
        // (no register copy of the whole row).
        if (gg >= L::NP && !waitw(pv_done + pb, ((gg - L::NP) / L::NP) & 1, gg)) { ok = false; continue; }
        if ((f16 || prev_f16) && gg >= 1 &&
            !waitw(pv_done + (gg - 1) % L::NP, ((gg - 1) / L::NP) & 1, gg)) { ok = false; continue; }
        // All 128 exponentials first (in place), then the conversions and the stores: one long
        // run of independent special-function instructions (measured 1 % faster than converting
        // and storing chunk by chunk).
        const float Cs = (kMixed && f16) ? C * R16 : C;
        const float2 Ct = make_float2(Cs, Cs);
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          const float2 Bc = kUA ? Bb[c >> 5] : B2;
          const float2 t = __ffma2_rn(make_float2(x[c], x[c + 1]), Ct, Bc);
          x[c] = ex2_approx(t.x);
          x[c + 1] = ex2_approx(t.y);
        }
        if (!f16) {
          unsigned char* prow = sP + pb * 16384 + row * 128;
          if constexpr (kUA)
            *reinterpret_cast<uint32_t*>(sm + L::OFF_PSFU + b2 * 512 + (row & 31) * 16 + (row >> 5) * 4) = psf_word;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {               // 16 keys per 16-byte chunk
            uint32_t w4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int c = ch * 16 + q * 4;
              w4[q] = cvt_e4m3x2(x[c], x[c + 1]) | (cvt_e4m3x2(x[c + 2], x[c + 3]) << 16);
            }
            *reinterpret_cast<uint4*>(prow + ((ch ^ (row & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        } else if constexpr (kMixed) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            unsigned char* prow = sP + h * 16384 + row * 128;     // atom h = keys 64h .. 64h+63
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {             // 8 keys per 16-byte chunk
              uint32_t w4[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int c = h * 64 + ch * 8 + q * 2;
                const __half2 hv = __floats2half2_rn(x[c], x[c + 1]);
                w4[q] = *reinterpret_cast<const uint32_t*>(&hv);
              }
              *reinterpret_cast<uint4*>(prow + ((ch ^ (row & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
          }
        }
        fence_proxy_async_smem();
        // O holds the item's tiles before j relative to m(j-1) = m_prev. Rows whose max rose
        // at this tile are brought to m_new once PV(gg-1) is done; a warp whose rows all kept
        // their max hands P on at once. Of the 16 ones columns only column D (l) is read, so
        // only it is rescaled. All loads are issued before one wait.
        const float alpha = (m_prev == -INFINITY || dead) ? 1.f : ex2_approx((m_prev - m_new) * C);
        if (j >= 1 && !__all_sync(0xffffffffu, alpha == 1.f)) {
          if (!waitw(pv_done + (gg - 1) % L::NP, ((gg - 1) / L::NP) & 1, gg)) { ok = false; continue; }
          tc_fence_after();
          const float2 A2 = make_float2(alpha, alpha);
          uint32_t o[D], ol;
#pragma unroll
          for (int cc = 0; cc < D; cc += 32) tmem_ld32(tO + cc, o + cc);
          tmem_ld1(tO + D, &ol);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < D; k += 2) {
            const float2 u = __fmul2_rn(make_float2(__uint_as_float(o[k]), __uint_as_float(o[k + 1])), A2);
            o[k] = __float_as_uint(u.x);
            o[k + 1] = __float_as_uint(u.y);
          }
          ol = __float_as_uint(__uint_as_float(ol) * alpha);
#pragma unroll
          for (int cc = 0; cc < D; cc += 32) tmem_st32(tO + cc, o + cc);
          tmem_st1(tO + D, &ol);
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + pb);
      }
      g = g0 + w.nt;
      if constexpr (kMixed) prev_last_f16 = bm_row[w.nt - 1] != 0;
      // ---- epilogue of this item: O / l (O and l already relative to the final max) ----
      // PV of the item's last tile covers every earlier MMA of its issuing thread; the group
      // that owns that tile waits for it (the next phase of its own barrier) and publishes the
      // final max, and the named barrier passes both on to the other group.
      const int owner = (g - 1) & 1;
      if (ok && grp == owner) {
        ok = waitw(pv_done + (g - 1) % L::NP, ((g - 1) / L::NP) & 1, g - 1);
        red_fin[(it & 1) * 128 + row] = m_last;
      }
      tc_fence_before();
      named_bar_sync(1, 256);
      const bool live = ok && !*abort_flag;
      if (live) {
        tc_fence_after();
        uint32_t lr[16];
        tmem_ld16(tO + D, lr);
        tmem_wait_ld();
        const float m_run = red_fin[(it & 1) * 128 + row];
        const float l_run = __uint_as_float(lr[0]);
        const float inv_l = __frcp_rn(l_run);     // O / l by Markstein's division (ptx.cuh)
        const bool store = qi < a.Nq;
        const int64_t orow = static_cast<int64_t>(w.bhq) * a.Nq + qi;
        // O is written once: streaming (evict-first) stores keep K and V in L2
#pragma unroll
        for (int cc = 0; cc < D / 2; cc += 32) {
          const int c = grp * (D / 2) + cc;
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
        if (store && grp == 0 && a.lse != nullptr)
          a.lse[orow] = m_run * C * kLn2 + logf(l_run * (1.f / 448.f));
      }
      // O has been read (every tcgen05.ld above waited): the next item's first PV may
      // overwrite it.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
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
