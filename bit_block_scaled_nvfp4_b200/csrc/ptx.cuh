// Thin inline-PTX wrappers for sm_100a: mbarriers, TMA tensor loads, tcgen05 (TMEM
// allocation, block-scaled and f16 MMAs, TMEM loads/stores, shared->TMEM scale copies),
// proxy fences and format conversions. Every wait is bounded by the global timer and reports
// a timeout through the library status word instead of spinning forever.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

namespace qk4v8 {

// ---------------------------------------------------------------------------------------
// Status word (device global). Bits: 1 = wait timeout, 2 = bounds check failed.
// ---------------------------------------------------------------------------------------
__device__ unsigned int g_status = 0;
constexpr unsigned int kStatusTimeout = 1u;
constexpr unsigned int kStatusBounds = 2u;

__device__ __forceinline__ void flag_error(unsigned int bits) { atomicOr(&g_status, bits); }

// First wait that timed out since the last read: kernel id << 56 | role << 48 |
// barrier id << 40 | (tile & 0xFFFFF) << 20 | (blockIdx.x & 0xFFFFF). Zero when none.
__device__ unsigned long long g_timeout_site = 0;
enum : uint32_t { kKernelFwd = 1, kKernelDecode = 2, kKernelSelfTest = 3 };
enum : uint32_t { kRoleProducer = 0, kRoleMma = 1, kRoleSoftmax = 2 };
__device__ __forceinline__ uint64_t wait_site(uint32_t kernel, uint32_t role, uint32_t bar_id,
                                              int tile) {
  return (static_cast<uint64_t>(kernel) << 56) | (static_cast<uint64_t>(role) << 48) |
         (static_cast<uint64_t>(bar_id & 0xFF) << 40) |
         (static_cast<uint64_t>(static_cast<uint32_t>(tile) & 0xFFFFFu) << 20) |
         static_cast<uint64_t>(blockIdx.x & 0xFFFFFu);
}
__device__ __forceinline__ void record_timeout(uint64_t site) {
  atomicCAS(&g_timeout_site, 0ull, static_cast<unsigned long long>(site));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
               ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\t"
               "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity to complete. Returns false (and sets the
// timeout status bit) when the limit passes first. The limit is counted in SM clock cycles
// (about a second at the B200's clocks) and read only every 32 polls, so the poll loop itself
// stays short.
constexpr long long kWaitLimitCycles = 2000000000ll;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > kWaitLimitCycles) {
      flag_error(kStatusTimeout);
      return false;
    }
  }
}

// Wait that gives up when *flag is set, and sets *flag when it times out itself. `site`
// (wait_site()) is recorded when this wait is the first to time out. A phase that has
// already completed is taken on the first poll (the common case in a running pipeline);
// only then is the flag read, and again every 32 polls (try_wait itself suspends the thread
// for a short, hardware-chosen time while the phase is pending).
__device__ __forceinline__ bool bounded_wait_slow(uint64_t* bar, uint32_t parity, volatile int* flag,
                                               uint64_t site) {
  const long long t0 = clock64();
  while (!*flag) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > kWaitLimitCycles) {
      flag_error(kStatusTimeout);
      record_timeout(site);
      *flag = 1;
      return false;
    }
  }
  return false;
}
__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, volatile int* flag,
                                             uint64_t site) {
  if (mbar_try_wait(bar, parity)) return true;
  return bounded_wait_slow(bar, parity, flag, site);
}
// The same with every lane polling until the phase completes (no divergent slow path), for
// waits while a thread holds many live values: a lane-0-only slow path there leaves the
// register allocator without room when the warp's register count is set by setmaxnreg.
__device__ __forceinline__ bool bounded_wait_warp_all(uint64_t* bar, uint32_t parity,
                                                      volatile int* flag, uint64_t site) {
  if (__any_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  const long long t0 = clock64();
  while (true) {
    if (__any_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    if (__any_sync(0xffffffffu, *flag != 0)) return false;
    if (__any_sync(0xffffffffu, clock64() - t0 > kWaitLimitCycles)) {
      if ((threadIdx.x & 31) == 0) {
        flag_error(kStatusTimeout);
        record_timeout(site);
        *flag = 1;
      }
      __syncwarp();
      return false;
    }
  }
}
// The same for a whole (converged) warp: every lane polls once (one instruction, so every
// lane sees the same phase); a pending phase is then waited for by lane 0 alone and the
// outcome broadcast, so that every lane agrees.
__device__ __forceinline__ bool bounded_wait_warp(uint64_t* bar, uint32_t parity,
                                                  volatile int* flag, uint64_t site) {
  if (__any_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = bounded_wait_slow(bar, parity, flag, site) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// ---------------------------------------------------------------------------------------
// Fences
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// A warpgroup's register count moved from the launch's per-thread count kLaunch to N (once, by
// all four warps of the warpgroup, at the start of its role): .inc above it, .dec below it,
// nothing when equal (an .inc or .dec the other way round is not a valid instruction). The
// warpgroups' counts must not add up to more than the launch allocated, or an .inc waits for
// registers that never free.
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N, int kLaunch>
__device__ __forceinline__ void setmaxnreg_to() {
  static_assert(N % 8 == 0 && N >= 24 && N <= 256 && kLaunch % 8 == 0, "setmaxnreg count");
  if constexpr (N > kLaunch) setmaxnreg_inc<N>();
  else if constexpr (N < kLaunch) setmaxnreg_dec<N>();
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------------------
// TMA tensor loads (no multicast)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
        "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
        "r"(x), "r"(y), "r"(z) : "memory");
}
// The same loads with an L2 eviction-priority policy (the .L2::cache_hint operand).
__device__ __forceinline__ void tma_load_3d_hint(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int x, int y, int z, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
        "r"(x), "r"(y), "r"(z), "l"(policy) : "memory");
}
// L2 eviction priority "evict first" as a cache-policy word (the value CUTLASS's SM90/SM100
// TMA copies pass for it), for data that is read once: its lines leave L2 before any
// others, so operands that are read again (K and V of a head, re-read by every query tile)
// stay.
constexpr uint64_t kL2EvictFirst = 0x12F0000000000000ull;
// 4-byte asynchronous global -> shared copy (zero-filled when `valid` is false).
__device__ __forceinline__ void cp_async4(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 4 : 0) : "memory");
}
// Arrive on `bar` once every cp.async issued so far by this thread has landed. The arrival
// counts against the barrier's expected count (set at init).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// 1-D bulk global -> shared copy completing on an mbarrier (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------------------
// tcgen05: TMEM allocation
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(dst_smem)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// ---------------------------------------------------------------------------------------
// tcgen05: shared-memory matrix descriptor (K-major canonical layouts)
//   bits  0-13 start address >> 4     bits 16-29 leading byte offset >> 4
//   bits 32-45 stride byte offset >> 4 bits 46-47 version (1 on sm_100)
//   bits 49-51 base offset (0)        bit  52    LBO mode (0)
//   bits 61-63 layout: 0 none, 2 128B swizzle, 4 64B swizzle, 6 32B swizzle
// ---------------------------------------------------------------------------------------
constexpr uint32_t kSwNone = 0, kSw128 = 2, kSw64 = 4, kSw32 = 6;

__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo_bytes,
                                               uint32_t sbo_bytes, uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}

// ---------------------------------------------------------------------------------------
// tcgen05: instruction descriptors
// ---------------------------------------------------------------------------------------
// Block-scaled kinds (mxf4nvf4, mxf8f6f4): bits 4-5 B scale id, 7-9 A format, 10-12 B
// format, 15/16 A/B major (0 = K), 17-22 N>>3, 23 scale format (0 UE4M3, 1 UE8M0),
// 24-28 M>>4, 29-30 A scale id, 31 K size (0 = dense default).
__host__ __device__ constexpr uint32_t idesc_block_scaled(uint32_t a_fmt, uint32_t b_fmt,
                                                          uint32_t scale_ue8m0, int M, int N) {
  return (a_fmt << 7) | (b_fmt << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (scale_ue8m0 << 23) | (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ uint32_t idesc_with_sf_ids(uint32_t idesc, uint32_t a_id,
                                                      uint32_t b_id) {
  return idesc | ((b_id & 3u) << 4) | ((a_id & 3u) << 29);
}
// kind::f16: bits 4-5 D format (1 = F32), 7-9 A format (0 F16, 1 BF16), 10-12 B format,
// 15/16 majors, 17-22 N>>3, 24-28 M>>4.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool bf16 = false) {
  return (1u << 4) | (bf16 ? (1u << 7) | (1u << 10) : 0u) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}
constexpr uint32_t kFmtE2M1_mxf4 = 1;   // E2M1 in kind::mxf4nvf4
constexpr uint32_t kFmtE4M3 = 0;        // E4M3 in kind::mxf8f6f4

// ---------------------------------------------------------------------------------------
// tcgen05: MMAs (issued by one thread)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
        "r"(sfb_tmem) : "memory");
}
__device__ __forceinline__ void mma_mxf8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
        "r"(sfb_tmem) : "memory");
}
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}
// Arrive on an mbarrier when every tcgen05 operation issued so far by this thread is done.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
      ::"r"(smem_u32(bar)) : "memory");
}
// Copy a 32-row x 128-bit block (512 contiguous bytes) from shared memory into TMEM,
// replicated into all four 32-lane sub-partitions (the scale-factor layout of M/N = 128).
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, const void* smem_chunk) {
  const uint64_t d = make_sdesc(smem_u32(smem_chunk), 0, 128, kSwNone);
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d)
               : "memory");
}

// ---------------------------------------------------------------------------------------
// tcgen05: TMEM <-> registers (32 lanes x 32-bit pattern; each thread owns one lane)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_ld1(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r[0]) : "r"(taddr));
}
__device__ __forceinline__ void tmem_st1(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(r[0]) : "memory");
}
#define QK4V8_R8(b) "=r"(r[b+0]), "=r"(r[b+1]), "=r"(r[b+2]), "=r"(r[b+3]), \
                    "=r"(r[b+4]), "=r"(r[b+5]), "=r"(r[b+6]), "=r"(r[b+7])
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : QK4V8_R8(0), QK4V8_R8(8) : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : QK4V8_R8(0), QK4V8_R8(8), QK4V8_R8(16), QK4V8_R8(24) : "r"(taddr));
}
#undef QK4V8_R8
#define QK4V8_W8(b) "r"(r[b+0]), "r"(r[b+1]), "r"(r[b+2]), "r"(r[b+3]), \
                    "r"(r[b+4]), "r"(r[b+5]), "r"(r[b+6]), "r"(r[b+7])
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), QK4V8_W8(0), QK4V8_W8(8) : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), QK4V8_W8(0), QK4V8_W8(8), QK4V8_W8(16), QK4V8_W8(24) : "memory");
}
#undef QK4V8_W8
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------------------
// Conversions
// ---------------------------------------------------------------------------------------
// Two floats -> two E4M3 codes (round to nearest even, saturating to +-448).
// Result: low byte = code of `lo`, high byte = code of `hi`.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// Markstein's correctly rounded division (round to nearest): with y = RN(1/b) and
// q = RN(a y), which is within one ulp of a/b, the residual r = a - b q is exact as one FMA
// and RN(q + r y) is RN(a/b), provided nothing under- or overflows.
__device__ __forceinline__ float div_markstein(float a, float b, float y) {
  const float q = __fmul_rn(a, y);
  const float r = __fmaf_rn(-b, q, a);
  return __fmaf_rn(r, y, q);
}

// Two E4M3 codes (low byte, high byte) -> half2 (exact).
__device__ __forceinline__ __half2 e4m3x2_to_half2(uint32_t codes16) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(static_cast<uint16_t>(codes16)));
  return *reinterpret_cast<__half2*>(&r);
}
// Two floats -> two E2M1 codes packed in one byte (low nibble = `lo`), RNE, saturating.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// Maximum of three floats in one instruction (sm_100a three-input max).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Self-test of the bounded-wait path: one warp waits on a barrier that nothing arrives at.
// The wait gives up after its time limit, records its site and the timeout status, and the
// kernel returns normally.
__global__ void __launch_bounds__(32) wait_timeout_selftest_kernel() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  bounded_wait_warp(&bar, 0, &flag, wait_site(kKernelSelfTest, kRoleProducer, 0, 0));
}

}  // namespace qk4v8
