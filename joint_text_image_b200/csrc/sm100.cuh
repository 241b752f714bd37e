// sm100.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) features the
// attention kernels use: mbarriers with bounded waits, TMA tensor loads,
// tcgen05 (TMEM allocation, MMA, commit, loads/stores) and shared-memory
// matrix descriptors.  Nothing here is specific to attention.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

namespace hia {

// Status word values written by device code (match hia_status).
constexpr int kStatusTimeout = 4;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// try_wait with a suspend-time hint: the thread sleeps until the phase
// completes or about hint_ns pass, instead of returning at once.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Shared per-CTA abort flag + the device status word.  A wait that expires
// records the timeout, raises the CTA's abort flag and returns false; every
// other wait in the CTA then gives up at once, so the CTA drains and exits
// instead of hanging.
struct WaitCtx {
  volatile int* abort_flag;  // shared memory
  int* status;               // global status word
  uint64_t limit_ns;
};

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (*w.abort_flag) return false;
    if ((it & 63) == 0 && globaltimer_ns() - t0 > w.limit_ns) {
      *w.abort_flag = 1;
      atomicExch(w.status, kStatusTimeout);
      return false;
    }
  }
}

// A wait on work the hardware finishes by itself (TMA copies, MMAs already
// issued).  Ignores the abort flag; bounded by time only.
__device__ __forceinline__ bool mbar_wait_hw(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 63 && globaltimer_ns() - t0 > w.limit_ns) {
      atomicExch(w.status, kStatusTimeout);
      return false;
    }
  }
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0, int c1,
                                            int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_u32(bar))
      : "memory");
}
// Untiled bulk copy global -> shared (16-byte aligned addresses, size % 16 == 0).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Make generic-proxy shared-memory writes visible to the async proxy (tensor core / TMA).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on `bar` once every tcgen05 op issued so far by this thread completes.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T  (kind::f16, operands described by descriptors)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]  (A: M rows in lanes, K packed along columns)
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets columns
// [col, col+32) of lane (lane_base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// tcgen05.ld writes its destination registers asynchronously: they hold the
// loaded values only after tcgen05.wait::ld.  To the compiler they are defined
// by the load statement itself, so it could schedule a use of them before the
// wait.  reg_fence (an empty statement that reads and rewrites the registers,
// ordered after the wait like every volatile asm) pins every later use after
// the wait; tmem_ld_wait_regs is the wait followed by that fence.
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[N]) {
  static_assert(N % 8 == 0, "whole groups of 8 registers");
#pragma unroll
  for (int i = 0; i < N; i += 8)
    asm volatile("" : "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]), "+r"(r[i + 5]),
                 "+r"(r[i + 6]), "+r"(r[i + 7]));
}
template <class... R>
__device__ __forceinline__ void tmem_ld_wait_regs(R&... regs) {
  tmem_ld_wait();
  (reg_fence(regs), ...);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator.
//   bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16), 10-12 B format
//   (1 = bf16), 15 A major (0 = K, 1 = MN), 16 B major, 17-22 N >> 3,
//   24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(a_mn_major) << 15) | (uint32_t(b_mn_major) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Shared-memory matrix descriptor with 128-byte swizzle (sm_100 version 1).
//   bits 0-13 start >> 4, 16-29 LBO >> 4, 32-45 SBO >> 4, 46-47 version = 1,
//   61-63 layout (2 = SWIZZLE_128B).
// K-major operand (rows x 64 bf16 per 128-byte row, 8-row atoms of 1 KB):
//   LBO unused (1), SBO = 1024.  MN-major operand: 64 MN-contiguous elements
//   per 128-byte row, K rows 128 B apart, LBO = byte distance between 64-wide
//   MN blocks, SBO = byte distance between 8-row K groups.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Issue a chain of kind::f16 MMAs whose descriptors are `base + offset`
// (offsets in 16-byte units, compile-time constants).  All descriptors are
// formed before the first MMA so the single issuing thread never waits on
// address arithmetic between MMAs (that dependency chain, not the tensor
// core, bounded the issue rate to ~100 clocks per MMA).
template <int NK>
__device__ __forceinline__ void mma_chain_ss(uint32_t d, uint64_t abase, const uint32_t (&aoff)[NK], uint64_t bbase,
                                             const uint32_t (&boff)[NK], uint32_t idesc, uint32_t acc_first) {
  uint64_t a[NK], b[NK];
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    a[i] = abase + aoff[i];
    b[i] = bbase + boff[i];
  }
#pragma unroll
  for (int i = 0; i < NK; ++i) mma_ss(d, a[i], b[i], idesc, i == 0 ? acc_first : 1u);
}
template <int NK>
__device__ __forceinline__ void mma_chain_ts(uint32_t d, uint32_t a_tmem, uint32_t a_step, uint64_t bbase,
                                             const uint32_t (&boff)[NK], uint32_t idesc, uint32_t acc_first) {
  uint64_t b[NK];
  uint32_t a[NK];
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    b[i] = bbase + boff[i];
    a[i] = a_tmem + uint32_t(i) * a_step;
  }
#pragma unroll
  for (int i = 0; i < NK; ++i) mma_ts(d, a[i], b[i], idesc, i == 0 ? acc_first : 1u);
}
// Warp-converged forms: the whole warp runs the surrounding code (so the
// descriptors live in uniform registers) and one elected lane issues.
__device__ __forceinline__ bool elect_one() {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "elect.sync _|P, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(r));
  return r != 0;
}
template <int NK>
__device__ __forceinline__ void mma_chain_ss_w(uint32_t d, uint64_t abase, const uint32_t (&aoff)[NK], uint64_t bbase,
                                               const uint32_t (&boff)[NK], uint32_t idesc, uint32_t acc_first) {
  uint64_t a[NK], b[NK];
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    a[i] = abase + aoff[i];
    b[i] = bbase + boff[i];
  }
  if (elect_one()) {
#pragma unroll
    for (int i = 0; i < NK; ++i) mma_ss(d, a[i], b[i], idesc, i == 0 ? acc_first : 1u);
  }
  __syncwarp();
}
template <int NK>
__device__ __forceinline__ void mma_chain_ts_w(uint32_t d, uint32_t a_tmem, uint32_t a_step, uint64_t bbase,
                                               const uint32_t (&boff)[NK], uint32_t idesc, uint32_t acc_first) {
  uint64_t b[NK];
  uint32_t a[NK];
#pragma unroll
  for (int i = 0; i < NK; ++i) {
    b[i] = bbase + boff[i];
    a[i] = a_tmem + uint32_t(i) * a_step;
  }
  if (elect_one()) {
#pragma unroll
    for (int i = 0; i < NK; ++i) mma_ts(d, a[i], b[i], idesc, i == 0 ? acc_first : 1u);
  }
  __syncwarp();
}
__device__ __forceinline__ void tc_commit_w(uint64_t* bar) {
  if (elect_one()) tc_commit(bar);
  __syncwarp();
}
// Offsets (16-byte units) of the K-steps of a K-major SW128 operand whose
// 64-wide K blocks are `block_bytes` apart: 32 bytes per 16-element step.
template <int NK>
struct KMajorSteps {
  uint32_t v[NK];
  __host__ __device__ constexpr KMajorSteps(uint32_t block_bytes) : v{} {
    for (int i = 0; i < NK; ++i) v[i] = (uint32_t(i >> 2) * block_bytes + uint32_t(i & 3) * 32u) >> 4;
  }
};
// Offsets of the K-steps of an MN-major SW128 operand: 16 K rows (2 KB) per step.
template <int NK>
struct MNMajorSteps {
  uint32_t v[NK];
  __host__ __device__ constexpr MNMajorSteps() : v{} {
    for (int i = 0; i < NK; ++i) v[i] = uint32_t(i) * (2048u >> 4);
  }
};

// ---------------------------------------------------------------- math
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 2^x for a pair of values on the FMA/ALU pipes (packed f32x2 arithmetic),
// for x <= 64: Cody-Waite split x = j + f with j = floor(x), f in [0, 1); 2^f
// from a cubic whose coefficients were fitted here to minimise the relative
// error on [0, 1) (max relative error 7.5e-5, well inside the bf16 rounding of
// P); 2^j is added to the exponent field.  Inputs are clamped at -125 (the
// cubic dips just below 1 at f = 0, so the exponent field must stay >= 2):
// x <= -125, -inf included, gives about 2^-125 = 2.4e-38 instead of 0, which
// is below anything a softmax row with a visible key can resolve.  Used for
// part of the softmax exponentials so that the MUFU unit (ex2.approx) is not
// the only source of exp2.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23: floor(x) lands in the low mantissa bits
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = __fadd2_rd(x, make_float2(kShift, kShift));
  const float2 j = __fadd2_rn(t, make_float2(-kShift, -kShift));  // floor(x), exact
  const float2 f = __ffma2_rn(j, make_float2(-1.0f, -1.0f), x);     // x - floor(x), exact
  float2 p = __ffma2_rn(make_float2(0x1.3f95cap-4f, 0x1.3f95cap-4f), f, make_float2(0x1.cefc18p-3f, 0x1.cefc18p-3f));
  p = __ffma2_rn(p, f, make_float2(0x1.64446cp-1f, 0x1.64446cp-1f));
  p = __ffma2_rn(p, f, make_float2(0x1.fff62cp-1f, 0x1.fff62cp-1f));
  // t's low mantissa bits hold floor(x) + 2^22; shifted left by 23 only the
  // low 9 bits of floor(x) survive: floor(x) << 23 modulo 2^32, the exponent step.
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// max of three (a NaN operand is ignored, as in fmaxf)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a
// 128-byte-swizzled tile whose rows are 128 bytes (1 KB atoms of 8 rows).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

}  // namespace hia

namespace hia {

// ---------------------------------------------------------------- bulk reduce
// global[dst .. dst+bytes) += shared[src ..] (fp32 add performed in L2).
__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the shared-memory sources of all but the newest N groups have been read.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until all but the newest N groups have completed (writes performed).
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// Named barrier over `count` threads (ids 1..15; 0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Per-warpgroup register budget (all four warps of a warpgroup execute it).
template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

}  // namespace hia
