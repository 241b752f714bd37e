// attn_bwd.cu -- recompute backward of the generalized-causal GQA attention.
//
// With P = softmax(scale * Qr Kr^T) over the visible pairs (the forward of
// HunyuanImage3Attention under build_joint_attention_mask), dO the incoming
// gradient and delta_q = dO_q . O_q:
//   dV  = P^T dO,   dP = dO V^T,   dS = P o (dP - delta),
//   dKr = scale dS^T Qr,   dQr = scale dS Kr,
// summed over the g query heads of each kv head; dK, dQ = R^T dKr, R^T dQr.
//
// bwd_pre: delta and LSE * log2(e) per row, padded to a multiple of 64 rows;
// it also zeroes the dQ accumulator and the split schedule's tickets.
// attn_bwd: one CTA per work-list entry and kv head: a (b, 128-key tile) over
// the query tiles that see its keys (a range of query tiles, since the row
// bound e(q) is non-decreasing), or, in a split schedule, one of the 2-4
// consecutive parts of that range for the longest tiles (the parts' fp32
// dK/dV are added in part order by the part that finishes last).  It keeps
// Kr and V in shared memory and dK, dV in TMEM, and walks the g heads x its
// query tiles.  Per query tile, with keys on the MMA M side:
//   S^T = Kr Qr^T, dP^T = V dO^T      (SS MMAs, M=128, N=64)
//   P^T = exp2(S^T * scale*log2e - lse2), dS^T = P^T o (dP^T - delta)
//   dV += P^T dO,  dK += dS^T Qr       (A = P^T / dS^T straight from TMEM)
//   dQ^T = Kr^T dS^T                   (A = Kr read as MN-major, B = dS^T in
//                                       shared memory)
// and dQ^T goes TMEM -> registers -> shared memory -> one bulk fp32
// reduce-add into the dq accumulator (the reduction runs in L2).
// Warps (512 threads): 0 TMA producer, 1 TMEM owner + S^T/dP^T MMA issuer,
// 2 dV/dK/dQ^T MMA issuer, 4-7 and
// 8-11 two softmax warpgroups that share every query tile, one half of its
// 64 query columns each (one key row per thread; then the dK and dV
// epilogues), 12-15 dQ writers (one head-dim lane per thread).  setmaxnreg moves registers from the producer/MMA and dQ
// warpgroups to the softmax warpgroups: 128*64 + 256*176 + 128*96 = 65536 = 512*128.
// P^T and dS^T become visible to the second MMA warp together (one barrier
// per tile).  TMEM: S^T[2] at 0/64, dP^T[2] at 128/192 (P^T, dS^T written over them as
// packed bf16, each column half inside the columns it was computed from), dV at 256, dK at 256 + D; dQ^T of buffer i is written over
// dP^T[i] after the dK MMA that read dS^T from there (MMAs run in issue
// order), so the next S^T never waits for the dQ writers.
#include <cuda.h>
#include <cuda_bf16.h>

#include "devctx.h"
#include "kernels.h"
#include "sm100.cuh"

namespace hia {
namespace {

constexpr int kThreads = 512;
constexpr int kLaunchRegs = 128;  // the setmaxnreg split below assumes 512 x 128 at launch
constexpr int kStages = 3;
constexpr int kFmaExpPairs = 4;  // of every 16 column pairs of P^T, this many use exp2_fma2
constexpr int BK = kBwdBK;  // 128 keys
constexpr int BQ = kBwdBQ;  // 64 query rows

template <int D>
struct BwdSmem {
  alignas(1024) __nv_bfloat16 k[BK * D];
  alignas(1024) __nv_bfloat16 v[BK * D];
  alignas(1024) __nv_bfloat16 q[kStages][BQ * D];
  alignas(1024) __nv_bfloat16 dout[kStages][BQ * D];
  alignas(1024) __nv_bfloat16 ds[2][BK * BQ];  // dS^T rows = keys, 64 q per 128-byte row
  alignas(1024) float dq[2][(BQ / 2) * D];     // half query tile of dQ, fp32 [32 q][D]
  alignas(16) float lse2[kStages][BQ];
  alignas(16) float delta[kStages][BQ];
  uint64_t bar_kv;
  uint64_t bar_full[kStages];
  uint64_t bar_empty[kStages];
  uint64_t bar_s_full[2];
  uint64_t bar_dp_full[2];
  uint64_t bar_ds_ready[2];
  uint64_t bar_dq_full[2];
  uint64_t bar_dq_empty[2];
  uint64_t bar_s_free[2];
  uint64_t bar_final;
  uint32_t tmem_base;
  int abort_flag;
  int split_ticket;  // split schedule: this half's ticket (0 first, 1 second to finish)
};

// S^T = Kr Qr^T and dP^T = V dO^T: A = 128-row tile (K-major, 64-wide D
// blocks 16 KB apart), B = 64-row tile (K-major, D blocks 8 KB apart); N = 64.
template <int D>
__device__ __forceinline__ void issue_kq(uint32_t d, uint64_t adesc, uint64_t bdesc) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, BQ, 0, 0);
  constexpr KMajorSteps<D / 16> sa(16384), sb(8192);
  mma_chain_ss_w<D / 16>(d, adesc, sa.v, bdesc, sb.v, idesc, 0u);
}

// dV += P^T dO or dK += dS^T Qr: A from TMEM (128 keys x 64 q, packed bf16:
// query rows 0-31 in columns [0, 16) of the buffer, rows 32-63 in [48, 64),
// each half where the softmax warpgroup of that half wrote it), B = 64-row
// tile read MN-major (N = D contiguous, D blocks 8 KB apart).
template <int D>
__device__ __forceinline__ void issue_acc(uint32_t d, uint32_t a_tmem, uint64_t bdesc, bool acc) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, 0, 1);
  constexpr MNMajorSteps<BQ / 16> st;
  static_assert(BQ == 64, "two 32-row query halves of two 16-row K-steps each");
  constexpr uint32_t aoff[4] = {0u, 8u, 48u, 56u};
  uint64_t bd[4];
  uint32_t ad[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    bd[i] = bdesc + st.v[i];
    ad[i] = a_tmem + aoff[i];
  }
  if (elect_one()) {
#pragma unroll
    for (int i = 0; i < 4; ++i) mma_ts(d, ad[i], bd[i], idesc, i == 0 ? (acc ? 1u : 0u) : 1u);
  }
  __syncwarp();
}

// dQ^T = Kr^T dS^T: M = 128 (head dims; for D = 64 the second 64-row block
// reads the V tile and its result lanes are ignored), N = 64 q, K = 128 keys.
// A = Kr tile read MN-major, B = dS^T tile read MN-major.
__device__ __forceinline__ void issue_dq(uint32_t d, uint64_t kt_mn_desc, uint64_t ds_desc) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, BQ, 1, 1);
  constexpr MNMajorSteps<BK / 16> st;
  mma_chain_ss_w<BK / 16>(d, kt_mn_desc, st.v, ds_desc, st.v, idesc, 0u);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  BwdSmem<D>& sm =
      *reinterpret_cast<BwdSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int bid = blockIdx.x;
  const int hkv = bid % p.Hkv;
  bid /= p.Hkv;
  // work entry: this CTA's query tiles [qt_first, qt_end) of kv tile kt (all
  // that see it, or part `part` of `parts` consecutive sub-ranges when split:
  // slot >= 0)
  const int32_t* we = p.work + kBwdWorkInts * bid;
  const int b = we[0], kt = we[1], qt_first = we[2], qt_end = we[3], slot = we[4], part = we[5], parts = we[6];
  // [full_first, full_end): the query tiles that see all of the kv tile
  const int32_t* te = p.tiles + 4 * (b * p.bKT + kt);
  const int full_first = te[2], full_end = te[3];
  const SampleDev smp = p.samples[b];
  const int n_qt = max(qt_end - qt_first, 0);
  const int n_it = n_qt * p.g;  // iteration i: head hkv*g + i / n_qt, query tile qt_first + i % n_qt

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_kv, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.bar_full[i], 1);
      mbar_init(&sm.bar_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.bar_s_full[i], 1);
      mbar_init(&sm.bar_dp_full[i], 1);
      mbar_init(&sm.bar_ds_ready[i], 8);   // one arrival per softmax warp (both warpgroups)
      mbar_init(&sm.bar_dq_full[i], 1);
      mbar_init(&sm.bar_dq_empty[i], 4);   // one arrival per dQ warp
      mbar_init(&sm.bar_s_free[i], 1);
    }
    mbar_init(&sm.bar_final, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtx wc{&sm.abort_flag, p.status, p.timeout_ns};
  // buffer i of S^T / dP^T as arithmetic (a runtime-indexed array would live in local memory)
  const auto tS = [tmem](int i) { return tmem + uint32_t(i) * 64u; };
  const auto tdP = [tmem](int i) { return tmem + 128u + uint32_t(i) * 64u; };
  const uint32_t tdV = tmem + 256, tdK = tmem + 256 + D;

  if (warp < 4) {
   regs_dec<64>();
   if (warp == 0) {
    // =============================== TMA producer
    if (lane == 0 && n_it > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      constexpr uint32_t kv_bytes = BK * D * 2, qd_bytes = BQ * D * 2;
      mbar_arrive_expect_tx(&sm.bar_kv, 2 * kv_bytes);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(&sm.k[c * BK * 64], &tm_k, &sm.bar_kv, c * 64, kt * BK, b * p.Hkv + hkv);
        tma_load_4d(&sm.v[c * BK * 64], &tm_v, &sm.bar_kv, c * 64, hkv, smp.off + kt * BK, p.packed ? 0 : b);
      }
      int issued = 0;
      for (int i = 0; i < n_it; ++i) {
        const int s = i % kStages, n = i / kStages;
        if (i >= kStages && !mbar_wait(&sm.bar_empty[s], (n - 1) & 1, wc)) break;
        const int hi = i / n_qt, qt = qt_first + i % n_qt;
        const int h = hkv * p.g + hi;
        mbar_arrive_expect_tx(&sm.bar_full[s], 2 * qd_bytes + 2 * BQ * 4);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(&sm.q[s][c * BQ * 64], &tm_q, &sm.bar_full[s], c * 64, qt * BQ, b * p.Hq + h);
          tma_load_5d(&sm.dout[s][c * BQ * 64], &tm_do, &sm.bar_full[s], c * 64, hi, hkv, smp.off + qt * BQ,
                      p.packed ? 0 : b);
        }
        const int64_t row = (int64_t(b) * p.Hq + h) * p.S_pad + int64_t(qt) * BQ;
        bulk_load(sm.lse2[s], p.lse2 + row, BQ * 4, &sm.bar_full[s]);
        bulk_load(sm.delta[s], p.delta + row, BQ * 4, &sm.bar_full[s]);
        issued = i + 1;
      }
      mbar_wait_hw(&sm.bar_kv, 0, wc);
      for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
        mbar_wait_hw(&sm.bar_full[i % kStages], (i / kStages) & 1, wc);
    }
  } else if (warp == 1 || warp == 2) {
    // =============================== MMA issuers
    // Two warps issue MMAs: a wait or fence in an issuing thread lets its
    // own short MMA queue drain, and the other thread's MMAs keep the tensor
    // core busy meanwhile.  Warp 1 issues S^T and dP^T (running up to two
    // query tiles ahead), warp 2 the dV, dK and dQ^T MMAs of each tile.  Each
    // issuing warp runs its loop converged (waits combined with __all_sync)
    // and one elected lane issues, so the descriptors are warp-uniform.
    if (n_it > 0) {
      constexpr uint32_t kQStep = (BQ * D * 2u) >> 4, kDsStep = (BK * BQ * 2u) >> 4;
      bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.bar_kv, 0, wc));
      if (warp == 1) {
        const uint64_t k_km = sdesc_sw128(smem_u32(sm.k), 16, 1024);
        const uint64_t v_km = sdesc_sw128(smem_u32(sm.v), 16, 1024);
        const uint64_t q_km = sdesc_sw128(smem_u32(sm.q[0]), 16, 1024);
        const uint64_t o_km = sdesc_sw128(smem_u32(sm.dout[0]), 16, 1024);
        for (int i = 0; ok && i < n_it; ++i) {
          const int b = i & 1, s = i % kStages;
          // S^T(i) reuses the buffer whose P^T(i-2) the dV MMA read; dP^T(i)
          // the buffer the dQ writers read dQ^T(i-2) from.
          if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_full[s], (i / kStages) & 1, wc))) { ok = false; break; }
          if (i >= 2 && !__all_sync(0xffffffffu, mbar_wait(&sm.bar_s_free[b], ((i >> 1) - 1) & 1, wc))) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_kq<D>(tS(b), k_km, q_km + uint32_t(s) * kQStep);
          tc_commit_w(&sm.bar_s_full[b]);
          if (i >= 2) {
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_dq_empty[b], ((i >> 1) - 1) & 1, wc))) {
              ok = false;
              break;
            }
            tc_fence_after();  // TMEM reuse after the dQ writers' loads
          }
          issue_kq<D>(tdP(b), v_km, o_km + uint32_t(s) * kQStep);
          tc_commit_w(&sm.bar_dp_full[b]);
        }
      } else {
        const uint64_t k_mn = sdesc_sw128(smem_u32(sm.k), D == 128 ? 16384u : smem_u32(sm.v) - smem_u32(sm.k), 1024);
        const uint64_t q_mn = sdesc_sw128(smem_u32(sm.q[0]), 8192, 1024);
        const uint64_t o_mn = sdesc_sw128(smem_u32(sm.dout[0]), 8192, 1024);
        const uint64_t ds_mn = sdesc_sw128(smem_u32(sm.ds[0]), 8192, 1024);
        for (int i = 0; ok && i < n_it; ++i) {
          const int b = i & 1, s = i % kStages;
          // P^T(i) and dS^T(i) are in TMEM and dS^T(i) in shared memory
          if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_ds_ready[b], (i >> 1) & 1, wc))) { ok = false; break; }
          tc_fence_after();
          issue_acc<D>(tdV, tS(b), o_mn + uint32_t(s) * kQStep, i > 0);
          tc_commit_w(&sm.bar_s_free[b]);
          issue_acc<D>(tdK, tdP(b), q_mn + uint32_t(s) * kQStep, i > 0);
          tc_commit_w(&sm.bar_empty[s]);  // the stage's Q and dO are no longer read
          issue_dq(tdP(b), k_mn, ds_mn + uint32_t(b) * kDsStep);  // over dS^T, after the dK MMA read it
          tc_commit_w(&sm.bar_dq_full[b]);
        }
        tc_commit_w(&sm.bar_final);
        mbar_wait_hw(&sm.bar_final, 0, wc);
      }
    }
   }
  } else if (warp < 12) {
    regs_inc<176>();
    // =============================== softmax: one key row per thread
    // Both warpgroups work on every query tile, each on one half of its 64
    // query columns (hq = 0: rows 0-31, hq = 1: rows 32-63), so a tile's P^T
    // and dS^T are ready in half the time.  Each half writes its packed bf16
    // P^T / dS^T inside the TMEM columns it has just read (columns [0, 16) or
    // [48, 64) of the buffer), never over the other half's scores.
    const int bf = (warp - 4) >> 2;  // warpgroup: query-column half here, dK / dV in the epilogue
    const int hq = bf;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int key = kt * BK + r;
    // this key is visible exactly to the query rows [vis_lo, vis_hi)
    const ImageDev* im = p.images + smp.img0;
    const int vis_lo = first_row(im, smp.n_img, smp.L, key);
    const int vis_hi = min(int(smp.rows), hidden_from(im, smp.n_img, key));
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const float cs = p.scale_log2;
    bool ok = true;
    for (int i = 0; i < n_it; ++i) {
      const int b = i & 1, s = i % kStages;
      const int qt = qt_first + i % n_qt;
      const bool partial = qt < full_first || qt >= full_end || (qt + 1) * BQ > smp.rows;
      // the stage's lse2/delta were written by TMA: acquire them through its barrier
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.bar_full[s], (i / kStages) & 1, wc) &&
                                       mbar_wait(&sm.bar_s_full[b], (i >> 1) & 1, wc));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld32(tS(b) + lane_off + uint32_t(hq * 32), sr);
      tmem_ld_wait_regs(sr);
      float pv[32];
      const float4* l2 = reinterpret_cast<const float4*>(sm.lse2[s]) + hq * 8;
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4) {
        const float4 l = l2[c4];
        // scale and subtract as packed f32x2 (two columns per instruction)
        const float2 xa = __ffma2_rn(make_float2(__uint_as_float(sr[4 * c4 + 0]), __uint_as_float(sr[4 * c4 + 1])),
                                     make_float2(cs, cs), make_float2(-l.x, -l.y));
        const float2 xb = __ffma2_rn(make_float2(__uint_as_float(sr[4 * c4 + 2]), __uint_as_float(sr[4 * c4 + 3])),
                                     make_float2(cs, cs), make_float2(-l.z, -l.w));
        // kFmaExpPairs of every 16 column pairs take exp2 on the FMA pipe (both
        // warpgroups share the MUFU unit on the same tile); masked columns are
        // zeroed below, whatever the emulation returned for them
        const float2 pa = ((2 * c4) % 16 < kFmaExpPairs) ? exp2_fma2(xa)
                                                         : make_float2(ex2_approx(xa.x), ex2_approx(xa.y));
        const float2 pb = ((2 * c4 + 1) % 16 < kFmaExpPairs) ? exp2_fma2(xb)
                                                             : make_float2(ex2_approx(xb.x), ex2_approx(xb.y));
        pv[4 * c4 + 0] = pa.x;
        pv[4 * c4 + 1] = pa.y;
        pv[4 * c4 + 2] = pb.x;
        pv[4 * c4 + 3] = pb.y;
      }
      if (partial) {
        const int q0 = qt * BQ + hq * 32;
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (q0 + c < vis_lo || q0 + c >= vis_hi) pv[c] = 0.f;
      }
      __syncwarp();  // converged before the warp-collective TMEM store
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(pv[2 * c], pv[2 * c + 1]);
      tmem_st16(tS(b) + lane_off + uint32_t(hq * 48), pk);

      ok = __all_sync(0xffffffffu, mbar_wait(&sm.bar_dp_full[b], (i >> 1) & 1, wc));
      if (!ok) break;
      tc_fence_after();
      tmem_ld32(tdP(b) + lane_off + uint32_t(hq * 32), sr);
      tmem_ld_wait_regs(sr);
      const float4* dl = reinterpret_cast<const float4*>(sm.delta[s]) + hq * 8;
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4) {
        const float4 d = dl[c4];
        pk[2 * c4] = pack_bf16x2(pv[4 * c4 + 0] * (__uint_as_float(sr[4 * c4 + 0]) - d.x),
                                 pv[4 * c4 + 1] * (__uint_as_float(sr[4 * c4 + 1]) - d.y));
        pk[2 * c4 + 1] = pack_bf16x2(pv[4 * c4 + 2] * (__uint_as_float(sr[4 * c4 + 2]) - d.z),
                                     pv[4 * c4 + 3] * (__uint_as_float(sr[4 * c4 + 3]) - d.w));
      }
      tmem_st16(tdP(b) + lane_off + uint32_t(hq * 48), pk);
      // dS^T row half -> shared memory: 16-byte chunks hq*4 .. hq*4+3 of the
      // 128-byte swizzled row of 64 query values
      uint8_t* dsrow = reinterpret_cast<uint8_t*>(sm.ds[b]);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(dsrow + sw128_offset(uint32_t(r), uint32_t(hq * 4 + c))) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();  // the warp's TMEM and shared-memory writes are done; one lane signals for it
      if (lane == 0) mbar_arrive(&sm.bar_ds_ready[b]);
    }
    // ---- epilogue: warpgroup 0 writes dK = R^T (scale dKr), warpgroup 1 dV
    bool have = n_it > 0 && ok;
    if (have) have = __all_sync(0xffffffffu, mbar_wait(&sm.bar_final, 0, wc));
    if (have) tc_fence_after();
    bool write_out = true;  // false: another part of a split kv tile writes dK/dV
    if (slot >= 0) {
      // Split kv tile: this CTA saw one of its `parts` query sub-ranges.
      // Every part writes its raw fp32 accumulator rows (dK in warpgroup 0,
      // dV in warpgroup 1) to its own partial, fences, and takes a ticket;
      // the part that finishes last adds all the partials in part order
      // (P_0 + P_1 + ..., its own from TMEM: the same bits whichever part is
      // last) into its TMEM and runs the common epilogue below.  No thread
      // waits on another CTA.
      const uint32_t tacc = (bf == 0 ? tdK : tdV) + lane_off;
      const int64_t unit = int64_t(slot) * p.Hkv + hkv;
      // a partial is BK x D fp32 stored as [D / 4][BK] float4: row r's float4
      // number q at q * BK + r, so a warp's 32 rows are 512 contiguous bytes
      const auto partial = [&](int j) {
        return reinterpret_cast<float4*>(p.part + ((unit * parts + j) * 2 + bf) * int64_t(BK * D)) + r;
      };
      float4* mine = partial(part);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        if (have) {
          tmem_ld32(tacc + uint32_t(c * 32), v);
          tmem_ld_wait_regs(v);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        }
        float4* d4 = mine + c * 8 * BK;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          d4[i * BK] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]), __uint_as_float(v[4 * i + 2]),
                              __uint_as_float(v[4 * i + 3]));
      }
      __threadfence();
      named_bar_sync(2, 256);  // both epilogue warpgroups' partial rows written and fenced
      if (threadIdx.x == 128) sm.split_ticket = atomicAdd(&p.part_cnt[unit], 1);
      named_bar_sync(2, 256);
      if (sm.split_ticket < parts - 1) {
        have = false;  // a later part finishes this kv tile
        write_out = false;
      } else {
        __threadfence();
      }
      if (have) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tacc + uint32_t(c * 32), v);
          tmem_ld_wait_regs(v);
          float sum[32];
#pragma unroll 1
          for (int j = 0; j < parts; ++j) {
            float x[32];
            if (j == part) {
#pragma unroll
              for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(v[i]);
            } else {
              const float4* o4 = partial(j) + c * 8 * BK;
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float4 a = __ldcg(o4 + i * BK);
                x[4 * i] = a.x;
                x[4 * i + 1] = a.y;
                x[4 * i + 2] = a.z;
                x[4 * i + 3] = a.w;
              }
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) sum[i] = j == 0 ? x[i] : sum[i] + x[i];
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(sum[i]);
          tmem_st32(tacc + uint32_t(c * 32), v);
        }
        tmem_st_wait();
      }
      if (write_out && threadIdx.x == 128) p.part_cnt[unit] = 0;  // ready for the next launch
    }
    const bool store = write_out && key < smp.rows;
    // dK / dV rows leave through shared memory: each thread stages its key
    // row's 16-byte chunks, XOR-swizzled by row so that a warp's 32 row writes
    // spread over the banks, then each warp writes its own 32 rows whole
    // (CPR lanes per row, 16 bytes each: coalesced 128-bit stores).
    constexpr int CPR = D / 8;  // 16-byte chunks per bf16 row
    const auto stage_chunk = [](uint8_t* tile, int row, int ch, uint4 v) {
      *reinterpret_cast<uint4*>(tile + row * (D * 2) + ((ch ^ (row & (CPR - 1))) * 16)) = v;
    };
    // rows of D * 2 bytes: a bf16 row, or half of an fp32 row; destination row
    // row0 + r of `base` (row_bytes apart) gets tile row r
    const auto store_rows = [&](const uint8_t* tile, uint8_t* base, int64_t row0, int64_t row_bytes) {
      constexpr int RPI = 32 / CPR;  // rows per warp store
      const int ch = lane % CPR;
#pragma unroll 4
      for (int rr = 0; rr < 32; rr += RPI) {
        const int row = quarter * 32 + rr + lane / CPR;
        if (write_out && kt * BK + row < smp.rows) {
          const uint4 v = *reinterpret_cast<const uint4*>(tile + row * (D * 2) + ((ch ^ (row & (CPR - 1))) * 16));
          *reinterpret_cast<uint4*>(base + (row0 + row) * row_bytes + ch * 16) = v;
        }
      }
    };
    if (bf == 0 && p.dk_acc) {
      // QK RMSNorm: the norm's backward needs the whole row, so write
      // scale * dK_n (gradient w.r.t. the normed rotated key row) in fp32 and
      // let the gradient epilogue kernel finish it
      // fp32 rows of D * 4 bytes, staged half a row (D * 2 bytes) at a time
      uint8_t* tile = reinterpret_cast<uint8_t*>(sm.k);  // K is no longer read: every MMA has finished
      uint8_t* abase = reinterpret_cast<uint8_t*>(p.dk_acc + (int64_t(b) * p.Hkv + hkv) * p.S_pad * D);
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          uint32_t ov[32];
          if (have) {
            tmem_ld32(tdK + lane_off + half * (D / 2) + c * 32, ov);
            tmem_ld_wait_regs(ov);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] = 0u;
          }
          if (store) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              stage_chunk(tile, r, c * 8 + i,
                          make_uint4(__float_as_uint(__uint_as_float(ov[4 * i]) * p.scale),
                                     __float_as_uint(__uint_as_float(ov[4 * i + 1]) * p.scale),
                                     __float_as_uint(__uint_as_float(ov[4 * i + 2]) * p.scale),
                                     __float_as_uint(__uint_as_float(ov[4 * i + 3]) * p.scale)));
          }
        }
        __syncwarp();
        store_rows(tile, abase + half * (D / 2) * 4, kt * BK, int64_t(D) * 4);
        __syncwarp();  // the tile is staged again for the second half
      }
    } else if (bf == 0) {
      const int kc = store ? key : 0;  // read only when storing
      const float* cp = p.cos_t + (int64_t(b) * p.S + kc) * D;
      const float* sp = p.sin_t + (int64_t(b) * p.S + kc) * D;
      uint8_t* tile = reinterpret_cast<uint8_t*>(sm.k);  // K is no longer read: every MMA has finished
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t lo[32], hi[32];
        if (have) {
          tmem_ld32(tdK + lane_off + c * 32, lo);
          tmem_ld32(tdK + lane_off + D / 2 + c * 32, hi);
          tmem_ld_wait_regs(lo, hi);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) lo[i] = hi[i] = 0u;
        }
        if (store) {
          uint32_t olo[16], ohi[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float a[2], bb[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int j = c * 32 + 2 * i + e;
              const float cj = __ldg(cp + j), sj = __ldg(sp + j);
              const float l = __uint_as_float(lo[2 * i + e]) * p.scale, u = __uint_as_float(hi[2 * i + e]) * p.scale;
              a[e] = fmaf(l, cj, u * sj);
              bb[e] = fmaf(u, cj, -l * sj);
            }
            olo[i] = pack_bf16x2(a[0], a[1]);
            ohi[i] = pack_bf16x2(bb[0], bb[1]);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            stage_chunk(tile, r, c * 4 + i, make_uint4(olo[4 * i], olo[4 * i + 1], olo[4 * i + 2], olo[4 * i + 3]));
            stage_chunk(tile, r, D / 16 + c * 4 + i,
                        make_uint4(ohi[4 * i], ohi[4 * i + 1], ohi[4 * i + 2], ohi[4 * i + 3]));
          }
        }
      }
      __syncwarp();
      store_rows(tile, reinterpret_cast<uint8_t*>(p.dk + int64_t(b) * p.dk_sb + int64_t(hkv) * p.dk_sh),
                 smp.off + kt * BK, p.dk_ss * 2);
    } else {
      uint8_t* tile = reinterpret_cast<uint8_t*>(sm.v);  // V is no longer read: every MMA has finished
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        if (have) {
          tmem_ld32(tdV + lane_off + c * 32, ov);
          tmem_ld_wait_regs(ov);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = 0u;
        }
        if (store) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            stage_chunk(tile, r, c * 4 + i,
                        make_uint4(pack_bf16x2(__uint_as_float(ov[8 * i]), __uint_as_float(ov[8 * i + 1])),
                                   pack_bf16x2(__uint_as_float(ov[8 * i + 2]), __uint_as_float(ov[8 * i + 3])),
                                   pack_bf16x2(__uint_as_float(ov[8 * i + 4]), __uint_as_float(ov[8 * i + 5])),
                                   pack_bf16x2(__uint_as_float(ov[8 * i + 6]), __uint_as_float(ov[8 * i + 7]))));
        }
      }
      __syncwarp();
      store_rows(tile, reinterpret_cast<uint8_t*>(p.dv + int64_t(b) * p.dv_sb + int64_t(hkv) * p.dv_sh),
                 smp.off + kt * BK, p.dv_ss * 2);
    }
  } else {
    // =============================== dQ writers: one head-dim lane per thread
    regs_dec<96>();
    const int quarter = warp & 3;
    const int d = quarter * 32 + lane;
    const bool leader = warp == 12 && lane == 0;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const bool live = quarter * 32 < D;  // warp-uniform (D = 64 uses lanes 0-63 only)
    for (int i = 0; i < n_it; ++i) {
      const int bf = i & 1;
      const int hi = i / n_qt, qt = qt_first + i % n_qt;
      const int h = hkv * p.g + hi;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_dq_full[bf], (i >> 1) & 1, wc))) break;
      tc_fence_after();
      uint32_t a[64];
      if (live) {
        tmem_ld32(tdP(bf) + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&a[0]));
        tmem_ld32(tdP(bf) + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(&a[32]));
        tmem_ld_wait_regs(a);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar_dq_empty[bf]);
      float* dst = p.dq_acc + ((int64_t(b) * p.Hq + h) * p.S_pad + int64_t(qt) * BQ) * D;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        // buffer hh was last handed to the bulk engine two groups ago
        if (leader) bulk_wait_group_read<1>();
        named_bar_sync(1, 128);
        if (live) {
          float* t = sm.dq[hh];
#pragma unroll
          for (int c = 0; c < 32; ++c) t[c * D + d] = __uint_as_float(a[hh * 32 + c]);
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (leader) {
          bulk_reduce_add_f32(dst + hh * (BQ / 2) * D, sm.dq[hh], (BQ / 2) * D * 4);
          bulk_commit_group();
        }
      }
    }
    if (leader) bulk_wait_group<0>();
  }
  __syncwarp();

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// delta = rowsum(dO o O) and lse2 = lse * log2(e) for every (b, h, q < S_pad);
// rows q >= the sample's rows get delta 0 and lse2 +inf (so they contribute
// nothing).  The same pass zeroes the fp32 dQ accumulator rows (b, h, q, :)
// that the attention kernel reduce-adds into.  One warp per (b, q) row: a
// lane group of D/8 lanes covers one head with 16-byte loads, so a warp
// reads 256/D heads per step, several steps in flight.
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const BwdPreParams p) {
  constexpr int LPH = D / 8;        // lanes per head (16-byte chunks of 8 bf16)
  constexpr int HPS = 32 / LPH;     // heads per step
  const int lane = threadIdx.x & 31;
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < p.n_cnt; i += blockDim.x) p.part_cnt[i] = 0;
  const int c = lane % LPH, hs = lane / LPH;
  const unsigned gmask = (LPH == 32 ? 0xffffffffu : ((1u << LPH) - 1u)) << (hs * LPH);
  // grid-stride over (b, q) rows: a fixed grid of resident warps
  for (int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; warp < p.B * p.S_pad;
       warp += (gridDim.x * blockDim.x) >> 5) {
  const int b = warp / p.S_pad, q = warp % p.S_pad;
  const SampleDev t = p.samples[b];
  const bool real = q < t.rows;  // beyond the sample's rows: padding past S, or past L when packed
  const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int h = hs; h < p.Hq; h += HPS) {
    const int64_t orow = (int64_t(b) * p.Hq + h) * p.S_pad + q;
    float4* acc = reinterpret_cast<float4*>(p.dq_acc + orow * D) + 2 * c;
    acc[0] = z4;
    acc[1] = z4;
    float dot = 0.f;
    if (real) {
      const __nv_bfloat16* o = p.o + int64_t(b) * p.o_sb + int64_t(t.off + q) * p.o_ss +
                               int64_t(h / p.g) * p.o_shkv + int64_t(h % p.g) * p.o_shq;
      const __nv_bfloat16* d = p.dout + int64_t(b) * p.d_sb + int64_t(t.off + q) * p.d_ss +
                               int64_t(h / p.g) * p.d_shkv + int64_t(h % p.g) * p.d_shq;
      const uint4 ov = __ldg(reinterpret_cast<const uint4*>(o) + c);
      const uint4 dv = __ldg(reinterpret_cast<const uint4*>(d) + c);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
      const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(o2[i]), y = __bfloat1622float2(d2[i]);
        dot = fmaf(x.x, y.x, dot);
        dot = fmaf(x.y, y.y, dot);
      }
    }
#pragma unroll
    for (int off = LPH / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(gmask, dot, off);
    if (c == 0) {
      p.delta[orow] = real ? dot : 0.f;
      p.lse2[orow] = real ? p.lse[int64_t(b) * p.lse_sb + int64_t(h) * p.lse_sh + t.off + q] * 1.4426950408889634f
                          : INFINITY;
    }
  }
  }
}

}  // namespace

cudaError_t launch_bwd_pre(const BwdPreParams& p, cudaStream_t st) {
  const int64_t warps = int64_t(p.B) * p.S_pad;
  if (warps == 0) return cudaSuccess;
  prof_begin(kBwdPre, st);
  const int blocks = int(warps < 148 * 64 ? (warps + 7) / 8 : 148 * 8);  // grid-stride beyond 8 blocks per SM
  if (p.D == 128)
    bwd_pre_kernel<128><<<blocks, 256, 0, st>>>(p);
  else
    bwd_pre_kernel<64><<<blocks, 256, 0, st>>>(p);
  prof_end(kBwdPre, st);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const BwdParams& p, int n_blocks, int D, cudaStream_t st) {
  if (n_blocks == 0) return cudaSuccess;
  static_assert(sizeof(BwdSmem<128>) + 1024 <= 232448, "shared memory budget");
  const size_t smem = D == 128 ? sizeof(BwdSmem<128>) + 1024 : sizeof(BwdSmem<64>) + 1024;
  const void* fn = D == 128 ? reinterpret_cast<const void*>(attn_bwd_kernel<128>)
                            : reinterpret_cast<const void*>(attn_bwd_kernel<64>);
  // once per device and context: the compiled register count (the setmaxnreg
  // split assumes kLaunchRegs) and the dynamic shared-memory opt-in
  static PerContext<int> ready[2];
  int ok = 0;
  const cudaError_t e = ready[D == 128].get(&ok, [&](int* out) {
    cudaFuncAttributes fa{};
    cudaError_t r = cudaFuncGetAttributes(&fa, fn);
    if (r != cudaSuccess) return r;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    r = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    *out = 1;
    return r;
  });
  if (e != cudaSuccess) return e;
  prof_begin(kAttnBwd, st);
  if (D == 128)
    attn_bwd_kernel<128><<<n_blocks, kThreads, smem, st>>>(tq, tk, tv, tdo, p);
  else
    attn_bwd_kernel<64><<<n_blocks, kThreads, smem, st>>>(tq, tk, tv, tdo, p);
  prof_end(kAttnBwd, st);
  return cudaGetLastError();
}

}  // namespace hia
