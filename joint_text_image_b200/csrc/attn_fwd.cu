// attn_fwd.cu -- forward of the generalized-causal GQA attention on sm_100a.
//
// Definition (hunyuan_image3.layers HunyuanImage3Attention.forward with the
// mask of hunyuan_image3.model build_joint_attention_mask): for every query
// row q and head h, O = softmax(scale * q_r . k_r over visible keys) V with
// q_r, k_r the RoPE-rotated rows and kv head h / g (grouped QKV).
//
// One CTA owns 128 query rows of two query heads of the same kv head (two
// M = 128 tiles), so every K/V tile it streams feeds two MMAs.  It walks the
// kv tiles the segment builder marked visible for that query tile: FULL tiles
// run without a mask, PARTIAL ones apply the predicate k <= e(q) in
// registers, fully masked and padded tiles are never loaded.
//
// Warp roles (384 threads):
//   warp 0      TMA producer: Q tiles once, then K tiles (3-stage ring) and V
//               tiles (2-stage ring)
//   warp 1      TMEM owner and tcgen05.mma issuer (the warp runs converged,
//               one elected lane issues)
//   warps 4-7   softmax / correction / epilogue of tile 0 (one row per thread)
//   warps 8-11  the same for tile 1
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 after it;
// P_t is written as packed bf16 over the first 64 columns of S_t and fed to
// the PV MMA straight from TMEM.  MMA order per kv tile j:
//   PV0(j), QK0(j+1), PV1(j), QK1(j+1)
// so the commit that publishes S_t(j+1) also proves PV_t(j) finished: the
// softmax warps may then rescale O_t and overwrite P_t without extra barriers.
// PV_t(j) is issued in two halves of 64 keys: the softmax warps signal once
// the first half of P_t is stored (and O_t rescaled) and again at the end, so
// the first half of the PV MMAs overlaps the second half of the exponentials.
#include <cuda.h>
#include <cuda_bf16.h>

#include "devctx.h"
#include "kernels.h"
#include "sm100.cuh"

namespace hia {
namespace {

constexpr int kThreads = 384;
// Register split (setmaxnreg): launch budget 384 x 168; warpgroup 0 (TMA, MMA)
// drops to 72, the two softmax warpgroups rise to 216:
// 128*72 + 256*216 = 64512 = 384*168.  The launcher checks the compiled count first.
constexpr int kLaunchRegs = 168;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only if the max grows by > 2^8
constexpr int kFmaExpPairs = 5;           // of every 16 column pairs, this many use exp2_fma2

constexpr int kKStages = 3;  // K(j+1) is awaited together with V(j), so K runs one stage deeper
constexpr int kVStages = 2;

template <int D>
struct FwdSmem {
  static constexpr int kTileElems = 128 * D;
  alignas(1024) __nv_bfloat16 q[2][kTileElems];
  alignas(1024) __nv_bfloat16 k[kKStages][kTileElems];
  alignas(1024) __nv_bfloat16 v[kVStages][kTileElems];
  uint64_t bar_q;
  uint64_t bar_k_full[kKStages];
  uint64_t bar_k_empty[kKStages];
  uint64_t bar_v_full[kVStages];
  uint64_t bar_v_empty[kVStages];
  uint64_t bar_s_full[2];
  uint64_t bar_p_half[2];
  uint64_t bar_p_ready[2];
  uint64_t bar_o_final[2];
  uint32_t tmem_base;
  int abort_flag;
};

// S_t = Q_t K^T: M = 128 query rows, N = 128 keys, K = D.  Both operands
// K-major, 64-wide D blocks 16 KB apart.
template <int D>
__device__ __forceinline__ void issue_qk(uint32_t tS, uint64_t qdesc, uint64_t kdesc) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
  constexpr KMajorSteps<D / 16> st(16384);
  mma_chain_ss_w<D / 16>(tS, qdesc, st.v, kdesc, st.v, idesc, 0u);
}

// O_t (+)= P_t V over one half of the kv tile (keys [64 half, 64 half + 64)):
// A = P_t from TMEM (packed bf16, 8 columns per 16 keys), B = V tile [128
// keys][D] read MN-major (D blocks 16 KB apart, 2 KB per 16 keys).
template <int D>
__device__ __forceinline__ void issue_pv_half(uint32_t tO, uint32_t tP, uint64_t vdesc, int half, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, 0, 1);
  constexpr MNMajorSteps<4> st;
  mma_chain_ts_w<4>(tO, tP + uint32_t(half * 32), 8u, vdesc + uint64_t(half * (4 * 2048 >> 4)), st.v, idesc,
                    accumulate ? 1u : 0u);
}

// P = exp2(S * scale*log2e - m) for column pairs [C0, C1) of one row of 128
// scores, packed to bf16 pairs, added to the row sum.  kFma: kFmaExpPairs of every 16 column pairs take
// exp2 on the FMA pipe, the rest on MUFU.
template <bool kFma, int C0, int C1>
__device__ __forceinline__ void exp_pack(const uint32_t (&sr)[128], float2 cs2, float2 nm2, uint32_t (&pk)[64],
                                         float2 (&ls)[2]) {
#pragma unroll
  for (int c = C0; c < C1; ++c) {
    const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), cs2, nm2);
    const float2 pv = (kFma && (c & 15) < kFmaExpPairs) ? exp2_fma2(x)
                                                        : make_float2(ex2_approx(x.x), ex2_approx(x.y));
    ls[c & 1] = __fadd2_rn(ls[c & 1], pv);
    pk[c] = pack_bf16x2(pv.x, pv.y);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  FwdSmem<D>& sm =
      *reinterpret_cast<FwdSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: (b, q tile) heaviest first, then kv head, then head pair
  int bid = blockIdx.x;
  const int hp = bid % p.n_hp;
  bid /= p.n_hp;
  const int hkv = bid % p.Hkv;
  bid /= p.Hkv;
  const int b = p.work[2 * bid], qt = p.work[2 * bid + 1];
  // the visible kv tiles of this query tile: entries kt | FULL << 16, in order
  const int32_t* tlist = p.list + p.tiles[2 * (b * p.nQT + qt)];
  const int n_vis = p.tiles[2 * (b * p.nQT + qt) + 1];
  const int h0 = hkv * p.g + 2 * hp;
  const int n_tiles = (2 * hp + 1 < p.g) ? 2 : 1;
  const SampleDev smp = p.samples[b];

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&sm.bar_k_full[i], 1);
      mbar_init(&sm.bar_k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&sm.bar_v_full[i], 1);
      mbar_init(&sm.bar_v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.bar_s_full[i], 1);
      mbar_init(&sm.bar_p_half[i], 4);   // one arrival per softmax warp
      mbar_init(&sm.bar_p_ready[i], 4);
      mbar_init(&sm.bar_o_final[i], 1);
    }
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

  if (warp < 4) {
   regs_dec<72>();
   if (warp == 0) {
    // =============================== TMA producer
    if (lane == 0 && n_vis > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      constexpr uint32_t tile_bytes = 128 * D * 2;
      mbar_arrive_expect_tx(&sm.bar_q, tile_bytes * n_tiles);
      for (int t = 0; t < n_tiles; ++t)
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(&sm.q[t][c * 128 * 64], &tm_q, &sm.bar_q, c * 64, qt * 128, b * p.Hq + h0 + t);
      int kiss = 0, viss = 0;
      for (int j = 0; j < n_vis; ++j) {
        const int ks = j % kKStages, vs = j % kVStages;
        const int kt = __ldg(tlist + j) & 0xffff;
        if (j >= kKStages && !mbar_wait(&sm.bar_k_empty[ks], ((j / kKStages) - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(&sm.bar_k_full[ks], tile_bytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(&sm.k[ks][c * 128 * 64], &tm_k, &sm.bar_k_full[ks], c * 64, kt * 128, b * p.Hkv + hkv);
        kiss = j + 1;
        if (j >= kVStages && !mbar_wait(&sm.bar_v_empty[vs], ((j / kVStages) - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(&sm.bar_v_full[vs], tile_bytes);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(&sm.v[vs][c * 128 * 64], &tm_v, &sm.bar_v_full[vs], c * 64, hkv, smp.off + kt * 128,
                      p.packed ? 0 : b);
        viss = j + 1;
      }
      // Drain: the copies this CTA issued must land before its shared memory
      // can be released, whatever the consumers did.
      mbar_wait_hw(&sm.bar_q, 0, wc);
      for (int j = (kiss > kKStages ? kiss - kKStages : 0); j < kiss; ++j)
        mbar_wait_hw(&sm.bar_k_full[j % kKStages], (j / kKStages) & 1, wc);
      for (int j = (viss > kVStages ? viss - kVStages : 0); j < viss; ++j)
        mbar_wait_hw(&sm.bar_v_full[j % kVStages], (j / kVStages) & 1, wc);
    }
  } else if (warp == 1) {
    // =============================== MMA issuer
    // The whole warp runs this loop (waits combined with __all_sync) and one
    // elected lane issues each MMA chain and commit, so the descriptors are
    // warp-uniform values.
    if (n_vis > 0) {
      const uint32_t tS[2] = {tmem, tmem + 128};
      const uint32_t tO[2] = {tmem + 256, tmem + 256 + D};
      // descriptor bases (start address of each buffer); stages are adjacent
      const uint64_t qd[2] = {sdesc_sw128(smem_u32(sm.q[0]), 16, 1024), sdesc_sw128(smem_u32(sm.q[1]), 16, 1024)};
      const uint64_t kd0 = sdesc_sw128(smem_u32(sm.k[0]), 16, 1024);
      const uint64_t vd0 = sdesc_sw128(smem_u32(sm.v[0]), 16384, 1024);
      constexpr uint32_t kStageStep = (128u * D * 2u) >> 4;  // one K or V stage, 16-byte units
      bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.bar_q, 0, wc) && mbar_wait(&sm.bar_k_full[0], 0, wc));
      if (ok) {
        for (int t = 0; t < n_tiles; ++t) {
          issue_qk<D>(tS[t], qd[t], kd0);
          tc_commit_w(&sm.bar_s_full[t]);
        }
        tc_commit_w(&sm.bar_k_empty[0]);
      }
      // Every wait/fence in the issuing thread lets the short MMA queue drain,
      // so each kv step has two synchronisation points, one per query tile:
      // (1) V(j), K(j+1) loaded and P0(j) written; (2) P1(j) written.
      for (int j = 0; ok && j < n_vis; ++j) {
        const int vs = j % kVStages, ks1 = (j + 1) % kKStages;
        const bool more = j + 1 < n_vis;
        for (int t = 0; t < n_tiles; ++t) {
          if (t == 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(&sm.bar_v_full[vs], (j / kVStages) & 1, wc) &&
                                             (!more || mbar_wait(&sm.bar_k_full[ks1], ((j + 1) / kKStages) & 1, wc)));
            if (!ok) break;
          }
          // PV_t(j) in two halves: the first as soon as P_t's first 64 keys are
          // stored, the second once the whole P_t is
          if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_p_half[t], j & 1, wc))) { ok = false; break; }
          tc_fence_after();
          issue_pv_half<D>(tO[t], tS[t], vd0 + uint32_t(vs) * kStageStep, 0, j > 0);
          if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_p_ready[t], j & 1, wc))) { ok = false; break; }
          tc_fence_after();
          issue_pv_half<D>(tO[t], tS[t], vd0 + uint32_t(vs) * kStageStep, 1, true);
          if (more) {
            issue_qk<D>(tS[t], qd[t], kd0 + uint32_t(ks1) * kStageStep);
            tc_commit_w(&sm.bar_s_full[t]);
          }
        }
        if (!ok) break;
        tc_commit_w(&sm.bar_v_empty[vs]);
        if (more) tc_commit_w(&sm.bar_k_empty[ks1]);
      }
      for (int t = 0; t < 2; ++t) tc_commit_w(&sm.bar_o_final[t]);
      // MMAs already issued must finish before TMEM can be released.
      mbar_wait_hw(&sm.bar_o_final[0], 0, wc);
    }
   }
  } else {
    regs_inc<216>();
    // =============================== softmax / epilogue
    // tcgen05.ld/st are warp-collective: every branch around them below is
    // warp-uniform (waits are combined with __all_sync, the O rescale is
    // decided per warp and applied per row with a factor of 1 where unneeded).
    const int t = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int q = qt * 128 + r;
    const int h = h0 + t;
    const bool active = t < n_tiles;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t tS = tmem + uint32_t(t * 128) + lane_off;
    const uint32_t tO = tmem + 256u + uint32_t(t * D) + lane_off;
    const ImageDev* im = p.images + smp.img0;
    const int e = row_bound(im, smp.n_img, smp.L, q);
    // context images this row no longer sees (only samples with several images)
    int n_hidden = 0;
    for (int i = 0; i < smp.n_img; ++i) n_hidden += (im[i].hidden && im[i].I1 <= q) ? 1 : 0;
    // warp-uniform: the masking loop below must not leave the warp diverged
    // before the warp-collective TMEM stores
    const bool warp_hidden = __any_sync(0xffffffffu, n_hidden > 0);
    const float cs = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = active;
    // the tile-list entry of the next kv tile is loaded one step ahead, off
    // the path from "S ready" to "P written"
    int32_t ent_next = n_vis > 0 ? __ldg(tlist) : 0;
    for (int j = 0; ok && j < n_vis; ++j) {
      const int32_t ent = ent_next;
      if (j + 1 < n_vis) ent_next = __ldg(tlist + j + 1);
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.bar_s_full[t], j & 1, wc));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_ld_wait_regs(sr);
      const bool full = (ent >> 16) != 0;
      if (!full) {
        const int k0 = (ent & 0xffff) * 128;
        const int lim = e - k0;  // key k0 + c is visible iff c <= lim and not hidden
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > lim) sr[c] = __float_as_uint(-INFINITY);
        for (int i = 0; warp_hidden && i < smp.n_img; ++i) {
          const bool hide = im[i].hidden && im[i].I1 <= q;  // per row: applied by selects
          const int lo = im[i].I0 - k0, n = im[i].I1 - im[i].I0;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (hide && unsigned(c - lo) < unsigned(n)) sr[c] = __float_as_uint(-INFINITY);
        }
      }
      __syncwarp();
      // row max with 8 independent partial maxima (short dependency chains)
      float mp[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) mp[c] = __uint_as_float(sr[c]);
#pragma unroll
      for (int c = 8; c < 128; c += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) mp[k] = fmax3(mp[k], __uint_as_float(sr[c + k]), __uint_as_float(sr[c + 8 + k]));
      const float xmax = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                               fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7]))) * cs;
      // Lazy O rescale: decided here, applied to O_t after P_t is stored (the
      // 128 scores are dead by then, which keeps the warp within its register
      // budget) and before the arrival that lets PV_t(j) accumulate into O_t.
      float f = 1.f;
      bool rescale = false;
      if (j == 0) {
        m = xmax;
      } else {
        const bool grow = xmax > m + kRescaleThreshold;
        rescale = __any_sync(0xffffffffu, grow);
        // selects, not a branch: the warp stays converged for the TMEM stores
        const float fg = ex2_approx(m - xmax);
        f = grow ? fg : 1.f;
        m = grow ? xmax : m;
      }
      uint32_t pk[64];
      float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      const float2 cs2 = make_float2(cs, cs), nm2 = make_float2(-m, -m);
      // FULL tiles have no masked entry: part of their exponentials run on the
      // FMA pipe.  PARTIAL tiles use MUFU only, whose ex2(-inf) is exactly 0,
      // so a masked key adds nothing (exp2_fma2 bottoms out at 2^-125).
      // First half of P (keys 0-63): stored, O_t rescaled if needed, then
      // signalled so that the first half of PV_t(j) runs while the second half
      // of the exponentials is computed.
      if (full)
        exp_pack<true, 0, 32>(sr, cs2, nm2, pk, ls);
      else
        exp_pack<false, 0, 32>(sr, cs2, nm2, pk, ls);
      tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
      if (rescale) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(tO + c * 32, ov);
          tmem_ld_wait_regs(ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * f);
          tmem_st32(tO + c * 32, ov);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();  // the warp's writes are done; one lane signals for it
      if (lane == 0) mbar_arrive(&sm.bar_p_half[t]);
      if (full)
        exp_pack<true, 32, 64>(sr, cs2, nm2, pk, ls);
      else
        exp_pack<false, 32, 64>(sr, cs2, nm2, pk, ls);
      l = l * f + ((ls[0].x + ls[1].x) + (ls[0].y + ls[1].y));
      tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar_p_ready[t]);
    }
    // ---- epilogue: O / l -> bf16 rows, LSE
    if (active) {
      bool have = n_vis > 0 && ok;
      if (have) have = __all_sync(0xffffffffu, mbar_wait(&sm.bar_o_final[t], 0, wc));
      if (have) tc_fence_after();
      const bool store = q < smp.rows;
      const float inv = (have && l > 0.f) ? 1.f / l : 0.f;
      // O / l -> bf16 rows staged in this tile's Q buffer (every MMA has
      // finished, so Q is no longer read), 16-byte chunks XOR-swizzled by row
      // so that a warp's 32 row writes hit distinct banks; then each warp
      // writes its own 32 rows whole: CPR lanes per row, 16 bytes each, so a
      // warp store covers 32 / CPR complete rows (coalesced 128-bit stores).
      constexpr int CPR = D / 8;  // 16-byte chunks per row
      uint8_t* tile = reinterpret_cast<uint8_t*>(sm.q[t]);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        if (have) {
          tmem_ld32(tO + c * 32, ov);
          tmem_ld_wait_regs(ov);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(ov[2 * i]) * inv, __uint_as_float(ov[2 * i + 1]) * inv);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int ch = (c * 4 + i) ^ (r & (CPR - 1));
          *reinterpret_cast<uint4*>(tile + r * (D * 2) + ch * 16) =
              make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      __syncwarp();
      {
        constexpr int RPI = 32 / CPR;  // rows per warp store
        const int ch = lane % CPR;
        const int64_t head_off = int64_t(b) * p.o_sb + int64_t(h / p.g) * p.o_shkv + int64_t(h % p.g) * p.o_shq;
#pragma unroll 4
        for (int rr = 0; rr < 32; rr += RPI) {
          const int row = quarter * 32 + rr + lane / CPR;
          const int qrow = qt * 128 + row;
          if (qrow < smp.rows) {
            const uint4 v = *reinterpret_cast<const uint4*>(tile + row * (D * 2) + ((ch ^ (row & (CPR - 1))) * 16));
            *reinterpret_cast<uint4*>(p.o + head_off + int64_t(smp.off + qrow) * p.o_ss + ch * 8) = v;
          }
        }
      }
      if (store)
        p.lse[int64_t(b) * p.lse_sb + int64_t(h) * p.lse_sh + smp.off + q] =
            (have && l > 0.f) ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }
  __syncwarp();

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_attn_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, int n_blocks, int D, cudaStream_t st) {
  if (n_blocks == 0) return cudaSuccess;
  static_assert(sizeof(FwdSmem<128>) + 1024 <= 232448, "shared memory budget");
  const size_t smem = D == 128 ? sizeof(FwdSmem<128>) + 1024 : sizeof(FwdSmem<64>) + 1024;
  const void* fn = D == 128 ? reinterpret_cast<const void*>(attn_fwd_kernel<128>)
                            : reinterpret_cast<const void*>(attn_fwd_kernel<64>);
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
  prof_begin(kAttnFwd, st);
  if (D == 128)
    attn_fwd_kernel<128><<<n_blocks, kThreads, smem, st>>>(tq, tk, tv, p);
  else
    attn_fwd_kernel<64><<<n_blocks, kThreads, smem, st>>>(tq, tk, tv, p);
  prof_end(kAttnFwd, st);
  return cudaGetLastError();
}

}  // namespace hia
