// moe.cu -- MoE feed-forward of a HunyuanImage-3.0 decoder block on sm_100a.
//
// Definition (technical report summary 3.1.1; hunyuan_image3.model
// build_moe_config and HunyuanImage3Block; hunyuan_image3.layers
// HunyuanSharedMLP; coverage page, Train: router in fp32): per token x,
//   p = softmax(x Wg^T) over the E routed experts, the topk largest chosen and
//   renormalized, out = sum_j w_j expert_{e_j}(x) + shared(x), every expert a
//   SwiGLU with fused [up; gate] projection (up first).
//
// Kernels, in launch order:
//   moe_prep      Wg (fp32) split into three bf16 parts hi + mid + lo = Wg
//                 exactly; the per-expert row counters cleared.
//   moe_router    logits = x [hi; mid; lo]^T as ONE tcgen05 GEMM (N = 3 Ep):
//                 x is exact in bf16 and each bf16 x bf16 product is exact
//                 in fp32, so the three partial sums added in fp32 give the
//                 logits to fp32 precision.  The epilogue (one token row per
//                 thread) takes the topk largest (ties: lower index),
//                 renormalizes, and claims a row slot per chosen expert with
//                 an atomic counter.
//   moe_scan      per-group row offsets (each group padded to 128 rows; the
//                 shared expert is group E, holding every token) and the
//                 table of 128-row tiles.
//   moe_gather    x rows copied into expert-sorted order; padding rows zeroed.
//   moe_gemm<UpGate>  act = silu(A W13_gate^T) * (A W13_up^T) -> bf16: a
//                 persistent grouped GEMM over (128-row tile, 128 up + 128
//                 gate columns); the SwiGLU runs in the epilogue.
//   moe_gemm<Down>    y = act W2^T -> bf16, tiles of 128 rows x 256 columns.
//   moe_combine   out = sum_j w_j y[row of (token, j)] + y[shared row], fp32.
//
// GEMM CTA: 192 threads.  Warp 0 TMA producer (4-stage ring of A 128 x 64 and
// B 256 x 64 bf16 tiles, 128-byte swizzle), warp 1 TMEM owner and the single
// tcgen05.mma issuer (M = 128, N = 256, K = 16 per instruction), warps 2-5
// epilogue (one accumulator row per thread).  TMEM holds two 128 x 256 fp32
// accumulators, so the epilogue of one tile overlaps the MMAs of the next.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "../../include/jointmoe.h"
#include "devctx.h"
#include "kernels.h"
#include "sm100.cuh"

namespace hia {
namespace {

constexpr int kMaxExperts = 80;
constexpr int kMaxTopk = 16;
constexpr int kTileRows = 128;
constexpr int kStages = 4;
constexpr int kGemmThreads = 192;
constexpr uint64_t kTimeoutNs = 2000000000ull;

// Device-resident routing tables (in the workspace).
struct MoeMeta {
  int32_t counts[kMaxExperts + 1];    // rows routed to each group (group E, the shared expert: T)
  int32_t offsets[kMaxExperts + 2];   // first row of each group in the sorted buffers (multiples of 128)
  int32_t n_mtiles;                   // 128-row tiles over all groups
};

__host__ __device__ inline int pad_rows(int n) { return (n + kTileRows - 1) / kTileRows * kTileRows; }

// ---------------------------------------------------------------- prep
// wsplit [3][Ep][H] bf16: hi = rn(w), mid = rn(w - hi), lo = rn(w - hi - mid).
// Each difference is exact in fp32 (w has 24 significant bits and each part
// takes 8 of them), so hi + mid + lo == w.  Rows E..Ep-1 are zero.
__global__ void moe_prep_kernel(const float* __restrict__ wg, int E, int Ep, int H, __nv_bfloat16* __restrict__ ws,
                                MoeMeta* meta) {
  const int64_t n = int64_t(Ep) * H;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int e = int(i / H);
    const float w = e < E ? wg[i] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    ws[i] = hi;
    ws[n + i] = mid;
    ws[2 * n + i] = __float2bfloat16_rn(r2);
  }
  if (blockIdx.x == 0)
    for (int g = threadIdx.x; g <= kMaxExperts; g += blockDim.x) meta->counts[g] = 0;
}

// ---------------------------------------------------------------- router
struct RouterParams {
  int T, H, E, Ep, topk;
  MoeMeta* meta;
  int32_t* ids;      // [T][topk]
  float* weights;    // [T][topk]
  int32_t* slot;     // [T][topk]: row of the token within its expert's group
  int* status;
  uint64_t timeout_ns;
};

constexpr int kRouterStages = 3;
constexpr int kRouterMaxN = 3 * kMaxExperts;  // 240

struct RouterSmem {
  alignas(1024) __nv_bfloat16 a[kRouterStages][kTileRows * 64];
  alignas(1024) __nv_bfloat16 b[kRouterStages][kRouterMaxN * 64];
  float logit[kTileRows][kMaxExperts + 1];
  uint64_t bar_full[kRouterStages];
  uint64_t bar_empty[kRouterStages];
  uint64_t bar_acc;
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(kGemmThreads, 1)
    moe_router_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                      const RouterParams p) {
  extern __shared__ uint8_t smem_raw[];
  RouterSmem& sm =
      *reinterpret_cast<RouterSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * kTileRows;
  const int nk = p.H / 64, N = 3 * p.Ep;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kRouterStages; ++i) {
      mbar_init(&sm.bar_full[i], 1);
      mbar_init(&sm.bar_empty[i], 1);
    }
    mbar_init(&sm.bar_acc, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtx wc{&sm.abort_flag, p.status, p.timeout_ns};

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_w);
      const uint32_t bytes = uint32_t(kTileRows * 64 * 2 + N * 64 * 2);
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kRouterStages;
        if (kb >= kRouterStages && !mbar_wait(&sm.bar_empty[s], ((kb / kRouterStages) - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(&sm.bar_full[s], bytes);
        tma_load_2d(sm.a[s], &tm_x, &sm.bar_full[s], kb * 64, row0);
        tma_load_2d(sm.b[s], &tm_w, &sm.bar_full[s], kb * 64, 0);
        issued = kb + 1;
      }
      for (int kb = std::max(issued - kRouterStages, 0); kb < issued; ++kb)
        mbar_wait_hw(&sm.bar_full[kb % kRouterStages], (kb / kRouterStages) & 1, wc);
    }
  } else if (warp == 1) {
    // MMA issuer: the warp runs converged, one elected lane issues
    {
      const uint32_t idesc = idesc_bf16_f32(kTileRows, N, 0, 0);
      constexpr KMajorSteps<4> st(0);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kRouterStages;
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_full[s], (kb / kRouterStages) & 1, wc))) break;
        tc_fence_after();
        mma_chain_ss_w<4>(tmem, sdesc_sw128(smem_u32(sm.a[s]), 16, 1024), st.v,
                          sdesc_sw128(smem_u32(sm.b[s]), 16, 1024), st.v, idesc, kb > 0 ? 1u : 0u);
        tc_commit_w(&sm.bar_empty[s]);
      }
      tc_commit_w(&sm.bar_acc);
      mbar_wait_hw(&sm.bar_acc, 0, wc);
    }
  } else {
    // epilogue: one token row per thread (TMEM lane quarter = warp % 4)
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int t = row0 + r;
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.bar_acc, 0, wc));
    if (ok) {
      tc_fence_after();
      float* lg = sm.logit[r];
      // columns [0, Ep) hi, [Ep, 2Ep) mid, [2Ep, 3Ep) lo: logits = (hi + mid) + lo
      for (int c = 0; c < N; c += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_off + uint32_t(c), v);
        tmem_ld_wait_regs(v);
        const int part = c / p.Ep, e0 = c % p.Ep;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float x = __uint_as_float(v[i]);
          lg[e0 + i] = part == 0 ? x : lg[e0 + i] + x;
        }
      }
      if (t < p.T) {
        int sel[kMaxTopk];
        float sl[kMaxTopk];
        for (int j = 0; j < p.topk; ++j) {
          float best = -INFINITY;
          int bi = 0;
          for (int e = 0; e < p.E; ++e) {
            const float x = lg[e];
            if (x > best) {  // strict: a tie keeps the lower expert index
              best = x;
              bi = e;
            }
          }
          sel[j] = bi;
          sl[j] = best;
          lg[bi] = -INFINITY;
        }
        // renormalized softmax over the chosen: w_j = exp(l_j - l_max) / sum
        float den = 0.f;
        for (int j = 0; j < p.topk; ++j) den += expf(sl[j] - sl[0]);
        for (int j = 0; j < p.topk; ++j) {
          const int64_t o = int64_t(t) * p.topk + j;
          p.ids[o] = sel[j];
          p.weights[o] = expf(sl[j] - sl[0]) / den;
          p.slot[o] = atomicAdd(&p.meta->counts[sel[j]], 1);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------- scan
// counts -> 128-aligned group offsets and the table of 128-row tiles:
// mtab[i] = (group, tile index within the group).  One block.
__global__ void moe_scan_kernel(MoeMeta* meta, int E, int T, int32_t* mtab) {
  __shared__ int first[kMaxExperts + 2];
  if (threadIdx.x == 0) {
    meta->counts[E] = T;
    int off = 0;
    for (int g = 0; g <= E; ++g) {
      meta->offsets[g] = off;
      first[g] = off / kTileRows;
      off += pad_rows(meta->counts[g]);
    }
    meta->offsets[E + 1] = off;
    meta->n_mtiles = off / kTileRows;
  }
  __syncthreads();
  for (int g = threadIdx.x; g <= E; g += blockDim.x) {
    const int n = pad_rows(meta->counts[g]) / kTileRows;
    for (int j = 0; j < n; ++j) {
      mtab[2 * (first[g] + j)] = g;
      mtab[2 * (first[g] + j) + 1] = j;
    }
  }
}

// ---------------------------------------------------------------- gather
// Row of (token t, choice j) = offsets[e] + slot; x[t] is read once and
// written to its topk rows (one warp per token, the row in registers in
// pieces of 16 chunks of 16 bytes per lane); the padding rows of every routed
// group are zeroed.
__global__ void __launch_bounds__(256) moe_gather_kernel(const __nv_bfloat16* __restrict__ x, int T, int H, int topk,
                                                         int E, const int32_t* __restrict__ ids,
                                                         const int32_t* __restrict__ slot, const MoeMeta* meta,
                                                         int32_t* __restrict__ rowidx, __nv_bfloat16* __restrict__ xp) {
  constexpr int kPiece = 16;  // 16-byte chunks per lane per pass
  const int lane = threadIdx.x & 31;
  const int nchunk = H / 8;  // 16-byte chunks per row
  const int64_t n_warps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int64_t w0 = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5;
  for (int64_t t = w0; t < T + int64_t(E) * kTileRows; t += n_warps) {
    if (t < T) {
      // this token's rows in the sorted order (lane j holds choice j's)
      const int my_row = lane < topk ? meta->offsets[ids[t * topk + lane]] + slot[t * topk + lane] : 0;
      if (lane < topk) rowidx[t * topk + lane] = my_row;
      const uint4* src = reinterpret_cast<const uint4*>(x + t * H);
      for (int c0 = 0; c0 < nchunk; c0 += 32 * kPiece) {
        uint4 v[kPiece];
#pragma unroll
        for (int i = 0; i < kPiece; ++i) {
          const int c = c0 + i * 32 + lane;
          if (c < nchunk) v[i] = __ldg(src + c);
        }
        for (int j = 0; j < topk; ++j) {
          uint4* dst = reinterpret_cast<uint4*>(xp + int64_t(__shfl_sync(0xffffffffu, my_row, j)) * H);
#pragma unroll
          for (int i = 0; i < kPiece; ++i) {
            const int c = c0 + i * 32 + lane;
            if (c < nchunk) dst[c] = v[i];
          }
        }
      }
    } else {
      const int g = int((t - T) / kTileRows), r = int((t - T) % kTileRows);
      const int n = meta->counts[g];
      if (n + r < pad_rows(n)) {
        uint4* dst = reinterpret_cast<uint4*>(xp + int64_t(meta->offsets[g] + n + r) * H);
        for (int c = lane; c < nchunk; c += 32) dst[c] = make_uint4(0, 0, 0, 0);
      }
    }
  }
}

// ---------------------------------------------------------------- grouped GEMM
enum GemmMode { kUpGate = 0, kDown = 1 };

struct GemmParams {
  const MoeMeta* meta;
  const int32_t* mtab;   // [n_mtiles][2]: (group, tile within group)
  __nv_bfloat16* out;    // act [rows][I] (UpGate) or y [rows][H] (Down)
  int64_t out_stride;    // elements
  int E, I, H;
  int nk;                // K / 64
  int nt;                // n-tiles per 128-row tile
  int* status;
  uint64_t timeout_ns;
};

struct GemmSmem {
  alignas(1024) __nv_bfloat16 a[kStages][kTileRows * 64];
  alignas(1024) __nv_bfloat16 b[kStages][256 * 64];
  uint64_t bar_full[kStages];
  uint64_t bar_empty[kStages];
  uint64_t bar_acc_full[2];
  uint64_t bar_acc_empty[2];
  uint64_t bar_final;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ float silu_f(float z) { return z / (1.f + __expf(-z)); }

// Tile t -> (group g, 128-row tile j of the group, column tile nt).  Tiles are
// ordered group by group and, inside a group, column-tile-major: the CTAs that
// run together (consecutive t) share each column tile of the group's weights,
// which is then read from HBM once, and the group's few row tiles stay in L2.
// Group g owns tiles [first_g * nt, first_g' * nt), first_g = offsets[g] / 128
// its first row tile, so the row tile t / nt lies inside group g.
__device__ __forceinline__ void decode_tile(const GemmParams& p, int t, int& g, int& j, int& nt) {
  g = p.mtab[2 * (t / p.nt)];
  const int first = p.meta->offsets[g] / kTileRows;
  const int mtg = p.meta->offsets[g + 1] / kTileRows - first;  // row tiles of the group
  const int local = t - first * p.nt;
  nt = local / mtg;
  j = local % mtg;
}

// tm_a: the sorted rows (x rows for UpGate, act rows for Down); tm_x: x itself
// (the shared expert's A rows in UpGate); tm_b: W13 as [(E+1)*2I][H] or W2 as
// [(E+1)*H][I].
template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ CUtensorMap tm_b, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  GemmSmem& sm = *reinterpret_cast<GemmSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = p.meta->n_mtiles * p.nt;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.bar_full[i], 1);
      mbar_init(&sm.bar_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.bar_acc_full[i], 1);
      mbar_init(&sm.bar_acc_empty[i], 128);
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

  if (warp == 0) {
    // =============================== TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      if (MODE == kUpGate) tma_prefetch_desc(&tm_x);
      constexpr uint32_t bytes = kTileRows * 64 * 2 + 256 * 64 * 2;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x) {
        int g, j, nt;
        decode_tile(p, tile, g, j, nt);
        const bool shared_x = MODE == kUpGate && g == p.E;  // the shared expert reads x directly
        const CUtensorMap* ma = shared_x ? &tm_x : &tm_a;
        const int arow = shared_x ? j * kTileRows : p.meta->offsets[g] + j * kTileRows;
        for (int kb = 0; kb < p.nk; ++kb, ++it) {
          const int s = it % kStages;
          if (it >= kStages && !mbar_wait(&sm.bar_empty[s], ((it / kStages) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.bar_full[s], bytes);
          tma_load_2d(sm.a[s], ma, &sm.bar_full[s], kb * 64, arow);
          if (MODE == kUpGate) {
            const int brow = g * 2 * p.I + nt * 128;
            tma_load_2d(sm.b[s], &tm_b, &sm.bar_full[s], kb * 64, brow);                      // up
            tma_load_2d(sm.b[s] + 128 * 64, &tm_b, &sm.bar_full[s], kb * 64, brow + p.I);    // gate
          } else {
            tma_load_2d(sm.b[s], &tm_b, &sm.bar_full[s], kb * 64, g * p.H + nt * 256);
          }
        }
      }
      // the copies in flight must land before shared memory is released
      for (int i = std::max(it - kStages, 0); i < it; ++i)
        mbar_wait_hw(&sm.bar_full[i % kStages], (i / kStages) & 1, wc);
    }
  } else if (warp == 1) {
    // =============================== MMA issuer
    // The warp runs converged (waits combined with __all_sync) and one elected
    // lane issues, so the descriptors are warp-uniform values.
    {
      constexpr uint32_t idesc = idesc_bf16_f32(kTileRows, 256, 0, 0);
      constexpr KMajorSteps<4> st(0);
      int it = 0, tl = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < n_tiles; tile += gridDim.x, ++tl) {
        const int buf = tl & 1;
        if (tl >= 2 && !__all_sync(0xffffffffu, mbar_wait(&sm.bar_acc_empty[buf], ((tl >> 1) - 1) & 1, wc))) break;
        tc_fence_after();
        const uint32_t acc = tmem + uint32_t(buf * 256);
        for (int kb = 0; kb < p.nk; ++kb, ++it) {
          const int s = it % kStages;
          if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_full[s], (it / kStages) & 1, wc))) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_chain_ss_w<4>(acc, sdesc_sw128(smem_u32(sm.a[s]), 16, 1024), st.v,
                            sdesc_sw128(smem_u32(sm.b[s]), 16, 1024), st.v, idesc, kb > 0 ? 1u : 0u);
          tc_commit_w(&sm.bar_empty[s]);
        }
        if (ok) tc_commit_w(&sm.bar_acc_full[buf]);
      }
      tc_commit_w(&sm.bar_final);
      mbar_wait_hw(&sm.bar_final, 0, wc);
    }
  } else {
    // =============================== epilogue: one accumulator row per thread
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    int tl = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tl) {
      const int buf = tl & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.bar_acc_full[buf], (tl >> 1) & 1, wc))) break;
      tc_fence_after();
      int g, j, nt;
      decode_tile(p, tile, g, j, nt);
      const int64_t row = p.meta->offsets[g] + j * kTileRows + r;
      const uint32_t acc = tmem + uint32_t(buf * 256) + lane_off;
      if (MODE == kUpGate) {
        // columns [0, 128) up, [128, 256) gate -> act[row][nt*128 + c]
        __nv_bfloat16* dst = p.out + row * p.out_stride + nt * 128;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t up[32], gt[32];
          tmem_ld32(acc + uint32_t(c), up);
          tmem_ld32(acc + uint32_t(128 + c), gt);
          tmem_ld_wait_regs(up, gt);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a0 = silu_f(__uint_as_float(gt[2 * i])) * __uint_as_float(up[2 * i]);
            const float a1 = silu_f(__uint_as_float(gt[2 * i + 1])) * __uint_as_float(up[2 * i + 1]);
            pk[i] = pack_bf16x2(a0, a1);
          }
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      } else {
        __nv_bfloat16* dst = p.out + row * p.out_stride + nt * 256;
#pragma unroll 1
        for (int c = 0; c < 256; c += 32) {
          uint32_t v[32];
          tmem_ld32(acc + uint32_t(c), v);
          tmem_ld_wait_regs(v);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.bar_acc_empty[buf]);
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

// ---------------------------------------------------------------- combine
// out[t] = sum_j w_j y[rowidx(t, j)] + y[offsets[E] + t] in fp32 (choices in
// order, then the shared expert), rounded to bf16.  One warp per token.
__global__ void __launch_bounds__(256) moe_combine_kernel(const __nv_bfloat16* __restrict__ y, int T, int H, int topk,
                                                          int E, const int32_t* __restrict__ rowidx,
                                                          const float* __restrict__ weights, const MoeMeta* meta,
                                                          __nv_bfloat16* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int nchunk = H / 8;
  const int64_t n_warps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int shared0 = meta->offsets[E];
  for (int64_t t = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5; t < T; t += n_warps) {
    const int my_row = lane < topk ? rowidx[t * topk + lane] : 0;
    const float my_w = lane < topk ? weights[t * topk + lane] : 0.f;
    // the rows of every choice (then the shared row), fetched once per token
    int rows[kMaxTopk + 1];
    float ws[kMaxTopk + 1];
#pragma unroll
    for (int j = 0; j <= kMaxTopk; ++j) {
      rows[j] = j < topk ? __shfl_sync(0xffffffffu, my_row, j) : shared0 + int(t);
      ws[j] = j < topk ? __shfl_sync(0xffffffffu, my_w, j) : 1.f;
    }
    for (int c = lane; c < nchunk; c += 32) {
      // all k + 1 loads of this chunk in flight before the sum (in order:
      // choices, then the shared expert)
      uint4 u[kMaxTopk + 1];
#pragma unroll
      for (int j = 0; j <= kMaxTopk; ++j)
        if (j <= topk) u[j] = __ldg(reinterpret_cast<const uint4*>(y + int64_t(rows[j]) * H) + c);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j <= kMaxTopk; ++j) {
        if (j > topk) break;
        const float w = j < topk ? ws[j] : 1.f;
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u[j]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(h2[i]);
          acc[2 * i] = fmaf(w, f.x, acc[2 * i]);
          acc[2 * i + 1] = fmaf(w, f.y, acc[2 * i + 1]);
        }
      }
      uint4 o;
      uint32_t* o32 = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i) o32[i] = pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
      reinterpret_cast<uint4*>(out + t * int64_t(H))[c] = o;
    }
  }
}

// ---------------------------------------------------------------- host side
int round16(int x) { return (x + 15) / 16 * 16; }

struct MoeWs {
  size_t wsplit, meta, slot, rowidx, mtab, xp, act, y, total;
  int64_t rows;    // rows of the sorted buffers
  int64_t mtiles;  // their 128-row tiles
};

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

MoeWs moe_ws(const hia_moe_dims& d) {
  MoeWs w{};
  const int Ep = round16(d.E);
  // every routed group pads at most 127 rows; the shared group holds T rows, padded
  w.rows = pad_rows(int(std::min<int64_t>(int64_t(d.T) * d.topk + int64_t(d.E) * (kTileRows - 1), 1ll << 30))) +
           pad_rows(d.T);
  w.mtiles = w.rows / kTileRows;
  size_t o = 0;
  w.wsplit = o;
  o = a256(o + size_t(3) * Ep * d.H * 2);
  w.meta = o;
  o = a256(o + sizeof(MoeMeta));
  w.slot = o;
  o = a256(o + size_t(d.T) * d.topk * 4);
  w.rowidx = o;
  o = a256(o + size_t(d.T) * d.topk * 4);
  w.mtab = o;
  o = a256(o + size_t(w.mtiles) * 8);
  w.xp = o;
  o = a256(o + size_t(w.rows) * d.H * 2);
  w.act = o;
  o = a256(o + size_t(w.rows) * d.I * 2);
  w.y = o;
  o = a256(o + size_t(w.rows) * d.H * 2);
  w.total = o;
  return w;
}

bool dims_ok(const hia_moe_dims* d) {
  return d && d->T >= 0 && d->T < (1 << 24) && d->H > 0 && d->H % 256 == 0 && d->H <= 65536 && d->I > 0 &&
         d->I % 128 == 0 && d->I <= 65536 && d->E >= 1 && d->E <= kMaxExperts && d->topk >= 1 &&
         d->topk <= std::min(d->E, kMaxTopk);
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int sm_count() {
  static PerContext<int> cache;
  int n = 0;
  if (cache.get(&n, [](int* out) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        return e != cudaSuccess ? e : cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev);
      }) != cudaSuccess)
    return 0;
  return n;
}

// dynamic shared memory opt-in, once per device and context
template <class K>
cudaError_t smem_optin(PerContext<int>& c, K kernel, size_t bytes) {
  int done = 0;
  return c.get(&done, [&](int* out) {
    *out = 1;
    return cudaFuncSetAttribute(reinterpret_cast<const void*>(kernel), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                int(bytes));
  });
}

}  // namespace

int* device_status_word();

}  // namespace hia

extern "C" size_t hia_moe_workspace_bytes(const hia_moe_dims* d) {
  if (!hia::dims_ok(d)) return 0;
  return hia::moe_ws(*d).total;
}

extern "C" int hia_moe_fwd(const hia_moe_dims* d, const void* x, const float* wg, const void* w13, const void* w2,
                           void* out, int32_t* ids, float* weights, void* ws, size_t ws_bytes, void* stream) {
  using namespace hia;
  if (!dims_ok(d)) return HIA_ERR_INVALID_ARG;
  if (d->T == 0) return HIA_OK;
  if (!x || !wg || !w13 || !w2 || !out || !ids || !weights || !ws) return HIA_ERR_INVALID_ARG;
  if (!al16(x) || !al16(wg) || !al16(w13) || !al16(w2) || !al16(out) || !al16(ids) || !al16(weights))
    return HIA_ERR_UNSUPPORTED;
  const MoeWs w = moe_ws(*d);
  if (ws_bytes < w.total || (reinterpret_cast<uintptr_t>(ws) & 255)) return HIA_ERR_INVALID_ARG;
  int* status = device_status_word();
  const int n_sm = sm_count();
  if (!status || n_sm <= 0) return HIA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int T = d->T, H = d->H, I = d->I, E = d->E, K = d->topk, Ep = round16(E);
  char* b = static_cast<char*>(ws);
  __nv_bfloat16* wsplit = reinterpret_cast<__nv_bfloat16*>(b + w.wsplit);
  MoeMeta* meta = reinterpret_cast<MoeMeta*>(b + w.meta);
  int32_t* slot = reinterpret_cast<int32_t*>(b + w.slot);
  int32_t* rowidx = reinterpret_cast<int32_t*>(b + w.rowidx);
  int32_t* mtab = reinterpret_cast<int32_t*>(b + w.mtab);
  __nv_bfloat16* xp = reinterpret_cast<__nv_bfloat16*>(b + w.xp);
  __nv_bfloat16* act = reinterpret_cast<__nv_bfloat16*>(b + w.act);
  __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(b + w.y);

  CUtensorMap tm_x, tm_ws, tm_xp, tm_w13, tm_act, tm_w2;
  if (!make_map_2d(&tm_x, x, H, T, uint64_t(H) * 2, 64, kTileRows) ||
      !make_map_2d(&tm_ws, wsplit, H, 3 * Ep, uint64_t(H) * 2, 64, uint32_t(3 * Ep)) ||
      !make_map_2d(&tm_xp, xp, H, w.rows, uint64_t(H) * 2, 64, kTileRows) ||
      !make_map_2d(&tm_w13, w13, H, uint64_t(E + 1) * 2 * I, uint64_t(H) * 2, 64, 128) ||
      !make_map_2d(&tm_act, act, I, w.rows, uint64_t(I) * 2, 64, kTileRows) ||
      !make_map_2d(&tm_w2, w2, I, uint64_t(E + 1) * H, uint64_t(I) * 2, 64, 256))
    return HIA_ERR_CUDA;

  const size_t router_smem = sizeof(RouterSmem) + 1024, gemm_smem = sizeof(GemmSmem) + 1024;
  static_assert(sizeof(RouterSmem) + 1024 <= 232448, "router shared memory");
  static_assert(sizeof(GemmSmem) + 1024 <= 232448, "gemm shared memory");
  static PerContext<int> opt_router, opt_up, opt_down;
  if (smem_optin(opt_router, moe_router_kernel, router_smem) != cudaSuccess ||
      smem_optin(opt_up, moe_gemm_kernel<kUpGate>, gemm_smem) != cudaSuccess ||
      smem_optin(opt_down, moe_gemm_kernel<kDown>, gemm_smem) != cudaSuccess)
    return HIA_ERR_CUDA;

  prof_begin(kMoePrep, st);
  moe_prep_kernel<<<std::min<int64_t>((int64_t(Ep) * H + 255) / 256, n_sm * 8), 256, 0, st>>>(wg, E, Ep, H, wsplit,
                                                                                             meta);
  prof_end(kMoePrep, st);

  RouterParams rp{T, H, E, Ep, K, meta, ids, weights, slot, status, kTimeoutNs};
  prof_begin(kMoeRouter, st);
  moe_router_kernel<<<(T + kTileRows - 1) / kTileRows, kGemmThreads, router_smem, st>>>(tm_x, tm_ws, rp);
  prof_end(kMoeRouter, st);

  prof_begin(kMoeScan, st);
  moe_scan_kernel<<<1, 128, 0, st>>>(meta, E, T, mtab);
  prof_end(kMoeScan, st);

  const int64_t gather_warps = int64_t(T) + int64_t(E) * kTileRows;
  prof_begin(kMoeGather, st);
  moe_gather_kernel<<<int(std::min<int64_t>((gather_warps + 7) / 8, n_sm * 8)), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), T, H, K, E, ids, slot, meta, rowidx, xp);
  prof_end(kMoeGather, st);

  GemmParams g1{meta, mtab, act, I, E, I, H, H / 64, I / 128, status, kTimeoutNs};
  prof_begin(kMoeUpGate, st);
  moe_gemm_kernel<kUpGate><<<n_sm, kGemmThreads, gemm_smem, st>>>(tm_xp, tm_x, tm_w13, g1);
  prof_end(kMoeUpGate, st);

  GemmParams g2{meta, mtab, y, H, E, I, H, I / 64, H / 256, status, kTimeoutNs};
  prof_begin(kMoeDown, st);
  moe_gemm_kernel<kDown><<<n_sm, kGemmThreads, gemm_smem, st>>>(tm_act, tm_act, tm_w2, g2);
  prof_end(kMoeDown, st);

  prof_begin(kMoeCombine, st);
  moe_combine_kernel<<<int(std::min<int64_t>((int64_t(T) + 7) / 8, n_sm * 8)), 256, 0, st>>>(
      y, T, H, K, E, rowidx, weights, meta, static_cast<__nv_bfloat16*>(out));
  prof_end(kMoeCombine, st);
  return cudaGetLastError() == cudaSuccess ? HIA_OK : HIA_ERR_CUDA;
}
