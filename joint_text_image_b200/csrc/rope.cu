// rope.cu -- generalized 2D RoPE: table builder and the rotation kernels.
//
// Paper review (xllm-io) 3.4 and Figure 5; technical report summary 3.1.3:
// 1D RoPE for text is [cos n t0, cos n t1, ..., sin n t0, sin n t1, ...];
// image tokens use [cos x t0, cos y t1, ..., sin x t0, sin y t1, ...] with the
// image's 1D positions reshaped to its h x w grid (row-major, as the UNet
// patch embedding orders them) between the text segments, text sitting on the
// diagonal x = y = n.  The tables are the fp32 [B, S, head_dim] cos/sin of
// HunyuanImage3Attention.forward: entry j and j + D/2 hold angle_j, and a
// vector is rotated as v*cos + rotate_half(v)*sin, rotate_half(v) =
// [-v[D/2:], v[:D/2]].
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "kernels.h"

namespace hia {

// K1: one warp per (b, n) row, lane l owns the angles j = l, l + 32, ... <
// D/2.  The row's position (and its image grid cell) is found once per row.
// Angle and cos/sin in fp64, rounded once to fp32: a text-only sample
// reproduces the 1D tables exactly.  The frequencies theta_j = base^(-2j/D)
// depend on j only: each block evaluates them once into shared memory.
__global__ void __launch_bounds__(256) rope2d_tables_kernel(const SampleDev* __restrict__ samples,
                                                            const ImageDev* __restrict__ images, int B, int S, int D,
                                                            double base, float* __restrict__ cos_out,
                                                            float* __restrict__ sin_out) {
  __shared__ double theta_s[128];
  const int half = D / 2;
  for (int j = threadIdx.x; j < half; j += blockDim.x) theta_s[j] = pow(base, -2.0 * double(j) / double(D));
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t row = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5;
  if (row < int64_t(B) * S) {
    const int b = int(row / S), n = int(row - int64_t(b) * S);
    const SampleDev t = samples[b];
    int x = n, y = n;
    const int im = image_of(images + t.img0, t.n_img, n);
    if (im >= 0) {  // each image on its own grid, origin at its first token
      const ImageDev g = images[t.img0 + im];
      const int i = n - g.I0;
      x = g.I0 + i % g.w;
      y = g.I0 + i / g.w;
    }
    for (int j = lane; j < half; j += 32) {
      const double a = double((j & 1) ? y : x) * theta_s[j];
      double sn, cs;
      sincos(a, &sn, &cs);
      const int64_t o = row * D + j;
      cos_out[o] = float(cs);
      cos_out[o + half] = float(cs);
      sin_out[o] = float(sn);
      sin_out[o + half] = float(sn);
    }
  }
}

// Row helpers shared by the rotation pre-pass and the gradient epilogue.  A
// warp owns one (b, s) row; lane = hs * CPH + c owns channels c*8 .. c*8+7 of
// the low half and the matching 8 of the high half of one head (CPH = D/16
// lanes per head, HPI = 32/CPH heads per pass).  A sum over one head's
// channels is a butterfly over the CPH lanes of the head's lane group.
template <int D>
struct RowLanes {
  static constexpr int CPH = D / 16;
  static constexpr int HPI = 32 / CPH;
  int c, hs;
  unsigned gmask;
  __device__ explicit RowLanes(int lane) : c(lane % CPH), hs(lane / CPH) {
    gmask = (CPH == 32 ? 0xffffffffu : ((1u << CPH) - 1u)) << (hs * CPH);
  }
  __device__ float head_sum(float v) const {
#pragma unroll
    for (int o = 1; o < CPH; o <<= 1) v += __shfl_xor_sync(gmask, v, o);
    return v;
  }
};

__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 x0 = __ldg(reinterpret_cast<const float4*>(p)), x1 = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w; v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
}

__device__ __forceinline__ void load8_bf16(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h2[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ uint4 pack8_bf16(const float (&v)[8]) {
  uint4 u;
  __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h2[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  return u;
}

// Rotation pre-pass: dst[b][h][s][:] = R(b,s) src[b,s,h,:] in fp32, rounded
// to bf16, for q and k in one launch.  With QK RMSNorm weights (w != nullptr)
// the rotated row x is replaced by w * x / sqrt(mean(x^2) + eps) before the
// rounding (HunyuanImage3Attention applies RoPE, then the per-head QK
// RMSNorm).  A warp owns one (b, s) row: the cos/sin of the row are read once
// and reused for every head of both tensors.
template <int D, bool NORM>
__device__ __forceinline__ void rotate_part(const RotatePart& a, const RowLanes<D>& L, int b, int s, int S,
                                            const SampleDev& t, const float (&cs)[8], const float (&sn)[8]) {
  constexpr bool norm = NORM;
  float wl[8], wh[8];
  if (norm) {
    load8(a.w + L.c * 8, wl);
    load8(a.w + D / 2 + L.c * 8, wh);
  }
#pragma unroll 2
  for (int h = L.hs; h < a.H; h += RowLanes<D>::HPI) {
    const int64_t so = int64_t(b) * a.src_sb + int64_t(t.off + s) * a.src_ss + int64_t(h / a.g) * a.src_shkv +
                       int64_t(h % a.g) * a.src_shq;
    const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(a.src) + so;
    float l[8], u[8], xl[8], xu[8];
    load8_bf16(src + L.c * 8, l);
    load8_bf16(src + D / 2 + L.c * 8, u);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      xl[k] = fmaf(l[k], cs[k], -u[k] * sn[k]);
      xu[k] = fmaf(u[k], cs[k], l[k] * sn[k]);
    }
    if (norm) {
      float ss = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) ss = fmaf(xl[k], xl[k], fmaf(xu[k], xu[k], ss));
      const float r = rsqrtf(L.head_sum(ss) * (1.0f / D) + a.eps);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        xl[k] = wl[k] * (xl[k] * r);
        xu[k] = wh[k] * (xu[k] * r);
      }
    }
    __nv_bfloat16* dst = a.dst + ((int64_t(b) * a.H + h) * S + s) * D;
    *reinterpret_cast<uint4*>(dst + L.c * 8) = pack8_bf16(xl);
    *reinterpret_cast<uint4*>(dst + D / 2 + L.c * 8) = pack8_bf16(xu);
  }
}

// NORM: the QK RMSNorm is applied (every part has weights); a separate
// instantiation keeps the plain rotation's register budget small.
template <int D, bool NORM>
__global__ void __launch_bounds__(256, NORM ? 2 : 3) rope_rotate_kernel(RotateArgs a) {
  const int lane = threadIdx.x & 31;
  const RowLanes<D> L(lane);
  const int n_rows = a.B * a.S;
  // grid-stride over (b, s) rows: a fixed grid of resident warps, no partial last wave
  for (int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; warp < n_rows; warp += (gridDim.x * blockDim.x) >> 5) {
    const int b = warp / a.S, s = warp % a.S;
    const SampleDev t = a.samples[b];
    if (s >= t.rows) {  // packed layout: the sample has no row s; keep the slab finite
      for (int p = 0; p < a.n_parts; ++p)
        for (int h = L.hs; h < a.part[p].H; h += RowLanes<D>::HPI) {
          __nv_bfloat16* dst = a.part[p].dst + ((int64_t(b) * a.part[p].H + h) * a.S + s) * D;
          *reinterpret_cast<uint4*>(dst + L.c * 8) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(dst + D / 2 + L.c * 8) = make_uint4(0, 0, 0, 0);
        }
      continue;
    }
    float cs[8], sn[8];
    load8(a.cos_t + (int64_t(b) * a.S + s) * D + L.c * 8, cs);
    load8(a.sin_t + (int64_t(b) * a.S + s) * D + L.c * 8, sn);
#pragma unroll
    for (int p = 0; p < 2; ++p)
      if (p < a.n_parts) rotate_part<D, NORM>(a.part[p], L, b, s, a.S, t, cs, sn);
  }
}

// Gradient epilogue for dq (and, with the QK RMSNorm, dk): for every row,
// v = scale * acc[b][h][s][:] is the gradient with respect to the attention's
// input row y.  Without the norm y = R x_in and the result is R^T v.  With it,
// y = w * xh, xh = x r, x = R x_in, r = 1/sqrt(mean(x^2) + eps): the gradient
// with respect to x is r (w v - xh <w v, xh> / D), then R^T; the weight
// gradient w += v * xh is summed per block into dw_part[blockIdx.x][:] in a
// fixed order (deterministic), and dw_reduce_kernel adds the blocks.
template <int D, bool NORM>
__global__ void __launch_bounds__(256, NORM ? 2 : 4) grad_finalize_kernel(GradFinalArgs a) {
  constexpr int CPH = RowLanes<D>::CPH, HPI = RowLanes<D>::HPI;
  __shared__ float red[8][32][16];
  const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const RowLanes<D> L(lane);
  constexpr bool norm = NORM;
  float dwl[8], dwh[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) dwl[k] = dwh[k] = 0.f;
  // grid-stride over (b, s) rows; which rows a block takes depends only on
  // (B, S), so its weight-gradient partial is summed in a fixed order
  for (int warp = blockIdx.x * 8 + wib; warp < a.B * a.S; warp += gridDim.x * 8) {
  const int b = warp / a.S, s = warp % a.S;
  if (s < a.samples[b].rows) {
    const int off = a.samples[b].off;
    float cs[8], sn[8], wl[8], wh[8];
    load8(a.cos_t + (int64_t(b) * a.S + s) * D + L.c * 8, cs);
    load8(a.sin_t + (int64_t(b) * a.S + s) * D + L.c * 8, sn);
    if (norm) {
      load8(a.w + L.c * 8, wl);
      load8(a.w + D / 2 + L.c * 8, wh);
    }
    for (int h = L.hs; h < a.H; h += HPI) {
      const float* src = a.acc + ((int64_t(b) * a.H + h) * a.S_pad + s) * D;
      float vl[8], vu[8];
      *reinterpret_cast<float4*>(vl) = *reinterpret_cast<const float4*>(src + L.c * 8);
      *reinterpret_cast<float4*>(vl + 4) = *reinterpret_cast<const float4*>(src + L.c * 8 + 4);
      *reinterpret_cast<float4*>(vu) = *reinterpret_cast<const float4*>(src + D / 2 + L.c * 8);
      *reinterpret_cast<float4*>(vu + 4) = *reinterpret_cast<const float4*>(src + D / 2 + L.c * 8 + 4);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        vl[k] *= a.scale;
        vu[k] *= a.scale;
      }
      if (norm) {
        const int64_t xo = int64_t(b) * a.x_sb + int64_t(off + s) * a.x_ss + int64_t(h / a.g) * a.x_shkv +
                           int64_t(h % a.g) * a.x_shq;
        const __nv_bfloat16* xin = reinterpret_cast<const __nv_bfloat16*>(a.x) + xo;
        float l[8], u[8], xl[8], xu[8];
        load8_bf16(xin + L.c * 8, l);
        load8_bf16(xin + D / 2 + L.c * 8, u);
        float ss = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          xl[k] = fmaf(l[k], cs[k], -u[k] * sn[k]);
          xu[k] = fmaf(u[k], cs[k], l[k] * sn[k]);
          ss = fmaf(xl[k], xl[k], fmaf(xu[k], xu[k], ss));
        }
        const float r = rsqrtf(L.head_sum(ss) * (1.0f / D) + a.eps);
        float dot = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          xl[k] *= r;  // xh
          xu[k] *= r;
          dwl[k] = fmaf(vl[k], xl[k], dwl[k]);
          dwh[k] = fmaf(vu[k], xu[k], dwh[k]);
          vl[k] *= wl[k];  // w v
          vu[k] *= wh[k];
          dot = fmaf(vl[k], xl[k], fmaf(vu[k], xu[k], dot));
        }
        const float m = L.head_sum(dot) * (1.0f / D);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          vl[k] = r * fmaf(-xl[k], m, vl[k]);
          vu[k] = r * fmaf(-xu[k], m, vu[k]);
        }
      }
      float ol[8], ou[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        ol[k] = fmaf(vl[k], cs[k], vu[k] * sn[k]);   // (R^T v)_j
        ou[k] = fmaf(vu[k], cs[k], -vl[k] * sn[k]);  // (R^T v)_{j+D/2}
      }
      const int64_t so = int64_t(b) * a.dst_sb + int64_t(off + s) * a.dst_ss + int64_t(h / a.g) * a.dst_shkv +
                         int64_t(h % a.g) * a.dst_shq;
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.dst) + so;
      *reinterpret_cast<uint4*>(dst + L.c * 8) = pack8_bf16(ol);
      *reinterpret_cast<uint4*>(dst + D / 2 + L.c * 8) = pack8_bf16(ou);
    }
  }
  }
  if (!norm) return;  // uniform across the block
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    red[wib][lane][k] = dwl[k];
    red[wib][lane][8 + k] = dwh[k];
  }
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    const int j = d % (D / 2), c = j / 8, k = (j % 8) + (d >= D / 2 ? 8 : 0);
    float t = 0.f;
    for (int w8 = 0; w8 < 8; ++w8)
      for (int h2 = 0; h2 < HPI; ++h2) t += red[w8][c + CPH * h2][k];
    a.dw_part[int64_t(blockIdx.x) * D + d] = t;
  }
}

// dw[d] = sum over blocks of dw_part[blk][d]: 32 channels x 32 block rows per
// CTA, a fixed strided split and a fixed tree (deterministic).
__global__ void __launch_bounds__(1024) dw_reduce_kernel(const float* __restrict__ part, int nblk, int D,
                                                         float* __restrict__ dw) {
  __shared__ float t[32][33];
  const int cx = threadIdx.x & 31, ry = threadIdx.x >> 5;
  const int d = blockIdx.x * 32 + cx;
  float s = 0.f;
  if (d < D)
    for (int i = ry; i < nblk; i += 32) s += part[int64_t(i) * D + d];
  t[ry][cx] = s;
  __syncthreads();
  for (int o = 16; o > 0; o >>= 1) {
    if (ry < o) t[ry][cx] += t[ry + o][cx];
    __syncthreads();
  }
  if (ry == 0 && d < D) dw[d] = t[0][cx];
}

// Blocks of the row-per-warp kernels: 8 warps each, one warp per row (the
// kernels' grid-stride loops then run once; the hardware block scheduler
// balances the rows).
int row_grid_blocks(int64_t rows) { return int((rows + 7) / 8); }

void launch_rope2d_tables(const SampleDev* samples, const ImageDev* images, int B, int S, int D, double base,
                          float* cos_out, float* sin_out, cudaStream_t st) {
  const int64_t rows = int64_t(B) * S;
  if (rows == 0) return;
  // one row per warp: rows < 2^31 (checked by the caller), so fewer than 2^28 blocks
  prof_begin(kRopeTables, st);
  rope2d_tables_kernel<<<row_grid_blocks(rows), 256, 0, st>>>(samples, images, B, S, D, base, cos_out, sin_out);
  prof_end(kRopeTables, st);
}

void launch_rope_rotate(const RotateArgs& a, int D, cudaStream_t st) {
  const int64_t warps = int64_t(a.B) * a.S;
  if (warps == 0) return;
  const int blocks = row_grid_blocks(warps);
  prof_begin(kRopeRotate, st);
  const bool norm = a.part[0].w != nullptr;
  if (D == 128) {
    if (norm) rope_rotate_kernel<128, true><<<blocks, 256, 0, st>>>(a);
    else rope_rotate_kernel<128, false><<<blocks, 256, 0, st>>>(a);
  } else {
    if (norm) rope_rotate_kernel<64, true><<<blocks, 256, 0, st>>>(a);
    else rope_rotate_kernel<64, false><<<blocks, 256, 0, st>>>(a);
  }
  prof_end(kRopeRotate, st);
}

int grad_finalize_blocks(int B, int S) { return row_grid_blocks(int64_t(B) * S); }

void launch_grad_finalize(const GradFinalArgs& a, int D, cudaStream_t st) {
  const int blocks = grad_finalize_blocks(a.B, a.S);
  if (blocks == 0) return;
  prof_begin(kGradFinalize, st);
  const bool norm = a.w != nullptr;
  if (D == 128) {
    if (norm) grad_finalize_kernel<128, true><<<blocks, 256, 0, st>>>(a);
    else grad_finalize_kernel<128, false><<<blocks, 256, 0, st>>>(a);
  } else {
    if (norm) grad_finalize_kernel<64, true><<<blocks, 256, 0, st>>>(a);
    else grad_finalize_kernel<64, false><<<blocks, 256, 0, st>>>(a);
  }
  prof_end(kGradFinalize, st);
}

void launch_dw_reduce(const float* part, int nblk, int D, float* dw, cudaStream_t st) {
  prof_begin(kDwReduce, st);
  dw_reduce_kernel<<<(D + 31) / 32, 1024, 0, st>>>(part, nblk, D, dw);
  prof_end(kDwReduce, st);
}

}  // namespace hia
