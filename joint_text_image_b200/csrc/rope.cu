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

#include "internal.h"
#include "kernels.h"

namespace hia {

// K1: one thread per (b, n, j < D/2).  Angle and cos/sin in fp64, rounded
// once to fp32: a text-only sample reproduces the 1D tables exactly.
__global__ void rope2d_tables_kernel(const SampleDev* __restrict__ samples, int B, int S, int D, double base,
                                     float* __restrict__ cos_out, float* __restrict__ sin_out) {
  const int half = D / 2;
  const int64_t total = int64_t(B) * S * half;
  for (int64_t idx = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; idx < total;
       idx += int64_t(gridDim.x) * blockDim.x) {
    const int j = int(idx % half);
    const int64_t bn = idx / half;
    const int n = int(bn % S);
    const int b = int(bn / S);
    const SampleDev t = samples[b];
    double x = n, y = n;
    if (n >= t.I0 && n < t.I1) {
      const int i = n - t.I0;
      x = double(t.I0 + i % t.w);
      y = double(t.I0 + i / t.w);
    }
    const double theta = pow(base, -2.0 * double(j) / double(D));
    const double a = ((j & 1) ? y : x) * theta;
    double sn, cs;
    sincos(a, &sn, &cs);
    const int64_t o = bn * D + j;
    cos_out[o] = float(cs);
    cos_out[o + half] = float(cs);
    sin_out[o] = float(sn);
    sin_out[o + half] = float(sn);
  }
}

// Rotation pre-pass: dst[b][h][s][:] = R(b,s) src[b,s,h,:] in fp32, rounded
// to bf16.  One warp per (b, s): each lane owns 8 channels of the low half
// and the matching 8 of the high half of one head; the cos/sin of the row are
// read once and reused for every head.  inverse = 1 applies R^T instead and
// reads fp32 input (used for dq).
template <int D>
__global__ void __launch_bounds__(256) rope_rotate_kernel(RotateArgs a) {
  constexpr int CPH = D / 16;  // 8-channel chunks per half-head
  constexpr int HPI = 32 / CPH;  // heads per warp iteration
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= a.B * a.S) return;
  const int b = warp / a.S, s = warp % a.S;
  const int c = lane % CPH, hs = lane / CPH;
  const float* cp = a.cos_t + (int64_t(b) * a.S + s) * D + c * 8;
  const float* sp = a.sin_t + (int64_t(b) * a.S + s) * D + c * 8;
  const float4 c0 = __ldg(reinterpret_cast<const float4*>(cp)), c1 = __ldg(reinterpret_cast<const float4*>(cp) + 1);
  const float4 s0 = __ldg(reinterpret_cast<const float4*>(sp)), s1 = __ldg(reinterpret_cast<const float4*>(sp) + 1);
  const float cs[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const float sn[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  for (int h = hs; h < a.H; h += HPI) {
    const int64_t so = int64_t(b) * a.src_sb + int64_t(s) * a.src_ss + int64_t(h / a.g) * a.src_shkv +
                       int64_t(h % a.g) * a.src_shq;
    const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(a.src) + so;
    const uint4 lo4 = *reinterpret_cast<const uint4*>(src + c * 8);
    const uint4 hi4 = *reinterpret_cast<const uint4*>(src + D / 2 + c * 8);
    const __nv_bfloat162* lo2 = reinterpret_cast<const __nv_bfloat162*>(&lo4);
    const __nv_bfloat162* hi2 = reinterpret_cast<const __nv_bfloat162*>(&hi4);
    uint4 olo, ohi;
    __nv_bfloat162* ol = reinterpret_cast<__nv_bfloat162*>(&olo);
    __nv_bfloat162* oh = reinterpret_cast<__nv_bfloat162*>(&ohi);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 l = __bfloat1622float2(lo2[i]);
      const float2 u = __bfloat1622float2(hi2[i]);
      const float cA = cs[2 * i], cB = cs[2 * i + 1], sA = sn[2 * i], sB = sn[2 * i + 1];
      const float nlA = fmaf(l.x, cA, -u.x * sA), nlB = fmaf(l.y, cB, -u.y * sB);
      const float nuA = fmaf(u.x, cA, l.x * sA), nuB = fmaf(u.y, cB, l.y * sB);
      ol[i] = __floats2bfloat162_rn(nlA, nlB);
      oh[i] = __floats2bfloat162_rn(nuA, nuB);
    }
    __nv_bfloat16* dst = a.dst + ((int64_t(b) * a.H + h) * a.S + s) * D;
    *reinterpret_cast<uint4*>(dst + c * 8) = olo;
    *reinterpret_cast<uint4*>(dst + D / 2 + c * 8) = ohi;
  }
}

// dq epilogue: dq[b,s,h,:] = R(b,s)^T (scale * acc[b][h][s][:]) in fp32,
// rounded to bf16 and written with the caller's strides.
template <int D>
__global__ void __launch_bounds__(256) dq_finalize_kernel(DqFinalArgs a) {
  constexpr int CPH = D / 16;
  constexpr int HPI = 32 / CPH;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= a.B * a.S) return;
  const int b = warp / a.S, s = warp % a.S;
  const int c = lane % CPH, hs = lane / CPH;
  const float* cp = a.cos_t + (int64_t(b) * a.S + s) * D + c * 8;
  const float* sp = a.sin_t + (int64_t(b) * a.S + s) * D + c * 8;
  const float4 c0 = __ldg(reinterpret_cast<const float4*>(cp)), c1 = __ldg(reinterpret_cast<const float4*>(cp) + 1);
  const float4 s0 = __ldg(reinterpret_cast<const float4*>(sp)), s1 = __ldg(reinterpret_cast<const float4*>(sp) + 1);
  const float cs[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const float sn[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  for (int h = hs; h < a.H; h += HPI) {
    const float* src = a.acc + ((int64_t(b) * a.H + h) * a.S_pad + s) * D;
    float lo[8], hi[8];
    *reinterpret_cast<float4*>(lo) = *reinterpret_cast<const float4*>(src + c * 8);
    *reinterpret_cast<float4*>(lo + 4) = *reinterpret_cast<const float4*>(src + c * 8 + 4);
    *reinterpret_cast<float4*>(hi) = *reinterpret_cast<const float4*>(src + D / 2 + c * 8);
    *reinterpret_cast<float4*>(hi + 4) = *reinterpret_cast<const float4*>(src + D / 2 + c * 8 + 4);
    uint4 olo, ohi;
    __nv_bfloat162* ol = reinterpret_cast<__nv_bfloat162*>(&olo);
    __nv_bfloat162* oh = reinterpret_cast<__nv_bfloat162*>(&ohi);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float r[4];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k = 2 * i + e;
        const float l = lo[k] * a.scale, u = hi[k] * a.scale;
        r[e] = fmaf(l, cs[k], u * sn[k]);        // (R^T v)_j
        r[2 + e] = fmaf(u, cs[k], -l * sn[k]);   // (R^T v)_{j+D/2}
      }
      ol[i] = __floats2bfloat162_rn(r[0], r[1]);
      oh[i] = __floats2bfloat162_rn(r[2], r[3]);
    }
    const int64_t so = int64_t(b) * a.dst_sb + int64_t(s) * a.dst_ss + int64_t(h / a.g) * a.dst_shkv +
                       int64_t(h % a.g) * a.dst_shq;
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.dst) + so;
    *reinterpret_cast<uint4*>(dst + c * 8) = olo;
    *reinterpret_cast<uint4*>(dst + D / 2 + c * 8) = ohi;
  }
}

void launch_rope2d_tables(const SampleDev* samples, int B, int S, int D, double base, float* cos_out,
                          float* sin_out, cudaStream_t st) {
  const int64_t total = int64_t(B) * S * (D / 2);
  if (total == 0) return;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 64) blocks = 148 * 64;
  prof_begin(kRopeTables, st);
  rope2d_tables_kernel<<<int(blocks), threads, 0, st>>>(samples, B, S, D, base, cos_out, sin_out);
  prof_end(kRopeTables, st);
}

void launch_rope_rotate(const RotateArgs& a, int D, cudaStream_t st) {
  const int64_t warps = int64_t(a.B) * a.S;
  if (warps == 0) return;
  const int blocks = int((warps + 7) / 8);
  prof_begin(kRopeRotate, st);
  if (D == 128) rope_rotate_kernel<128><<<blocks, 256, 0, st>>>(a);
  else rope_rotate_kernel<64><<<blocks, 256, 0, st>>>(a);
  prof_end(kRopeRotate, st);
}

void launch_dq_finalize(const DqFinalArgs& a, int D, cudaStream_t st) {
  const int64_t warps = int64_t(a.B) * a.S;
  if (warps == 0) return;
  const int blocks = int((warps + 7) / 8);
  prof_begin(kDqFinalize, st);
  if (D == 128) dq_finalize_kernel<128><<<blocks, 256, 0, st>>>(a);
  else dq_finalize_kernel<64><<<blocks, 256, 0, st>>>(a);
  prof_end(kDqFinalize, st);
}

}  // namespace hia
