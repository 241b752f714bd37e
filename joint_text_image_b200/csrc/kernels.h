// kernels.h -- argument blocks and launchers of the device kernels.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"

namespace hia {

// One tensor of the rotation pre-pass: src rows rotated (and optionally
// RMS-normed) into dst.
struct RotatePart {
  const void* src;  // bf16 [B,S,heads,D] with strides (elements)
  int64_t src_sb, src_ss, src_shkv, src_shq;
  int g;            // heads per stride_hkv group (1 for k)
  int H;            // heads
  const float* w;   // QK RMSNorm weight [D], or nullptr: no norm
  float eps;
  __nv_bfloat16* dst;  // [B][H][S][D]
};

struct RotateArgs {
  const SampleDev* samples;  // rows / off of every sample (layout of src)
  const float* cos_t;
  const float* sin_t;
  RotatePart part[2];        // q and k, rotated by one launch
  int n_parts;
  int B, S;
};

struct GradFinalArgs {
  const SampleDev* samples;  // rows / off of every sample (layout of x and dst)
  const float* acc;  // fp32 [B][H][S_pad][D]: gradient w.r.t. the attention's input rows (times 1/scale)
  int S_pad;
  float scale;
  const float* cos_t;
  const float* sin_t;
  const void* x;     // the layer input rows (q or k), bf16 with strides; read only with the norm
  int64_t x_sb, x_ss, x_shkv, x_shq;
  const float* w;    // QK RMSNorm weight [D], or nullptr: no norm
  float eps;
  float* dw_part;    // [grad_finalize_blocks][D] per-block weight-gradient partials (with the norm)
  void* dst;         // bf16 with strides
  int64_t dst_sb, dst_ss, dst_shkv, dst_shq;
  int g;
  int B, S, H;
};

struct FwdParams {
  const SampleDev* samples;
  const ImageDev* images;
  const int32_t* tiles;  // [B][nQT][2]: (first entry of list, count)
  const int32_t* list;   // kv tile entries kt | FULL << 16
  const int32_t* work;   // [n_work][2]
  int B, S, Hq, Hkv, g, nQT, n_hp;
  __nv_bfloat16* o;
  int64_t o_sb, o_ss, o_shkv, o_shq;
  float* lse;        // element b * lse_sb + h * lse_sh + off + q
  int64_t lse_sb, lse_sh;
  int packed;        // 1: V is a packed tensor map (row = off + s, batch coordinate 0)
  float scale_log2;  // softmax scale * log2(e)
  int* status;
  uint64_t timeout_ns;
};

struct BwdPreParams {
  const __nv_bfloat16* o;
  int64_t o_sb, o_ss, o_shkv, o_shq;
  const __nv_bfloat16* dout;
  int64_t d_sb, d_ss, d_shkv, d_shq;
  const SampleDev* samples;
  const float* lse;     // element b * lse_sb + h * lse_sh + off + q
  int64_t lse_sb, lse_sh;
  float* lse2;          // [B][Hq][S_pad]: lse * log2(e); +inf beyond S
  float* delta;         // [B][Hq][S_pad]: rowsum(dout * o); 0 beyond S
  float* dq_acc;        // [B][Hq][S_pad][D]: zeroed by this pass
  int* part_cnt;        // [n_cnt] split-schedule tickets: zeroed by this pass
  int n_cnt;
  int B, S, S_pad, Hq, g, D;
};

struct BwdParams {
  const SampleDev* samples;
  const ImageDev* images;
  const int32_t* tiles;  // [B][bKT][4]: (qt_first, qt_end, full_first, full_end)
  const int32_t* work;   // [n_work][kBwdWorkInts]: (b, kt, qt_lo, qt_hi, slot, part, parts, 0)
  float* part;           // split tiles' fp32 partials [slot][Hkv][part < parts][dK, dV][D / 4][128] float4
  int* part_cnt;         // [slot][Hkv] tickets (zeroed by bwd_pre)
  int B, S, S_pad, Hq, Hkv, g, bQT, bKT;
  const float* lse2;
  const float* delta;
  float* dq_acc;
  const float* cos_t;
  const float* sin_t;
  __nv_bfloat16* dk;
  int64_t dk_sb, dk_ss, dk_sh;
  float* dk_acc;      // non-null (QK RMSNorm): write scale * dK_n rows fp32 [B][Hkv][S_pad][D] here instead of dk
  int packed;         // 1: V and dO are packed tensor maps (row = off + s, batch coordinate 0)
  __nv_bfloat16* dv;
  int64_t dv_sb, dv_ss, dv_sh;
  float scale;        // softmax scale
  float scale_log2;   // scale * log2(e)
  int* status;
  uint64_t timeout_ns;
};

// 2D bf16 tensor map [rows][cols] (row stride in bytes, a multiple of 16),
// 128-byte swizzle, box box_rows x box_cols (box_cols * 2 = 128 bytes).
bool make_map_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t row_stride_bytes,
                 uint32_t box_cols, uint32_t box_rows);

// Host-side argument checks of the forward (everything but the workspace):
// HIA_OK, or the status hia_attn_fwd_ex would return for these arguments.
int fwd_check_args(const hia_segments* g, int Hq, int Hkv, int D, const hia_tensor& q, const hia_tensor& k,
                   const hia_tensor& v, const float* c, const float* s, float scale, const hia_qk_norm* norm,
                   const hia_tensor& o, const float* lse);

// Profiling brackets around one kernel launch (no-ops unless profiling is on).
enum KernelId {
  kRopeTables = 0, kRopeRotate, kAttnFwd, kBwdPre, kAttnBwd, kGradFinalize, kDwReduce,
  kMoePrep, kMoeRouter, kMoeScan, kMoeGather, kMoeUpGate, kMoeDown, kMoeCombine, kNumKernels
};
void prof_begin(KernelId id, cudaStream_t st);
void prof_end(KernelId id, cudaStream_t st);

void launch_rope2d_tables(const SampleDev* samples, const ImageDev* images, int B, int S, int D, double base,
                          float* cos_out,
                          float* sin_out, cudaStream_t st);
void launch_rope_rotate(const RotateArgs& a, int D, cudaStream_t st);
int grad_finalize_blocks(int B, int S);
void launch_grad_finalize(const GradFinalArgs& a, int D, cudaStream_t st);
void launch_dw_reduce(const float* part, int nblk, int D, float* dw, cudaStream_t st);
cudaError_t launch_attn_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, int n_blocks, int D, cudaStream_t st);
cudaError_t launch_bwd_pre(const BwdPreParams& p, cudaStream_t st);
cudaError_t launch_attn_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, const BwdParams& p, int n_blocks, int D, cudaStream_t st);
cudaError_t launch_wait_probe(int* status, uint64_t timeout_ns, cudaStream_t st);
cudaError_t launch_exp2_probe(const float* x, float* y, int n, cudaStream_t st);

}  // namespace hia
