// host_step.cpp -- one training step of the attention from host buffers.
//
// A hia_step owns the device copies of one step's tensors (contiguous
// [B, S, heads, D] bf16, lse [B, Hq, S] fp32), the RoPE tables of its segment
// descriptor and both workspaces.  hia_attn_step_host enqueues, on the
// caller's stream: the host->device copies of q, k, v, the forward, the
// backward and the device->host copies of dq, dk, dv.  dout is uploaded and
// o, lse are downloaded on the step's own copy stream, so those copies run
// under the forward and the backward.  The caller's stream waits for the copy
// stream before its next operation, so its completion covers every copy.
#include <cuda_runtime.h>

#include "internal.h"

struct hia_step {
  const hia_segments* seg = nullptr;
  int Hq = 0, Hkv = 0, D = 0;
  size_t q_bytes = 0, kv_bytes = 0, lse_bytes = 0;
  void* q = nullptr;
  void* k = nullptr;
  void* v = nullptr;
  void* dout = nullptr;
  void* o = nullptr;
  float* lse = nullptr;
  void* dq = nullptr;
  void* dk = nullptr;
  void* dv = nullptr;
  float* cos_t = nullptr;
  float* sin_t = nullptr;
  void* ws_fwd = nullptr;
  size_t ws_fwd_bytes = 0;
  void* ws_bwd = nullptr;
  size_t ws_bwd_bytes = 0;
  cudaStream_t copy = nullptr;
  cudaEvent_t ev_start = nullptr, ev_fwd = nullptr, ev_dout = nullptr, ev_copy_done = nullptr;
};

namespace {

void release(hia_step* st) {
  void* bufs[] = {st->q, st->k, st->v, st->dout, st->o, st->lse, st->dq, st->dk, st->dv,
                  st->cos_t, st->sin_t, st->ws_fwd, st->ws_bwd};
  for (void* p : bufs)
    if (p) cudaFree(p);
  cudaEvent_t evs[] = {st->ev_start, st->ev_fwd, st->ev_dout, st->ev_copy_done};
  for (cudaEvent_t e : evs)
    if (e) cudaEventDestroy(e);
  if (st->copy) cudaStreamDestroy(st->copy);
  delete st;
}

// contiguous [B, S, heads, D]; for q-head tensors head h = (h / g, h % g)
hia_tensor dense(void* p, int S, int heads, int D, int g) {
  hia_tensor t;
  t.ptr = p;
  t.stride_b = int64_t(S) * heads * D;
  t.stride_s = int64_t(heads) * D;
  t.stride_hkv = int64_t(g) * D;
  t.stride_hq = g > 1 ? D : 0;
  return t;
}

int cuda_ok(cudaError_t e) { return e == cudaSuccess ? HIA_OK : HIA_ERR_CUDA; }

}  // namespace

extern "C" int hia_step_create(const hia_segments* seg, int Hq, int Hkv, int D, double rope_base,
                               hia_step** out) {
  if (!seg || !out || Hq <= 0 || Hkv <= 0 || !(rope_base > 0)) return HIA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0 || (D != 64 && D != 128)) return HIA_ERR_UNSUPPORTED;
  if (seg->packed) return HIA_ERR_UNSUPPORTED;  // the step's buffers use the padded layout
  if (!seg->dbuf) return HIA_ERR_NOT_ON_DEVICE;
  *out = nullptr;
  hia_step* st = new hia_step;
  st->seg = seg;
  st->Hq = Hq;
  st->Hkv = Hkv;
  st->D = D;
  const size_t BS = size_t(seg->B) * seg->S;
  st->q_bytes = BS * Hq * D * 2;
  st->kv_bytes = BS * Hkv * D * 2;
  st->lse_bytes = BS * Hq * 4;
  st->ws_fwd_bytes = hia_attn_fwd_workspace_bytes(seg, Hq, Hkv, D);
  st->ws_bwd_bytes = hia_attn_bwd_workspace_bytes(seg, Hq, Hkv, D);
  bool ok = cudaMalloc(&st->q, st->q_bytes) == cudaSuccess && cudaMalloc(&st->k, st->kv_bytes) == cudaSuccess &&
            cudaMalloc(&st->v, st->kv_bytes) == cudaSuccess && cudaMalloc(&st->dout, st->q_bytes) == cudaSuccess &&
            cudaMalloc(&st->o, st->q_bytes) == cudaSuccess &&
            cudaMalloc(reinterpret_cast<void**>(&st->lse), st->lse_bytes) == cudaSuccess &&
            cudaMalloc(&st->dq, st->q_bytes) == cudaSuccess && cudaMalloc(&st->dk, st->kv_bytes) == cudaSuccess &&
            cudaMalloc(&st->dv, st->kv_bytes) == cudaSuccess &&
            cudaMalloc(reinterpret_cast<void**>(&st->cos_t), BS * D * 4) == cudaSuccess &&
            cudaMalloc(reinterpret_cast<void**>(&st->sin_t), BS * D * 4) == cudaSuccess &&
            cudaMalloc(&st->ws_fwd, st->ws_fwd_bytes > 0 ? st->ws_fwd_bytes : 1) == cudaSuccess &&
            cudaMalloc(&st->ws_bwd, st->ws_bwd_bytes > 0 ? st->ws_bwd_bytes : 1) == cudaSuccess &&
            cudaStreamCreateWithFlags(&st->copy, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&st->ev_start, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&st->ev_fwd, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&st->ev_dout, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&st->ev_copy_done, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    release(st);
    return HIA_ERR_CUDA;
  }
  // the RoPE tables depend only on the segments: compute them once
  int rc = hia_rope2d_tables(seg, D, rope_base, st->cos_t, st->sin_t, st->copy);
  if (rc == HIA_OK) rc = cuda_ok(cudaStreamSynchronize(st->copy));
  if (rc != HIA_OK) {
    release(st);
    return rc;
  }
  *out = st;
  return HIA_OK;
}

extern "C" void hia_step_destroy(hia_step* st) {
  if (!st) return;
  cudaStreamSynchronize(st->copy);
  release(st);
}

extern "C" int hia_attn_step_host(hia_step* st, const void* q, const void* k, const void* v, const void* dout,
                                  float scale, void* o, float* lse, void* dq, void* dk, void* dv, void* stream) {
  if (!st || !q || !k || !v || !dout || !o || !lse || !dq || !dk || !dv) return HIA_ERR_INVALID_ARG;
  const hia_segments* seg = st->seg;
  const int S = seg->S, Hq = st->Hq, Hkv = st->Hkv, D = st->D, g = Hq / Hkv;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaStream_t c = st->copy;
  const hia_tensor tq = dense(st->q, S, Hq, D, g), tk = dense(st->k, S, Hkv, D, 1), tv = dense(st->v, S, Hkv, D, 1);
  const hia_tensor to = dense(st->o, S, Hq, D, g), tdo = dense(st->dout, S, Hq, D, g);
  const hia_tensor tdq = dense(st->dq, S, Hq, D, g), tdk = dense(st->dk, S, Hkv, D, 1),
                   tdv = dense(st->dv, S, Hkv, D, 1);
  // the copy stream starts after everything already queued on the caller's
  // stream (a previous step's use of these buffers included)
  if (cudaEventRecord(st->ev_start, s) != cudaSuccess || cudaStreamWaitEvent(c, st->ev_start, 0) != cudaSuccess)
    return HIA_ERR_CUDA;
  int rc = cuda_ok(cudaMemcpyAsync(st->q, q, st->q_bytes, cudaMemcpyHostToDevice, s));
  if (rc == HIA_OK) rc = cuda_ok(cudaMemcpyAsync(st->k, k, st->kv_bytes, cudaMemcpyHostToDevice, s));
  if (rc == HIA_OK) rc = cuda_ok(cudaMemcpyAsync(st->v, v, st->kv_bytes, cudaMemcpyHostToDevice, s));
  // dout is needed only by the backward: upload it under the forward
  if (rc == HIA_OK) rc = cuda_ok(cudaMemcpyAsync(st->dout, dout, st->q_bytes, cudaMemcpyHostToDevice, c));
  if (rc == HIA_OK) rc = cuda_ok(cudaEventRecord(st->ev_dout, c));
  if (rc == HIA_OK)
    rc = hia_attn_fwd(seg, Hq, Hkv, D, tq, tk, tv, st->cos_t, st->sin_t, scale, to, st->lse, st->ws_fwd,
                      st->ws_fwd_bytes, s);
  // o and lse go down under the backward
  if (rc == HIA_OK) rc = cuda_ok(cudaEventRecord(st->ev_fwd, s));
  if (rc == HIA_OK) rc = cuda_ok(cudaStreamWaitEvent(c, st->ev_fwd, 0));
  if (rc == HIA_OK) rc = cuda_ok(cudaMemcpyAsync(o, st->o, st->q_bytes, cudaMemcpyDeviceToHost, c));
  if (rc == HIA_OK) rc = cuda_ok(cudaMemcpyAsync(lse, st->lse, st->lse_bytes, cudaMemcpyDeviceToHost, c));
  if (rc == HIA_OK) rc = cuda_ok(cudaStreamWaitEvent(s, st->ev_dout, 0));
  if (rc == HIA_OK)
    // the backward reads the rotated q and k the forward left in its workspace
    rc = hia_attn_bwd_reuse_fwd(seg, Hq, Hkv, D, tq, tk, tv, st->cos_t, st->sin_t, scale, nullptr, to, st->lse,
                                tdo, tdq, tdk, tdv, nullptr, nullptr, st->ws_fwd, st->ws_fwd_bytes, st->ws_bwd,
                                st->ws_bwd_bytes, s);
  if (rc == HIA_OK) rc = cuda_ok(cudaMemcpyAsync(dq, st->dq, st->q_bytes, cudaMemcpyDeviceToHost, s));
  if (rc == HIA_OK) rc = cuda_ok(cudaMemcpyAsync(dk, st->dk, st->kv_bytes, cudaMemcpyDeviceToHost, s));
  if (rc == HIA_OK) rc = cuda_ok(cudaMemcpyAsync(dv, st->dv, st->kv_bytes, cudaMemcpyDeviceToHost, s));
  // the caller's stream completes only after the copy stream's work
  if (cudaEventRecord(st->ev_copy_done, c) != cudaSuccess || cudaStreamWaitEvent(s, st->ev_copy_done, 0) != cudaSuccess)
    return HIA_ERR_CUDA;
  return rc;
}
