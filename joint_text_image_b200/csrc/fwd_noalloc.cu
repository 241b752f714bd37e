// fwd_noalloc.cu -- hia_attn_fwd_noalloc: the forward for callers that may not
// allocate device memory.
//
// Who needs it: code that runs inside a host runtime which owns every byte of
// device memory and hands a plug-in only its input and output buffers (no
// allocator, no workspace), and code that must not call cudaMalloc/cudaFree in
// the middle of a step because those calls synchronize the device and can
// stall every other stream.  hia_attn_fwd needs a caller-provided workspace
// for the RoPE-rotated q and k; this variant uses a fixed array compiled into
// the library instead and allocates nothing itself.
//
// The array is a file-scope __device__ variable of kScratchBytes (64 MiB).
// Every GPU that loads this part of the library holds it until the process
// exits.  In host code its name is only a host-side stand-in, so the device
// address is looked up with cudaGetSymbolAddress (with the device current)
// and passed to the kernels: once per device, and again if the device's
// context has been replaced (after cudaDeviceReset the old address is stale).
#include <cuda_runtime.h>

#include "devctx.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = size_t(64) << 20;  // 64 MiB

static __device__ __align__(256) unsigned char g_fwd_scratch[kScratchBytes];

// Device address of g_fwd_scratch in the current device's context.  The
// first lookup in a context also loads the module that holds the array,
// which is why the first call on each device should come before any stream
// capture.
int scratch_address(void** out) {
  static hia::PerContext<void*> cache;
  const cudaError_t e = cache.get(out, [](void** p) { return cudaGetSymbolAddress(p, g_fwd_scratch); });
  return (e == cudaSuccess && *out) ? HIA_OK : HIA_ERR_CUDA;
}

}  // namespace

extern "C" int hia_attn_fwd_noalloc(const hia_segments* seg, int Hq, int Hkv, int D, hia_tensor q, hia_tensor k,
                                    hia_tensor v, const float* cos_t, const float* sin_t, float scale,
                                    hia_tensor o, float* lse, void* stream) {
  // The same argument checks as hia_attn_fwd, in the same order, before the
  // size limit: a bad argument reports its own error.
  int rc = hia::fwd_check_args(seg, Hq, Hkv, D, q, k, v, cos_t, sin_t, scale, nullptr, o, lse);
  if (rc != HIA_OK) return rc;
  if (seg->B == 0 || seg->S == 0) return HIA_OK;
  // The scratch holds the rotated q and k (hia_attn_fwd's workspace).
  if (hia_attn_fwd_workspace_bytes(seg, Hq, Hkv, D) > kScratchBytes) return HIA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if ((rc = scratch_address(&scratch)) != HIA_OK) return rc;
  // Nothing in the scratch has to start at zero: the rotation pass rewrites
  // every element the attention kernel reads.  Calls share the array, so two
  // calls whose work overlaps on the GPU (different streams, or different
  // host threads without ordering) race on it; order them on one stream.
  return hia_attn_fwd(seg, Hq, Hkv, D, q, k, v, cos_t, sin_t, scale, o, lse, scratch, kScratchBytes, stream);
}
