// devctx.h -- per-device, per-context host state of the library.
//
// Some host state belongs to one CUDA context: the device address of a
// __device__ variable, or a kernel attribute set with cudaFuncSetAttribute.
// A process can lose a context (cudaDeviceReset) and get a new one on the
// same device, where the old values are stale.  PerContext<T> keeps one value
// per device, tagged with the identity of the context it was computed in, and
// computes it again when the current context is a different one.
#pragma once
#include <cuda_runtime.h>

#include <mutex>

namespace hia {

// Identity of the context current on the calling thread (unique for the life
// of the process: a context created after cudaDeviceReset gets a new one), or
// 0 if no context is current yet.
unsigned long long current_context_id();

template <class T>
class PerContext {
 public:
  // The value for the current device and context; `make(T*)` (returning a
  // cudaError_t) computes it the first time, and again after a context change.
  template <class F>
  cudaError_t get(T* out, F make) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu_);
    unsigned long long id = current_context_id();
    if (id != 0 && slot_[dev].ctx == id) {
      *out = slot_[dev].value;
      return cudaSuccess;
    }
    T v{};
    const cudaError_t e = make(&v);
    if (e != cudaSuccess) return e;
    id = current_context_id();  // make() may have created the context
    slot_[dev].ctx = id;
    slot_[dev].value = v;
    *out = v;
    return cudaSuccess;
  }

 private:
  static constexpr int kMaxDevices = 64;
  struct Slot {
    unsigned long long ctx = 0;
    T value{};
  };
  std::mutex mu_;
  Slot slot_[kMaxDevices];
};

}  // namespace hia
