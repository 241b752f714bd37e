// api.cu -- the C ABI of libjointattn: argument checks, device copies of the
// segment descriptor, TMA tensor maps, workspace layout and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <algorithm>
#include <functional>
#include <initializer_list>
#include <queue>
#include <cstring>
#include <mutex>

#include "devctx.h"
#include "kernels.h"

namespace hia {

unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext c = nullptr;
  if (get_current(&c) != CUDA_SUCCESS || !c) return 0;
  unsigned long long id = 0;
  return get_id(c, &id) == CUDA_SUCCESS ? id : 0;
}

}  // namespace hia

namespace {

using hia::SampleDev;

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per barrier wait

__device__ int g_status;  // per-device status word (HIA_OK or HIA_ERR_DEVICE_TIMEOUT)

// Device address of g_status in the current device's context.
int* status_ptr() {
  static hia::PerContext<int*> cache;
  int* p = nullptr;
  if (cache.get(&p, [](int** out) { return cudaGetSymbolAddress(reinterpret_cast<void**>(out), g_status); }) !=
      cudaSuccess)
    return nullptr;
  return p;
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

// bf16 tensor map with 128-byte swizzle and a box of 64 x rows along dims 0/`row_dim`.
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
              const uint32_t* box) {
  EncodeFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t d[5], s[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) s[i] = strides_bytes[i];
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cuuint32_t(rank), const_cast<void*>(base), d, s, bx, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

namespace hia {

int* device_status_word() { return status_ptr(); }

bool make_map_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t row_stride_bytes,
                 uint32_t box_cols, uint32_t box_rows) {
  uint64_t dims[2] = {cols, rows};
  uint64_t st[1] = {row_stride_bytes};
  uint32_t box[2] = {box_cols, box_rows};
  return make_map(m, base, 2, dims, st, box);
}

}  // namespace hia

namespace {

// [rows = S][D] per (b, head) slab of a [B*H][S][D] workspace tensor.
bool make_ws_map(CUtensorMap* m, const void* base, int D, int S, int BH, uint32_t rows = 128) {
  uint64_t dims[3] = {uint64_t(D), uint64_t(S), uint64_t(BH)};
  uint64_t st[2] = {uint64_t(D) * 2, uint64_t(S) * D * 2};
  uint32_t box[3] = {64, rows, 1};
  return make_map(m, base, 3, dims, st, box);
}

// Batch stride of a map: a packed tensor is one batch of total_rows rows (its
// stride_b is 0, so the map gets the extent of the whole tensor instead).
uint64_t batch_stride_bytes(const hia_tensor& t, int S, int B) {
  return (B == 1 && t.stride_b == 0) ? uint64_t(S) * uint64_t(t.stride_s) * 2 : uint64_t(t.stride_b) * 2;
}

// User tensor with Hkv heads: dims (D, Hkv, S, B), box rows along S.  A packed
// tensor is mapped with S = total_rows and B = 1.
bool make_kv_map(CUtensorMap* m, const hia_tensor& t, int D, int Hkv, int S, int B, uint32_t rows) {
  uint64_t dims[4] = {uint64_t(D), uint64_t(Hkv), uint64_t(S), uint64_t(B)};
  uint64_t st[3] = {uint64_t(t.stride_hkv) * 2, uint64_t(t.stride_s) * 2, batch_stride_bytes(t, S, B)};
  uint32_t box[4] = {64, 1, rows, 1};
  return make_map(m, t.ptr, 4, dims, st, box);
}

// User tensor with Hq heads: dims (D, g, Hkv, S, B), box rows along S.
bool make_q_map(CUtensorMap* m, const hia_tensor& t, int D, int g, int Hkv, int S, int B, uint32_t rows) {
  uint64_t dims[5] = {uint64_t(D), uint64_t(g), uint64_t(Hkv), uint64_t(S), uint64_t(B)};
  uint64_t st[4] = {uint64_t(t.stride_hq) * 2, uint64_t(t.stride_hkv) * 2, uint64_t(t.stride_s) * 2,
                    batch_stride_bytes(t, S, B)};
  uint32_t box[5] = {64, 1, 1, rows, 1};
  return make_map(m, t.ptr, 5, dims, st, box);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Checks shared by fwd and bwd.  heads_g: g for Hq-head tensors, 1 for Hkv-head tensors.
int check_tensor(const hia_tensor& t, bool q_heads, int B, int S, int g) {
  if (!t.ptr) return (B == 0 || S == 0) ? HIA_OK : HIA_ERR_INVALID_ARG;
  if (t.stride_b < 0 || t.stride_s < 0 || t.stride_hkv < 0 || t.stride_hq < 0) return HIA_ERR_INVALID_ARG;
  if (!aligned16(t.ptr)) return HIA_ERR_UNSUPPORTED;
  if ((t.stride_b * 2) % 16 || (t.stride_s * 2) % 16 || (t.stride_hkv * 2) % 16) return HIA_ERR_UNSUPPORTED;
  if (q_heads && g > 1 && (t.stride_hq * 2) % 16) return HIA_ERR_UNSUPPORTED;
  return HIA_OK;
}

int check_common(const hia_segments* seg, int Hq, int Hkv, int D, const float* c, const float* s) {
  if (!seg || Hq <= 0 || Hkv <= 0) return HIA_ERR_INVALID_ARG;
  if (Hq % Hkv) return HIA_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return HIA_ERR_UNSUPPORTED;
  if (seg->B == 0 || seg->S == 0) return HIA_OK;
  if (!c || !s) return HIA_ERR_INVALID_ARG;
  if (!aligned16(c) || !aligned16(s)) return HIA_ERR_UNSUPPORTED;
  if (seg->device < 0) return HIA_ERR_NOT_ON_DEVICE;
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != seg->device) return HIA_ERR_NOT_ON_DEVICE;
  return HIA_OK;
}

struct FwdWs {
  size_t q_off, k_off, total;
};
FwdWs fwd_ws(const hia_segments* seg, int Hq, int Hkv, int D) {
  FwdWs w{};
  const size_t BS = size_t(seg->B) * seg->S;
  w.q_off = 0;
  w.k_off = align256(BS * Hq * D * 2);
  w.total = w.k_off + align256(BS * Hkv * D * 2);
  return w;
}

int S_pad64(int S) { return (S + 63) / 64 * 64; }

struct BwdWs {
  size_t q_off, k_off, lse_off, delta_off, dq_off, dk_off, dw_off, part_off, cnt_off, total;
};
// The dK accumulator and the weight-gradient partials are used only with the
// QK RMSNorm; the size always includes them so one workspace serves both.
// The partials of split kv tiles are sized for the schedule `sc`.
BwdWs bwd_ws(const hia_segments* seg, int Hq, int Hkv, int D, const hia_segments::BwdSched& sc) {
  BwdWs w{};
  const size_t BS = size_t(seg->B) * seg->S;
  const size_t BSp = size_t(seg->B) * S_pad64(seg->S);
  w.q_off = 0;
  w.k_off = align256(BS * Hq * D * 2);
  w.lse_off = w.k_off + align256(BS * Hkv * D * 2);
  w.delta_off = w.lse_off + align256(BSp * Hq * 4);
  w.dq_off = w.delta_off + align256(BSp * Hq * 4);
  w.dk_off = w.dq_off + align256(BSp * Hq * D * 4);
  w.dw_off = w.dk_off + align256(BSp * Hkv * D * 4);
  w.part_off = w.dw_off + align256(size_t(2) * hia::grad_finalize_blocks(seg->B, seg->S) * D * 4);
  // split kv tiles: per (slot, kv head) every part's fp32 dK and dV partials, and a ticket counter
  w.cnt_off = w.part_off + align256(size_t(sc.n_slots) * Hkv * sc.parts * 2 * hia::kBwdBK * D * 4);
  w.total = w.cnt_off + align256(size_t(sc.n_slots) * Hkv * 4);
  return w;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? HIA_OK : HIA_ERR_CUDA; }

// Finish time of a backward work list dispatched in order to the first free
// SM (the block scheduler's policy), one CTA per (entry, kv head), in units of
// one query-tile iteration of a whole kv tile.  A CTA costs its query tiles
// times g plus a fixed part (K/V load, TMEM setup, dK/dV epilogue: about nine
// iterations); a part of a split kv tile runs its iterations 20% slower and
// the last part (the one that usually adds the partials) costs 22.5 more.  The
// constants are fitted to per-CTA timings (globaltimer stamps) and backward
// times of the 1024px, 1024px_bwd, mixed and multi_image workloads under every
// schedule: the estimate's pick was within 1% of the fastest measured one on
// each.
double bwd_makespan(const std::vector<int32_t>& work, int Hkv, int g, int n_sm) {
  constexpr double kCtaCost = 9.0, kPartSlowdown = 1.2, kMergeCost = 22.5;
  std::priority_queue<double, std::vector<double>, std::greater<double>> sms;
  for (int i = 0; i < n_sm; ++i) sms.push(0.0);
  double span = 0.0;
  for (size_t e = 0; e + hia::kBwdWorkInts <= work.size(); e += hia::kBwdWorkInts) {
    const double it = double(work[e + 3] - work[e + 2]) * g;
    const bool split = work[e + 4] >= 0;
    const double c = split ? it * kPartSlowdown + kCtaCost + (work[e + 5] == work[e + 6] - 1 ? kMergeCost : 0.0)
                           : it + kCtaCost;
    for (int h = 0; h < Hkv; ++h) {
      const double t = sms.top() + c;
      sms.pop();
      sms.push(t);
      span = std::max(span, t);
    }
  }
  return span;
}

int device_sm_count() {
  static hia::PerContext<int> cache;
  int n = 0;
  if (cache.get(&n, [](int* out) {
        int dev = 0;
        const cudaError_t e = cudaGetDevice(&dev);
        return e != cudaSuccess ? e : cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev);
      }) != cudaSuccess)
    return 148;
  return n;
}

// The backward schedule a launch uses (an index into bwd_sched): the one the
// estimate finishes soonest among those the mode admits (all of them for
// AUTO, the split ones for ALWAYS, those cutting tiles into k parts for
// PARTS_k), the whole list for NEVER or when the mode admits none.
int choose_bwd_sched(const hia_segments* gc, int Hkv, int gq, int n_sm) {
  hia_segments* g = const_cast<hia_segments*>(gc);
  std::lock_guard<std::mutex> lk(g->choice_mu);
  const int mode = g->bwd_split_mode;
  if (mode == HIA_BWD_SPLIT_NEVER || g->bwd_sched.size() <= 1) return 0;
  const auto key = std::make_tuple(mode, Hkv, gq, n_sm);
  auto it = g->choice.find(key);
  if (it != g->choice.end()) return it->second;
  int best = 0;  // the whole list when the mode admits none
  double best_span = -1.0;
  for (int i = 0; i < int(g->bwd_sched.size()); ++i) {
    const int parts = g->bwd_sched[i].parts;
    const bool admitted = mode == HIA_BWD_SPLIT_AUTO || (mode == HIA_BWD_SPLIT_ALWAYS && parts > 1) ||
                          (mode >= HIA_BWD_SPLIT_PARTS_2 && parts == mode - HIA_BWD_SPLIT_PARTS_2 + 2);
    if (!admitted) continue;
    const double span = bwd_makespan(g->bwd_sched[i].work, Hkv, gq, n_sm);
    if (best_span < 0.0 || span < best_span) {  // ties: the earlier (less split) schedule
      best = i;
      best_span = span;
    }
  }
  g->choice[key] = best;
  return best;
}

int check_norm(const hia_qk_norm* n) {
  if (!n) return HIA_OK;
  if (!n->wq || !n->wk || !std::isfinite(n->eps) || n->eps < 0.f) return HIA_ERR_INVALID_ARG;
  if (!aligned16(n->wq) || !aligned16(n->wk)) return HIA_ERR_UNSUPPORTED;
  return HIA_OK;
}

// q and k rotated (and, with the norm, normed) into the workspace by one launch.
void rotate_qk(const hia_segments* seg, int Hq, int Hkv, int D, const hia_tensor& q, const hia_tensor& k,
               const float* c, const float* s, const hia_qk_norm* norm, __nv_bfloat16* qr, __nv_bfloat16* kr,
               cudaStream_t st) {
  hia::RotateArgs a{};
  a.samples = seg->d_samples;
  a.cos_t = c;
  a.sin_t = s;
  a.B = seg->B;
  a.S = seg->S;
  a.n_parts = 2;
  const hia_tensor* src[2] = {&q, &k};
  const int heads[2] = {Hq, Hkv}, groups[2] = {Hq / Hkv, 1};
  __nv_bfloat16* dst[2] = {qr, kr};
  for (int i = 0; i < 2; ++i) {
    hia::RotatePart& p = a.part[i];
    p.src = src[i]->ptr;
    p.src_sb = src[i]->stride_b;
    p.src_ss = src[i]->stride_s;
    p.src_shkv = src[i]->stride_hkv;
    p.src_shq = src[i]->stride_hq;
    p.g = groups[i];
    p.H = heads[i];
    p.w = norm ? (i == 0 ? norm->wq : norm->wk) : nullptr;
    p.eps = norm ? norm->eps : 0.f;
    p.dst = dst[i];
  }
  hia::launch_rope_rotate(a, D, st);
}

// Packed layout: row s of sample b is at (off_b + s) * stride_s; the batch
// stride is not used.
void packed_view(const hia_segments* g, std::initializer_list<hia_tensor*> ts) {
  if (!g->packed) return;
  for (hia_tensor* t : ts) t->stride_b = 0;
}

// The tensor maps' sequence extent and batch count.
int map_rows(const hia_segments* g) { return g->packed ? int(g->total_rows) : g->S; }
int map_batches(const hia_segments* g) { return g->packed ? 1 : g->B; }


}  // namespace

extern "C" int hia_segments_upload(hia_segments* g, void* stream) {
  if (!g) return HIA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HIA_ERR_CUDA;
  if (g->dbuf && g->device != dev) return HIA_ERR_INVALID_ARG;
  const size_t n_s = g->samples.size() * sizeof(SampleDev), n_i = g->images.size() * sizeof(hia::ImageDev);
  const size_t n_ft = g->fwd_tiles.size() * 4, n_fl = g->fwd_list.size() * 4, n_fw = g->fwd_work.size() * 4;
  const size_t n_bt = g->bwd_tiles.size() * 4;
  const size_t o_s = 0, o_i = align256(n_s), o_ft = o_i + align256(n_i), o_fl = o_ft + align256(n_ft),
               o_fw = o_fl + align256(n_fl), o_bt = o_fw + align256(n_fw), o_bw = o_bt + align256(n_bt);
  std::vector<size_t> o_sched(g->bwd_sched.size());
  size_t total = o_bw;
  for (size_t i = 0; i < g->bwd_sched.size(); ++i) {
    o_sched[i] = total;
    total += align256(g->bwd_sched[i].work.size() * 4);
  }
  total += 256;
  if (!g->dbuf) {
    if (cudaMalloc(&g->dbuf, total) != cudaSuccess) {
      g->dbuf = nullptr;
      return HIA_ERR_CUDA;
    }
  }
  char* base = static_cast<char*>(g->dbuf);
  cudaError_t e = cudaSuccess;
  if (n_s) e = cudaMemcpyAsync(base + o_s, g->samples.data(), n_s, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess && n_i) e = cudaMemcpyAsync(base + o_i, g->images.data(), n_i, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess && n_ft) e = cudaMemcpyAsync(base + o_ft, g->fwd_tiles.data(), n_ft, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess && n_fl) e = cudaMemcpyAsync(base + o_fl, g->fwd_list.data(), n_fl, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess && n_fw) e = cudaMemcpyAsync(base + o_fw, g->fwd_work.data(), n_fw, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess && n_bt) e = cudaMemcpyAsync(base + o_bt, g->bwd_tiles.data(), n_bt, cudaMemcpyHostToDevice, st);
  for (size_t i = 0; i < g->bwd_sched.size(); ++i) {
    const std::vector<int32_t>& w = g->bwd_sched[i].work;
    if (e == cudaSuccess && !w.empty())
      e = cudaMemcpyAsync(base + o_sched[i], w.data(), w.size() * 4, cudaMemcpyHostToDevice, st);
  }
  if (e != cudaSuccess) return HIA_ERR_CUDA;
  g->device = dev;
  g->d_samples = reinterpret_cast<const SampleDev*>(base + o_s);
  g->d_images = reinterpret_cast<const hia::ImageDev*>(base + o_i);
  g->d_fwd_tiles = reinterpret_cast<const int32_t*>(base + o_ft);
  g->d_fwd_list = reinterpret_cast<const int32_t*>(base + o_fl);
  g->d_fwd_work = reinterpret_cast<const int32_t*>(base + o_fw);
  g->d_bwd_tiles = reinterpret_cast<const int32_t*>(base + o_bt);
  for (size_t i = 0; i < g->bwd_sched.size(); ++i)
    g->bwd_sched[i].d_work = reinterpret_cast<const int32_t*>(base + o_sched[i]);
  return HIA_OK;
}

extern "C" void hia_segments_destroy(hia_segments* g) {
  if (!g) return;
  if (g->dbuf) {
    int cur = 0;
    cudaGetDevice(&cur);
    if (cur != g->device) cudaSetDevice(g->device);
    cudaFree(g->dbuf);
    if (cur != g->device) cudaSetDevice(cur);
  }
  delete g;
}

extern "C" int hia_segments_bwd_choice(const hia_segments* g, int Hkv, int gq, int n_sm, int* index) {
  if (!g || Hkv <= 0 || gq <= 0 || n_sm <= 0 || !index) return HIA_ERR_INVALID_ARG;
  *index = choose_bwd_sched(g, Hkv, gq, n_sm);
  return HIA_OK;
}

extern "C" int hia_segments_set_bwd_split(hia_segments* g, int mode) {
  if (!g || mode < HIA_BWD_SPLIT_AUTO || mode > HIA_BWD_SPLIT_PARTS_4) return HIA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g->choice_mu);
  g->bwd_split_mode = mode;
  return HIA_OK;
}

extern "C" int hia_rope2d_tables(const hia_segments* g, int D, double base, float* c, float* s, void* stream) {
  if (!g || D < 2 || D > 256 || (D & 1) || !(base > 0.0) || !std::isfinite(base)) return HIA_ERR_INVALID_ARG;
  if (g->B == 0 || g->S == 0) return HIA_OK;
  if (!c || !s) return HIA_ERR_INVALID_ARG;
  if (int64_t(g->B) * g->S >= (int64_t(1) << 31)) return HIA_ERR_UNSUPPORTED;  // one warp per row: grid size
  if (g->device < 0) return HIA_ERR_NOT_ON_DEVICE;
  hia::launch_rope2d_tables(g->d_samples, g->d_images, g->B, g->S, D, base, c, s, static_cast<cudaStream_t>(stream));
  return cuda_status(cudaGetLastError());
}

extern "C" size_t hia_attn_fwd_workspace_bytes(const hia_segments* g, int Hq, int Hkv, int D) {
  if (!g || Hq <= 0 || Hkv <= 0 || D <= 0) return 0;
  return fwd_ws(g, Hq, Hkv, D).total;
}

extern "C" size_t hia_attn_bwd_workspace_bytes(const hia_segments* g, int Hq, int Hkv, int D) {
  if (!g || Hq <= 0 || Hkv <= 0 || D <= 0) return 0;
  const int si = choose_bwd_sched(g, Hkv, std::max(1, Hq / Hkv), device_sm_count());
  return bwd_ws(g, Hq, Hkv, D, g->bwd_sched[si]).total;
}

extern "C" int hia_attn_fwd(const hia_segments* g, int Hq, int Hkv, int D, hia_tensor q, hia_tensor k,
                            hia_tensor v, const float* c, const float* s, float scale, hia_tensor o, float* lse,
                            void* ws, size_t ws_bytes, void* stream) {
  return hia_attn_fwd_ex(g, Hq, Hkv, D, q, k, v, c, s, scale, nullptr, o, lse, ws, ws_bytes, stream);
}

namespace hia {

int fwd_check_args(const hia_segments* g, int Hq, int Hkv, int D, const hia_tensor& q, const hia_tensor& k,
                   const hia_tensor& v, const float* c, const float* s, float scale, const hia_qk_norm* norm,
                   const hia_tensor& o, const float* lse) {
  int rc = check_common(g, Hq, Hkv, D, c, s);
  if (rc) return rc;
  if ((rc = check_norm(norm))) return rc;
  if (g->B == 0 || g->S == 0) return HIA_OK;
  if (!std::isfinite(scale) || !(scale > 0.f)) return HIA_ERR_INVALID_ARG;
  const int gq = Hq / Hkv;
  if ((rc = check_tensor(q, true, g->B, g->S, gq)) || (rc = check_tensor(k, false, g->B, g->S, 1)) ||
      (rc = check_tensor(v, false, g->B, g->S, 1)) || (rc = check_tensor(o, true, g->B, g->S, gq)))
    return rc;
  if (!q.ptr || !k.ptr || !v.ptr || !o.ptr || !lse) return HIA_ERR_INVALID_ARG;
  return HIA_OK;
}

}  // namespace hia

extern "C" int hia_attn_fwd_ex(const hia_segments* g, int Hq, int Hkv, int D, hia_tensor q, hia_tensor k,
                               hia_tensor v, const float* c, const float* s, float scale, const hia_qk_norm* norm,
                               hia_tensor o, float* lse, void* ws, size_t ws_bytes, void* stream) {
  int rc = hia::fwd_check_args(g, Hq, Hkv, D, q, k, v, c, s, scale, norm, o, lse);
  if (rc) return rc;
  if (g->B == 0 || g->S == 0) return HIA_OK;
  if (!ws) return HIA_ERR_INVALID_ARG;
  const int gq = Hq / Hkv;
  packed_view(g, {&q, &k, &v, &o});
  const FwdWs w = fwd_ws(g, Hq, Hkv, D);
  if (ws_bytes < w.total || (reinterpret_cast<uintptr_t>(ws) & 255)) return HIA_ERR_INVALID_ARG;
  int* status = status_ptr();
  if (!status) return HIA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* wb = static_cast<char*>(ws);
  __nv_bfloat16* qr = reinterpret_cast<__nv_bfloat16*>(wb + w.q_off);
  __nv_bfloat16* kr = reinterpret_cast<__nv_bfloat16*>(wb + w.k_off);

  CUtensorMap tq, tk, tv;
  if (!make_ws_map(&tq, qr, D, g->S, g->B * Hq) || !make_ws_map(&tk, kr, D, g->S, g->B * Hkv) ||
      !make_kv_map(&tv, v, D, Hkv, map_rows(g), map_batches(g), 128))
    return HIA_ERR_CUDA;

  rotate_qk(g, Hq, Hkv, D, q, k, c, s, norm, qr, kr, st);

  hia::FwdParams p{};
  p.samples = g->d_samples;
  p.images = g->d_images;
  p.tiles = g->d_fwd_tiles;
  p.list = g->d_fwd_list;
  p.work = g->d_fwd_work;
  p.B = g->B;
  p.S = g->S;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.g = gq;
  p.nQT = g->nQT;
  p.n_hp = (gq + 1) / 2;
  p.o = static_cast<__nv_bfloat16*>(o.ptr);
  p.o_sb = o.stride_b;
  p.o_ss = o.stride_s;
  p.o_shkv = o.stride_hkv;
  p.o_shq = o.stride_hq;
  p.lse = lse;
  p.lse_sb = g->packed ? 0 : int64_t(Hq) * g->S;
  p.lse_sh = g->packed ? g->total_rows : g->S;
  p.packed = g->packed ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = status;
  p.timeout_ns = kDefaultTimeoutNs;
  const int64_t n_blocks = int64_t(g->B) * g->nQT * Hkv * p.n_hp;
  if (n_blocks > (1ll << 31) - 1) return HIA_ERR_UNSUPPORTED;
  return cuda_status(hia::launch_attn_fwd(tq, tk, tv, p, int(n_blocks), D, st));
}

extern "C" int hia_get_device_status(void* stream) {
  int* sp = status_ptr();
  if (!sp) return HIA_ERR_CUDA;
  int h = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&h, sp, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return HIA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return HIA_ERR_CUDA;
  if (h != 0) {
    const int z = 0;
    if (cudaMemcpyAsync(sp, &z, sizeof(int), cudaMemcpyHostToDevice, st) != cudaSuccess) return HIA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return HIA_ERR_CUDA;
  }
  return h == 0 ? HIA_OK : HIA_ERR_DEVICE_TIMEOUT;
}

extern "C" int hia_debug_wait_timeout(uint64_t timeout_ns, void* stream) {
  if (timeout_ns < 1 || timeout_ns > 1000000000ull) return HIA_ERR_INVALID_ARG;
  int* sp = status_ptr();
  if (!sp) return HIA_ERR_CUDA;
  return cuda_status(hia::launch_wait_probe(sp, timeout_ns, static_cast<cudaStream_t>(stream)));
}

extern "C" int hia_debug_exp2(const float* x, float* y, int n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return HIA_ERR_INVALID_ARG;
  return cuda_status(hia::launch_exp2_probe(x, y, n, static_cast<cudaStream_t>(stream)));
}

extern "C" int hia_attn_bwd(const hia_segments* g, int Hq, int Hkv, int D, hia_tensor q, hia_tensor k,
                            hia_tensor v, const float* c, const float* s, float scale, hia_tensor o,
                            const float* lse, hia_tensor dout, hia_tensor dq, hia_tensor dk, hia_tensor dv,
                            void* ws, size_t ws_bytes, void* stream) {
  return hia_attn_bwd_ex(g, Hq, Hkv, D, q, k, v, c, s, scale, nullptr, o, lse, dout, dq, dk, dv, nullptr, nullptr,
                         ws, ws_bytes, stream);
}

extern "C" int hia_attn_bwd_ex(const hia_segments* g, int Hq, int Hkv, int D, hia_tensor q, hia_tensor k,
                               hia_tensor v, const float* c, const float* s, float scale, const hia_qk_norm* norm,
                               hia_tensor o, const float* lse, hia_tensor dout, hia_tensor dq, hia_tensor dk,
                               hia_tensor dv, float* dwq, float* dwk, void* ws, size_t ws_bytes, void* stream) {
  return hia_attn_bwd_reuse_fwd(g, Hq, Hkv, D, q, k, v, c, s, scale, norm, o, lse, dout, dq, dk, dv, dwq, dwk,
                                nullptr, 0, ws, ws_bytes, stream);
}

extern "C" int hia_attn_bwd_reuse_fwd(const hia_segments* g, int Hq, int Hkv, int D, hia_tensor q, hia_tensor k,
                                      hia_tensor v, const float* c, const float* s, float scale,
                                      const hia_qk_norm* norm, hia_tensor o, const float* lse, hia_tensor dout,
                                      hia_tensor dq, hia_tensor dk, hia_tensor dv, float* dwq, float* dwk,
                                      const void* fws, size_t fws_bytes, void* ws, size_t ws_bytes,
                                      void* stream) {
  int rc = check_common(g, Hq, Hkv, D, c, s);
  if (rc) return rc;
  if ((rc = check_norm(norm))) return rc;
  if (norm && (!dwq || !dwk)) return HIA_ERR_INVALID_ARG;
  if (g->B == 0 || g->S == 0) return HIA_OK;
  if (!std::isfinite(scale) || !(scale > 0.f)) return HIA_ERR_INVALID_ARG;
  const int gq = Hq / Hkv;
  if ((rc = check_tensor(q, true, g->B, g->S, gq)) || (rc = check_tensor(k, false, g->B, g->S, 1)) ||
      (rc = check_tensor(v, false, g->B, g->S, 1)) || (rc = check_tensor(o, true, g->B, g->S, gq)) ||
      (rc = check_tensor(dout, true, g->B, g->S, gq)) || (rc = check_tensor(dq, true, g->B, g->S, gq)) ||
      (rc = check_tensor(dk, false, g->B, g->S, 1)) || (rc = check_tensor(dv, false, g->B, g->S, 1)))
    return rc;
  if (!q.ptr || !k.ptr || !v.ptr || !o.ptr || !lse || !dout.ptr || !dq.ptr || !dk.ptr || !dv.ptr || !ws)
    return HIA_ERR_INVALID_ARG;
  packed_view(g, {&q, &k, &v, &o, &dout, &dq, &dk, &dv});
  // the schedule; a workspace sized for another choice (another device's SM
  // count, or before the mode changed) that does not hold its partials runs
  // the whole list, which needs none
  int si = choose_bwd_sched(g, Hkv, gq, device_sm_count());
  if (ws_bytes < bwd_ws(g, Hq, Hkv, D, g->bwd_sched[si]).total) si = 0;
  const hia_segments::BwdSched& sched = g->bwd_sched[si];
  const BwdWs w = bwd_ws(g, Hq, Hkv, D, sched);
  if (ws_bytes < w.total || (reinterpret_cast<uintptr_t>(ws) & 255)) return HIA_ERR_INVALID_ARG;
  const FwdWs fw = fwd_ws(g, Hq, Hkv, D);
  if (fws && (fws_bytes < fw.total || (reinterpret_cast<uintptr_t>(fws) & 255)))
    return HIA_ERR_INVALID_ARG;
  int* status = status_ptr();
  if (!status) return HIA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* wb = static_cast<char*>(ws);
  // the rotated q and k: the forward's (reused as they are) or rotated here
  __nv_bfloat16* qr = reinterpret_cast<__nv_bfloat16*>(
      fws ? static_cast<char*>(const_cast<void*>(fws)) + fw.q_off : wb + w.q_off);
  __nv_bfloat16* kr = reinterpret_cast<__nv_bfloat16*>(
      fws ? static_cast<char*>(const_cast<void*>(fws)) + fw.k_off : wb + w.k_off);
  float* lse2 = reinterpret_cast<float*>(wb + w.lse_off);
  float* delta = reinterpret_cast<float*>(wb + w.delta_off);
  float* dq_acc = reinterpret_cast<float*>(wb + w.dq_off);
  float* dk_acc = reinterpret_cast<float*>(wb + w.dk_off);
  float* dw_part = reinterpret_cast<float*>(wb + w.dw_off);
  float* part = reinterpret_cast<float*>(wb + w.part_off);
  int* part_cnt = reinterpret_cast<int*>(wb + w.cnt_off);
  const int S_pad = S_pad64(g->S);

  CUtensorMap tq, tk, tv, tdo;
  if (!make_ws_map(&tq, qr, D, g->S, g->B * Hq, 64) || !make_ws_map(&tk, kr, D, g->S, g->B * Hkv, 128) ||
      !make_kv_map(&tv, v, D, Hkv, map_rows(g), map_batches(g), 128) ||
      !make_q_map(&tdo, dout, D, gq, Hkv, map_rows(g), map_batches(g), 64))
    return HIA_ERR_CUDA;

  if (!fws) rotate_qk(g, Hq, Hkv, D, q, k, c, s, norm, qr, kr, st);

  hia::BwdPreParams pp{};
  pp.o = static_cast<const __nv_bfloat16*>(o.ptr);
  pp.o_sb = o.stride_b;
  pp.o_ss = o.stride_s;
  pp.o_shkv = o.stride_hkv;
  pp.o_shq = o.stride_hq;
  pp.dout = static_cast<const __nv_bfloat16*>(dout.ptr);
  pp.d_sb = dout.stride_b;
  pp.d_ss = dout.stride_s;
  pp.d_shkv = dout.stride_hkv;
  pp.d_shq = dout.stride_hq;
  pp.samples = g->d_samples;
  pp.lse = lse;
  pp.lse_sb = g->packed ? 0 : int64_t(Hq) * g->S;
  pp.lse_sh = g->packed ? g->total_rows : g->S;
  pp.lse2 = lse2;
  pp.delta = delta;
  pp.dq_acc = dq_acc;
  pp.part_cnt = part_cnt;
  pp.n_cnt = sched.n_slots * Hkv;
  pp.B = g->B;
  pp.S = g->S;
  pp.S_pad = S_pad;
  pp.Hq = Hq;
  pp.g = gq;
  pp.D = D;
  if ((rc = cuda_status(hia::launch_bwd_pre(pp, st)))) return rc;

  hia::BwdParams p{};
  p.samples = g->d_samples;
  p.images = g->d_images;
  p.tiles = g->d_bwd_tiles;
  p.work = sched.d_work;
  p.part = part;
  p.part_cnt = part_cnt;
  p.B = g->B;
  p.S = g->S;
  p.S_pad = S_pad;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.g = gq;
  p.bQT = g->bQT;
  p.bKT = g->bKT;
  p.lse2 = lse2;
  p.delta = delta;
  p.dq_acc = dq_acc;
  p.cos_t = c;
  p.sin_t = s;
  p.dk = static_cast<__nv_bfloat16*>(dk.ptr);
  p.dk_sb = dk.stride_b;
  p.dk_ss = dk.stride_s;
  p.dk_sh = dk.stride_hkv;
  p.dv = static_cast<__nv_bfloat16*>(dv.ptr);
  p.dv_sb = dv.stride_b;
  p.dv_ss = dv.stride_s;
  p.dv_sh = dv.stride_hkv;
  p.dk_acc = norm ? dk_acc : nullptr;
  p.packed = g->packed ? 1 : 0;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = status;
  p.timeout_ns = kDefaultTimeoutNs;
  const int64_t n_entries = int64_t(sched.work.size()) / hia::kBwdWorkInts;
  const int64_t n_blocks = n_entries * Hkv;
  if (n_blocks > (1ll << 31) - 1) return HIA_ERR_UNSUPPORTED;
  if ((rc = cuda_status(hia::launch_attn_bwd(tq, tk, tv, tdo, p, int(n_blocks), D, st)))) return rc;

  // dq = R^T (norm backward of) scale * dq_acc; with the norm also dk from dk_acc and the weight gradients
  const int nblk = hia::grad_finalize_blocks(g->B, g->S);
  hia::GradFinalArgs fa{};
  fa.samples = g->d_samples;
  fa.acc = dq_acc;
  fa.S_pad = S_pad;
  fa.scale = scale;
  fa.cos_t = c;
  fa.sin_t = s;
  fa.x = q.ptr;
  fa.x_sb = q.stride_b;
  fa.x_ss = q.stride_s;
  fa.x_shkv = q.stride_hkv;
  fa.x_shq = q.stride_hq;
  fa.w = norm ? norm->wq : nullptr;
  fa.eps = norm ? norm->eps : 0.f;
  fa.dw_part = dw_part;
  fa.dst = dq.ptr;
  fa.dst_sb = dq.stride_b;
  fa.dst_ss = dq.stride_s;
  fa.dst_shkv = dq.stride_hkv;
  fa.dst_shq = dq.stride_hq;
  fa.g = gq;
  fa.B = g->B;
  fa.S = g->S;
  fa.H = Hq;
  hia::launch_grad_finalize(fa, D, st);
  if (norm) {
    hia::launch_dw_reduce(dw_part, nblk, D, dwq, st);
    hia::GradFinalArgs fk = fa;
    fk.acc = dk_acc;
    fk.scale = 1.f;  // the epilogue already applied the softmax scale
    fk.x = k.ptr;
    fk.x_sb = k.stride_b;
    fk.x_ss = k.stride_s;
    fk.x_shkv = k.stride_hkv;
    fk.x_shq = 0;
    fk.w = norm->wk;
    fk.dw_part = dw_part + size_t(nblk) * D;
    fk.dst = dk.ptr;
    fk.dst_sb = dk.stride_b;
    fk.dst_ss = dk.stride_s;
    fk.dst_shkv = dk.stride_hkv;
    fk.dst_shq = 0;
    fk.g = 1;
    fk.H = Hkv;
    hia::launch_grad_finalize(fk, D, st);
    hia::launch_dw_reduce(dw_part + size_t(nblk) * D, nblk, D, dwk, st);
  }
  return cuda_status(cudaGetLastError());
}
