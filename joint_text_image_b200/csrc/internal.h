// internal.h -- library-private types shared by the host code and the kernels.
#pragma once
#include <cstdint>
#include <vector>

#include "../../include/jointattn.h"

#ifdef __CUDACC__
#define HIA_HD __host__ __device__
#else
#define HIA_HD
#endif

namespace hia {

// Tile geometry.  Forward: 128 query rows x 128 keys.  Backward: 128 keys
// (the MMA M side) x 64 query rows.
constexpr int kFwdBM = 128;
constexpr int kFwdBN = 128;
constexpr int kBwdBK = 128;
constexpr int kBwdBQ = 64;

// Per-sample bounds on the device: I0 = image start, I1 = image end,
// L = valid length, w = image width (unused by the attention kernels),
// rows = the sample's rows in the caller's tensors (S for the padded layout,
// L for the packed one), off = the sample's first row in a packed tensor
// (0 for the padded layout).  Row s of sample b sits at
// b * stride_b + (off + s) * stride_s; a packed layout has stride_b = 0.
struct SampleDev {
  int32_t I0, I1, L, w, rows, off;
};

// Row bound e(q): the last visible key of query q (keys k <= e(q) visible).
HIA_HD inline int32_t row_bound(int32_t I0, int32_t I1, int32_t L, int32_t q) {
  if (L <= 0) return -1;
  int32_t e = (q >= I0 && q < I1) ? I1 - 1 : q;
  return e < L - 1 ? e : L - 1;
}

}  // namespace hia

struct hia_segments {
  int B = 0, S = 0;
  bool packed = false;      // samples stored back to back (no padding rows); S = max L
  int64_t total_rows = 0;   // packed: sum of L; padded: B * S
  std::vector<hia::SampleDev> samples;
  // forward tile table [B][nQT]: (n_full, n_visible) over 128-key tiles.
  int nQT = 0, nKT = 0;
  std::vector<int32_t> fwd_tiles;   // 2 per entry
  std::vector<int32_t> fwd_work;    // (b, qt) pairs, heaviest first
  // backward tile table [B][bKT]: (qt_first, qt_full) over 64-row query tiles.
  int bQT = 0, bKT = 0;
  std::vector<int32_t> bwd_tiles;   // 2 per entry
  std::vector<int32_t> bwd_work;    // (b, kt) pairs, heaviest first
  int64_t pairs = 0;
  hia_segments_info_t info{};
  // device copies (one allocation)
  int device = -1;
  void* dbuf = nullptr;
  const hia::SampleDev* d_samples = nullptr;
  const int32_t* d_fwd_tiles = nullptr;
  const int32_t* d_fwd_work = nullptr;
  const int32_t* d_bwd_tiles = nullptr;
  const int32_t* d_bwd_work = nullptr;
};
