// internal.h -- library-private types shared by the host code and the kernels.
#pragma once
#include <cstdint>
#include <map>
#include <mutex>
#include <tuple>
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
constexpr int kBwdWorkInts = 8;  // ints per backward work-list entry
constexpr int kBwdMaxParts = 4;  // a split kv tile's query range is cut into at most this many parts

// One image of a sample: tokens [I0, I1) on a grid of width w (row-major).
// hidden = 1 for a context image: every image of a sample but its last is
// masked from all tokens after its span (technical report summary 3.1.2,
// training sequences with several generated images).
struct ImageDev {
  int32_t I0, I1, w, hidden;
};

// Per-sample data on the device: L = valid length, rows = the sample's rows
// in the caller's tensors (S for the padded layout, L for the packed one),
// off = the sample's first row in a packed tensor (0 for the padded layout),
// images [img0, img0 + n_img) of the image array.  Row s of sample b sits at
// b * stride_b + (off + s) * stride_s; a packed layout has stride_b = 0.
struct SampleDev {
  int32_t L, rows, off, img0, n_img, pad_;
};

// Index of the image holding token n, or -1.
HIA_HD inline int image_of(const ImageDev* im, int n_img, int32_t n) {
  for (int i = 0; i < n_img; ++i)
    if (im[i].I0 <= n && n < im[i].I1) return i;
  return -1;
}

// Row bound e(q): keys k <= e(q) are visible unless hidden (below); e is
// non-decreasing in q.  Text rows end at themselves, image rows at their
// image's last token, padded rows at L - 1.
HIA_HD inline int32_t row_bound(const ImageDev* im, int n_img, int32_t L, int32_t q) {
  if (L <= 0) return -1;
  const int i = image_of(im, n_img, q);
  const int32_t e = i >= 0 ? im[i].I1 - 1 : q;
  return e < L - 1 ? e : L - 1;
}

// End of the context image holding key k (k is hidden from every row q >= it),
// or INT32_MAX when k is not in a context image.
HIA_HD inline int32_t hidden_from(const ImageDev* im, int n_img, int32_t k) {
  const int i = image_of(im, n_img, k);
  return (i >= 0 && im[i].hidden) ? im[i].I1 : 0x7fffffff;
}

// First row that sees key k (e is non-decreasing: rows of k's image see it
// from the image's first row on, other keys from their own row on), or
// INT32_MAX for a padded key.  Key k is visible exactly to the rows
// [first_row(k), hidden_from(k)).
HIA_HD inline int32_t first_row(const ImageDev* im, int n_img, int32_t L, int32_t k) {
  if (k >= L) return 0x7fffffff;
  const int i = image_of(im, n_img, k);
  return i >= 0 ? im[i].I0 : k;
}

// The mask: key k visible from query q iff k <= e(q) and q < hidden_from(k).
HIA_HD inline bool visible(const ImageDev* im, int n_img, int32_t L, int32_t q, int32_t k) {
  return k <= row_bound(im, n_img, L, q) && q < hidden_from(im, n_img, k);
}

}  // namespace hia

struct hia_segments {
  int B = 0, S = 0;
  bool packed = false;      // samples stored back to back (no padding rows); S = max L
  int64_t total_rows = 0;   // packed: sum of L; padded: B * S
  std::vector<hia::SampleDev> samples;
  std::vector<hia::ImageDev> images;
  // forward tile lists over 128 x 128 tiles: for (b, qt), fwd_tiles holds
  // (first entry, count) of fwd_list, whose entries kt | FULL << 16 name the
  // visible kv tiles in increasing order (FULL: every pair visible).
  int nQT = 0, nKT = 0;
  std::vector<int32_t> fwd_tiles;   // 2 per (b, qt)
  std::vector<int32_t> fwd_list;
  std::vector<int32_t> fwd_work;    // (b, qt) pairs, heaviest first
  // backward tile table [B][bKT] over 64-row query tiles: (qt_first, qt_end,
  // full_first, full_end): the query tiles [qt_first, qt_end) see the key
  // tile, those in [full_first, full_end) see all of it.
  int bQT = 0, bKT = 0;
  std::vector<int32_t> bwd_tiles;   // 4 per entry
  // backward schedules: work lists of kBwdWorkInts per entry, (b, kt, qt_lo,
  // qt_hi, slot, part, parts, 0), heaviest first.  bwd_sched[0]: every (b, kv
  // tile) over its whole query range (slot -1, parts 1).  bwd_sched[i > 0]:
  // the same, except that the kv tiles whose query range is at least a given
  // fraction of the longest are cut into `parts` consecutive sub-ranges (part
  // 0 .. parts-1) sharing a slot: each writes its fp32 dK/dV partial, and the
  // one that finishes last adds the partials in part order and writes dK/dV.
  struct BwdSched {
    std::vector<int32_t> work;
    int parts = 1;
    int n_slots = 0;                  // kv tiles split
    const int32_t* d_work = nullptr;  // device copy
  };
  std::vector<BwdSched> bwd_sched;
  int bwd_split_mode = 0;           // HIA_BWD_SPLIT_*
  // launch-time choice of a schedule, per (mode, Hkv, g, SM count)
  std::mutex choice_mu;
  std::map<std::tuple<int, int, int, int>, int> choice;
  int64_t pairs = 0;
  hia_segments_info_t info{};
  // device copies (one allocation)
  int device = -1;
  void* dbuf = nullptr;
  const hia::SampleDev* d_samples = nullptr;
  const hia::ImageDev* d_images = nullptr;
  const int32_t* d_fwd_tiles = nullptr;
  const int32_t* d_fwd_list = nullptr;
  const int32_t* d_fwd_work = nullptr;
  const int32_t* d_bwd_tiles = nullptr;
};
