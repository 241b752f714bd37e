// segments.cpp -- host-side segment-descriptor builder.
//
// Replaces the dense [B,1,S,S] boolean mask of build_joint_attention_mask
// (hunyuan_image3.model: causal text, bidirectional image span, padded keys
// masked out; technical report summary 3.1.2) by per-sample bounds and
// per-tile work lists.  The rule "k < L and (k <= q or q, k in one image)"
// equals "k <= e(q)" with the non-decreasing row bound
// e(q) = min(L-1, q in an image ? the image's last token : q): text rows end
// at themselves, image rows at their image's last token, padded rows at L-1.
// With several images per sample, every image but the last is a context
// image, masked from all tokens after its span (3.1.2, training sequences
// with several generated images): k is then also hidden from q when k lies
// in a context image that ends at or before q.  The builder counts the
// visible pairs of every (q-tile, kv-tile) pair: FULL when all are visible,
// skipped when none is, PARTIAL otherwise.
#include <algorithm>
#include <cstring>
#include <new>

#include "internal.h"

using hia::ImageDev;
using hia::row_bound;

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

namespace {

// One sample before layout: images (text before each, h, w) in order, then
// the suffix.
struct SampleSpec {
  std::vector<hia_image> images;
  int32_t suffix = 0;
};

// Visible keys of row q in [k0, k1]: [0, e(q)] minus the context images that
// end at or before q.
int64_t visible_in(const ImageDev* im, int n, int32_t L, int32_t q, int32_t k0, int32_t k1) {
  const int32_t e = row_bound(im, n, L, q);
  int64_t c = std::max<int64_t>(0, int64_t(std::min(k1, e)) - k0 + 1);
  for (int i = 0; i < n; ++i)
    if (im[i].hidden && im[i].I1 <= q) c -= std::max(0, std::min(k1 + 1, im[i].I1) - std::max(k0, im[i].I0));
  return c;
}

int build(const std::vector<SampleSpec>& spec, int S, bool packed, hia_segments** out) {
  const int B = int(spec.size());
  hia_segments* g = new (std::nothrow) hia_segments();
  if (!g) return HIA_ERR_INVALID_ARG;
  g->B = B;
  g->S = S;
  g->packed = packed;
  g->samples.resize(B);
  int64_t off = 0;
  for (int b = 0; b < B; ++b) {
    const SampleSpec& x = spec[b];
    const int n = int(x.images.size());
    int64_t pos = 0;
    const int32_t img0 = int32_t(g->images.size());
    for (int j = 0; j < n; ++j) {
      const hia_image& im = x.images[j];
      if (im.text_before < 0 || im.img_h <= 0 || im.img_w <= 0) {
        delete g;
        return HIA_ERR_INVALID_ARG;
      }
      const int64_t I0 = pos + im.text_before, I1 = I0 + int64_t(im.img_h) * im.img_w;
      if (I1 > S) {
        delete g;
        return HIA_ERR_INVALID_ARG;
      }
      g->images.push_back({int32_t(I0), int32_t(I1), im.img_w, j < n - 1 ? 1 : 0});
      pos = I1;
    }
    const int64_t L = pos + x.suffix;
    if (x.suffix < 0 || L > S) {
      delete g;
      return HIA_ERR_INVALID_ARG;
    }
    const int32_t rows = packed ? int32_t(L) : S;
    // the padded layout addresses sample b through stride_b: its first row is row 0
    g->samples[b] = {int32_t(L), rows, packed ? int32_t(off) : 0, img0, n, 0};
    off += rows;
  }
  if (off >= (int64_t(1) << 31)) {
    delete g;
    return HIA_ERR_INVALID_ARG;
  }
  g->total_rows = off;
  auto imgs = [&](int b) { return g->images.data() + g->samples[b].img0; };

  // visible pairs: sum over the sample's query rows of its visible keys
  int64_t pairs = 0;
  for (int b = 0; b < B; ++b) {
    const auto& t = g->samples[b];
    for (int q = 0; q < t.rows; ++q) pairs += visible_in(imgs(b), t.n_img, t.L, q, 0, S - 1);
  }
  g->pairs = pairs;

  // forward tiles: 128 x 128; per (b, qt) the list of visible kv tiles
  using hia::kFwdBM;
  using hia::kFwdBN;
  g->nQT = ceil_div(S, kFwdBM);
  g->nKT = ceil_div(S, kFwdBN);
  g->fwd_tiles.assign(size_t(B) * g->nQT * 2, 0);
  int64_t nfull = 0, npart = 0, nskip = 0;
  for (int b = 0; b < B; ++b) {
    const auto& t = g->samples[b];
    for (int qt = 0; qt < g->nQT; ++qt) {
      const int q0 = qt * kFwdBM, q1 = std::min(q0 + kFwdBM, int(t.rows)) - 1;
      g->fwd_tiles[(size_t(b) * g->nQT + qt) * 2 + 0] = int32_t(g->fwd_list.size());
      int count = 0;
      for (int kt = 0; q0 <= q1 && kt < g->nKT; ++kt) {
        const int k0 = kt * kFwdBN, k1 = std::min(k0 + kFwdBN, S) - 1;
        int64_t vis = 0;
        for (int q = q0; q <= q1; ++q) vis += visible_in(imgs(b), t.n_img, t.L, q, k0, k1);
        if (vis == 0) continue;
        const bool full = k1 - k0 + 1 == kFwdBN && vis == int64_t(q1 - q0 + 1) * kFwdBN;
        g->fwd_list.push_back(kt | (full ? (1 << 16) : 0));
        ++count;
        (full ? nfull : npart) += 1;
      }
      g->fwd_tiles[(size_t(b) * g->nQT + qt) * 2 + 1] = count;
      nskip += g->nKT - count;
    }
  }
  std::vector<int> order(size_t(B) * g->nQT);
  for (size_t i = 0; i < order.size(); ++i) order[i] = int(i);
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int c) { return g->fwd_tiles[size_t(a) * 2 + 1] > g->fwd_tiles[size_t(c) * 2 + 1]; });
  g->fwd_work.resize(order.size() * 2);
  for (size_t i = 0; i < order.size(); ++i) {
    g->fwd_work[i * 2 + 0] = order[i] / g->nQT;
    g->fwd_work[i * 2 + 1] = order[i] % g->nQT;
  }

  // backward tiles: 128 keys x 64 query rows.  The query tiles that see a kv
  // tile form a range (keys in a context image are seen only by its own
  // rows, other keys by every later row); the FULL ones (every pair visible,
  // a whole 64-row tile) are taken as their first contiguous run, the rest of
  // the range is PARTIAL (the mask is evaluated there).
  using hia::kBwdBK;
  using hia::kBwdBQ;
  g->bQT = ceil_div(S, kBwdBQ);
  g->bKT = ceil_div(S, kBwdBK);
  g->bwd_tiles.assign(size_t(B) * g->bKT * 4, 0);
  std::vector<int64_t> bwd_cost(size_t(B) * g->bKT, 0);
  for (int b = 0; b < B; ++b) {
    const auto& t = g->samples[b];
    const int nq = ceil_div(t.rows, kBwdBQ);
    for (int kt = 0; kt < g->bKT; ++kt) {
      const int k0 = kt * kBwdBK, k1 = std::min(k0 + kBwdBK, S) - 1;
      int first = -1, last = -1, f0 = -1, f1 = -1;
      for (int qt = 0; qt < nq; ++qt) {
        const int q0 = qt * kBwdBQ, q1 = std::min(q0 + kBwdBQ, int(t.rows)) - 1;
        int64_t vis = 0;
        for (int q = q0; q <= q1; ++q) vis += visible_in(imgs(b), t.n_img, t.L, q, k0, k1);
        if (vis == 0) continue;
        if (first < 0) first = qt;
        last = qt;
        const bool full = q1 - q0 + 1 == kBwdBQ && k1 - k0 + 1 == kBwdBK && vis == int64_t(kBwdBQ) * kBwdBK;
        if (full && (f0 < 0 || f1 == qt)) {
          if (f0 < 0) f0 = qt;
          f1 = qt + 1;
        }
      }
      int32_t* e = &g->bwd_tiles[(size_t(b) * g->bKT + kt) * 4];
      e[0] = first < 0 ? 0 : first;
      e[1] = first < 0 ? 0 : last + 1;
      e[2] = f0 < 0 ? 0 : f0;
      e[3] = f0 < 0 ? 0 : f1;
      bwd_cost[size_t(b) * g->bKT + kt] = e[1] - e[0];
    }
  }
  order.assign(size_t(B) * g->bKT, 0);
  for (size_t i = 0; i < order.size(); ++i) order[i] = int(i);
  std::stable_sort(order.begin(), order.end(), [&](int a, int c) { return bwd_cost[a] > bwd_cost[c]; });
  // Schedules: the whole list, and for parts in {2, 3, 4} and a threshold
  // of 95, 90 or 85% of the longest query range, the list with every kv tile
  // at or above the threshold cut into `parts` sub-ranges (of at least two
  // query tiles each).  The launch picks one by a list-scheduling estimate.
  struct BwdJob {
    int64_t cost;
    int32_t b, kt, lo, hi, slot, part, parts;
  };
  int64_t max_cost = 0;
  for (int u : order) max_cost = std::max(max_cost, bwd_cost[u]);
  auto make = [&](int parts, int64_t threshold) {
    hia_segments::BwdSched sc;
    sc.parts = parts;
    std::vector<BwdJob> js;
    for (int u : order) {
      const int b = u / g->bKT, kt = u % g->bKT;
      const int32_t* e = &g->bwd_tiles[size_t(u) * 4];
      const int64_t c = bwd_cost[u];
      if (parts > 1 && c >= threshold && c >= 2 * parts) {
        for (int j = 0; j < parts; ++j) {
          const int lo = e[0] + int(c * j / parts), hi = e[0] + int(c * (j + 1) / parts);
          js.push_back({hi - lo, b, kt, lo, hi, sc.n_slots, j, parts});
        }
        ++sc.n_slots;
      } else {
        js.push_back({c, b, kt, e[0], e[1], -1, 0, 1});
      }
    }
    std::stable_sort(js.begin(), js.end(), [](const BwdJob& x, const BwdJob& y) { return x.cost > y.cost; });
    for (const BwdJob& j : js) sc.work.insert(sc.work.end(), {j.b, j.kt, j.lo, j.hi, j.slot, j.part, j.parts, 0});
    return sc;
  };
  g->bwd_sched.clear();
  g->bwd_sched.push_back(make(1, 0));
  int split_units = 0;
  for (int parts = 2; parts <= hia::kBwdMaxParts; ++parts) {
    int prev_slots = -1;
    for (int pct : {95, 90, 85}) {
      const int64_t threshold = (max_cost * pct + 99) / 100;
      hia_segments::BwdSched sc = make(parts, threshold);
      if (sc.n_slots == 0 || sc.n_slots == prev_slots) continue;  // nothing split, or the same tiles again
      prev_slots = sc.n_slots;
      if (parts == 2) split_units = std::max(split_units, sc.n_slots);
      g->bwd_sched.push_back(std::move(sc));
    }
  }

  hia_segments_info_t& in = g->info;
  in.B = B;
  in.S = S;
  in.visible_pairs = pairs;
  in.fwd_q_tiles = g->nQT;
  in.fwd_kv_tiles = g->nKT;
  in.fwd_tiles_full = nfull;
  in.fwd_tiles_partial = npart;
  in.fwd_tiles_skipped = nskip;
  in.bwd_q_tiles = g->bQT;
  in.bwd_kv_tiles = g->bKT;
  in.packed = packed ? 1 : 0;
  in.bwd_split_units = split_units;
  in.total_rows = g->total_rows;
  *out = g;
  return HIA_OK;
}

// The one-image form: prefix, one image (none when h = w = 0), suffix.
int from_samples(const hia_sample* s, int B, std::vector<SampleSpec>* spec) {
  spec->resize(B);
  for (int b = 0; b < B; ++b) {
    const hia_sample& x = s[b];
    if (x.prefix_len < 0 || x.img_h < 0 || x.img_w < 0 || x.suffix_len < 0 || ((x.img_h == 0) != (x.img_w == 0)))
      return HIA_ERR_INVALID_ARG;
    SampleSpec& o = (*spec)[b];
    if (x.img_h > 0) {
      o.images.push_back({x.prefix_len, x.img_h, x.img_w});
      o.suffix = x.suffix_len;
    } else {
      const int64_t t = int64_t(x.prefix_len) + x.suffix_len;
      if (t >= (int64_t(1) << 31)) return HIA_ERR_INVALID_ARG;
      o.suffix = int32_t(t);
    }
  }
  return HIA_OK;
}

int64_t max_length(const std::vector<SampleSpec>& spec) {
  int64_t S = 0;
  for (const SampleSpec& x : spec) {
    int64_t L = x.suffix;
    for (const hia_image& im : x.images) L += int64_t(im.text_before) + int64_t(im.img_h) * im.img_w;
    S = std::max(S, L);
  }
  return S;
}

}  // namespace

extern "C" int hia_segments_build(const hia_sample* s, int B, int S, hia_segments** out) {
  if (!out || B < 0 || (B > 0 && !s) || B >= (1 << 20)) return HIA_ERR_INVALID_ARG;
  *out = nullptr;
  if (S < 0 || S >= (1 << 24)) return HIA_ERR_INVALID_ARG;
  std::vector<SampleSpec> spec;
  int rc = from_samples(s, B, &spec);
  return rc ? rc : build(spec, S, false, out);
}

extern "C" int hia_segments_build_packed(const hia_sample* s, int B, hia_segments** out) {
  if (!out || B < 0 || (B > 0 && !s) || B >= (1 << 20)) return HIA_ERR_INVALID_ARG;
  *out = nullptr;
  std::vector<SampleSpec> spec;
  int rc = from_samples(s, B, &spec);
  if (rc) return rc;
  const int64_t S = max_length(spec);
  if (S >= (1 << 24)) return HIA_ERR_INVALID_ARG;
  return build(spec, int(S), true, out);
}

extern "C" int hia_segments_build_multi(const hia_image* images, const int32_t* n_images,
                                        const int32_t* suffix_len, int B, int S, int packed,
                                        hia_segments** out) {
  if (!out || B < 0 || (B > 0 && (!n_images || !suffix_len)) || B >= (1 << 20)) return HIA_ERR_INVALID_ARG;
  *out = nullptr;
  std::vector<SampleSpec> spec(B);
  int64_t k = 0;
  for (int b = 0; b < B; ++b) {
    if (n_images[b] < 0 || n_images[b] > (1 << 16) || suffix_len[b] < 0) return HIA_ERR_INVALID_ARG;
    if (n_images[b] > 0 && !images) return HIA_ERR_INVALID_ARG;
    spec[b].images.assign(images + k, images + k + n_images[b]);
    spec[b].suffix = suffix_len[b];
    k += n_images[b];
  }
  if (packed) {
    const int64_t L = max_length(spec);
    if (L >= (1 << 24)) return HIA_ERR_INVALID_ARG;
    S = int(L);
  } else if (S < 0 || S >= (1 << 24)) {
    return HIA_ERR_INVALID_ARG;
  }
  return build(spec, S, packed != 0, out);
}

extern "C" int hia_segments_info(const hia_segments* g, hia_segments_info_t* info) {
  if (!g || !info) return HIA_ERR_INVALID_ARG;
  *info = g->info;
  return HIA_OK;
}

extern "C" int hia_segments_layout(const hia_segments* g, int32_t* rows, int32_t* offsets) {
  if (!g || (g->B > 0 && (!rows || !offsets))) return HIA_ERR_INVALID_ARG;
  for (int b = 0; b < g->B; ++b) {
    rows[b] = g->samples[b].rows;
    offsets[b] = g->samples[b].off;
  }
  return HIA_OK;
}

extern "C" int hia_segments_row_bound(const hia_segments* g, int32_t* e) {
  if (!g || (!e && g->B * int64_t(g->S) > 0)) return HIA_ERR_INVALID_ARG;
  for (int b = 0; b < g->B; ++b) {
    const auto& t = g->samples[b];
    const ImageDev* im = g->images.data() + t.img0;
    for (int q = 0; q < g->S; ++q) e[int64_t(b) * g->S + q] = row_bound(im, t.n_img, t.L, q);
  }
  return HIA_OK;
}

extern "C" int hia_segments_mask(const hia_segments* g, uint8_t* m) {
  if (!g || (!m && g->B * int64_t(g->S) > 0)) return HIA_ERR_INVALID_ARG;
  const int64_t S = g->S;
  for (int b = 0; b < g->B; ++b) {
    const auto& t = g->samples[b];
    const ImageDev* im = g->images.data() + t.img0;
    for (int64_t q = 0; q < S; ++q) {
      uint8_t* row = m + (int64_t(b) * S + q) * S;
      int64_t e = row_bound(im, t.n_img, t.L, int32_t(q));
      std::memset(row, 0, size_t(S));
      if (e >= 0) std::memset(row, 1, size_t(e + 1));
      for (int i = 0; i < t.n_img; ++i)  // context images ended before this row
        if (im[i].hidden && im[i].I1 <= q) std::memset(row + im[i].I0, 0, size_t(im[i].I1 - im[i].I0));
    }
  }
  return HIA_OK;
}

extern "C" int hia_segments_tile_classes(const hia_segments* g, uint8_t* cls) {
  if (!g || (!cls && g->B * int64_t(g->nQT) > 0)) return HIA_ERR_INVALID_ARG;
  for (int b = 0; b < g->B; ++b) {
    const auto& t = g->samples[b];
    for (int qt = 0; qt < g->nQT; ++qt) {
      uint8_t* row = cls + (size_t(b) * g->nQT + qt) * g->nKT;
      for (int kt = 0; kt < g->nKT; ++kt) row[kt] = kt * hia::kFwdBN >= t.L ? HIA_TILE_PADDED : HIA_TILE_SKIP;
      const int first = g->fwd_tiles[(size_t(b) * g->nQT + qt) * 2 + 0];
      const int count = g->fwd_tiles[(size_t(b) * g->nQT + qt) * 2 + 1];
      for (int j = 0; j < count; ++j) {
        const int32_t x = g->fwd_list[first + j];
        row[x & 0xffff] = (x >> 16) ? HIA_TILE_FULL : HIA_TILE_PARTIAL;
      }
    }
  }
  return HIA_OK;
}

extern "C" int hia_segments_bwd_schedule(const hia_segments* g, int index, int32_t* parts, int64_t* n_entries,
                                         int32_t* entries) {
  if (!g || index < 0 || index >= int(g->bwd_sched.size()) || !parts || !n_entries) return HIA_ERR_INVALID_ARG;
  const hia_segments::BwdSched& sc = g->bwd_sched[size_t(index)];
  *parts = sc.parts;
  *n_entries = int64_t(sc.work.size()) / hia::kBwdWorkInts;
  if (entries && !sc.work.empty()) std::memcpy(entries, sc.work.data(), sc.work.size() * sizeof(int32_t));
  return HIA_OK;
}

extern "C" const char* hia_status_string(int s) {
  switch (s) {
    case HIA_OK: return "ok";
    case HIA_ERR_INVALID_ARG: return "invalid argument";
    case HIA_ERR_UNSUPPORTED: return "unsupported configuration (head_dim, head ratio or alignment)";
    case HIA_ERR_CUDA: return "CUDA error";
    case HIA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case HIA_ERR_NOT_ON_DEVICE: return "segments not uploaded to the device";
    case HIA_ERR_SCRATCH_LIMIT: return "problem exceeds the fixed 64 MiB scratch of hia_attn_fwd_noalloc";
    default: return "unknown status";
  }
}
