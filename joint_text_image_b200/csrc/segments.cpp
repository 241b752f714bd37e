// segments.cpp -- host-side segment-descriptor builder.
//
// Replaces the dense [B,1,S,S] boolean mask of build_joint_attention_mask
// (hunyuan_image3.model: causal text, bidirectional image span, padded keys
// masked out; technical report summary 3.1.2) by per-sample bounds and a
// per-tile classification.  The rule "k < L and (k <= q or q, k both in the
// image span)" equals "k <= e(q)" with the non-decreasing row bound
// e(q) = min(L-1, q in [I0,I1) ? I1-1 : q): text rows end at themselves,
// image rows at the image's last token, suffix rows at themselves, padded
// rows at L-1.  Monotone e makes every row's visible set a prefix, so a
// (q-tile, k-tile) pair is FULL when its last key is <= e(first row), skipped
// when its first key is > e(last row), and PARTIAL otherwise.
#include <algorithm>
#include <cstring>
#include <new>

#include "internal.h"

using hia::row_bound;

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Shared by the padded and the packed layouts.  A sample's query and key
// rows are [0, rows) with rows = S (padded: rows >= L are padding) or L
// (packed: the next sample follows at once); every loop over rows below stops
// at rows, so a packed descriptor has no padded query rows and no work on
// them.
static int build(const hia_sample* s, int B, int S, bool packed, hia_segments** out) {
  hia_segments* g = new (std::nothrow) hia_segments();
  if (!g) return HIA_ERR_INVALID_ARG;
  g->B = B;
  g->S = S;
  g->packed = packed;
  g->samples.resize(B);
  int64_t off = 0;
  for (int b = 0; b < B; ++b) {
    const hia_sample& x = s[b];
    if (x.prefix_len < 0 || x.img_h < 0 || x.img_w < 0 || x.suffix_len < 0 || ((x.img_h == 0) != (x.img_w == 0))) {
      delete g;
      return HIA_ERR_INVALID_ARG;
    }
    int64_t n = int64_t(x.img_h) * x.img_w;
    int64_t L = int64_t(x.prefix_len) + n + x.suffix_len;
    if (L > S) {
      delete g;
      return HIA_ERR_INVALID_ARG;
    }
    const int32_t rows = packed ? int32_t(L) : S;
    // the padded layout addresses sample b through stride_b: its first row is row 0
    g->samples[b] = {x.prefix_len, int32_t(x.prefix_len + n), int32_t(L), x.img_w, rows,
                     packed ? int32_t(off) : 0};
    off += rows;
  }
  if (off >= (int64_t(1) << 31)) {
    delete g;
    return HIA_ERR_INVALID_ARG;
  }
  g->total_rows = off;

  // visible pairs: sum over the sample's query rows of e(q) + 1
  int64_t pairs = 0;
  for (int b = 0; b < B; ++b) {
    const auto& t = g->samples[b];
    for (int q = 0; q < t.rows; ++q) pairs += row_bound(t.I0, t.I1, t.L, q) + 1;
  }
  g->pairs = pairs;

  // forward tiles: 128 x 128
  using hia::kFwdBM;
  using hia::kFwdBN;
  g->nQT = ceil_div(S, kFwdBM);
  g->nKT = ceil_div(S, kFwdBN);
  g->fwd_tiles.assign(size_t(B) * g->nQT * 2, 0);
  int64_t nfull = 0, npart = 0, nskip = 0;
  for (int b = 0; b < B; ++b) {
    const auto& t = g->samples[b];
    for (int qt = 0; qt < g->nQT; ++qt) {
      int q0 = qt * kFwdBM, q1 = std::min(q0 + kFwdBM, int(t.rows)) - 1;
      if (q0 >= t.rows) {  // packed: no rows here
        nskip += g->nKT;
        continue;
      }
      int e0 = row_bound(t.I0, t.I1, t.L, q0), e1 = row_bound(t.I0, t.I1, t.L, q1);
      int n_vis = e1 < 0 ? 0 : ceil_div(e1 + 1, kFwdBN);
      int n_full = e0 < 0 ? 0 : (e0 + 1) / kFwdBN;
      n_full = std::min(n_full, n_vis);
      g->fwd_tiles[(size_t(b) * g->nQT + qt) * 2 + 0] = n_full;
      g->fwd_tiles[(size_t(b) * g->nQT + qt) * 2 + 1] = n_vis;
      nfull += n_full;
      npart += n_vis - n_full;
      nskip += g->nKT - n_vis;
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

  // backward tiles: 128 keys x 64 query rows.  For kv tile kt the visited
  // query tiles are [qt_first, ceil(rows / 64)) (a suffix, by monotone e);
  // those from qt_full on are FULL (all rows < rows and e(first row) >= last
  // key).
  using hia::kBwdBK;
  using hia::kBwdBQ;
  g->bQT = ceil_div(S, kBwdBQ);
  g->bKT = ceil_div(S, kBwdBK);
  g->bwd_tiles.assign(size_t(B) * g->bKT * 2, 0);
  std::vector<int64_t> bwd_cost(size_t(B) * g->bKT, 0);
  for (int b = 0; b < B; ++b) {
    const auto& t = g->samples[b];
    const int R = t.rows, nq = ceil_div(R, kBwdBQ);
    int first = 0, full = 0;  // non-decreasing in kt: two pointers
    for (int kt = 0; kt < g->bKT; ++kt) {
      int k0 = kt * kBwdBK, k1 = k0 + kBwdBK - 1;
      while (first < nq && row_bound(t.I0, t.I1, t.L, std::min((first + 1) * kBwdBQ, R) - 1) < k0) ++first;
      while (full < nq && !((full + 1) * kBwdBQ <= R && row_bound(t.I0, t.I1, t.L, full * kBwdBQ) >= k1)) ++full;
      int f = std::max(full, first);
      g->bwd_tiles[(size_t(b) * g->bKT + kt) * 2 + 0] = first;
      g->bwd_tiles[(size_t(b) * g->bKT + kt) * 2 + 1] = f;
      bwd_cost[size_t(b) * g->bKT + kt] = nq - first;
    }
  }
  order.assign(size_t(B) * g->bKT, 0);
  for (size_t i = 0; i < order.size(); ++i) order[i] = int(i);
  std::stable_sort(order.begin(), order.end(), [&](int a, int c) { return bwd_cost[a] > bwd_cost[c]; });
  g->bwd_work.resize(order.size() * 2);
  for (size_t i = 0; i < order.size(); ++i) {
    g->bwd_work[i * 2 + 0] = order[i] / g->bKT;
    g->bwd_work[i * 2 + 1] = order[i] % g->bKT;
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
  in.total_rows = g->total_rows;
  *out = g;
  return HIA_OK;
}

static int check_args(const hia_sample* s, int B, hia_segments** out) {
  if (!out || B < 0 || (B > 0 && !s)) return HIA_ERR_INVALID_ARG;
  *out = nullptr;
  if (B >= (1 << 20)) return HIA_ERR_INVALID_ARG;
  return HIA_OK;
}

extern "C" int hia_segments_build(const hia_sample* s, int B, int S, hia_segments** out) {
  int rc = check_args(s, B, out);
  if (rc) return rc;
  if (S < 0 || S >= (1 << 24)) return HIA_ERR_INVALID_ARG;
  return build(s, B, S, false, out);
}

extern "C" int hia_segments_build_packed(const hia_sample* s, int B, hia_segments** out) {
  int rc = check_args(s, B, out);
  if (rc) return rc;
  int64_t S = 0;
  for (int b = 0; b < B; ++b) {
    const hia_sample& x = s[b];
    if (x.prefix_len < 0 || x.img_h < 0 || x.img_w < 0 || x.suffix_len < 0) return HIA_ERR_INVALID_ARG;
    S = std::max(S, int64_t(x.prefix_len) + int64_t(x.img_h) * x.img_w + x.suffix_len);
  }
  if (S >= (1 << 24)) return HIA_ERR_INVALID_ARG;
  return build(s, B, int(S), true, out);
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
    for (int q = 0; q < g->S; ++q) e[int64_t(b) * g->S + q] = row_bound(t.I0, t.I1, t.L, q);
  }
  return HIA_OK;
}

extern "C" int hia_segments_mask(const hia_segments* g, uint8_t* m) {
  if (!g || (!m && g->B * int64_t(g->S) > 0)) return HIA_ERR_INVALID_ARG;
  const int64_t S = g->S;
  for (int b = 0; b < g->B; ++b) {
    const auto& t = g->samples[b];
    for (int64_t q = 0; q < S; ++q) {
      uint8_t* row = m + (int64_t(b) * S + q) * S;
      int64_t e = row_bound(t.I0, t.I1, t.L, int32_t(q));
      std::memset(row, 0, size_t(S));
      if (e >= 0) std::memset(row, 1, size_t(e + 1));
    }
  }
  return HIA_OK;
}

extern "C" int hia_segments_tile_classes(const hia_segments* g, uint8_t* cls) {
  if (!g || (!cls && g->B * int64_t(g->nQT) > 0)) return HIA_ERR_INVALID_ARG;
  for (int b = 0; b < g->B; ++b) {
    const auto& t = g->samples[b];
    for (int qt = 0; qt < g->nQT; ++qt) {
      int n_full = g->fwd_tiles[(size_t(b) * g->nQT + qt) * 2 + 0];
      int n_vis = g->fwd_tiles[(size_t(b) * g->nQT + qt) * 2 + 1];
      for (int kt = 0; kt < g->nKT; ++kt) {
        uint8_t c;
        if (kt < n_full) c = HIA_TILE_FULL;
        else if (kt < n_vis) c = HIA_TILE_PARTIAL;
        else if (kt * hia::kFwdBN >= t.L) c = HIA_TILE_PADDED;
        else c = HIA_TILE_SKIP;
        cls[(size_t(b) * g->nQT + qt) * g->nKT + kt] = c;
      }
    }
  }
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
