/*
 * jointattn.h -- C ABI of libjointattn: the generalized-causal GQA
 * self-attention of a unified text+image decoder (HunyuanImage-3.0), with the
 * generalized 2D RoPE applied to Q and K, forward and recompute backward, for
 * NVIDIA B200 (sm_100a).
 *
 * Conventions for every entry point
 *   - Return value: an hia_status (HIA_OK = 0).  All argument checks run on the
 *     host before anything is launched; on error nothing is launched and no
 *     output is touched.
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *     default stream).  Every device call is asynchronous on that stream; the
 *     library never synchronizes the device and never allocates inside
 *     hia_attn_fwd / hia_attn_bwd (the caller passes the workspace).
 *   - Ownership: the caller owns every device buffer (tensors, tables,
 *     workspace).  The library owns only hia_segments objects, which the
 *     caller frees with hia_segments_destroy.
 *   - Dtypes: bf16 for q, k, v, o, dout, dq, dk, dv; fp32 for cos, sin, lse.
 *   - Shapes: B samples, padded length S, Hq query heads, Hkv key/value heads
 *     (Hq % Hkv == 0, g = Hq / Hkv query heads per kv head), head_dim D in
 *     {64, 128}.
 *
 * Citations name the page title and the section or API item they come from.
 */
#ifndef JOINTATTN_H
#define JOINTATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HIA_OK = 0,
    HIA_ERR_INVALID_ARG = 1,    /* null pointer, negative size, bad geometry, short workspace */
    HIA_ERR_UNSUPPORTED = 2,    /* D not in {64,128}, Hq % Hkv != 0, misaligned pointer/stride */
    HIA_ERR_CUDA = 3,           /* a CUDA runtime/driver call failed */
    HIA_ERR_DEVICE_TIMEOUT = 4, /* a kernel's bounded wait expired (see hia_get_device_status) */
    HIA_ERR_NOT_ON_DEVICE = 5,  /* hia_segments used on the device before hia_segments_upload */
    HIA_ERR_SCRATCH_LIMIT = 6   /* problem larger than hia_attn_fwd_noalloc's fixed scratch */
} hia_status;

/* One sample of the batch.  Layout (HunyuanImage-3.0 coverage page, Cache
 * Contract; hunyuan_image3.model HunyuanImage3ForCausalMM.forward, input_ids):
 *   [0, prefix_len)                 text, ending in the <timestep> token
 *   [prefix_len, prefix_len + h*w)  image tokens, row-major (h, w) order
 *   [.., L = prefix + h*w + suffix) suffix text (e.g. <eoi>)
 *   [L, S)                          right padding
 * img_h = img_w = 0 is a text-only sample.  Equivalent to the reference
 * mask builder's arguments with image_starts = prefix_len, num_image_tokens =
 * h*w (here allowed to differ per sample) and valid_lengths = L. */
typedef struct {
    int32_t prefix_len;
    int32_t img_h;
    int32_t img_w;
    int32_t suffix_len;
} hia_sample;

/* One image of a sample with several images: text_before text tokens, then
 * an img_h x img_w image (row-major, img_h, img_w > 0). */
typedef struct {
    int32_t text_before;
    int32_t img_h;
    int32_t img_w;
} hia_image;

/* A strided [B, S, heads, D] bf16 (or fp32) device tensor.  Strides are in
 * elements; the last dimension is contiguous.  For a tensor with Hq heads,
 * head h lives at ptr + (h / g) * stride_hkv + (h % g) * stride_hq, which
 * covers both a plain [B,S,Hq,D] tensor (stride_hkv = g*D, stride_hq = D) and
 * the fused KV-head-grouped QKV projection output [B,S,Hkv,g+2,D]
 * (hunyuan_image3.layers HunyuanImage3Attention: per kv head, its g query
 * heads then one key and one value head).  For a tensor with Hkv heads, head
 * h lives at ptr + h * stride_hkv and stride_hq is ignored.  Every stride in
 * bytes and the pointer must be multiples of 16. */
typedef struct {
    void* ptr;
    int64_t stride_b;
    int64_t stride_s;
    int64_t stride_hkv;
    int64_t stride_hq;
} hia_tensor;

/* Opaque segment descriptor, owned by the library. */
typedef struct hia_segments hia_segments;

/* Summary numbers of a descriptor. */
typedef struct {
    int32_t B, S;
    int64_t visible_pairs;       /* sum over b and query rows q < S of (e_b(q) + 1) */
    int32_t fwd_q_tiles;         /* ceil(S / 128) */
    int32_t fwd_kv_tiles;        /* ceil(S / 128) */
    int64_t fwd_tiles_full;      /* (b, q-tile, kv-tile) triples, 128 x 128 tiles */
    int64_t fwd_tiles_partial;
    int64_t fwd_tiles_skipped;   /* fully masked, incl. padded keys: never loaded */
    int32_t bwd_q_tiles;         /* ceil(S / 64) */
    int32_t bwd_kv_tiles;        /* ceil(S / 128) */
    int32_t packed;              /* 1: built by hia_segments_build_packed */
    int32_t bwd_split_units;     /* kv tiles a split schedule can cut into parts (see hia_segments_set_bwd_split) */
    int64_t total_rows;          /* rows of a tensor in this layout: B*S, or the sum of L when packed */
} hia_segments_info_t;

/* Tile classes reported by hia_segments_tile_classes. */
enum {
    HIA_TILE_SKIP = 0,       /* every pair masked (causal future or image-block edge) */
    HIA_TILE_FULL = 1,       /* every pair visible: no predicate evaluated */
    HIA_TILE_PARTIAL = 2,    /* mixed: per-pair predicate k <= e(q) in registers */
    HIA_TILE_PADDED = 3      /* keys all at or beyond L (right padding): skipped */
};

/* Build the segment descriptor that replaces the dense [B,1,S,S] boolean
 * mask (hunyuan_image3.model build_joint_attention_mask: causal text,
 * bidirectional image span, padded keys masked out; technical report summary
 * 3.1.2; paper review 3.3).  With I0 = prefix_len, I1 = I0 + h*w and
 * L = I1 + suffix_len, key k is visible from query q iff k <= e(q) where
 *   e(q) = min(L - 1, (I0 <= q < I1) ? I1 - 1 : q),
 * a non-decreasing row bound (padded query rows see every real key).  From it
 * the builder classifies every (q-tile, kv-tile) as FULL, PARTIAL or skipped
 * and orders the work heaviest first.  Host only: no CUDA call is made.
 * samples: host array of B entries.  S >= max L.  On success *out receives a
 * new object.  Errors: HIA_ERR_INVALID_ARG (null, B < 0, S < 0, negative
 * lengths, exactly one of img_h/img_w zero, L > S, S >= 2^24). */
int hia_segments_build(const hia_sample* samples, int B, int S, hia_segments** out);

/* The same descriptor for the PACKED (varlen) layout: the samples are stored
 * back to back with no padding rows, sample b's rows starting at row
 * off_b = L_0 + ... + L_{b-1} of a [total_rows, heads, D] tensor
 * (total_rows = sum of L).  Every hia_tensor passed with such a descriptor
 * addresses row s of sample b at ptr + (off_b + s) * stride_s (stride_b is
 * ignored), lse is fp32 [Hq, total_rows], and the RoPE tables stay
 * [B, S, D] with S = max L.  There are no padded query rows: nothing is
 * computed, read or written past a sample's L.  Errors as hia_segments_build
 * (S >= 2^24 or total_rows >= 2^31 refused). */
int hia_segments_build_packed(const hia_sample* samples, int B, hia_segments** out);

/* Samples with any number of images (technical report summary 3.1.2: in
 * a training sequence with several generated images, an image already in
 * context is masked from the tokens after it; positions 3.1.3).  Sample b is
 * n_images[b] entries of `images` (consecutive, in order: each is its text
 * then its image), then suffix_len[b] text tokens.  Reading of the pages:
 * every image of a sample but its last is a context image, hidden from all
 * tokens after its span; the last image follows the one-image rule, so one
 * image per sample is exactly hia_segments_build.  Each image sits on its own
 * 2D grid (x = I0 + column, y = I0 + row); text keeps x = y = its index (the
 * pages also shift positions after a generated image, by an amount they do
 * not give: not modelled).  packed != 0 builds the packed layout (S is then
 * computed as max L and ignored).  Errors: HIA_ERR_INVALID_ARG (null
 * arrays, negative counts or lengths, an image with h or w <= 0, L > S). */
int hia_segments_build_multi(const hia_image* images, const int32_t* n_images, const int32_t* suffix_len,
                             int B, int S, int packed, hia_segments** out);

/* Copy the per-sample bounds, tile tables and work lists to the current
 * device (allocated once per object; asynchronous on `stream`).  Must
 * precede hia_rope2d_tables / hia_attn_fwd / hia_attn_bwd. */
int hia_segments_upload(hia_segments* seg, void* stream);

/* Free the object and its device copies (the device copies are freed with
 * cudaFree, which synchronizes).  NULL is a no-op. */
void hia_segments_destroy(hia_segments* seg);

int hia_segments_info(const hia_segments* seg, hia_segments_info_t* info);

/* Scheduling of the backward (a property of the library, not of the method:
 * the result is the same either way, and deterministic).  One CTA of the
 * backward handles one (sample, kv head, 128-key tile) over every query tile
 * that sees it, so CTAs differ in length by up to the whole query range and
 * the last ones can leave SMs idle at the end.  Besides that whole schedule,
 * the descriptor holds split schedules: for parts k in {2, 3, 4} and a
 * threshold of 95, 90 or 85% of the longest query range, every kv tile at or
 * above the threshold is cut into k consecutive query sub-ranges (of at least
 * two 64-row tiles each), each run by its own CTA that writes fp32 partials
 * of dK and dV; the part that finishes last adds the k partials in part
 * order (bitwise the same whichever part is last) and writes dK and dV.
 *   HIA_BWD_SPLIT_AUTO (default): each backward launch takes the schedule a
 *     list-scheduling estimate (heaviest first, on the device's SM count, for
 *     its number of kv heads and g) finishes soonest.
 *   HIA_BWD_SPLIT_NEVER: the whole schedule.
 *   HIA_BWD_SPLIT_ALWAYS: the estimate's best split schedule.
 *   HIA_BWD_SPLIT_PARTS_2 / _3 / _4: the estimate's best schedule cutting
 *     tiles into exactly 2 / 3 / 4 parts.
 * A mode that admits no schedule of the descriptor (nothing long enough to
 * split) runs the whole one.  The choice is made per (mode, kv heads, g, SM
 * count); hia_attn_bwd_workspace_bytes sizes the partials for the choice on
 * the current device, and a workspace too small for a later choice (another
 * device, or the mode changed after sizing) runs the whole schedule.
 * Errors: HIA_ERR_INVALID_ARG (null, unknown mode). */
enum {
  HIA_BWD_SPLIT_AUTO = 0,
  HIA_BWD_SPLIT_NEVER = 1,
  HIA_BWD_SPLIT_ALWAYS = 2,
  HIA_BWD_SPLIT_PARTS_2 = 3,
  HIA_BWD_SPLIT_PARTS_3 = 4,
  HIA_BWD_SPLIT_PARTS_4 = 5
};
int hia_segments_set_bwd_split(hia_segments* seg, int mode);

/* Inspection of the backward schedules (host only, no CUDA call).
 * hia_segments_bwd_schedule: schedule `index` (0 = the whole one; the
 * others in order of parts, then of decreasing threshold): *parts (1 for the
 * whole schedule), *n_entries, and, if entries is not NULL, its work list,
 * int32 [n_entries][8] = (b, kv tile, first query tile, end query tile,
 * slot (-1 unless split), part, parts, 0), in launch order (one CTA per
 * entry and kv head).  HIA_ERR_INVALID_ARG past the last schedule.
 * hia_segments_bwd_choice: the schedule index a launch with Hkv kv heads, g
 * query heads per kv head and n_sm SMs takes under the current mode. */
int hia_segments_bwd_schedule(const hia_segments* seg, int index, int32_t* parts, int64_t* n_entries,
                              int32_t* entries);
int hia_segments_bwd_choice(const hia_segments* seg, int Hkv, int g, int n_sm, int* index);

/* Host copies for tests and inspection.  row_bound: int32 [B, S] e_b(q)
 * (-1 for a sample with L = 0).  mask: uint8 [B, S, S] (1 = visible) rendered
 * from e, for a bit-exact comparison with the reference rule.  classes:
 * uint8 [B, fwd_q_tiles, fwd_kv_tiles] with HIA_TILE_* values. */
int hia_segments_row_bound(const hia_segments* seg, int32_t* row_bound);
/* Per-sample layout, int32 [B] each: rows = the sample's rows in a tensor of
 * this layout (S padded, L packed) and offsets = its first row (0 padded,
 * L_0 + ... + L_{b-1} packed).  The packed offsets are what a caller uses to
 * cut its packed tensors per sample. */
int hia_segments_layout(const hia_segments* seg, int32_t* rows, int32_t* offsets);
int hia_segments_mask(const hia_segments* seg, uint8_t* mask);
int hia_segments_tile_classes(const hia_segments* seg, uint8_t* classes);

/* Generalized 2D RoPE tables (paper review 3.4 and Figure 5; technical report
 * summary 3.1.3): cos, sin fp32 [B, S, D] device buffers written on `stream`.
 * Token n of a sample sits at (x, y) = (n, n) unless it is image token
 * i = n - I0, which sits at x = I0 + (i % w), y = I0 + (i / w).  For
 * j < D/2, angle_j = (j even ? x : y) * base^(-2j/D), and
 * cos[b,n,j] = cos[b,n,j+D/2] = cos(angle_j), likewise sin (the cos block /
 * sin block layout of the [B, S, head_dim] tables taken by
 * HunyuanImage3Attention.forward).  Angles and cos/sin are evaluated in fp64
 * and rounded once to fp32, so a text-only sample gives exactly the 1D RoPE
 * tables.  D even, 2 <= D <= 256, base > 0.  Errors: HIA_ERR_INVALID_ARG
 * (null seg or buffers, D or base out of range), HIA_ERR_UNSUPPORTED
 * (B * S >= 2^31 table rows), HIA_ERR_NOT_ON_DEVICE, HIA_ERR_CUDA. */
int hia_rope2d_tables(const hia_segments* seg, int D, double base, float* cos_out,
                      float* sin_out, void* stream);

/* Bytes of device workspace hia_attn_fwd needs (256-byte aligned pointer). */
size_t hia_attn_fwd_workspace_bytes(const hia_segments* seg, int Hq, int Hkv, int D);

/* Forward of the masked GQA attention with RoPE applied to q and k
 * (HunyuanImage3Attention.forward: q_r = q*cos + rotate_half(q)*sin, the same
 * for k; rotate_half(v) = [-v[D/2:], v[:D/2]]; v is not rotated; scores
 * scale * q_r . k_r over visible pairs; softmax; output P v).
 *   q [B,S,Hq,D], k, v [B,S,Hkv,D], o [B,S,Hq,D] (bf16, hia_tensor strides);
 *   cos, sin fp32 [B,S,D] (from hia_rope2d_tables or the caller's own);
 *   lse fp32 [B,Hq,S] contiguous: natural-log sum of exp(scaled scores) per
 *   row (-inf, with o = 0, for a row with no visible key, i.e. L = 0);
 *   scale: usually 1/sqrt(D).  Padded query rows are computed like any row.
 * Q and K are rotated once into the workspace (bf16, [B,H,S,D]) by a
 * bandwidth-bound pre-pass; the attention kernel streams them with TMA into
 * tcgen05 MMAs.  Errors: HIA_ERR_INVALID_ARG, HIA_ERR_UNSUPPORTED,
 * HIA_ERR_NOT_ON_DEVICE, HIA_ERR_CUDA (launch failure). */
int hia_attn_fwd(const hia_segments* seg, int Hq, int Hkv, int D, hia_tensor q, hia_tensor k,
                 hia_tensor v, const float* cos_t, const float* sin_t, float scale,
                 hia_tensor o, float* lse, void* workspace, size_t workspace_bytes,
                 void* stream);

/* Per-head QK RMSNorm applied after RoPE (HunyuanImage3Attention with
 * use_qk_norm: RoPE is applied before the per-head QK RMSNorm; HunyuanRMSNorm
 * normalizes over the last axis with eps and scales by its weight).  With a
 * norm, the attention uses y = w * x / sqrt(mean(x^2) + eps) of every rotated
 * q row (w = wq) and k row (w = wk), x = R q or R k, computed in fp32 and
 * rounded once to bf16.  wq, wk: fp32 [D] device pointers, 16-byte aligned;
 * eps >= 0 (the layer's default is 1e-5). */
typedef struct {
    const float* wq;
    const float* wk;
    float eps;
} hia_qk_norm;

/* hia_attn_fwd with an optional QK RMSNorm (norm == NULL: none, identical to
 * hia_attn_fwd).  Same workspace.  Extra errors: HIA_ERR_INVALID_ARG for a
 * null weight or a negative or non-finite eps, HIA_ERR_UNSUPPORTED for a
 * misaligned weight pointer. */
int hia_attn_fwd_ex(const hia_segments* seg, int Hq, int Hkv, int D, hia_tensor q, hia_tensor k,
                    hia_tensor v, const float* cos_t, const float* sin_t, float scale,
                    const hia_qk_norm* norm, hia_tensor o, float* lse, void* workspace,
                    size_t workspace_bytes, void* stream);

/* hia_attn_fwd for callers that cannot allocate device memory.  (No
 * counterpart on the pages: this is a property of the library, not of the
 * method.)  Some callers may not call cudaMalloc at all: a plug-in inside a
 * host runtime that owns all device memory and passes it only its inputs and
 * outputs, or a step that must not call cudaMalloc/cudaFree midway because
 * they synchronize the device.  This entry point takes the same inputs and
 * outputs as hia_attn_fwd but no workspace: the rotated q and k go into a
 * fixed 64 MiB array compiled into the library (a __device__ variable), which
 * every GPU that loads the library holds until the process exits.  It calls
 * no cudaMalloc, cudaFree or other allocating routine.
 *   - Limit: hia_attn_fwd_workspace_bytes(seg, Hq, Hkv, D) must not exceed
 *     64 MiB = 67,108,864 bytes (B*S*(Hq+Hkv)*D*2 bytes
 *     plus 256-byte alignment; e.g. one 1024px sample, S = 5122, Hq = 32, Hkv = 8,
 *     D = 128 needs 52.5 MB).  Larger problems return HIA_ERR_SCRATCH_LIMIT
 *     before anything is launched.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current), which also loads the
 *     library module holding it; make that first call before any stream
 *     capture on the device.  The address belongs to the device's context:
 *     if the context is replaced (cudaDeviceReset, then new work), the next
 *     call sees the new context and looks the address up again, so that call
 *     too should come before any capture.
 *   - Argument errors are checked first, exactly as hia_attn_fwd checks
 *     them; only a problem with valid arguments can get the size error.
 *   - All calls share the one array and it keeps the last call's contents
 *     (nothing in it needs to start at zero: every element that is read is
 *     first rewritten by the same call).  Calls whose GPU work overlaps, e.g.
 *     on two streams, race on it: issue them on one stream or order them.
 * Errors: those of hia_attn_fwd, plus HIA_ERR_SCRATCH_LIMIT. */
int hia_attn_fwd_noalloc(const hia_segments* seg, int Hq, int Hkv, int D, hia_tensor q, hia_tensor k,
                         hia_tensor v, const float* cos_t, const float* sin_t, float scale,
                         hia_tensor o, float* lse, void* stream);

/* Bytes of device workspace hia_attn_bwd and hia_attn_bwd_ex need (the
 * size covers the QK RMSNorm's extra accumulators either way, and the fp32
 * partials of the backward schedule chosen for the current device and the
 * descriptor's mode: see hia_segments_set_bwd_split). */
size_t hia_attn_bwd_workspace_bytes(const hia_segments* seg, int Hq, int Hkv, int D);

/* Recompute backward of hia_attn_fwd: given o and lse from the forward and
 * dout = dL/do, writes dq [B,S,Hq,D], dk, dv [B,S,Hkv,D] (bf16), i.e. the
 * gradients w.r.t. the un-rotated q and k (dq = R^T dq_r, dk = R^T dk_r) and
 * v, summed over the g query heads of each kv head.  Same conventions and
 * errors as hia_attn_fwd. */
int hia_attn_bwd(const hia_segments* seg, int Hq, int Hkv, int D, hia_tensor q, hia_tensor k,
                 hia_tensor v, const float* cos_t, const float* sin_t, float scale,
                 hia_tensor o, const float* lse, hia_tensor dout, hia_tensor dq,
                 hia_tensor dk, hia_tensor dv, void* workspace, size_t workspace_bytes,
                 void* stream);

/* hia_attn_bwd with an optional QK RMSNorm: norm must be the one given to
 * the forward that produced o and lse.  With a norm, dq and dk are the
 * gradients with respect to the un-rotated, un-normed q and k (through the
 * norm and R^T), and dwq, dwk (fp32 [D] device, overwritten) receive the
 * gradients of wq and wk summed over every row and head, in a fixed order
 * (deterministic).  norm == NULL: identical to hia_attn_bwd; dwq, dwk are
 * ignored.  Errors as hia_attn_fwd_ex, plus HIA_ERR_INVALID_ARG for null
 * dwq/dwk with a norm. */
int hia_attn_bwd_ex(const hia_segments* seg, int Hq, int Hkv, int D, hia_tensor q, hia_tensor k,
                    hia_tensor v, const float* cos_t, const float* sin_t, float scale,
                    const hia_qk_norm* norm, hia_tensor o, const float* lse, hia_tensor dout,
                    hia_tensor dq, hia_tensor dk, hia_tensor dv, float* dwq, float* dwk,
                    void* workspace, size_t workspace_bytes, void* stream);

/* hia_attn_bwd_ex that reuses the rotated (and, with a norm, normed) q and
 * k which the forward left in its workspace, instead of computing them again
 * (the rotation is the same arithmetic either way: R q and R k in fp32,
 * rounded once to bf16).  fwd_workspace: the workspace of the
 * hia_attn_fwd / hia_attn_fwd_ex call that produced o and lse, with the same
 * seg, heads, D, q, k, cos, sin and norm, not written since;
 * fwd_workspace_bytes >= hia_attn_fwd_workspace_bytes and 256-byte aligned.
 * A caller that keeps the forward workspace alive until the backward trades
 * that memory (B*S*(Hq+Hkv)*D*2 bytes) for one rotation pass per step.
 * fwd_workspace == NULL: identical to hia_attn_bwd_ex.  The backward
 * workspace is still required (its dQ accumulator and row statistics).
 * Errors as hia_attn_bwd_ex, plus HIA_ERR_INVALID_ARG for a short or
 * misaligned fwd_workspace. */
int hia_attn_bwd_reuse_fwd(const hia_segments* seg, int Hq, int Hkv, int D, hia_tensor q, hia_tensor k,
                           hia_tensor v, const float* cos_t, const float* sin_t, float scale,
                           const hia_qk_norm* norm, hia_tensor o, const float* lse, hia_tensor dout,
                           hia_tensor dq, hia_tensor dk, hia_tensor dv, float* dwq, float* dwk,
                           const void* fwd_workspace, size_t fwd_workspace_bytes, void* workspace,
                           size_t workspace_bytes, void* stream);

/* ---- One training step from HOST buffers.  (No counterpart on the pages:
 * a convenience of the library for callers that hold their tensors in host
 * memory.)  A hia_step owns, on the device current at creation, the device
 * copies of one step's tensors in the plain contiguous layout (q, dout, o,
 * dq: [B,S,Hq,D] bf16; k, v, dk, dv: [B,S,Hkv,D] bf16; lse: [B,Hq,S] fp32),
 * the RoPE tables of `seg` (computed once, at creation, with `rope_base`) and
 * both workspaces (the backward reuses the forward's rotated q and k).  `seg` must stay alive and uploaded while the step exists.
 * Returns HIA_ERR_INVALID_ARG for null pointers, non-positive head counts
 * or rope_base, HIA_ERR_UNSUPPORTED unless D is 64 or 128 and Hq a multiple
 * of Hkv, HIA_ERR_NOT_ON_DEVICE if `seg` was not uploaded, HIA_ERR_CUDA if
 * an allocation fails (nothing is left allocated). */
typedef struct hia_step hia_step;
int hia_step_create(const hia_segments* seg, int Hq, int Hkv, int D, double rope_base, hia_step** out);
/* Waits for the step's own copy stream, then frees everything it owns. */
void hia_step_destroy(hia_step* st);

/* Enqueue one forward + backward on `stream` from host buffers (all
 * pointers below are HOST pointers, in the layouts above): copies q, k, v,
 * dout to the device, runs hia_attn_fwd and hia_attn_bwd, copies o, lse, dq,
 * dk, dv back.  dout is uploaded, and o and lse downloaded, on the step's own
 * copy stream so that they overlap the kernels; `stream` waits for that
 * stream at the end, so once `stream` reaches this point every output is in
 * host memory.  Asynchronous: host buffers must stay valid until then.
 * Pinned (page-locked) host memory makes the copies asynchronous; pageable
 * memory works but the copies then block the calling thread.  Two steps
 * enqueued on two streams overlap one step's copies with the other's
 * kernels.  Errors: HIA_ERR_INVALID_ARG (null pointer), the errors of
 * hia_attn_fwd / hia_attn_bwd, HIA_ERR_CUDA. */
int hia_attn_step_host(hia_step* st, const void* q, const void* k, const void* v, const void* dout,
                       float scale, void* o, float* lse, void* dq, void* dk, void* dv, void* stream);

/* Read and clear the device status word of the current device (synchronizes
 * `stream`).  Returns HIA_OK, HIA_ERR_DEVICE_TIMEOUT if any kernel's bounded
 * wait expired since the last call, or HIA_ERR_CUDA. */
int hia_get_device_status(void* stream);

/* Test hook for the bounded-wait machinery: launches one block that waits on
 * an mbarrier nothing ever arrives on, with the given limit in nanoseconds;
 * the wait expires, records HIA_ERR_DEVICE_TIMEOUT in the status word and the
 * kernel returns normally.  timeout_ns in [1, 10^9]. */
int hia_debug_wait_timeout(uint64_t timeout_ns, void* stream);

/* Test hook for the softmax's FMA-pipe exponential: y[i] = 2^x[i] for n
 * fp32 device values, computed as the forward kernel computes part of its
 * exponentials (Cody-Waite range reduction, cubic for 2^f on [0, 1);
 * relative error <= 1e-4 for x in [-125, 64]; x < -125, -inf included,
 * gives about 2^-125). Returns HIA_ERR_INVALID_ARG for n < 0 or null
 * pointers with n > 0; launch errors as HIA_ERR_CUDA. */
int hia_debug_exp2(const float* x, float* y, int n, void* stream);

const char* hia_status_string(int status);

/* Per-kernel device timing, for benchmarks.  Between hia_profile_begin() and
 * hia_profile_end(), every kernel the library launches from any thread is
 * bracketed by a pair of CUDA events recorded on its launch stream (event
 * objects are created once and reused; recording adds no device work).
 * hia_profile_end synchronizes those events and fills up to max_entries
 * records, one per kernel name, with the launch count and the summed
 * event-to-event time; *n_out receives the number of records.  Kernel names:
 * "rope2d_tables", "rope_rotate", "attn_fwd", "bwd_pre", "attn_bwd",
 * "grad_finalize", "dw_reduce".  Not a library-wide profiler: no other state
 * changes. */
typedef struct {
    char name[32];
    int32_t launches;
    double total_ms;
} hia_kernel_time;

int hia_profile_begin(void);
int hia_profile_end(hia_kernel_time* out, int max_entries, int* n_out);

#ifdef __cplusplus
}
#endif

#endif /* JOINTATTN_H */
