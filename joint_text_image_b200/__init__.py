"""libjointattn: generalized-causal GQA attention with generalized 2D RoPE
(HunyuanImage-3.0) for B200 / sm_100a.

Thin ctypes binding over the C ABI in ``include/jointattn.h``: these functions
only marshal arguments (torch tensors -> pointers and strides, the current
torch CUDA stream); every step runs in the library's CUDA kernels.  There is no
CPU fallback: if ``libjointattn.so`` is missing or fails to load, every call
raises.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "HiaError", "Segments", "lib", "hia_segments_build", "hia_rope2d_tables", "hia_attn_fwd",
    "hia_attn_bwd", "hia_attn_fwd_workspace_bytes", "hia_attn_bwd_workspace_bytes",
    "hia_get_device_status", "hia_debug_wait_timeout", "hia_profile_begin", "hia_profile_end",
    "Step", "hia_step_create", "hia_attn_step_host", "hia_segments_build_packed", "hia_segments_build_multi",
    "LIB_PATH",
    "EXPORTED_SYMBOLS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libjointattn.so")

EXPORTED_SYMBOLS = (
    "hia_segments_build", "hia_segments_upload", "hia_segments_destroy", "hia_segments_info",
    "hia_segments_row_bound", "hia_segments_mask", "hia_segments_tile_classes", "hia_rope2d_tables",
    "hia_attn_fwd_workspace_bytes", "hia_attn_fwd", "hia_attn_bwd_workspace_bytes", "hia_attn_bwd",
    "hia_get_device_status", "hia_debug_wait_timeout", "hia_status_string", "hia_profile_begin",
    "hia_profile_end", "hia_attn_fwd_noalloc", "hia_debug_exp2", "hia_step_create", "hia_step_destroy",
    "hia_attn_step_host", "hia_attn_fwd_ex", "hia_attn_bwd_ex", "hia_segments_build_packed",
    "hia_segments_layout", "hia_segments_build_multi", "hia_attn_bwd_reuse_fwd",
    "hia_moe_workspace_bytes", "hia_moe_fwd", "hia_segments_set_bwd_split", "hia_segments_bwd_schedule",
    "hia_segments_bwd_choice",
)


class HiaError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        super().__init__(f"{what}: {_status_string(code)} (status {code})")


class _Sample(ctypes.Structure):
    _fields_ = [("prefix_len", ctypes.c_int32), ("img_h", ctypes.c_int32),
                ("img_w", ctypes.c_int32), ("suffix_len", ctypes.c_int32)]


class _Tensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("stride_b", ctypes.c_int64), ("stride_s", ctypes.c_int64),
                ("stride_hkv", ctypes.c_int64), ("stride_hq", ctypes.c_int64)]


class SegmentsInfo(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("S", ctypes.c_int32), ("visible_pairs", ctypes.c_int64),
                ("fwd_q_tiles", ctypes.c_int32), ("fwd_kv_tiles", ctypes.c_int32),
                ("fwd_tiles_full", ctypes.c_int64), ("fwd_tiles_partial", ctypes.c_int64),
                ("fwd_tiles_skipped", ctypes.c_int64), ("bwd_q_tiles", ctypes.c_int32),
                ("bwd_kv_tiles", ctypes.c_int32), ("packed", ctypes.c_int32), ("bwd_split_units", ctypes.c_int32),
                ("total_rows", ctypes.c_int64)]


class _QkNorm(ctypes.Structure):
    _fields_ = [("wq", ctypes.c_void_p), ("wk", ctypes.c_void_p), ("eps", ctypes.c_float)]


class _Image(ctypes.Structure):
    _fields_ = [("text_before", ctypes.c_int32), ("img_h", ctypes.c_int32), ("img_w", ctypes.c_int32)]


class _MoeDims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32), ("E", ctypes.c_int32),
                ("topk", ctypes.c_int32)]


class _KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int32), ("total_ms", ctypes.c_double)]


_lib = None


def lib():
    """The loaded libjointattn.so (raises if it is missing: no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                              "or python joint_text_image_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        P, I, Z, T = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, _Tensor
        L.hia_segments_build.argtypes = [ctypes.POINTER(_Sample), I, I, ctypes.POINTER(P)]
        L.hia_segments_build_packed.argtypes = [ctypes.POINTER(_Sample), I, ctypes.POINTER(P)]
        L.hia_segments_build_multi.argtypes = [ctypes.POINTER(_Image), P, P, I, I, I, ctypes.POINTER(P)]
        L.hia_segments_upload.argtypes = [P, P]
        L.hia_segments_destroy.argtypes = [P]
        L.hia_segments_destroy.restype = None
        L.hia_segments_info.argtypes = [P, ctypes.POINTER(SegmentsInfo)]
        L.hia_segments_set_bwd_split.argtypes = [P, I]
        L.hia_segments_bwd_schedule.argtypes = [P, I, P, P, P]
        L.hia_segments_bwd_choice.argtypes = [P, I, I, I, P]
        L.hia_segments_row_bound.argtypes = [P, P]
        L.hia_segments_layout.argtypes = [P, P, P]
        L.hia_segments_mask.argtypes = [P, P]
        L.hia_segments_tile_classes.argtypes = [P, P]
        L.hia_rope2d_tables.argtypes = [P, I, ctypes.c_double, P, P, P]
        L.hia_attn_fwd_workspace_bytes.argtypes = [P, I, I, I]
        L.hia_attn_fwd_workspace_bytes.restype = Z
        L.hia_attn_bwd_workspace_bytes.argtypes = [P, I, I, I]
        L.hia_attn_bwd_workspace_bytes.restype = Z
        L.hia_attn_fwd.argtypes = [P, I, I, I, T, T, T, P, P, ctypes.c_float, T, P, P, Z, P]
        L.hia_attn_bwd.argtypes = [P, I, I, I, T, T, T, P, P, ctypes.c_float, T, P, T, T, T, T, P, Z, P]
        L.hia_attn_bwd_reuse_fwd.argtypes = [P, I, I, I, T, T, T, P, P, ctypes.c_float, P, T, P, T, T, T, T, P, P,
                                             P, Z, P, Z, P]
        L.hia_moe_workspace_bytes.argtypes = [ctypes.POINTER(_MoeDims)]
        L.hia_moe_workspace_bytes.restype = Z
        L.hia_moe_fwd.argtypes = [ctypes.POINTER(_MoeDims), P, P, P, P, P, P, P, P, Z, P]
        L.hia_get_device_status.argtypes = [P]
        L.hia_debug_wait_timeout.argtypes = [ctypes.c_uint64, P]
        QN = ctypes.POINTER(_QkNorm)
        L.hia_attn_fwd_ex.argtypes = [P, I, I, I, T, T, T, P, P, ctypes.c_float, QN, T, P, P, Z, P]
        L.hia_attn_bwd_ex.argtypes = [P, I, I, I, T, T, T, P, P, ctypes.c_float, QN, T, P, T, T, T, T, P, P, P,
                                      Z, P]
        L.hia_attn_fwd_noalloc.argtypes = [P, I, I, I, T, T, T, P, P, ctypes.c_float, T, P, P]
        L.hia_debug_exp2.argtypes = [P, P, I, P]
        L.hia_step_create.argtypes = [P, I, I, I, ctypes.c_double, ctypes.POINTER(P)]
        L.hia_step_destroy.argtypes = [P]
        L.hia_step_destroy.restype = None
        L.hia_attn_step_host.argtypes = [P, P, P, P, P, ctypes.c_float, P, P, P, P, P, P]
        L.hia_profile_begin.argtypes = []
        L.hia_profile_end.argtypes = [ctypes.POINTER(_KernelTime), I, ctypes.POINTER(I)]
        L.hia_status_string.argtypes = [I]
        L.hia_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _status_string(code):
    try:
        return lib().hia_status_string(int(code)).decode()
    except Exception:  # library missing: still report the code
        return "status"


def _check(rc, what):
    if rc != 0:
        raise HiaError(rc, what)


def _stream(device=None):
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


class Segments:
    """Owner of a library hia_segments object (host tables + device copies)."""

    def __init__(self, samples, S, packed=False):
        """samples: (prefix, img_h, img_w, suffix) per sample, or, for several
        images, (images, suffix) with images a list of (text_before, h, w)."""
        h = ctypes.c_void_p()
        multi = any(len(x) == 2 for x in samples)
        if multi:
            norm = [x if len(x) == 2 else (([(x[0], x[1], x[2])], x[3]) if x[1] * x[2] > 0 else ([], x[0] + x[3]))
                    for x in samples]
            imgs = [im for (ims, _) in norm for im in ims]
            iarr = (_Image * max(1, len(imgs)))(*[_Image(*map(int, im)) for im in imgs])
            import numpy as np
            n_img = np.asarray([len(ims) for (ims, _) in norm] or [0], dtype=np.int32)
            suf = np.asarray([sf for (_, sf) in norm] or [0], dtype=np.int32)
            _check(lib().hia_segments_build_multi(iarr, n_img.ctypes.data_as(ctypes.c_void_p),
                                                  suf.ctypes.data_as(ctypes.c_void_p), len(samples), int(S),
                                                  int(bool(packed)), ctypes.byref(h)), "hia_segments_build_multi")
            self.samples = [([tuple(map(int, im)) for im in ims], int(sf)) for (ims, sf) in norm]
            self.lengths = [sum(t + hh * ww for (t, hh, ww) in ims) + sf for (ims, sf) in self.samples]
        else:
            arr = (_Sample * max(1, len(samples)))(*[_Sample(*map(int, x)) for x in samples])
            if packed:
                _check(lib().hia_segments_build_packed(arr, len(samples), ctypes.byref(h)),
                       "hia_segments_build_packed")
            else:
                _check(lib().hia_segments_build(arr, len(samples), int(S), ctypes.byref(h)), "hia_segments_build")
            self.samples = [tuple(map(int, x)) for x in samples]
            self.lengths = [p + hh * ww + sf for (p, hh, ww, sf) in self.samples]
        self.handle = h
        inf = self.info()
        self.B, self.S = len(samples), int(inf.S)
        self.packed = bool(inf.packed)
        self.total_rows = int(inf.total_rows)
        self.rows, self.offsets = self.layout()
        self.on_device = False

    def upload(self):
        _check(lib().hia_segments_upload(self.handle, _stream()), "hia_segments_upload")
        self.on_device = True
        return self

    def info(self) -> SegmentsInfo:
        out = SegmentsInfo()
        _check(lib().hia_segments_info(self.handle, ctypes.byref(out)), "hia_segments_info")
        return out

    def layout(self):
        """(rows, offsets) per sample, from the library: a sample's rows in a
        tensor of this layout and its first row."""
        import numpy as np
        r = np.zeros(max(self.B, 1), dtype=np.int32)
        o = np.zeros(max(self.B, 1), dtype=np.int32)
        _check(lib().hia_segments_layout(self.handle, r.ctypes.data_as(ctypes.c_void_p),
                                         o.ctypes.data_as(ctypes.c_void_p)), "hia_segments_layout")
        return [int(x) for x in r[:self.B]], [int(x) for x in o[:self.B]]

    def row_bound(self):
        import numpy as np
        e = np.zeros((self.B, self.S), dtype=np.int32)
        _check(lib().hia_segments_row_bound(self.handle, e.ctypes.data_as(ctypes.c_void_p)), "row_bound")
        return e

    def set_bwd_split(self, mode):
        """Backward schedule (hia_segments_set_bwd_split): 0 auto (default),
        1 never split, 2 the best split schedule, 3 / 4 / 5 the best one
        cutting the longest kv tiles into exactly 2 / 3 / 4 parts."""
        _check(lib().hia_segments_set_bwd_split(self.handle, int(mode)), "hia_segments_set_bwd_split")
        return self

    def bwd_schedules(self):
        """Every backward schedule of the descriptor as (parts, entries):
        entries int32 [n, 8] = (b, kv tile, first query tile, end query tile,
        slot, part, parts, 0) in launch order (hia_segments_bwd_schedule)."""
        import numpy as np
        out = []
        while True:
            parts, n = ctypes.c_int32(0), ctypes.c_int64(0)
            rc = lib().hia_segments_bwd_schedule(self.handle, len(out), ctypes.byref(parts), ctypes.byref(n), None)
            if rc != 0:
                return out
            e = np.zeros((max(n.value, 1), 8), dtype=np.int32)
            _check(lib().hia_segments_bwd_schedule(self.handle, len(out), ctypes.byref(parts), ctypes.byref(n),
                                                   e.ctypes.data_as(ctypes.c_void_p)), "hia_segments_bwd_schedule")
            out.append((parts.value, e[:n.value]))

    def bwd_choice(self, Hkv, g, n_sm):
        """Index into bwd_schedules() of the schedule a backward launch takes
        (hia_segments_bwd_choice)."""
        i = ctypes.c_int(0)
        _check(lib().hia_segments_bwd_choice(self.handle, int(Hkv), int(g), int(n_sm), ctypes.byref(i)),
               "hia_segments_bwd_choice")
        return i.value

    def mask(self):
        import numpy as np
        m = np.zeros((self.B, self.S, self.S), dtype=np.uint8)
        _check(lib().hia_segments_mask(self.handle, m.ctypes.data_as(ctypes.c_void_p)), "mask")
        return m

    def tile_classes(self):
        import numpy as np
        inf = self.info()
        c = np.zeros((self.B, inf.fwd_q_tiles, inf.fwd_kv_tiles), dtype=np.uint8)
        _check(lib().hia_segments_tile_classes(self.handle, c.ctypes.data_as(ctypes.c_void_p)), "tile_classes")
        return c

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value and _lib is not None:
            _lib.hia_segments_destroy(h)
            self.handle = None


def hia_segments_build(samples, S, upload=True) -> Segments:
    """Segment descriptor for samples [(prefix, img_h, img_w, suffix)] padded to S."""
    seg = Segments(samples, S)
    return seg.upload() if upload else seg


def hia_segments_build_packed(samples, upload=True) -> Segments:
    """Segment descriptor for the packed (varlen) layout: samples back to back,
    tensors [total_rows, heads, D], lse [Hq, total_rows]."""
    seg = Segments(samples, 0, packed=True)
    return seg.upload() if upload else seg


def hia_segments_build_multi(samples, S=0, packed=False, upload=True) -> Segments:
    """Segment descriptor for samples with any number of images: each sample
    (images, suffix), images a list of (text_before, img_h, img_w); every
    image but a sample's last is hidden from all tokens after it."""
    seg = Segments([x if len(x) == 2 else x for x in samples], S, packed=packed)
    return seg.upload() if upload else seg


def _view(seg, x):
    """A packed [T,H,D] (or grouped [T,Hkv,g,D]) tensor as one batch row."""
    return x.unsqueeze(0) if (x is not None and seg.packed) else x


def _t(x, q_heads, g):
    """hia_tensor from a [B,S,H,D] torch view (or a [B,S,Hkv,g+2,D] fused slice)."""
    if x is None:
        return _Tensor(None, 0, 0, 0, 0)
    if x.dim() == 4:
        sb, ss, sh, sd = x.stride()
        if sd != 1:
            raise ValueError("last dimension must be contiguous")
        return _Tensor(x.data_ptr(), sb, ss, sh * g if q_heads else sh, sh if q_heads else 0)
    if x.dim() == 5:  # [B, S, Hkv, g, D] grouped view
        sb, ss, shkv, shq, sd = x.stride()
        if sd != 1:
            raise ValueError("last dimension must be contiguous")
        return _Tensor(x.data_ptr(), sb, ss, shkv, shq)
    raise ValueError("expected a 4-D [B,S,H,D] or 5-D [B,S,Hkv,g,D] tensor")


def _heads(x):
    return x.shape[2] * (x.shape[3] if x.dim() == 5 else 1)


def hia_rope2d_tables(seg: Segments, D: int, base: float = 10000.0, out=None):
    """fp32 cos, sin [B, S, D] on the current CUDA device."""
    import torch
    if out is None:
        out = (torch.empty(seg.B, seg.S, D, device="cuda", dtype=torch.float32),
               torch.empty(seg.B, seg.S, D, device="cuda", dtype=torch.float32))
    c, s = out
    _check(lib().hia_rope2d_tables(seg.handle, int(D), float(base), c.data_ptr(), s.data_ptr(), _stream()),
           "hia_rope2d_tables")
    return c, s


def hia_attn_fwd_workspace_bytes(seg: Segments, Hq, Hkv, D):
    return int(lib().hia_attn_fwd_workspace_bytes(seg.handle, Hq, Hkv, D))


def hia_attn_bwd_workspace_bytes(seg: Segments, Hq, Hkv, D):
    return int(lib().hia_attn_bwd_workspace_bytes(seg.handle, Hq, Hkv, D))


def _ws(nbytes, workspace):
    import torch
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError("workspace too small")
        return workspace
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")


def _norm(qk_norm, D):
    """qk_norm = (wq, wk, eps) with fp32 [D] CUDA weights -> pointer to a
    hia_qk_norm (or None); the tensors are kept alive by the caller."""
    if qk_norm is None:
        return None
    wq, wk, eps = qk_norm
    for w in (wq, wk):
        if not w.is_cuda or w.dtype.itemsize != 4 or not w.dtype.is_floating_point or w.numel() != D \
                or not w.is_contiguous():
            raise ValueError("QK-norm weights must be contiguous fp32 CUDA tensors of D elements")
    return ctypes.pointer(_QkNorm(wq.data_ptr(), wk.data_ptr(), float(eps)))


def hia_attn_fwd(seg: Segments, q, k, v, cos, sin, scale=None, o=None, lse=None, workspace=None,
                 qk_norm=None):
    """Forward.  q [B,S,Hq,D], k, v [B,S,Hkv,D] bf16 CUDA tensors (or grouped
    5-D views).  Returns (o [B,S,Hq,D] bf16, lse [B,Hq,S] fp32).  qk_norm:
    optional (wq, wk, eps), fp32 [D] CUDA weights of the per-head RMSNorm
    applied after RoPE (hia_attn_fwd_ex)."""
    import torch
    Hq, Hkv, D = _heads(_view(seg, q)), _heads(_view(seg, k)), q.shape[-1]
    g = Hq // Hkv
    if scale is None:
        scale = D ** -0.5
    if o is None:
        shape = (seg.total_rows, Hq, D) if seg.packed else (seg.B, seg.S, Hq, D)
        o = torch.empty(shape, device=q.device, dtype=torch.bfloat16)
    if lse is None:
        shape = (Hq, seg.total_rows) if seg.packed else (seg.B, Hq, seg.S)
        lse = torch.empty(shape, device=q.device, dtype=torch.float32)
    o_ret = o
    q, k, v, o = (_view(seg, x) for x in (q, k, v, o))
    nb = hia_attn_fwd_workspace_bytes(seg, Hq, Hkv, D)
    ws = _ws(nb, workspace)
    if qk_norm is None:
        _check(lib().hia_attn_fwd(seg.handle, Hq, Hkv, D, _t(q, True, g), _t(k, False, 1), _t(v, False, 1),
                                  cos.data_ptr(), sin.data_ptr(), float(scale), _t(o, True, g), lse.data_ptr(),
                                  ws.data_ptr(), nb, _stream()), "hia_attn_fwd")
    else:
        _check(lib().hia_attn_fwd_ex(seg.handle, Hq, Hkv, D, _t(q, True, g), _t(k, False, 1), _t(v, False, 1),
                                     cos.data_ptr(), sin.data_ptr(), float(scale), _norm(qk_norm, D),
                                     _t(o, True, g), lse.data_ptr(), ws.data_ptr(), nb, _stream()),
               "hia_attn_fwd_ex")
    return o_ret, lse


def hia_attn_bwd(seg: Segments, q, k, v, cos, sin, o, lse, dout, scale=None, dq=None, dk=None, dv=None,
                 workspace=None, qk_norm=None, fwd_workspace=None):
    """Recompute backward.  Returns (dq, dk, dv) bf16; with qk_norm (the
    forward's (wq, wk, eps)) returns (dq, dk, dv, dwq, dwk), dwq/dwk fp32 [D]
    (hia_attn_bwd_ex).  fwd_workspace: the workspace tensor of the forward
    that produced o and lse, untouched since; its rotated q and k are reused
    (hia_attn_bwd_reuse_fwd)."""
    import torch
    Hq, Hkv, D = _heads(_view(seg, q)), _heads(_view(seg, k)), q.shape[-1]
    g = Hq // Hkv
    if scale is None:
        scale = D ** -0.5
    lead = (seg.total_rows,) if seg.packed else (seg.B, seg.S)
    if dq is None:
        dq = torch.empty(*lead, Hq, D, device=q.device, dtype=torch.bfloat16)
    if dk is None:
        dk = torch.empty(*lead, Hkv, D, device=q.device, dtype=torch.bfloat16)
    if dv is None:
        dv = torch.empty(*lead, Hkv, D, device=q.device, dtype=torch.bfloat16)
    ret = (dq, dk, dv)
    q, k, v, o, dout, dq, dk, dv = (_view(seg, x) for x in (q, k, v, o, dout, dq, dk, dv))
    nb = hia_attn_bwd_workspace_bytes(seg, Hq, Hkv, D)
    ws = _ws(nb, workspace)
    if fwd_workspace is not None:
        nf = hia_attn_fwd_workspace_bytes(seg, Hq, Hkv, D)
        if fwd_workspace.numel() * fwd_workspace.element_size() < nf:
            raise ValueError("forward workspace too small")
        dwq = dwk = None
        if qk_norm is not None:
            dwq = torch.empty(D, device=q.device, dtype=torch.float32)
            dwk = torch.empty(D, device=q.device, dtype=torch.float32)
        _check(lib().hia_attn_bwd_reuse_fwd(
            seg.handle, Hq, Hkv, D, _t(q, True, g), _t(k, False, 1), _t(v, False, 1), cos.data_ptr(),
            sin.data_ptr(), float(scale), _norm(qk_norm, D), _t(o, True, g), lse.data_ptr(), _t(dout, True, g),
            _t(dq, True, g), _t(dk, False, 1), _t(dv, False, 1), dwq.data_ptr() if dwq is not None else None,
            dwk.data_ptr() if dwk is not None else None, fwd_workspace.data_ptr(), nf, ws.data_ptr(), nb,
            _stream()), "hia_attn_bwd_reuse_fwd")
        return ret if qk_norm is None else (*ret, dwq, dwk)
    if qk_norm is None:
        _check(lib().hia_attn_bwd(seg.handle, Hq, Hkv, D, _t(q, True, g), _t(k, False, 1), _t(v, False, 1),
                                  cos.data_ptr(), sin.data_ptr(), float(scale), _t(o, True, g), lse.data_ptr(),
                                  _t(dout, True, g), _t(dq, True, g), _t(dk, False, 1), _t(dv, False, 1),
                                  ws.data_ptr(), nb, _stream()), "hia_attn_bwd")
        return ret
    dwq = torch.empty(D, device=q.device, dtype=torch.float32)
    dwk = torch.empty(D, device=q.device, dtype=torch.float32)
    _check(lib().hia_attn_bwd_ex(seg.handle, Hq, Hkv, D, _t(q, True, g), _t(k, False, 1), _t(v, False, 1),
                                 cos.data_ptr(), sin.data_ptr(), float(scale), _norm(qk_norm, D), _t(o, True, g),
                                 lse.data_ptr(), _t(dout, True, g), _t(dq, True, g), _t(dk, False, 1),
                                 _t(dv, False, 1), dwq.data_ptr(), dwk.data_ptr(), ws.data_ptr(), nb, _stream()),
           "hia_attn_bwd_ex")
    return (*ret, dwq, dwk)


class Step:
    """Owner of a library hia_step: device buffers, RoPE tables and workspaces
    for training steps fed from host memory (hia_attn_step_host)."""

    def __init__(self, seg: "Segments", Hq, Hkv, D, base=10000.0):
        self.seg, self.Hq, self.Hkv, self.D = seg, Hq, Hkv, D
        h = ctypes.c_void_p()
        _check(lib().hia_step_create(seg.handle, int(Hq), int(Hkv), int(D), float(base), ctypes.byref(h)),
               "hia_step_create")
        self.handle = h

    def __del__(self):
        if getattr(self, "handle", None) and _lib is not None:
            _lib.hia_step_destroy(self.handle)
            self.handle = None


def hia_step_create(seg: "Segments", Hq, Hkv, D, base=10000.0) -> Step:
    return Step(seg, Hq, Hkv, D, base)


def hia_attn_step_host(step: Step, q, k, v, dout, o, lse, dq, dk, dv, scale=None, stream=None):
    """One forward + backward from host tensors (contiguous CPU tensors; pin
    them for asynchronous copies): q, dout [B,S,Hq,D], k, v [B,S,Hkv,D] bf16
    in; o, dq [B,S,Hq,D], dk, dv [B,S,Hkv,D] bf16 and lse [B,Hq,S] fp32 out.
    Enqueued on `stream` (default: the current CUDA stream)."""
    import torch
    B, S, Hq, Hkv, D = step.seg.B, step.seg.S, step.Hq, step.Hkv, step.D
    want = ((q, (B, S, Hq, D), torch.bfloat16), (k, (B, S, Hkv, D), torch.bfloat16),
            (v, (B, S, Hkv, D), torch.bfloat16), (dout, (B, S, Hq, D), torch.bfloat16),
            (o, (B, S, Hq, D), torch.bfloat16), (lse, (B, Hq, S), torch.float32),
            (dq, (B, S, Hq, D), torch.bfloat16), (dk, (B, S, Hkv, D), torch.bfloat16),
            (dv, (B, S, Hkv, D), torch.bfloat16))
    for t, shape, dt in want:
        if t.is_cuda or not t.is_contiguous() or tuple(t.shape) != shape or t.dtype != dt:
            raise ValueError(f"hia_attn_step_host takes contiguous host tensors {shape} {dt}")
    if scale is None:
        scale = step.D ** -0.5
    st = _stream() if stream is None else ctypes.c_void_p(stream.cuda_stream)
    _check(lib().hia_attn_step_host(step.handle, q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(),
                                    float(scale), o.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                    dv.data_ptr(), st), "hia_attn_step_host")


def hia_get_device_status():
    return int(lib().hia_get_device_status(_stream()))


def hia_debug_wait_timeout(timeout_ns: int):
    _check(lib().hia_debug_wait_timeout(int(timeout_ns), _stream()), "hia_debug_wait_timeout")


def hia_profile_begin():
    """Start per-kernel CUDA-event timing of every library launch."""
    _check(lib().hia_profile_begin(), "hia_profile_begin")


def hia_profile_end():
    """Stop timing; returns {kernel name: (launches, total_ms)}."""
    arr = (_KernelTime * 16)()
    n = ctypes.c_int(0)
    _check(lib().hia_profile_end(arr, 16, ctypes.byref(n)), "hia_profile_end")
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms)) for i in range(min(n.value, 16))}


def hia_moe_workspace_bytes(T, H, I, E, topk):
    return int(lib().hia_moe_workspace_bytes(ctypes.byref(_MoeDims(T, H, I, E, topk))))


def hia_moe_fwd(x, wg, w13, w2, topk, out=None, workspace=None):
    """MoE feed-forward of one block (jointmoe.h): x bf16 [T, H], wg fp32
    [E, H], w13 bf16 [E + 1, 2I, H] ([up; gate], index E the shared expert),
    w2 bf16 [E + 1, H, I], all contiguous CUDA tensors.  Returns (out bf16
    [T, H], topk_ids int32 [T, topk], topk_weights fp32 [T, topk])."""
    import torch
    T, H = x.shape
    E = wg.shape[0]
    I = w13.shape[1] // 2
    for t, dt in ((x, torch.bfloat16), (wg, torch.float32), (w13, torch.bfloat16), (w2, torch.bfloat16)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != dt:
            raise ValueError("hia_moe_fwd takes contiguous CUDA tensors (x, w13, w2 bf16; wg fp32)")
    if tuple(w13.shape) != (E + 1, 2 * I, H) or tuple(w2.shape) != (E + 1, H, I) or wg.shape[1] != H:
        raise ValueError("inconsistent MoE weight shapes")
    dims = _MoeDims(T, H, I, E, int(topk))
    nb = int(lib().hia_moe_workspace_bytes(ctypes.byref(dims)))
    if nb == 0:
        raise HiaError(1, "hia_moe_workspace_bytes")
    ws = _ws(nb, workspace)
    if out is None:
        out = torch.empty(T, H, device=x.device, dtype=torch.bfloat16)
    ids = torch.empty(T, topk, device=x.device, dtype=torch.int32)
    w = torch.empty(T, topk, device=x.device, dtype=torch.float32)
    _check(lib().hia_moe_fwd(ctypes.byref(dims), x.data_ptr(), wg.data_ptr(), w13.data_ptr(), w2.data_ptr(),
                             out.data_ptr(), ids.data_ptr(), w.data_ptr(), ws.data_ptr(), nb, _stream()),
           "hia_moe_fwd")
    return out, ids, w
