"""hia_attn_fwd_noalloc: the forward for callers that cannot allocate.

Some callers may not call cudaMalloc: a plug-in inside a host runtime that owns
all device memory and gives it only its inputs and outputs, or a step that must
not allocate midway because cudaMalloc/cudaFree synchronize the device.  This
entry point keeps its scratch (the RoPE-rotated q and k) in a fixed 64 MiB
array compiled into the library instead of a caller workspace.

The test calls it through the C ABI several times in a row on different
problems (so each call finds the previous call's data in the shared array) and
checks every output against the regular hia_attn_fwd, which uses a caller
workspace, within the forward tolerances of the other tests.  It also checks
that a problem larger than the array is refused before anything is launched.
The file name makes pytest collect it last.
"""
import numpy as np
import pytest
import torch

import joint_text_image_b200 as jt
from joint_text_image_b200 import synth
from helpers import LSE_MAX, O_MAX, O_MEAN

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 6  # HIA_ERR_SCRATCH_LIMIT


def _noalloc(seg, q, k, v, c, s, scale):
    Hq, Hkv, D = q.shape[2], k.shape[2], q.shape[3]
    g = Hq // Hkv
    o = torch.empty_like(q)
    lse = torch.empty(seg.B, Hq, seg.S, device=q.device, dtype=torch.float32)
    rc = jt.lib().hia_attn_fwd_noalloc(seg.handle, Hq, Hkv, D, jt._t(q, True, g), jt._t(k, False, 1),
                                       jt._t(v, False, 1), c.data_ptr(), s.data_ptr(), float(scale),
                                       jt._t(o, True, g), lse.data_ptr(), jt._stream())
    return rc, o, lse


def _problem(name, seed):
    wl = synth.workload(name)
    q, k, v = (t.cuda() for t in synth.tensors(wl, seed))
    seg = jt.hia_segments_build(wl.samples, wl.S)
    c, s = jt.hia_rope2d_tables(seg, wl.D, wl.base)
    o_ref, lse_ref = jt.hia_attn_fwd(seg, q, k, v, c, s, wl.scale)
    return wl, seg, (q, k, v, c, s), o_ref, lse_ref


def _close(o, lse, o_ref, lse_ref):
    d = (o.float() - o_ref.float()).abs()
    assert float(d.max()) <= O_MAX and float(d.mean()) <= O_MEAN
    fin = torch.isfinite(lse_ref)
    assert torch.equal(torch.isfinite(lse), fin)
    assert float((lse[fin] - lse_ref[fin]).abs().max()) <= LSE_MAX


def test_noalloc_matches_workspace_forward_on_consecutive_calls():
    assert torch.cuda.is_available()
    probs = [_problem("256px", 0), _problem("tiny", 1)]
    outs = []
    for wl, seg, (q, k, v, c, s), _, _ in probs + probs[:1]:
        rc, o, lse = _noalloc(seg, q, k, v, c, s, wl.scale)
        assert rc == 0, jt.lib().hia_status_string(rc)
        outs.append((o, lse))
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 0
    for (o, lse), (_, _, _, o_ref, lse_ref) in zip(outs, probs + probs[:1]):
        _close(o, lse, o_ref, lse_ref)


def test_noalloc_refuses_problems_beyond_the_scratch():
    # one text-only sample of 20000 tokens, 32 + 8 heads, D = 128: 205 MB of rotated q/k
    seg = jt.hia_segments_build([(20000, 0, 0, 0)], 20000)
    z = jt._Tensor(None, 0, 0, 0, 0)
    rc = jt.lib().hia_attn_fwd_noalloc(seg.handle, 32, 8, 128, z, z, z, None, None, 0.088, z, None, None)
    assert rc == SCRATCH_LIMIT
    assert b"64 MiB" in jt.lib().hia_status_string(rc)


def test_noalloc_packed_layout_matches_workspace_forward():
    """The fixed-scratch forward on a packed descriptor (samples back to back)."""
    import joint_text_image_b200 as jt
    from joint_text_image_b200 import synth
    wl = synth.workload("256px")
    q, k, v = synth.tensors(wl, 4)
    seg = jt.hia_segments_build_packed(wl.samples)
    pack = lambda x: torch.cat([x[b, :L] for b, L in enumerate(seg.lengths)], 0).contiguous().cuda()
    qp, kp, vp = pack(q), pack(k), pack(v)
    c, s = jt.hia_rope2d_tables(seg, wl.D)
    o_ref, lse_ref = jt.hia_attn_fwd(seg, qp, kp, vp, c, s)
    o = torch.empty_like(o_ref)
    lse = torch.empty_like(lse_ref)
    g = wl.Hq // wl.Hkv
    rc = jt.lib().hia_attn_fwd_noalloc(seg.handle, wl.Hq, wl.Hkv, wl.D, jt._t(qp.unsqueeze(0), True, g),
                                       jt._t(kp.unsqueeze(0), False, 1), jt._t(vp.unsqueeze(0), False, 1),
                                       c.data_ptr(), s.data_ptr(), wl.scale, jt._t(o.unsqueeze(0), True, g),
                                       lse.data_ptr(), jt._stream())
    torch.cuda.synchronize()
    assert rc == 0
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
