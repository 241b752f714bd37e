"""hia_attn_fwd_noalloc: the forward for callers that cannot allocate.

Some callers may not call cudaMalloc: a plug-in inside a host runtime that owns
all device memory and gives it only its inputs and outputs, or a step that must
not allocate midway because cudaMalloc/cudaFree synchronize the device.  This
entry point keeps its scratch (the RoPE-rotated q and k) in a fixed 64 MiB
array compiled into the library instead of a caller workspace.

The test calls it through the C ABI several times in a row on different
problems (so each call finds the previous call's data in the shared array) and
checks every output bit for bit against the regular hia_attn_fwd, which runs
the same kernels on the same inputs with a caller workspace.  After a first
call has loaded the library's module, later calls must leave the device's
free memory unchanged.  A problem larger than the array is refused before
anything is launched, and a bad argument reports its own error first.
The file name makes pytest collect it last.
"""
import pytest
import torch

import joint_text_image_b200 as jt
from joint_text_image_b200 import synth

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 6  # HIA_ERR_SCRATCH_LIMIT


def _problem(name, seed):
    wl = synth.workload(name)
    q, k, v = (t.cuda() for t in synth.tensors(wl, seed))
    seg = jt.hia_segments_build(wl.samples, wl.S)
    c, s = jt.hia_rope2d_tables(seg, wl.D, wl.base)
    o_ref, lse_ref = jt.hia_attn_fwd(seg, q, k, v, c, s, wl.scale)
    return wl, seg, (q, k, v, c, s), o_ref, lse_ref


def _same(o, lse, o_ref, lse_ref):
    # same kernels, same inputs, same launch shapes: identical bits
    assert torch.equal(o, o_ref)
    assert torch.equal(lse, lse_ref)


def test_noalloc_matches_workspace_forward_on_consecutive_calls():
    assert torch.cuda.is_available()
    probs = [_problem("256px", 0), _problem("tiny", 1)]
    order = probs + probs[:1] + probs[1:]
    # outputs allocated up front, so that only the library could change the free memory below
    outs = [(torch.empty_like(p[3]), torch.empty_like(p[4])) for p in order]
    torch.cuda.synchronize()

    def call(i):
        wl, seg, (q, k, v, c, s), _, _ = order[i]
        o, lse = outs[i]
        g = wl.Hq // wl.Hkv
        rc = jt.lib().hia_attn_fwd_noalloc(seg.handle, wl.Hq, wl.Hkv, wl.D, jt._t(q, True, g), jt._t(k, False, 1),
                                           jt._t(v, False, 1), c.data_ptr(), s.data_ptr(), float(wl.scale),
                                           jt._t(o, True, g), lse.data_ptr(), jt._stream())
        assert rc == 0, jt.lib().hia_status_string(rc)

    call(0)  # the first call may load the module that holds the fixed array
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for i in range(1, len(order)):
        call(i)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0, "a call changed the device's free memory"
    assert jt.hia_get_device_status() == 0
    for (o, lse), (_, _, _, o_ref, lse_ref) in zip(outs, order):
        _same(o, lse, o_ref, lse_ref)


def _big_problem():
    # one text-only sample of 20000 tokens, 32 + 8 heads, D = 128: 205 MB of rotated q/k
    S = 20000
    seg = jt.hia_segments_build([(S, 0, 0, 0)], S)
    q = torch.zeros(1, S, 32, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(1, S, 8, 128, dtype=torch.bfloat16, device="cuda")
    c, s = jt.hia_rope2d_tables(seg, 128)
    lse = torch.empty(1, 32, S, device="cuda")
    return seg, q, kv, c, s, lse


def test_noalloc_refuses_problems_beyond_the_scratch():
    seg, q, kv, c, s, lse = _big_problem()
    o = torch.empty_like(q)
    assert jt.hia_attn_fwd_workspace_bytes(seg, 32, 8, 128) > 64 << 20
    rc = jt.lib().hia_attn_fwd_noalloc(seg.handle, 32, 8, 128, jt._t(q, True, 4), jt._t(kv, False, 1),
                                       jt._t(kv, False, 1), c.data_ptr(), s.data_ptr(), 0.088,
                                       jt._t(o, True, 4), lse.data_ptr(), jt._stream())
    assert rc == SCRATCH_LIMIT
    assert b"64 MiB" in jt.lib().hia_status_string(rc)


def test_noalloc_argument_errors_come_before_the_size_limit():
    """Same errors as hia_attn_fwd for bad arguments, even on a problem that
    is also too large for the fixed array."""
    seg, q, kv, c, s, lse = _big_problem()
    o = torch.empty_like(q)
    L = jt.lib()
    args = lambda Hq, Hkv, D, cc: (seg.handle, Hq, Hkv, D, jt._t(q, True, 4), jt._t(kv, False, 1),
                                   jt._t(kv, False, 1), cc, s.data_ptr(), 0.088, jt._t(o, True, 4),
                                   lse.data_ptr(), jt._stream())
    assert L.hia_attn_fwd_noalloc(*args(32, 7, 128, c.data_ptr())) == 2   # Hq % Hkv != 0: UNSUPPORTED
    assert L.hia_attn_fwd_noalloc(*args(32, 8, 96, c.data_ptr())) == 2    # D = 96: UNSUPPORTED
    assert L.hia_attn_fwd_noalloc(*args(32, 8, 128, None)) == 1           # null cos: INVALID_ARG
    assert L.hia_attn_fwd_noalloc(None, 32, 8, 128, *args(32, 8, 128, 0)[4:]) == 1


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
