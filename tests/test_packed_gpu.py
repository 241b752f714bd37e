"""GPU: the packed (varlen) layout against the padded one and the fp64
oracle.  Same kernels: a sample's rows see the same keys in both layouts and
masked keys contribute exact zeros, so o, lse, dk, dv of the real rows are
bitwise equal to the padded run with zero dout on the padded rows."""
import numpy as np
import pytest
import torch

import joint_text_image_b200 as jt
from joint_text_image_b200 import synth
from helpers import check_bwd, check_fwd, gpu_tables

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "needs a GPU"
    jt.lib()


def pack(x, lens):
    return torch.cat([x[b, :L] for b, L in enumerate(lens)], dim=0).contiguous()


def unpack(x, lens, S):
    out = torch.zeros((len(lens), S) + tuple(x.shape[1:]), dtype=x.dtype)
    off = 0
    for b, L in enumerate(lens):
        out[b, :L] = x[off:off + L]
        off += L
    return out


def padded_inputs(wl, seed=0):
    """The workload's tensors with dout zeroed on padded rows (a padded row
    then adds nothing to dk, dv)."""
    q, k, v, do = synth.tensors(wl, seed, grad=True)
    lens = [p + h * w + s for p, h, w, s in wl.samples]
    for b, L in enumerate(lens):
        do[b, L:] = 0
    return q, k, v, do, lens


# The bitwise comparisons below hold for one backward schedule: under the
# automatic choice the two layouts (different query ranges per kv tile) may
# pick different ones, and a split kv tile sums its parts' fp32 partials in a
# different order than one accumulation.  Both run the unsplit schedule.
NEVER_SPLIT = 1


def run_padded(wl, q, k, v, do):
    seg = jt.hia_segments_build(wl.samples, wl.S).set_bwd_split(NEVER_SPLIT)
    c, s = gpu_tables(seg, wl.D, wl.base)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = jt.hia_attn_fwd(seg, qd, kd, vd, c, s, wl.scale)
    dq, dk, dv = jt.hia_attn_bwd(seg, qd, kd, vd, c, s, o, lse, dod, wl.scale)
    torch.cuda.synchronize()
    return [t.cpu() for t in (o, lse, dq, dk, dv)]


def run_packed(wl, q, k, v, do, lens, split=NEVER_SPLIT):
    seg = jt.hia_segments_build_packed(wl.samples).set_bwd_split(split)
    assert seg.S <= wl.S
    c, s = gpu_tables(seg, wl.D, wl.base)
    qp, kp, vp, dop = (pack(t, lens).cuda() for t in (q, k, v, do))
    o, lse = jt.hia_attn_fwd(seg, qp, kp, vp, c, s, wl.scale)
    dq, dk, dv = jt.hia_attn_bwd(seg, qp, kp, vp, c, s, o, lse, dop, wl.scale)
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 0
    assert o.shape == (sum(lens), wl.Hq, wl.D) and lse.shape == (wl.Hq, sum(lens))
    return seg, [t.cpu() for t in (o, lse, dq, dk, dv)]


@pytest.mark.parametrize("name", ["tiny", "256px", "mixed"])
def test_packed_equals_padded_on_real_rows(name):
    wl = synth.workload(name)
    q, k, v, do, lens = padded_inputs(wl)
    po, plse, pdq, pdk, pdv = run_padded(wl, q, k, v, do)
    _, (o, lse, dq, dk, dv) = run_packed(wl, q, k, v, do, lens)
    off = 0
    for b, L in enumerate(lens):
        assert torch.equal(o[off:off + L], po[b, :L])
        assert torch.equal(lse[:, off:off + L], plse[b, :, :L])
        assert torch.equal(dk[off:off + L], pdk[b, :L]) and torch.equal(dv[off:off + L], pdv[b, :L])
        a, r = dq[off:off + L].float(), pdq[b, :L].float()
        assert (a - r).norm() <= 1e-3 * max(r.norm(), 1e-30)  # dq: order of its fp32 reductions
        off += L


@pytest.mark.parametrize("name,split", [("tiny", 0), ("256px", 0), ("256px", 2)])
def test_packed_parity_with_oracle(oracle_mod, name, split):
    """split 2: the split backward schedule forced on, in the packed layout."""
    wl = synth.workload(name)
    q, k, v, do, lens = padded_inputs(wl, 1)
    seg, (o, lse, dq, dk, dv) = run_packed(wl, q, k, v, do, lens, split=split)
    S = wl.S
    # the oracle on the padded equivalent, compared on real rows only
    rows_ok = np.zeros((wl.B, S), dtype=bool)
    for b, L in enumerate(lens):
        rows_ok[b, :L] = True
    o_pad = unpack(o, lens, S).float().numpy()
    lse_pad = np.full((wl.B, wl.Hq, S), -np.inf, dtype=np.float32)
    off = 0
    for b, L in enumerate(lens):
        lse_pad[b, :, :L] = lse[:, off:off + L].numpy()
        off += L
    o_ref, lse_ref, _ = oracle_mod.attn_fwd(wl.samples, q.double().numpy(), k.double().numpy(),
                                            v.double().numpy(), wl.scale, wl.base)
    err = np.abs(o_pad - o_ref)[rows_ok]
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
    lerr = np.abs(lse_pad - lse_ref).transpose(0, 2, 1)[rows_ok]
    assert lerr.max() <= 1e-2
    grads = tuple(unpack(t, lens, S).float().numpy() for t in (dq, dk, dv))
    check_bwd(oracle_mod, wl, (q, k, v, do), grads)


def test_packed_text_and_empty_samples():
    """A text-only and an empty sample between image samples: the empty one
    owns no rows, nothing past the total is touched (guard rows stay intact)."""
    samples = [(40, 4, 8, 2), (0, 0, 0, 0), (150, 0, 0, 0), (1, 8, 8, 1)]
    lens = [p + h * w + s for p, h, w, s in samples]
    T, Hq, Hkv, D = sum(lens), 4, 2, 128
    g = torch.Generator().manual_seed(5)
    mk = lambda H: torch.randn(T + 8, H, D, generator=g).bfloat16().cuda()
    q, k, v, do = mk(Hq), mk(Hkv), mk(Hkv), mk(Hq)
    seg = jt.hia_segments_build_packed(samples)
    c, s = gpu_tables(seg, D)
    o = torch.full((T + 8, Hq, D), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((Hq, T), 7.0, device="cuda")
    jt.hia_attn_fwd(seg, q[:T], k[:T], v[:T], c, s, o=o[:T], lse=lse)
    dq = torch.full_like(o, 7.0)
    dk = torch.full((T + 8, Hkv, D), 7.0, dtype=torch.bfloat16, device="cuda")
    dv = torch.full_like(dk, 7.0)
    jt.hia_attn_bwd(seg, q[:T], k[:T], v[:T], c, s, o[:T], lse, do[:T], dq=dq[:T], dk=dk[:T], dv=dv[:T])
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 0
    for t in (o, dq, dk, dv):
        assert torch.isfinite(t[:T].float()).all()
        assert (t[T:].float() == 7.0).all()  # rows past the packed total untouched
    assert torch.isfinite(lse).all()
    # the text-only sample is causal attention over its own rows
    b0 = lens[0] + lens[1]
    qq, kk, vv = (x[b0:b0 + lens[2]].float() for x in (q, k, v))
    cs, sn = c[2, :lens[2]], s[2, :lens[2]]
    rot = lambda x: x * cs[:, None] + torch.cat([-x[..., D // 2:], x[..., :D // 2]], -1) * sn[:, None]
    qr, kr = rot(qq).bfloat16().float(), rot(kk).bfloat16().float()
    kr = kr.repeat_interleave(Hq // Hkv, dim=1)
    vv = vv.repeat_interleave(Hq // Hkv, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        qr.transpose(0, 1), kr.transpose(0, 1), vv.transpose(0, 1), is_causal=True).transpose(0, 1)
    assert (o[b0:b0 + lens[2]].float() - ref).abs().max() <= 2e-2
