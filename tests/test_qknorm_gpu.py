"""GPU parity of the per-head QK RMSNorm after RoPE (hia_attn_fwd_ex /
hia_attn_bwd_ex) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import joint_text_image_b200 as jt
from joint_text_image_b200 import synth
from helpers import check_bwd, check_fwd, gpu_tables, sample_rows

pytestmark = pytest.mark.gpu

EPS = 1e-5


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "needs a GPU"
    jt.lib()


def weights(D, seed=0):
    g = torch.Generator().manual_seed(1000 + seed)
    wq = (torch.rand(D, generator=g, dtype=torch.float64) + 0.5).float().double()
    wk = (torch.rand(D, generator=g, dtype=torch.float64) + 0.5).float().double()
    return wq, wk  # fp32-representable, so the oracle sees the kernels' exact weights


def run(wl, wq, wk, bwd=True, split=0):
    q, k, v, do = synth.tensors(wl, 0, grad=True)
    seg = jt.hia_segments_build(wl.samples, wl.S).set_bwd_split(split)
    c, s = gpu_tables(seg, wl.D, wl.base)
    norm = (wq.float().cuda(), wk.float().cuda(), EPS)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = jt.hia_attn_fwd(seg, qd, kd, vd, c, s, wl.scale, qk_norm=norm)
    out = None
    if bwd:
        out = jt.hia_attn_bwd(seg, qd, kd, vd, c, s, o, lse, dod, wl.scale, qk_norm=norm)
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 0
    return (q, k, v, do), o.float().cpu().numpy(), lse.cpu().numpy(), out


@pytest.mark.parametrize("name,split", [("tiny", 0), ("256px", 0), ("256px", 2)])
def test_qknorm_fwd_bwd_parity(oracle_mod, name, split):
    """split 2: the split backward schedule forced on, whose combine feeds the
    norm's fp32 dk accumulator."""
    wl = synth.workload(name)
    wq, wk = weights(wl.D)
    ref_norm = (wq.numpy(), wk.numpy(), EPS)
    (q, k, v, do), o, lse, (dq, dk, dv, dwq, dwk) = run(wl, wq, wk, split=split)
    check_fwd(oracle_mod, wl, q, k, v, o, lse, qk_norm=ref_norm)
    f = lambda t: t.float().cpu().numpy()
    check_bwd(oracle_mod, wl, (q, k, v, do), (f(dq), f(dk), f(dv)), qk_norm=ref_norm,
              dw=(dwq.cpu().numpy(), dwk.cpu().numpy()))


def test_qknorm_full_size_sampled(oracle_mod):
    """1024px backward workload: forward on sampled rows of every segment,
    backward on two (b, kv head) groups in full."""
    wl = synth.workload("1024px_bwd")
    wq, wk = weights(wl.D, 1)
    ref_norm = (wq.numpy(), wk.numpy(), EPS)
    (q, k, v, do), o, lse, (dq, dk, dv, dwq, dwk) = run(wl, wq, wk)
    check_fwd(oracle_mod, wl, q, k, v, o, lse, rows=sample_rows(wl, 4), qk_norm=ref_norm)
    groups = np.zeros((wl.B, wl.Hkv), dtype=bool)
    groups[0, 2] = groups[0, 7] = True
    f = lambda t: t.float().cpu().numpy()
    check_bwd(oracle_mod, wl, (q, k, v, do), (f(dq), f(dk), f(dv)), groups=groups, qk_norm=ref_norm)
    assert torch.isfinite(dwq).all() and torch.isfinite(dwk).all()


def test_qknorm_weight_gradients_deterministic():
    wl = synth.workload("256px")
    wq, wk = weights(wl.D, 2)
    a = run(wl, wq, wk)[3]
    b = run(wl, wq, wk)[3]
    # dk, dv, dwk never pass through the dq accumulator's unordered fp32 reductions
    for i in (1, 2, 4):
        assert torch.equal(a[i], b[i])


def test_qknorm_unit_weights_eps0_on_unit_rms_rows_matches_plain():
    """With w = 1, eps = 0 and rows of RMS 1 the norm is the identity (R keeps
    the RMS): the forward equals the plain one to bf16 rounding."""
    wl = synth.workload("tiny")
    q, k, v = synth.tensors(wl, 3)
    q = (q.float() / q.float().pow(2).mean(-1, keepdim=True).sqrt()).bfloat16()
    k = (k.float() / k.float().pow(2).mean(-1, keepdim=True).sqrt()).bfloat16()
    seg = jt.hia_segments_build(wl.samples, wl.S)
    c, s = gpu_tables(seg, wl.D, wl.base)
    one = torch.ones(wl.D, device="cuda", dtype=torch.float32)
    o1, l1 = jt.hia_attn_fwd(seg, q.cuda(), k.cuda(), v.cuda(), c, s, wl.scale, qk_norm=(one, one, 0.0))
    o0, l0 = jt.hia_attn_fwd(seg, q.cuda(), k.cuda(), v.cuda(), c, s, wl.scale)
    torch.cuda.synchronize()
    assert (o1.float() - o0.float()).abs().max() <= 2e-2
    assert (l1 - l0).abs().max() <= 1e-2


def test_qknorm_rejects_bad_arguments():
    wl = synth.workload("tiny")
    q, k, v = (t.cuda() for t in synth.tensors(wl, 0))
    seg = jt.hia_segments_build(wl.samples, wl.S)
    c, s = gpu_tables(seg, wl.D, wl.base)
    w = torch.ones(wl.D + 4, device="cuda", dtype=torch.float32)
    with pytest.raises(jt.HiaError) as e:
        jt.hia_attn_fwd(seg, q, k, v, c, s, qk_norm=(w[:wl.D], w[:wl.D], -1.0))
    assert e.value.code == 1  # HIA_ERR_INVALID_ARG
    with pytest.raises(jt.HiaError) as e:
        jt.hia_attn_fwd(seg, q, k, v, c, s, qk_norm=(w[1:wl.D + 1], w[:wl.D], 1e-5))
    assert e.value.code == 2  # HIA_ERR_UNSUPPORTED: misaligned weight
    with pytest.raises(ValueError):
        jt.hia_attn_fwd(seg, q, k, v, c, s, qk_norm=(w, w, 1e-5))
