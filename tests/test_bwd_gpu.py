"""GPU parity of the recompute backward (dQ, dK, dV through the 2D RoPE)
against the fp64 oracle gradients."""
import numpy as np
import pytest
import torch

import joint_text_image_b200 as jt
from joint_text_image_b200 import synth
from helpers import check_bwd, run_fwd_bwd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "needs a GPU"
    jt.lib()


@pytest.mark.parametrize("name", ["tiny", "256px"])
def test_bwd_full_parity(oracle_mod, name):
    wl = synth.workload(name)
    inputs, grads = run_fwd_bwd(wl)
    check_bwd(oracle_mod, wl, inputs, grads)


def test_bwd_1024px_sampled_groups(oracle_mod):
    """Full-size training backward; the oracle computes two (b, kv head) groups
    (8 query heads) in full."""
    wl = synth.workload("1024px_bwd")
    inputs, grads = run_fwd_bwd(wl)
    groups = np.zeros((wl.B, wl.Hkv), dtype=bool)
    groups[0, 0] = groups[0, 5] = True
    check_bwd(oracle_mod, wl, inputs, grads, groups=groups)
    for gr in grads:
        assert np.all(np.isfinite(gr))


def test_bwd_bench_workload_groups_of_each_sample(oracle_mod):
    """The workload the benchmark times (1024px: B=2, S=5554, right-padded;
    sample 1 has 305 padded query rows whose dO is non-zero, and tail kv
    tiles past its L): two complete (b, kv head) groups of each sample
    against the oracle, whole-tensor and block by block."""
    wl = synth.workload("1024px")
    assert wl.B == 2 and wl.S > min(P + h * w + s for (P, h, w, s) in wl.samples)
    inputs, grads = run_fwd_bwd(wl)
    groups = np.zeros((wl.B, wl.Hkv), dtype=bool)
    groups[0, 0] = groups[0, 5] = groups[1, 2] = groups[1, 7] = True
    check_bwd(oracle_mod, wl, inputs, grads, groups=groups)
    for gr in grads:
        assert np.all(np.isfinite(gr))


@pytest.mark.parametrize("samples,S,Hq,Hkv,D", [
    ([(5, 3, 3, 2)], 19, 4, 1, 64),
    ([(100, 10, 13, 7), (0, 0, 0, 0), (250, 0, 0, 0), (0, 16, 16, 2)], 261, 6, 2, 128),
    ([(129, 1, 127, 1), (0, 11, 23, 0)], 300, 2, 2, 128),
    ([(1, 0, 0, 0)], 1, 2, 1, 64),
    ([(64, 8, 16, 0)], 256, 8, 2, 128),
    ([(7, 9, 30, 1)], 290, 4, 4, 64),
])
def test_bwd_edge_cases(oracle_mod, samples, S, Hq, Hkv, D):
    wl = synth.custom(samples, Hq, Hkv, D, S=S)
    inputs, grads = run_fwd_bwd(wl, seed=4)
    check_bwd(oracle_mod, wl, inputs, grads)
    for b, (P, h, w, s) in enumerate(samples):
        if P + h * w + s == 0:
            for gr in grads:
                assert np.all(gr[b] == 0)


def test_bwd_fused_qkv_layout(oracle_mod):
    wl = synth.custom([(40, 6, 6, 3), (10, 4, 9, 0)], 8, 2, 128)
    g = 4
    gen = torch.Generator().manual_seed(6)
    fused = torch.randn(wl.B, wl.S, wl.Hkv, g + 2, wl.D, generator=gen).to(torch.bfloat16)
    do = torch.randn(wl.B, wl.S, wl.Hq, wl.D, generator=gen).to(torch.bfloat16)
    fc, dod = fused.cuda(), do.cuda()
    seg = jt.hia_segments_build(wl.samples, wl.S)
    c, s = jt.hia_rope2d_tables(seg, wl.D)
    qv, kv, vv = fc[:, :, :, :g], fc[:, :, :, g], fc[:, :, :, g + 1]
    o, lse = jt.hia_attn_fwd(seg, qv, kv, vv, c, s)
    dq, dk, dv = jt.hia_attn_bwd(seg, qv, kv, vv, c, s, o, lse, dod)
    torch.cuda.synchronize()
    q = fused[:, :, :, :g].reshape(wl.B, wl.S, wl.Hq, wl.D)
    f = lambda t: t.float().cpu().numpy()
    check_bwd(oracle_mod, wl, (q, fused[:, :, :, g], fused[:, :, :, g + 1], do), (f(dq), f(dk), f(dv)))


def test_bwd_deterministic_dkdv():
    """dK and dV are accumulated in TMEM inside one CTA: bitwise repeatable."""
    wl = synth.workload("256px")
    _, g1 = run_fwd_bwd(wl)
    _, g2 = run_fwd_bwd(wl)
    assert np.array_equal(g1[1], g2[1]) and np.array_equal(g1[2], g2[2])


@pytest.mark.parametrize("norm", [False, True])
def test_bwd_reusing_forward_workspace(oracle_mod, norm):
    """hia_attn_bwd_reuse_fwd reads the rotated (and normed) q, k from the
    forward's workspace: dk, dv equal the plain backward's bit for bit, dq
    (unordered fp32 reduce-adds) to rounding, and all match the oracle.  The
    backward workspace starts filled with NaN bytes and is used twice: its
    dQ accumulator must be cleared by the library on every call."""
    wl = synth.workload("256px")
    q, k, v, do = synth.tensors(wl, 3, grad=True)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    seg = jt.hia_segments_build(wl.samples, wl.S)
    c, s = jt.hia_rope2d_tables(seg, wl.D, wl.base)
    qk = None
    if norm:
        gw = torch.Generator().manual_seed(11)
        qk = (torch.rand(wl.D, generator=gw) + 0.5, torch.rand(wl.D, generator=gw) + 0.5, 1e-5)
    qkd = None if qk is None else (qk[0].cuda(), qk[1].cuda(), qk[2])
    wsf = torch.empty(jt.hia_attn_fwd_workspace_bytes(seg, wl.Hq, wl.Hkv, wl.D), dtype=torch.uint8, device="cuda")
    wsb = torch.full((jt.hia_attn_bwd_workspace_bytes(seg, wl.Hq, wl.Hkv, wl.D),), 0xFF, dtype=torch.uint8,
                     device="cuda")
    o, lse = jt.hia_attn_fwd(seg, qd, kd, vd, c, s, wl.scale, workspace=wsf, qk_norm=qkd)
    plain = jt.hia_attn_bwd(seg, qd, kd, vd, c, s, o, lse, dod, wl.scale, qk_norm=qkd)
    reuse1 = jt.hia_attn_bwd(seg, qd, kd, vd, c, s, o, lse, dod, wl.scale, workspace=wsb, qk_norm=qkd,
                             fwd_workspace=wsf)
    reuse2 = jt.hia_attn_bwd(seg, qd, kd, vd, c, s, o, lse, dod, wl.scale, workspace=wsb, qk_norm=qkd,
                             fwd_workspace=wsf)
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 0
    for r in (reuse1, reuse2):
        assert torch.equal(r[1], plain[1]) and torch.equal(r[2], plain[2])
        rel = float((r[0].float() - plain[0].float()).norm() / plain[0].float().norm())
        assert rel <= 1e-5, rel
    f = lambda t: t.float().cpu().numpy()
    ref_norm = None if qk is None else (qk[0].numpy(), qk[1].numpy(), qk[2])
    check_bwd(oracle_mod, wl, (q, k, v, do), (f(reuse2[0]), f(reuse2[1]), f(reuse2[2])), qk_norm=ref_norm)


def _fwd_bwd_with_split(wl, mode, seed=0):
    q, k, v, do = synth.tensors(wl, seed, grad=True)
    seg = jt.hia_segments_build(wl.samples, wl.S).set_bwd_split(mode)
    c, s = jt.hia_rope2d_tables(seg, wl.D, wl.base)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = jt.hia_attn_fwd(seg, qd, kd, vd, c, s, wl.scale)
    dq, dk, dv = jt.hia_attn_bwd(seg, qd, kd, vd, c, s, o, lse, dod, wl.scale)
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 0
    f = lambda t: t.float().cpu().numpy()
    return seg, (q, k, v, do), (f(dq), f(dk), f(dv))


def _chosen_parts(seg, wl):
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    return seg.bwd_schedules()[seg.bwd_choice(wl.Hkv, wl.Hq // wl.Hkv, n_sm)][0]


@pytest.mark.parametrize("name,mode", [("256px", 2), ("256px", 4), ("mixed_small", 3), ("mixed_small", 4),
                                       ("mixed_small", 5)])
def test_bwd_split_schedule_parity(oracle_mod, name, mode):
    """A split schedule forced on: mode 2 the estimate's best split one, 3 / 4
    / 5 the longest kv tiles' query ranges cut into 2 / 3 / 4 parts (each part
    a CTA writing fp32 dK/dV partials, added in part order by the part that
    finishes last): against the oracle in full and block by block, dk/dv
    bitwise repeatable."""
    if name == "mixed_small":
        wl = synth.custom([(300, 12, 20, 5), (0, 0, 0, 0), (700, 0, 0, 0), (64, 16, 16, 2)], 8, 2, 128)
    else:
        wl = synth.workload(name)
    seg, inputs, g1 = _fwd_bwd_with_split(wl, mode)
    assert seg.info().bwd_split_units > 0
    parts = _chosen_parts(seg, wl)
    assert parts == mode - 1 if mode >= 3 else parts > 1
    check_bwd(oracle_mod, wl, inputs, g1)
    _, _, g2 = _fwd_bwd_with_split(wl, mode)
    assert np.array_equal(g1[1], g2[1]) and np.array_equal(g1[2], g2[2])


@pytest.mark.parametrize("mode", [2, 4])
def test_bwd_split_schedule_full_size(oracle_mod, mode):
    """The single-sample training backward (1024px_bwd) with a split schedule
    forced on (the best split one, which cuts the longest tiles in four, and
    the best three-part one): two complete (b, kv head) groups against the
    oracle, one of them a kv head whose prefix tiles are split."""
    wl = synth.workload("1024px_bwd")
    seg, inputs, grads = _fwd_bwd_with_split(wl, mode)
    assert seg.info().bwd_split_units > 0
    assert _chosen_parts(seg, wl) == (4 if mode == 2 else 3)
    groups = np.zeros((wl.B, wl.Hkv), dtype=bool)
    groups[0, 1] = groups[0, 6] = True
    check_bwd(oracle_mod, wl, inputs, grads, groups=groups)
