"""GPU parity for samples with several images (hia_segments_build_multi):
the forward and backward against the fp64 oracle, the one-image form against
the canonical builder, and the packed layout against the padded one."""
import numpy as np
import pytest
import torch

import joint_text_image_b200 as jt
from helpers import GRAD_REL, LSE_MAX, O_MAX, O_MEAN

pytestmark = pytest.mark.gpu

# Two context images and a last one, text in between; a sample whose only
# image is followed by a second; a text-only sample; image at position 0.
SAMPLES = [
    ([(33, 8, 16), (20, 16, 8), (7, 12, 12)], 2),
    ([(150, 16, 16), (1, 4, 32)], 40),
    ([], 300),
    ([(0, 10, 10), (64, 6, 6)], 3),
]


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "needs a GPU"
    jt.lib()


def length(x):
    return sum(t + h * w for t, h, w in x[0]) + x[1]


def inputs(S, Hq, Hkv, D, seed=0):
    g = torch.Generator().manual_seed(seed)
    B = len(SAMPLES)
    q = torch.randn(B, S, Hq, D, generator=g).bfloat16()
    k = torch.randn(B, S, Hkv, D, generator=g).bfloat16()
    v = torch.randn(B, S, Hkv, D, generator=g).bfloat16()
    do = torch.randn(B, S, Hq, D, generator=g).bfloat16()
    return q, k, v, do


def run(seg, q, k, v, do, scale):
    D = q.shape[-1]
    c, s = jt.hia_rope2d_tables(seg, D)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = jt.hia_attn_fwd(seg, qd, kd, vd, c, s, scale)
    dq, dk, dv = jt.hia_attn_bwd(seg, qd, kd, vd, c, s, o, lse, dod, scale)
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 0
    return [t.cpu() for t in (o, lse, dq, dk, dv)], (c.cpu(), s.cpu())


@pytest.mark.parametrize("D,split", [(128, 0), (64, 0), (128, 2), (64, 2)])
def test_multi_image_parity_with_oracle(oracle_mod, D, split):
    S = max(length(x) for x in SAMPLES) + 17
    Hq, Hkv = 4, 2
    q, k, v, do = inputs(S, Hq, Hkv, D)
    seg = jt.hia_segments_build_multi(SAMPLES, S).set_bwd_split(split)
    (o, lse, dq, dk, dv), (c, s) = run(seg, q, k, v, do, D ** -0.5)
    # tables: each image on its own grid, within one fp32 ulp of the oracle
    cr, sr = oracle_mod.rope_tables(SAMPLES, S, D)
    for got, ref in ((c, cr), (s, sr)):
        ref32 = ref.astype(np.float32)
        assert np.all(np.abs(got.numpy().astype(np.float64) - ref32) <= np.spacing(np.abs(ref32)))
    f64 = lambda t: t.double().numpy()
    o_ref, lse_ref, _ = oracle_mod.attn_fwd(SAMPLES, f64(q), f64(k), f64(v), D ** -0.5)
    err = np.abs(o.float().numpy() - o_ref)
    assert err.max() <= O_MAX and err.mean() <= O_MEAN
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse.numpy()), fin)
    assert np.abs(lse.numpy()[fin] - lse_ref[fin]).max() <= LSE_MAX
    refs = oracle_mod.attn_bwd(SAMPLES, f64(q), f64(k), f64(v), f64(do), D ** -0.5)[:3]
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        rel = np.linalg.norm(got.float().numpy() - ref) / np.linalg.norm(ref)
        assert rel <= GRAD_REL, (name, rel)


def test_multi_packed_equals_padded():
    S = max(length(x) for x in SAMPLES) + 9
    q, k, v, do = inputs(S, 4, 2, 128, seed=1)
    lens = [length(x) for x in SAMPLES]
    for b, L in enumerate(lens):
        do[b, L:] = 0  # padded rows then add nothing to dk, dv
    # one backward schedule for both layouts (bitwise dk, dv; see test_packed_gpu)
    pad, _ = run(jt.hia_segments_build_multi(SAMPLES, S).set_bwd_split(1), q, k, v, do, 128 ** -0.5)
    seg = jt.hia_segments_build_multi(SAMPLES, packed=True).set_bwd_split(1)
    pack = lambda x: torch.cat([x[b, :L] for b, L in enumerate(lens)], 0).contiguous()
    c, s = jt.hia_rope2d_tables(seg, 128)
    qp, kp, vp, dop = (pack(t).cuda() for t in (q, k, v, do))
    o, lse = jt.hia_attn_fwd(seg, qp, kp, vp, c, s)
    dq, dk, dv = jt.hia_attn_bwd(seg, qp, kp, vp, c, s, o, lse, dop)
    torch.cuda.synchronize()
    o, lse, dq, dk, dv = (t.cpu() for t in (o, lse, dq, dk, dv))
    off = 0
    for b, L in enumerate(lens):
        assert torch.equal(o[off:off + L], pad[0][b, :L]) and torch.equal(lse[:, off:off + L], pad[1][b, :, :L])
        assert torch.equal(dk[off:off + L], pad[3][b, :L]) and torch.equal(dv[off:off + L], pad[4][b, :L])
        a, r = dq[off:off + L].float(), pad[2][b, :L].float()
        assert (a - r).norm() <= 1e-3 * max(r.norm(), 1e-30)
        off += L


def test_one_image_multi_form_equals_canonical():
    canon = [(40, 8, 8, 2), (0, 0, 0, 0), (90, 0, 0, 0), (0, 12, 12, 5)]
    multi = [([(40, 8, 8)], 2), ([], 0), ([], 90), ([(0, 12, 12)], 5)]
    S = 160
    q, k, v, do = inputs(S, 4, 2, 128, seed=2)
    a, _ = run(jt.hia_segments_build(canon, S), q, k, v, do, 128 ** -0.5)
    b, _ = run(jt.hia_segments_build_multi(multi, S), q, k, v, do, 128 ** -0.5)
    for i in (0, 1, 3, 4):  # o, lse, dk, dv bitwise; dq up to its reduction order
        assert torch.equal(a[i], b[i])
    assert (a[2].float() - b[2].float()).norm() <= 1e-3 * a[2].float().norm()


@pytest.mark.parametrize("split", [0, 2])
def test_multi_packed_with_qk_norm_against_oracle(oracle_mod, split):
    """All three options at once: several images per sample, the packed
    layout and the QK RMSNorm, against the oracle on the padded equivalent;
    with the automatic backward schedule and with the split one forced on."""
    S = max(length(x) for x in SAMPLES) + 5
    Hq, Hkv, D, eps = 4, 2, 128, 1e-5
    q, k, v, do = inputs(S, Hq, Hkv, D, seed=3)
    lens = [length(x) for x in SAMPLES]
    for b, L in enumerate(lens):
        do[b, L:] = 0
    g = torch.Generator().manual_seed(9)
    wq = (torch.rand(D, generator=g, dtype=torch.float64) + 0.5).float()
    wk = (torch.rand(D, generator=g, dtype=torch.float64) + 0.5).float()
    seg = jt.hia_segments_build_multi(SAMPLES, packed=True).set_bwd_split(split)
    pack = lambda x: torch.cat([x[b, :L] for b, L in enumerate(lens)], 0).contiguous()
    c, s = jt.hia_rope2d_tables(seg, D)
    qp, kp, vp, dop = (pack(t).cuda() for t in (q, k, v, do))
    norm = (wq.cuda(), wk.cuda(), eps)
    o, lse = jt.hia_attn_fwd(seg, qp, kp, vp, c, s, qk_norm=norm)
    dq, dk, dv, dwq, dwk = jt.hia_attn_bwd(seg, qp, kp, vp, c, s, o, lse, dop, qk_norm=norm)
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 0
    ref_norm = (wq.double().numpy(), wk.double().numpy(), eps)
    f64 = lambda t: t.double().numpy()
    o_ref, lse_ref, _ = oracle_mod.attn_fwd(SAMPLES, f64(q), f64(k), f64(v), D ** -0.5, qk_norm=ref_norm)
    rdq, rdk, rdv, rdwq, rdwk, _ = oracle_mod.attn_bwd_qknorm(SAMPLES, f64(q), f64(k), f64(v), f64(do), ref_norm,
                                                              D ** -0.5)
    off = 0
    errs, grads = [], {"dq": ([], []), "dk": ([], []), "dv": ([], [])}
    for b, L in enumerate(lens):
        errs.append(np.abs(o[off:off + L].float().cpu().numpy() - o_ref[b, :L]).ravel())
        lr = lse_ref[b, :, :L]
        assert np.abs(lse[:, off:off + L].cpu().numpy() - lr).max() <= LSE_MAX
        for name, got, ref in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
            grads[name][0].append(got[off:off + L].float().cpu().numpy().ravel())
            grads[name][1].append(ref[b, :L].ravel())
        off += L
    e = np.concatenate(errs)
    assert e.max() <= O_MAX and e.mean() <= O_MEAN
    for name, (a, r) in grads.items():
        a, r = np.concatenate(a), np.concatenate(r)
        assert np.linalg.norm(a - r) / np.linalg.norm(r) <= GRAD_REL, name
    for got, ref in ((dwq, rdwq), (dwk, rdwk)):
        assert np.linalg.norm(got.cpu().numpy() - ref) / np.linalg.norm(ref) <= GRAD_REL


def test_multi_image_forward_repeated_with_held_allocations(oracle_mod):
    """The several-images step (D = 128) repeated with differently sized
    allocations held alive between calls, so that the inputs, tables,
    workspaces and outputs land at other addresses each time, and with a
    backward between forwards.  Warps that run the per-row hidden-image
    masking once returned wrong forward rows on some boxes in exactly this
    pattern (every row of such a warp, the same values every call: the warp
    reached the warp-collective TMEM stores diverged); each forward must
    match the oracle."""
    S = max(length(x) for x in SAMPLES) + 17
    Hq, Hkv, D = 4, 2, 128
    q, k, v, do = inputs(S, Hq, Hkv, D)
    f64 = lambda t: t.double().numpy()
    o_ref = oracle_mod.attn_fwd(SAMPLES, f64(q), f64(k), f64(v), D ** -0.5)[0]
    rng = np.random.default_rng(0)
    held = []
    for it in range(8):
        held.append(torch.full((int(rng.integers(1, 3_000_000)),), float("nan"), device="cuda"))
        if len(held) > 6:
            held.pop(0)
        seg = jt.hia_segments_build_multi(SAMPLES, S).set_bwd_split([0, 2, 1][it % 3])
        c, s = jt.hia_rope2d_tables(seg, D)
        qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
        o, lse = jt.hia_attn_fwd(seg, qd, kd, vd, c, s, D ** -0.5)
        torch.cuda.synchronize()
        assert jt.hia_get_device_status() == 0
        err = np.abs(o.float().cpu().numpy() - o_ref)
        assert err.max() <= O_MAX and err.mean() <= O_MEAN, (it, float(err.max()))
        jt.hia_attn_bwd(seg, qd, kd, vd, c, s, o, lse, dod, D ** -0.5)
        torch.cuda.synchronize()
        assert jt.hia_get_device_status() == 0


def _random_case(rng):
    """A random batch of samples with up to three images each (text gaps,
    image sizes and tails drawn at random; empty and text-only samples
    included), a random GQA group size and head dim."""
    B = int(rng.integers(1, 4))
    samples = []
    for _ in range(B):
        segs = []
        for _ in range(int(rng.integers(0, 4))):
            segs.append((int(rng.integers(0, 81)), int(rng.integers(1, 17)), int(rng.integers(1, 17))))
        samples.append((segs, int(rng.integers(0, 41))))
    S = max(max(length(x) for x in samples), 1) + int(rng.integers(0, 41))
    Hkv = int(rng.integers(1, 4))
    g = int(rng.integers(1, 5))
    D = int(rng.choice([64, 128]))
    return samples, S, g * Hkv, Hkv, D


@pytest.mark.parametrize("case", range(16))
def test_multi_image_random_configs(oracle_mod, case):
    """Seeded random several-images batches (ragged lengths, empty samples,
    g from 1 to 4, D = 64 or 128, both backward schedules): forward and
    backward against the oracle."""
    rng = np.random.default_rng(1000 + case)
    samples, S, Hq, Hkv, D = _random_case(rng)
    g = torch.Generator().manual_seed(case)
    B = len(samples)
    q = torch.randn(B, S, Hq, D, generator=g).bfloat16()
    k = torch.randn(B, S, Hkv, D, generator=g).bfloat16()
    v = torch.randn(B, S, Hkv, D, generator=g).bfloat16()
    do = torch.randn(B, S, Hq, D, generator=g).bfloat16()
    seg = jt.hia_segments_build_multi(samples, S).set_bwd_split(2 * (case % 2))
    (o, lse, dq, dk, dv), _ = run(seg, q, k, v, do, D ** -0.5)
    f64 = lambda t: t.double().numpy()
    o_ref, lse_ref, _ = oracle_mod.attn_fwd(samples, f64(q), f64(k), f64(v), D ** -0.5)
    err = np.abs(o.float().numpy() - o_ref)
    assert err.max() <= O_MAX and err.mean() <= O_MEAN, (samples, S, Hq, Hkv, D, float(err.max()))
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse.numpy()), fin)
    if fin.any():
        assert np.abs(lse.numpy()[fin] - lse_ref[fin]).max() <= LSE_MAX
    refs = oracle_mod.attn_bwd(samples, f64(q), f64(k), f64(v), f64(do), D ** -0.5)[:3]
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        nr = np.linalg.norm(ref)
        diff = np.linalg.norm(got.float().numpy() - ref)
        assert (diff <= GRAD_REL * nr) if nr > 0 else diff == 0, (name, samples, S, Hq, Hkv, D)


@pytest.mark.parametrize("case", range(8))
def test_multi_image_random_packed_and_norm(oracle_mod, case):
    """Seeded random several-images batches in the packed layout, half of them
    with the QK RMSNorm, against the oracle on the padded equivalent (padded
    rows get zero dO, so they add nothing to dk, dv)."""
    rng = np.random.default_rng(2000 + case)
    samples, S, Hq, Hkv, D = _random_case(rng)
    lens = [length(x) for x in samples]
    if sum(lens) == 0:
        samples[0] = ([(3, 2, 2)], 1)
        lens = [length(x) for x in samples]
        S = max(S, lens[0])
    g = torch.Generator().manual_seed(100 + case)
    B = len(samples)
    q = torch.randn(B, S, Hq, D, generator=g).bfloat16()
    k = torch.randn(B, S, Hkv, D, generator=g).bfloat16()
    v = torch.randn(B, S, Hkv, D, generator=g).bfloat16()
    do = torch.randn(B, S, Hq, D, generator=g).bfloat16()
    for b, L in enumerate(lens):
        do[b, L:] = 0
    norm = case % 2 == 1
    eps = 1e-5
    wq = (torch.rand(D, generator=g, dtype=torch.float64) + 0.5).float()
    wk = (torch.rand(D, generator=g, dtype=torch.float64) + 0.5).float()
    seg = jt.hia_segments_build_multi(samples, packed=True).set_bwd_split(2 * ((case // 2) % 2))
    pack = lambda x: torch.cat([x[b, :L] for b, L in enumerate(lens)], 0).contiguous()
    c, s = jt.hia_rope2d_tables(seg, D)
    qp, kp, vp, dop = (pack(t).cuda() for t in (q, k, v, do))
    qn = (wq.cuda(), wk.cuda(), eps) if norm else None
    o, lse = jt.hia_attn_fwd(seg, qp, kp, vp, c, s, qk_norm=qn)
    out = jt.hia_attn_bwd(seg, qp, kp, vp, c, s, o, lse, dop, qk_norm=qn)
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 0
    dq, dk, dv = out[:3]
    f64 = lambda t: t.double().numpy()
    ref_norm = (wq.double().numpy(), wk.double().numpy(), eps) if norm else None
    o_ref, lse_ref, _ = oracle_mod.attn_fwd(samples, f64(q), f64(k), f64(v), D ** -0.5, qk_norm=ref_norm)
    if norm:
        rdq, rdk, rdv, rdwq, rdwk, _ = oracle_mod.attn_bwd_qknorm(samples, f64(q), f64(k), f64(v), f64(do), ref_norm,
                                                                  D ** -0.5)
    else:
        rdq, rdk, rdv = oracle_mod.attn_bwd(samples, f64(q), f64(k), f64(v), f64(do), D ** -0.5)[:3]
    off = 0
    errs, grads = [], {"dq": ([], []), "dk": ([], []), "dv": ([], [])}
    for b, L in enumerate(lens):
        errs.append(np.abs(o[off:off + L].float().cpu().numpy() - o_ref[b, :L]).ravel())
        lr = lse_ref[b, :, :L]
        assert np.abs(lse[:, off:off + L].cpu().numpy() - lr).max() <= LSE_MAX
        for name, got, ref in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
            grads[name][0].append(got[off:off + L].float().cpu().numpy().ravel())
            grads[name][1].append(ref[b, :L].ravel())
        off += L
    e = np.concatenate(errs)
    assert e.max() <= O_MAX and e.mean() <= O_MEAN, (samples, Hq, Hkv, D, norm)
    for name, (a, r) in grads.items():
        a, r = np.concatenate(a), np.concatenate(r)
        assert np.linalg.norm(a - r) <= GRAD_REL * np.linalg.norm(r), (name, samples, Hq, Hkv, D, norm)
    if norm:
        for got, ref in ((out[3], rdwq), (out[4], rdwk)):
            assert np.linalg.norm(got.cpu().numpy() - ref) <= GRAD_REL * np.linalg.norm(ref)
