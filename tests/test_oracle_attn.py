"""Pins for the oracle's attention forward and backward: a library attention
routine (torch SDPA, fp64 CPU) on the same rotated inputs, closed-form
special cases, and central finite differences through the 2D RoPE."""
import numpy as np
import pytest
import torch


def _sdpa_ref(oracle_mod, samples, qr, kr, v, scale, grad_out=None):
    """torch scaled_dot_product_attention with the oracle's bool mask (the
    mask itself is pinned by the hand-written fixtures).  GQA: head h reads kv
    head h // g (HunyuanImage3Attention's grouped QKV)."""
    B, S, Hq, D = qr.shape
    g = Hq // kr.shape[2]
    m = torch.from_numpy(oracle_mod.mask(samples, S).astype(bool))[:, None]
    q = torch.from_numpy(qr).permute(0, 2, 1, 3).requires_grad_(grad_out is not None)
    k = torch.from_numpy(kr).permute(0, 2, 1, 3).requires_grad_(grad_out is not None)
    vv = torch.from_numpy(v).permute(0, 2, 1, 3).requires_grad_(grad_out is not None)
    ke = k.repeat_interleave(g, dim=1)
    ve = vv.repeat_interleave(g, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(q, ke, ve, attn_mask=m, scale=scale)
    if grad_out is None:
        return o.permute(0, 2, 1, 3).detach().numpy()
    o.backward(torch.from_numpy(grad_out).permute(0, 2, 1, 3))
    return (o.permute(0, 2, 1, 3).detach().numpy(), q.grad.permute(0, 2, 1, 3).numpy(),
            k.grad.permute(0, 2, 1, 3).numpy(), vv.grad.permute(0, 2, 1, 3).numpy())


SAMPLES = [(5, 2, 3, 2), (3, 0, 0, 4), (0, 3, 3, 1), (2, 1, 4, 0)]


def _inputs(rng, S, Hq, Hkv, D, B):
    return (rng.standard_normal((B, S, Hq, D)), rng.standard_normal((B, S, Hkv, D)),
            rng.standard_normal((B, S, Hkv, D)), rng.standard_normal((B, S, Hq, D)))


def test_fwd_matches_library_sdpa(oracle_mod):
    rng = np.random.default_rng(0)
    S, Hq, Hkv, D = 15, 4, 2, 16
    q, k, v, _ = _inputs(rng, S, Hq, Hkv, D, len(SAMPLES))
    o, lse, _ = oracle_mod.attn_fwd(SAMPLES, q, k, v, rotate=False)
    ref = _sdpa_ref(oracle_mod, SAMPLES, q, k, v, D ** -0.5)
    assert np.allclose(o, ref, atol=1e-12)


def test_lse_closed_form(oracle_mod):
    """LSE = log sum_k exp(scale q.k) over the visible keys of each row."""
    rng = np.random.default_rng(3)
    S, D = 9, 8
    smp = [(2, 2, 2, 1)]
    q, k, v, _ = _inputs(rng, S, 1, 1, D, 1)
    m = oracle_mod.mask(smp, S)[0].astype(bool)
    _, lse, _ = oracle_mod.attn_fwd(smp, q, k, v, rotate=False)
    sc = 0.5 ** 1.5 * q[0, :, 0] @ k[0, :, 0].T
    for i in range(S):
        want = np.log(np.sum(np.exp(sc[i][m[i]])))
        assert abs(lse[0, 0, i] - want) < 1e-12


def test_first_row_is_v0_and_zero_k_is_mean(oracle_mod):
    rng = np.random.default_rng(4)
    smp = [(3, 2, 2, 1)]
    S, D = 10, 8
    q, k, v, _ = _inputs(rng, S, 2, 1, D, 1)
    o, _, _ = oracle_mod.attn_fwd(smp, q, k, v)
    assert np.array_equal(o[0, 0, 0], v[0, 0, 0]) and np.array_equal(o[0, 0, 1], v[0, 0, 0])
    o0, _, _ = oracle_mod.attn_fwd(smp, q, np.zeros_like(k), v)
    m = oracle_mod.mask(smp, S)[0].astype(bool)
    for i in range(S):
        assert np.allclose(o0[0, i, 0], v[0, m[i], 0].mean(axis=0), atol=1e-14)


def test_empty_sample_gives_zero_and_neg_inf(oracle_mod):
    rng = np.random.default_rng(5)
    q, k, v, do = _inputs(rng, 4, 2, 1, 8, 1)
    o, lse, _ = oracle_mod.attn_fwd([(0, 0, 0, 0)], q, k, v)
    assert np.all(o == 0) and np.all(np.isneginf(lse))
    dq, dk, dv, _ = oracle_mod.attn_bwd([(0, 0, 0, 0)], q, k, v, do)
    assert np.all(dq == 0) and np.all(dk == 0) and np.all(dv == 0)


def test_rows_and_groups_subsets(oracle_mod):
    rng = np.random.default_rng(6)
    S, Hq, Hkv, D = 15, 4, 2, 16
    q, k, v, do = _inputs(rng, S, Hq, Hkv, D, len(SAMPLES))
    o, lse, _ = oracle_mod.attn_fwd(SAMPLES, q, k, v)
    rows = [0, 7, 14]
    gs = np.zeros((len(SAMPLES), Hkv), dtype=bool)
    gs[1, 1] = gs[3, 0] = True
    o2, lse2, _ = oracle_mod.attn_fwd(SAMPLES, q, k, v, rows=rows, groups=gs)
    for b, hk in [(1, 1), (3, 0)]:
        hs = slice(hk * 2, hk * 2 + 2)
        assert np.array_equal(o2[b, rows, hs], o[b, rows, hs])
        assert np.array_equal(lse2[b, hs][:, rows], lse[b, hs][:, rows])
    dq, dk, dv, _ = oracle_mod.attn_bwd(SAMPLES, q, k, v, do)
    dq2, dk2, dv2, _ = oracle_mod.attn_bwd(SAMPLES, q, k, v, do, groups=gs)
    assert np.array_equal(dk2[1, :, 1], dk[1, :, 1]) and np.array_equal(dq2[3, :, 0:2], dq[3, :, 0:2])


def test_bwd_matches_library_autograd(oracle_mod):
    """Attention core (inputs already rotated) vs torch autograd of SDPA."""
    rng = np.random.default_rng(7)
    S, Hq, Hkv, D = 15, 4, 2, 16
    q, k, v, do = _inputs(rng, S, Hq, Hkv, D, len(SAMPLES))
    dq, dk, dv, _ = oracle_mod.attn_bwd(SAMPLES, q, k, v, do, rotate=False)
    _, gq, gk, gv = _sdpa_ref(oracle_mod, SAMPLES, q, k, v, D ** -0.5, grad_out=do)
    assert np.allclose(dq, gq, atol=1e-12)
    assert np.allclose(dk, gk, atol=1e-12)
    assert np.allclose(dv, gv, atol=1e-12)


@pytest.mark.parametrize("D", [4, 8])
def test_bwd_finite_differences_through_rope(oracle_mod, D):
    """Central differences (h = 1e-6, fp64) of loss = sum(O * dO) w.r.t. the
    raw (un-rotated) q, k, v: pins the gradient and the inverse rotation."""
    rng = np.random.default_rng(8 + D)
    smp = [(3, 2, 2, 1)]
    S, Hq, Hkv = 11, 2, 1          # prefix 3, 2x2 image, suffix 1, 3 padded rows
    q, k, v, do = _inputs(rng, S, Hq, Hkv, D, 1)
    q, k, v = q * 2.0, k * 2.0, v
    dq, dk, dv, _ = oracle_mod.attn_bwd(smp, q, k, v, do)
    loss = lambda qq, kk, vv: float(np.sum(oracle_mod.attn_fwd(smp, qq, kk, vv, nthreads=1)[0] * do))
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.linalg.norm(fd - g) / np.linalg.norm(g)
        assert err < 1e-6, (name, err)


def test_bwd_row_subsets_are_partial_sums(oracle_mod):
    """dQ of a row depends on that row only; dK, dV are sums over query rows,
    so disjoint row subsets add up to the full gradient."""
    rng = np.random.default_rng(9)
    S, Hq, Hkv, D = 15, 4, 2, 16
    q, k, v, do = _inputs(rng, S, Hq, Hkv, D, len(SAMPLES))
    dq, dk, dv, _ = oracle_mod.attn_bwd(SAMPLES, q, k, v, do)
    ra, rb = list(range(0, S, 2)), list(range(1, S, 2))
    dqa, dka, dva, _ = oracle_mod.attn_bwd(SAMPLES, q, k, v, do, rows=ra)
    dqb, dkb, dvb, _ = oracle_mod.attn_bwd(SAMPLES, q, k, v, do, rows=rb)
    assert np.array_equal(dqa[:, ra], dq[:, ra]) and np.all(dqa[:, rb] == 0)
    assert np.allclose(dka + dkb, dk, atol=1e-13) and np.allclose(dva + dvb, dv, atol=1e-13)
