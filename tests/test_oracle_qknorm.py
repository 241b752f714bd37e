"""Pins for the oracle's per-head QK RMSNorm (RoPE first, then the norm, as
the HunyuanImage3Attention layer states): library routines in torch fp64
(transformers' rotary helper, torch.nn.functional.rms_norm, SDPA, autograd),
the norm's scale invariance, its reduction to the plain attention on
unit-RMS rows, and central finite differences for the weights."""
import numpy as np
import pytest
import torch

SAMPLES = [(5, 2, 3, 2), (3, 0, 0, 4), (0, 3, 3, 1)]


def _inputs(rng, S, Hq, Hkv, D, B):
    return (rng.standard_normal((B, S, Hq, D)), rng.standard_normal((B, S, Hkv, D)),
            rng.standard_normal((B, S, Hkv, D)), rng.standard_normal((B, S, Hq, D)))


def _library_ref(oracle_mod, samples, q, k, v, do, wq, wk, eps):
    """torch fp64: transformers' apply_rotary_pos_emb with the oracle's tables
    (pinned by test_oracle_rope), F.rms_norm over the head vector, SDPA with
    the oracle's mask (pinned by the hand-written fixtures), autograd."""
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    B, S, Hq, D = q.shape
    g = Hq // k.shape[2]
    c, s = oracle_mod.rope_tables(samples, S, D)
    c, s = torch.from_numpy(c), torch.from_numpy(s)
    tq, tk, tv = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
    twq, twk = torch.from_numpy(wq).requires_grad_(True), torch.from_numpy(wk).requires_grad_(True)
    qr, _ = apply_rotary_pos_emb(tq, tq, c, s, unsqueeze_dim=2)
    kr, _ = apply_rotary_pos_emb(tk, tk, c, s, unsqueeze_dim=2)
    qn = torch.nn.functional.rms_norm(qr, (D,), weight=twq, eps=eps)
    kn = torch.nn.functional.rms_norm(kr, (D,), weight=twk, eps=eps)
    m = torch.from_numpy(oracle_mod.mask(samples, S).astype(bool))[:, None]
    o = torch.nn.functional.scaled_dot_product_attention(
        qn.permute(0, 2, 1, 3), kn.permute(0, 2, 1, 3).repeat_interleave(g, dim=1),
        tv.permute(0, 2, 1, 3).repeat_interleave(g, dim=1), attn_mask=m, scale=D ** -0.5).permute(0, 2, 1, 3)
    o.backward(torch.from_numpy(do))
    return (o.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy(), twq.grad.numpy(),
            twk.grad.numpy())


@pytest.mark.parametrize("eps", [1e-5, 0.0])
def test_qknorm_matches_library_autograd(oracle_mod, eps):
    rng = np.random.default_rng(20)
    S, Hq, Hkv, D = 15, 4, 2, 16
    q, k, v, do = _inputs(rng, S, Hq, Hkv, D, len(SAMPLES))
    wq, wk = 1.0 + 0.3 * rng.standard_normal(D), 1.0 + 0.3 * rng.standard_normal(D)
    o, _, _ = oracle_mod.attn_fwd(SAMPLES, q, k, v, qk_norm=(wq, wk, eps))
    dq, dk, dv, dwq, dwk, _ = oracle_mod.attn_bwd_qknorm(SAMPLES, q, k, v, do, (wq, wk, eps))
    ro, rdq, rdk, rdv, rdwq, rdwk = _library_ref(oracle_mod, SAMPLES, q, k, v, do, wq, wk, eps)
    for got, want in ((o, ro), (dq, rdq), (dk, rdk), (dv, rdv), (dwq, rdwq), (dwk, rdwk)):
        assert np.allclose(got, want, atol=1e-11, rtol=1e-11)


def test_qknorm_is_scale_invariant(oracle_mod):
    """With eps = 0 the norm removes any positive per-row scale of q and k."""
    rng = np.random.default_rng(21)
    S, Hq, Hkv, D = 15, 4, 2, 16
    q, k, v, _ = _inputs(rng, S, Hq, Hkv, D, len(SAMPLES))
    wq, wk = rng.uniform(0.5, 1.5, D), rng.uniform(0.5, 1.5, D)
    o, lse, _ = oracle_mod.attn_fwd(SAMPLES, q, k, v, qk_norm=(wq, wk, 0.0))
    sq = rng.uniform(0.1, 10.0, q.shape[:3] + (1,))
    sk = rng.uniform(0.1, 10.0, k.shape[:3] + (1,))
    o2, lse2, _ = oracle_mod.attn_fwd(SAMPLES, q * sq, k * sk, v, qk_norm=(wq, wk, 0.0))
    assert np.allclose(o2, o, atol=1e-12) and np.allclose(lse2, lse, atol=1e-12, equal_nan=True)


def test_qknorm_on_unit_rms_rows_is_plain_attention(oracle_mod):
    """Unit weights, eps = 0 and rows of RMS 1 (R is orthogonal, so R q keeps
    the RMS): the norm is the identity and the plain attention results."""
    rng = np.random.default_rng(22)
    S, Hq, Hkv, D = 15, 4, 2, 16
    q, k, v, do = _inputs(rng, S, Hq, Hkv, D, len(SAMPLES))
    q = q / np.sqrt(np.mean(q * q, axis=-1, keepdims=True))
    k = k / np.sqrt(np.mean(k * k, axis=-1, keepdims=True))
    one = np.ones(D)
    o, lse, _ = oracle_mod.attn_fwd(SAMPLES, q, k, v, qk_norm=(one, one, 0.0))
    o0, lse0, _ = oracle_mod.attn_fwd(SAMPLES, q, k, v)
    assert np.allclose(o, o0, atol=1e-12) and np.allclose(lse, lse0, atol=1e-12)
    dq, dk, dv, _, _, _ = oracle_mod.attn_bwd_qknorm(SAMPLES, q, k, v, do, (one, one, 0.0))
    dq0, dk0, dv0, _ = oracle_mod.attn_bwd(SAMPLES, q, k, v, do)
    # the norm's Jacobian at a unit-RMS row is the projection I - x x^T / D
    assert np.allclose(dv, dv0, atol=1e-12)
    for got, plain, x in ((dq, dq0, q), (dk, dk0, k)):
        want = plain - x * np.sum(plain * x, axis=-1, keepdims=True) / D
        assert np.allclose(got, want, atol=1e-11)


def test_qknorm_weight_gradients_finite_differences(oracle_mod):
    """Central differences (h = 1e-6) of loss = sum(O * dO) w.r.t. wq, wk and q."""
    rng = np.random.default_rng(23)
    smp = [(3, 2, 2, 1)]
    S, Hq, Hkv, D = 11, 2, 1, 8
    q, k, v, do = _inputs(rng, S, Hq, Hkv, D, 1)
    wq, wk, eps = 1.0 + 0.2 * rng.standard_normal(D), 1.0 + 0.2 * rng.standard_normal(D), 1e-5
    dq, _, _, dwq, dwk, _ = oracle_mod.attn_bwd_qknorm(smp, q, k, v, do, (wq, wk, eps))

    def loss(qq, a, b):
        return float(np.sum(oracle_mod.attn_fwd(smp, qq, k, v, nthreads=1, qk_norm=(a, b, eps))[0] * do))

    h = 1e-6
    for name, x, gref in (("wq", wq, dwq), ("wk", wk, dwk), ("q", q, dq)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            ap = {"wq": (q, xp, wk), "wk": (q, wq, xp), "q": (xp, wq, wk)}[name]
            am = {"wq": (q, xm, wk), "wk": (q, wq, xm), "q": (xm, wq, wk)}[name]
            fd[idx] = (loss(*ap) - loss(*am)) / (2 * h)
        err = np.linalg.norm(fd - gref) / np.linalg.norm(gref)
        assert err < 1e-6, (name, err)


def test_qknorm_argument_checks(oracle_mod):
    rng = np.random.default_rng(24)
    q, k, v, do = _inputs(rng, 6, 2, 1, 8, 1)
    with pytest.raises(ValueError):
        oracle_mod.attn_fwd([(2, 1, 2, 1)], q, k, v, qk_norm=(np.ones(8), np.ones(8), -1.0))
