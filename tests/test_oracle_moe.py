"""Pins of the MoE oracle (oracle/moe.py) against what the pages and the
mathematics fix, independent of the oracle's own code:

  - routing weights in closed form: renormalizing the top-k of a softmax
    cancels its denominator, so w_k = exp(l_k) / sum_{j in top-k} exp(l_j);
    logits chosen as logs of small integers give rational weights worked out
    by hand (build_moe_config: softmax over all experts, top-k, renormalized);
  - the tie rule (lower expert index first), on hand-built ties;
  - k = E reduces to a plain softmax (library routine);
  - the selected set equals the k largest logits (library partition);
  - the SwiGLU expert on scalars in closed form, which fixes the [up; gate]
    order (HunyuanSharedMLP: gate_and_up_proj holds [up; gate], up first),
    and on vectors against torch.nn.functional.silu;
  - the whole block against a dense mixture written with torch library
    routines (softmax, topk, silu, matmul over every expert), shared expert
    added with weight 1 (HunyuanImage3Block);
  - special cases: one expert per token (weight exactly 1), routed outputs
    zero (only the shared expert remains), token permutation, row subsets,
    a given selection.
"""
import math

import numpy as np
import pytest
import torch

from oracle import moe


def _eye_router(logit_rows):
    """x = logits, wg = I: the router sees exactly these logits."""
    x = np.asarray(logit_rows, dtype=np.float64)
    return x, np.eye(x.shape[1])


# (logits, k, expected ids, expected weights) -- worked by hand
HAND_CASES = [
    ([0.0, math.log(3), math.log(2), -10.0], 2, [1, 2], [3 / 5, 2 / 5]),
    ([math.log(2), math.log(2), 0.0, 0.0], 2, [0, 1], [1 / 2, 1 / 2]),       # tie at the top
    ([math.log(3), 0.0, 0.0, -1.0], 2, [0, 1], [3 / 4, 1 / 4]),              # tie for second: index 1 first
    ([0.0, math.log(4), math.log(2), math.log(3)], 3, [1, 3, 2], [4 / 9, 3 / 9, 2 / 9]),
    ([5.0, 5.0, 5.0, 5.0, 5.0, 5.0], 4, [0, 1, 2, 3], [1 / 4] * 4),          # all tied
    ([-1.0, 2.0, 0.5], 1, [1], [1.0]),                                       # one expert: weight 1
]


@pytest.mark.parametrize("logits,k,ids,weights", HAND_CASES)
def test_router_hand_worked_cases(logits, k, ids, weights):
    x, wg = _eye_router([logits])
    got_ids, got_w, probs, got_logits = moe.router(x, wg, k)
    assert got_ids[0].tolist() == ids
    np.testing.assert_allclose(got_w[0], weights, rtol=0, atol=1e-15)
    np.testing.assert_allclose(got_logits[0], logits, atol=0)
    np.testing.assert_allclose(probs.sum(), 1.0, atol=1e-15)


def test_router_weights_closed_form_and_k_largest():
    rng = np.random.default_rng(0)
    T, H, E, k = 50, 16, 64, 8
    x = rng.standard_normal((T, H))
    wg = rng.standard_normal((E, H)) / 4
    ids, w, probs, logits = moe.router(x, wg, k)
    for t in range(T):
        # the selected set is the k largest logits (library partition; no ties in random data)
        assert set(ids[t]) == set(np.argpartition(-logits[t], k)[:k].tolist())
        assert np.all(np.diff(logits[t][ids[t]]) <= 0)  # descending
        ex = np.exp(logits[t][ids[t]])
        np.testing.assert_allclose(w[t], ex / ex.sum(), rtol=1e-13)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-14)


def test_router_top_all_is_softmax():
    rng = np.random.default_rng(1)
    x, wg = rng.standard_normal((20, 8)), rng.standard_normal((6, 8))
    ids, w, _, logits = moe.router(x, wg, 6)
    ref = torch.softmax(torch.from_numpy(logits), dim=1).numpy()
    np.testing.assert_allclose(np.take_along_axis(ref, ids, axis=1), w, rtol=1e-13)


def test_router_shift_invariance():
    """Adding the same amount to every logit (an extra input channel) changes nothing."""
    rng = np.random.default_rng(2)
    x, wg = rng.standard_normal((30, 12)), rng.standard_normal((16, 12))
    ids, w, _, _ = moe.router(x, wg, 4)
    x2 = np.concatenate([x, np.ones((30, 1))], axis=1)
    wg2 = np.concatenate([wg, np.full((16, 1), 7.5)], axis=1)
    ids2, w2, _, _ = moe.router(x2, wg2, 4)
    assert np.array_equal(ids, ids2)
    np.testing.assert_allclose(w, w2, rtol=1e-12)


def test_swiglu_scalar_closed_form_fixes_up_gate_order():
    # H = I = 1: up = a x, gate = b x, y = c * silu(b x) * (a x)
    a, b, c, xv = 1.0, 2.0, 1.5, 1.0
    w13 = np.array([[a], [b]])  # [up; gate]
    w2 = np.array([[c]])
    y = moe.expert(np.array([[xv]]), w13, w2)[0, 0]
    assert y == pytest.approx(c * (b * xv / (1 + math.exp(-b * xv))) * (a * xv), rel=1e-15)
    swapped = c * (a * xv / (1 + math.exp(-a * xv))) * (b * xv)
    assert abs(y - swapped) > 0.1
    # silu(0) = 0: a zero gate silences the expert whatever the up projection
    assert moe.expert(np.array([[3.0]]), np.array([[5.0], [0.0]]), np.array([[1.0]]))[0, 0] == 0.0


def test_swiglu_vectors_against_torch_silu():
    rng = np.random.default_rng(3)
    H, I, n = 10, 6, 7
    x, w13, w2 = rng.standard_normal((n, H)), rng.standard_normal((2 * I, H)), rng.standard_normal((H, I))
    tx, t13, t2 = (torch.from_numpy(v) for v in (x, w13, w2))
    up, gate = tx @ t13[:I].T, tx @ t13[I:].T
    ref = (torch.nn.functional.silu(gate) * up) @ t2.T
    np.testing.assert_allclose(moe.expert(x, w13, w2), ref.numpy(), rtol=1e-12, atol=1e-12)


def _random_block(seed, T=40, H=12, I=5, E=8):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H))
    wg = rng.standard_normal((E, H)) / 3
    w13 = rng.standard_normal((E + 1, 2 * I, H)) / math.sqrt(H)
    w2 = rng.standard_normal((E + 1, H, I)) / math.sqrt(I)
    return x, wg, w13, w2


def test_block_equals_dense_mixture_from_torch():
    x, wg, w13, w2 = _random_block(4)
    E, I, k = wg.shape[0], w13.shape[1] // 2, 3
    tx = torch.from_numpy(x)
    p = torch.softmax(tx @ torch.from_numpy(wg).T, dim=1)
    top, idx = torch.topk(p, k, dim=1)
    gates = torch.zeros_like(p).scatter(1, idx, top / top.sum(dim=1, keepdim=True))
    out = torch.zeros_like(tx)
    for e in range(E + 1):
        t13, t2 = torch.from_numpy(w13[e]), torch.from_numpy(w2[e])
        y = (torch.nn.functional.silu(tx @ t13[I:].T) * (tx @ t13[:I].T)) @ t2.T
        out += (gates[:, e:e + 1] if e < E else 1.0) * y
    got, ids, w = moe.moe_fwd(x, wg, w13, w2, k)
    np.testing.assert_allclose(got, out.numpy(), rtol=1e-12, atol=1e-12)
    assert np.array_equal(np.sort(ids, axis=1), np.sort(idx.numpy(), axis=1))


def test_one_expert_per_token_and_shared_only():
    x, wg, w13, w2 = _random_block(5)
    E = wg.shape[0]
    # top-1: weight exactly 1, output = own expert + shared
    got, ids, w = moe.moe_fwd(x, wg, w13, w2, 1)
    assert np.all(w == 1.0)
    for t in range(x.shape[0]):
        ref = moe.expert(x[t:t + 1], w13[ids[t, 0]], w2[ids[t, 0]]) + moe.expert(x[t:t + 1], w13[E], w2[E])
        np.testing.assert_allclose(got[t:t + 1], ref, rtol=1e-13, atol=1e-14)
    # routed down projections zero: only the shared expert remains
    w2z = w2.copy()
    w2z[:E] = 0.0
    got, _, _ = moe.moe_fwd(x, wg, w13, w2z, 4)
    np.testing.assert_allclose(got, moe.expert(x, w13[E], w2[E]), rtol=1e-14, atol=1e-15)


def test_permutation_subset_and_given_selection():
    x, wg, w13, w2 = _random_block(6)
    k = 2
    full, ids, w = moe.moe_fwd(x, wg, w13, w2, k)
    perm = np.random.default_rng(7).permutation(x.shape[0])
    pf, _, _ = moe.moe_fwd(x[perm], wg, w13, w2, k)
    np.testing.assert_allclose(pf, full[perm], rtol=1e-13, atol=1e-14)
    rows = [3, 0, 17, 39]
    sub, sub_ids, _ = moe.moe_fwd(x, wg, w13, w2, k, tokens=rows)
    np.testing.assert_allclose(sub, full[rows], rtol=1e-13, atol=1e-14)
    assert np.array_equal(sub_ids, ids[rows])
    # the oracle's own selection given back: the same result
    same, _, _ = moe.moe_fwd(x, wg, w13, w2, k, ids=ids)
    np.testing.assert_allclose(same, full, rtol=0, atol=0)
    # another selection: weights are those experts' probabilities, renormalized
    other = ids[:, ::-1].copy()
    other[:, 1] = (ids[:, 0] + 1) % wg.shape[0]
    _, _, wo = moe.moe_fwd(x, wg, w13, w2, k, ids=other)
    _, _, probs, _ = moe.router(x, wg, k)
    p = np.take_along_axis(probs, other, axis=1)
    np.testing.assert_allclose(wo, p / p.sum(axis=1, keepdims=True), rtol=1e-14)
