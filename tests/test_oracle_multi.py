"""Pins for the oracle's multi-image sequences (technical report summary
3.1.2: with several generated images, an image already in context is hidden
from the tokens after it): hand-written
masks, the reduction to the one-image layout, hand-derived positions, the
row-bound-minus-hidden-spans form the kernels use, and a library attention
routine on the multi-image mask."""
import numpy as np
import pytest
import torch

from conftest import read_golden


def golden_cases():
    out = []
    for c in read_golden("mask_multi_image.txt"):
        h = c["head"]
        name, S, rest = h[0], int(h[1]), h[2:]
        i = rest.index("suffix")
        images = [tuple(map(int, rest[j:j + 3])) for j in range(0, i, 3)]
        want = np.array([[int(ch) for ch in r] for r in c["rows"]], dtype=np.uint8)
        out.append((name, S, images, int(rest[i + 1]), want))
    return out


@pytest.mark.parametrize("case", golden_cases(), ids=lambda c: c[0])
def test_mask_golden(oracle_mod, case):
    _, S, images, suffix, want = case
    assert want.shape == (S, S)
    assert np.array_equal(oracle_mod.mask([(images, suffix)], S)[0], want)


def test_one_image_multi_form_is_the_canonical_layout(oracle_mod):
    rng = np.random.default_rng(30)
    canon = [(5, 2, 3, 2), (3, 0, 0, 4), (0, 3, 3, 1)]
    multi = [([(5, 2, 3)], 2), ([], 7), ([(0, 3, 3)], 1)]
    S, D = 15, 8
    assert np.array_equal(oracle_mod.mask(canon, S), oracle_mod.mask(multi, S))
    for a, b in zip(oracle_mod.positions(canon, S), oracle_mod.positions(multi, S)):
        assert np.array_equal(a, b)
    q, k, v = (rng.standard_normal((3, S, 2, D)) for _ in range(3))
    o1, l1, _ = oracle_mod.attn_fwd(canon, q, k, v)
    o2, l2, _ = oracle_mod.attn_fwd(multi, q, k, v)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_positions_hand_derived(oracle_mod):
    """t t A A t B B s pad, A 1x2 at I0 = 2, B 2x1 at I0 = 5: image tokens at
    (I0 + column, I0 + row) of their own grid, every other token at (n, n)."""
    x, y = oracle_mod.positions([([(2, 1, 2), (1, 2, 1)], 1)], 9)
    assert list(x[0]) == [0, 1, 2, 3, 4, 5, 5, 7, 8]
    assert list(y[0]) == [0, 1, 2, 2, 4, 5, 6, 7, 8]


def _random_layouts(rng, n):
    out = []
    for _ in range(n):
        m = int(rng.integers(0, 4))
        images = [(int(rng.integers(0, 4)), int(rng.integers(1, 4)), int(rng.integers(1, 4))) for _ in range(m)]
        out.append((images, int(rng.integers(0, 4))))
    return out


def test_mask_is_row_bound_minus_hidden_spans(oracle_mod):
    """The form the kernels evaluate: k visible from q iff k <= e(q) and k is
    not in a context image (every image but the last) whose span ends at or
    before q, with e(q) = min(L-1, end of q's image - 1 if q is in an image,
    else q) non-decreasing."""
    rng = np.random.default_rng(31)
    for images, suffix in _random_layouts(rng, 60):
        spans, pos = [], 0
        for (t, h, w) in images:
            spans.append((pos + t, pos + t + h * w))
            pos += t + h * w
        L = pos + suffix
        S = L + int(rng.integers(0, 3))
        m = oracle_mod.mask([(images, suffix)], S)[0].astype(bool)
        e_prev = -1
        for q in range(S):
            e = q
            for (a, b) in spans:
                if a <= q < b:
                    e = b - 1
            e = min(e, L - 1)
            assert e >= e_prev
            e_prev = e
            want = np.zeros(S, dtype=bool)
            want[:e + 1] = True
            for (a, b) in spans[:-1]:
                if b <= q:
                    want[a:b] = False
            assert np.array_equal(m[q], want), (images, suffix, q)


def test_multi_image_attention_matches_library(oracle_mod):
    """Forward and backward on a multi-image layout (inputs already rotated)
    against torch SDPA + autograd in fp64 with the oracle's mask."""
    rng = np.random.default_rng(32)
    samples = [([(2, 1, 2), (1, 2, 1)], 1), ([(0, 2, 2), (2, 1, 3), (1, 1, 1)], 2)]
    S, Hq, Hkv, D = 16, 4, 2, 8
    B = len(samples)
    q, do = (rng.standard_normal((B, S, Hq, D)) for _ in range(2))
    k, v = (rng.standard_normal((B, S, Hkv, D)) for _ in range(2))
    o, _, _ = oracle_mod.attn_fwd(samples, q, k, v, rotate=False)
    dq, dk, dv, _ = oracle_mod.attn_bwd(samples, q, k, v, do, rotate=False)
    m = torch.from_numpy(oracle_mod.mask(samples, S).astype(bool))[:, None]
    tq = torch.from_numpy(q).permute(0, 2, 1, 3).requires_grad_(True)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).requires_grad_(True)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).requires_grad_(True)
    g = Hq // Hkv
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk.repeat_interleave(g, 1), tv.repeat_interleave(g, 1),
                                                           attn_mask=m, scale=D ** -0.5)
    ref.backward(torch.from_numpy(do).permute(0, 2, 1, 3))
    assert np.allclose(o, ref.permute(0, 2, 1, 3).detach().numpy(), atol=1e-12)
    for got, t in ((dq, tq), (dk, tk), (dv, tv)):
        assert np.allclose(got, t.grad.permute(0, 2, 1, 3).numpy(), atol=1e-12)


def test_bad_multi_geometry_refused(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.mask([([(1, 0, 2)], 1)], 8)   # an image needs h, w > 0
    with pytest.raises(ValueError):
        oracle_mod.mask([([(1, 2, 2)], 1)], 5)   # L = 6 > S


def test_mask_columns_are_row_intervals(oracle_mod):
    """The backward's form: key k is seen exactly by the rows
    [first(k), end(k)), first(k) = its image's first token (or k itself for
    text), end(k) = the end of its image when that is a context image (else S);
    padded keys by no row."""
    rng = np.random.default_rng(33)
    for images, suffix in _random_layouts(rng, 60):
        spans, pos = [], 0
        for (t, h, w) in images:
            spans.append((pos + t, pos + t + h * w))
            pos += t + h * w
        L = pos + suffix
        S = L + int(rng.integers(0, 3))
        m = oracle_mod.mask([(images, suffix)], S)[0].astype(bool)
        for k in range(S):
            want = np.zeros(S, dtype=bool)
            if k < L:
                first, end = k, S
                for i, (a, b) in enumerate(spans):
                    if a <= k < b:
                        first = a
                        if i < len(spans) - 1:
                            end = b
                want[first:end] = True
            assert np.array_equal(m[:, k], want), (images, suffix, k)
