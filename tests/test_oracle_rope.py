"""Pins for the oracle's generalized 2D RoPE (paper review 3.4, Figure 5;
technical report summary 3.1.3; HunyuanImage3Attention cos/sin tables)."""
import numpy as np
import torch

from conftest import read_golden


def test_hand_derived_positions(oracle_mod):
    for c in read_golden("rope_positions.txt"):
        P, h, w, s, S = map(int, c["head"])
        want = np.array([[int(t) for t in r.split()] for r in c["rows"]])
        x, y = oracle_mod.positions([(P, h, w, s)], S)
        assert np.array_equal(x[0], want[:, 0]) and np.array_equal(y[0], want[:, 1])


def test_text_only_equals_library_1d_rope(oracle_mod):
    """No image tokens: the tables must be standard 1D RoPE.  Compared with the
    transformers Llama rotary embedding (default rope, base 10000, half-split
    cos/sin layout), a library routine independent of the oracle."""
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding
    D, S = 64, 48
    cfg = LlamaConfig(hidden_size=D * 4, num_attention_heads=4, head_dim=D,
                      max_position_embeddings=4096)
    c_ref, s_ref = LlamaRotaryEmbedding(cfg)(torch.zeros(1, S, D), torch.arange(S)[None])
    c, s = oracle_mod.rope_tables([(S, 0, 0, 0)], S, D, 10000.0)
    # the library computes in fp32; positions < 48 keep its angle error < 1e-5
    assert np.allclose(c[0], c_ref[0].double().numpy(), atol=2e-5)
    assert np.allclose(s[0], s_ref[0].double().numpy(), atol=2e-5)


def test_2d_reduces_exactly_to_1d_without_image(oracle_mod):
    """Exact (bitwise) reduction: a sample with h*w = 0 gives the same tables
    as the diagonal positions of text tokens in any other sample."""
    D, S = 128, 40
    c1, s1 = oracle_mod.rope_tables([(30, 0, 0, 10)], S, D)
    c2, s2 = oracle_mod.rope_tables([(S, 0, 0, 0)], S, D)
    c3, s3 = oracle_mod.rope_tables([(5, 3, 3, 2)], S, D)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
    # text rows of the image sample (before the image, after it) equal 1D rows
    for n in list(range(5)) + list(range(14, S)):
        assert np.array_equal(c3[0, n], c2[0, n]) and np.array_equal(s3[0, n], s2[0, n])


def test_row_and_column_sharing(oracle_mod):
    """Image tokens of one column share the x (even-j) angles; tokens of one
    row share the y (odd-j) angles; halves j and j + D/2 are equal."""
    D, P, h, w = 16, 4, 3, 5
    S = P + h * w + 1
    c, s = oracle_mod.rope_tables([(P, h, w, 1)], S, D)
    c = c[0]
    assert np.array_equal(c[:, : D // 2], c[:, D // 2:])
    tok = lambda r, cc: P + r * w + cc
    for r in range(h):
        for cc in range(w):
            assert np.array_equal(c[tok(r, cc), 0:D // 2:2], c[tok(0, cc), 0:D // 2:2])
            assert np.array_equal(c[tok(r, cc), 1:D // 2:2], c[tok(r, 0), 1:D // 2:2])
    # top-left image token sits on the diagonal at I0: same as text position P
    ct, _ = oracle_mod.rope_tables([(S, 0, 0, 0)], S, D)
    assert np.array_equal(c[tok(0, 0)], ct[0, P])


def test_apply_matches_library_rotate_half(oracle_mod):
    """R q equals q*cos + rotate_half(q)*sin as the transformers Llama helper
    applies it, given the oracle's tables."""
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    rng = np.random.default_rng(0)
    smp = [(3, 2, 3, 2)]
    S, H, D = 11, 2, 8
    x = rng.standard_normal((1, S, H, D))
    c, s = oracle_mod.rope_tables(smp, S, D)
    got = oracle_mod.rope_apply(smp, x)
    xt = torch.from_numpy(x)
    ref, _ = apply_rotary_pos_emb(xt, xt, torch.from_numpy(c), torch.from_numpy(s), unsqueeze_dim=2)
    assert np.allclose(got, ref.numpy(), atol=1e-14)


def test_orthogonal_and_inverse(oracle_mod):
    rng = np.random.default_rng(1)
    smp = [(4, 3, 2, 1)]
    x = rng.standard_normal((1, 12, 3, 32))
    y = oracle_mod.rope_apply(smp, x)
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), atol=1e-12)
    assert np.allclose(oracle_mod.rope_apply(smp, y, inverse=True), x, atol=1e-12)


def test_relative_position_invariance(oracle_mod):
    """<R(p+t) q, R(p'+t) k> = <R(p) q, R(p') k> for a 2D shift t.  Shifting
    the whole image block by t = (d, d) is a prefix change of d tokens, which
    moves every image position by (d, d)."""
    rng = np.random.default_rng(2)
    D, h, w = 32, 3, 4
    q = rng.standard_normal(D)
    k = rng.standard_normal(D)
    def rot_pair(P, i, j):
        S = P + h * w
        x = np.zeros((1, S, 2, D))
        x[0, P + i, 0] = q
        x[0, P + j, 1] = k
        y = oracle_mod.rope_apply([(P, h, w, 0)], x)
        return float(y[0, P + i, 0] @ y[0, P + j, 1])
    for (i, j) in [(0, 11), (5, 2), (7, 7), (3, 8)]:
        a = rot_pair(2, i, j)
        for P in (3, 9, 40):
            assert abs(rot_pair(P, i, j) - a) < 1e-12 * max(1.0, abs(a))
