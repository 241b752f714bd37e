"""Pins for the oracle's mask (build_joint_attention_mask; 3.1.2; 3.3)."""
import numpy as np
import pytest

from conftest import read_golden
from joint_text_image_b200 import synth


def test_hand_written_masks(oracle_mod):
    cases = read_golden("mask_cases.txt")
    assert len(cases) >= 6
    for c in cases:
        name, P, h, w, s, S = c["head"][0], *map(int, c["head"][1:])
        want = np.array([[int(ch) for ch in row] for row in c["rows"]], dtype=np.uint8)
        assert want.shape == (S, S), name
        got = oracle_mod.mask([(P, h, w, s)], S)[0]
        assert np.array_equal(got, want), name


def closed_form_pairs(P, h, w, s, S):
    """Sum over query rows of the visible-key count, by segment:
    text rows q < P see q+1 keys; each image row sees P+n keys; suffix row q
    sees q+1; each padded row sees all L real keys."""
    n = h * w
    L = P + n + s
    return P * (P + 1) // 2 + n * (P + n) + sum(q + 1 for q in range(P + n, L)) + (S - L) * L


def test_tiny_pair_count_worked_example(oracle_mod):
    # 15 text + <timestep> = 16, 8x8 image, suffix 2: 136 + 5120 + 163 = 5419.
    assert closed_form_pairs(16, 8, 8, 2, 82) == 5419
    assert int(oracle_mod.mask([(16, 8, 8, 2)], 82).sum()) == 5419


@pytest.mark.parametrize("name", ["256px", "mixed"])
def test_pair_counts_closed_form(oracle_mod, name):
    wl = synth.workload(name)
    m = oracle_mod.mask(wl.samples, wl.S)
    for b, smp in enumerate(wl.samples):
        assert int(m[b].sum()) == closed_form_pairs(*smp, wl.S)


def test_mask_is_prefix_of_monotone_bound(oracle_mod):
    """Every row's visible set is a prefix [0, e(q)] and e is non-decreasing."""
    samples = [(5, 3, 4, 2), (0, 2, 2, 0), (7, 0, 0, 3), (1, 1, 5, 1)]
    S = 22
    m = oracle_mod.mask(samples, S)
    for b in range(len(samples)):
        prev = -1
        for q in range(S):
            row = m[b, q]
            e = int(row.sum()) - 1
            assert np.all(row[: e + 1] == 1) and np.all(row[e + 1:] == 0)
            assert e >= prev
            prev = e


def test_text_only_is_causal_and_pad_keys_masked(oracle_mod):
    S, L = 9, 6
    m = oracle_mod.mask([(L, 0, 0, 0)], S)[0]
    want = np.tril(np.ones((S, S), dtype=np.uint8))
    want[:, L:] = 0
    assert np.array_equal(m, want)
