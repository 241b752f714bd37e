"""CPU tests of the packed (varlen) segment descriptor: sizes, pair counts
and the tile classification, against the oracle's literal mask restricted to
each sample's own rows."""
import numpy as np
import pytest

import joint_text_image_b200 as jt
from joint_text_image_b200 import build as jbuild
from joint_text_image_b200 import synth

CASES = [
    [(3, 2, 2, 1)],
    [(0, 0, 0, 0), (5, 0, 0, 0)],
    [(100, 10, 13, 7), (0, 0, 0, 0), (250, 0, 0, 0), (0, 16, 16, 2)],
    [(130, 8, 16, 2), (1, 1, 1, 0), (64, 4, 32, 3)],
]


@pytest.fixture(scope="module", autouse=True)
def built():
    jbuild.build()


def lengths(samples):
    return [p + h * w + s for p, h, w, s in samples]


def brute_classes(mask_b, L, S, nQT, nKT):
    """Tile classes from the literal mask over the sample's rows [0, L):
    1 FULL (every key of a whole 128-key tile visible to every row),
    2 PARTIAL (some visible), 0/3 otherwise."""
    out = np.zeros((nQT, nKT), dtype=np.uint8)
    for qt in range(nQT):
        rows = np.arange(qt * 128, min(qt * 128 + 128, L))
        for kt in range(nKT):
            keys = np.arange(kt * 128, min(kt * 128 + 128, S))
            if len(rows) == 0:
                continue
            vis = mask_b[np.ix_(rows, keys)]
            if vis.all() and len(keys) == 128:
                out[qt, kt] = 1
            elif vis.any():
                out[qt, kt] = 2
    return out


@pytest.mark.parametrize("samples", CASES + [synth.workload("mixed").samples])
def test_packed_descriptor(oracle_mod, samples):
    seg = jt.hia_segments_build_packed(samples, upload=False)
    inf = seg.info()
    L = lengths(samples)
    S = max(L)
    assert inf.packed == 1 and inf.S == S and inf.total_rows == sum(L)
    assert seg.offsets == [sum(L[:b]) for b in range(len(L))] and seg.rows == L
    m = oracle_mod.mask(samples, S)
    # visible pairs over each sample's own rows only (no padded query rows)
    assert inf.visible_pairs == sum(int(m[b, :L[b]].sum()) for b in range(len(L)))
    cls = seg.tile_classes()
    for b in range(len(L)):
        want = brute_classes(m[b].astype(bool), L[b], S, inf.fwd_q_tiles, inf.fwd_kv_tiles)
        got = cls[b].copy()
        got[(got == 0) | (got == 3)] = 0
        assert np.array_equal(got, want), b


def test_packed_pairs_closed_form():
    """sum over q < L of (e(q) + 1) = P(P+1)/2 + n(P+n) + sum over the suffix
    rows of (row + 1): the padded closed form without the pad * L term."""
    samples = [(100, 10, 13, 7), (250, 0, 0, 0), (0, 16, 16, 2)]
    seg = jt.hia_segments_build_packed(samples, upload=False)
    want = 0
    for p, h, w, s in samples:
        n = h * w
        want += p * (p + 1) // 2 + n * (p + n) + sum(p + n + i + 1 for i in range(s))
    assert seg.info().visible_pairs == want


def test_padded_descriptor_reports_layout():
    seg = jt.hia_segments_build([(3, 2, 2, 1), (5, 0, 0, 0)], 16, upload=False)
    inf = seg.info()
    # the padded layout reaches sample b through stride_b: every first row is 0
    assert inf.packed == 0 and inf.total_rows == 2 * 16 and seg.offsets == [0, 0] and seg.rows == [16, 16]


def test_packed_rejects_bad_samples():
    with pytest.raises(jt.HiaError):
        jt.hia_segments_build_packed([(3, 2, 0, 1)], upload=False)
    with pytest.raises(jt.HiaError):
        jt.hia_segments_build_packed([(-1, 0, 0, 1)], upload=False)
