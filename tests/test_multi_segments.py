"""CPU tests of the segment descriptor for samples with several images: the
library's mask, pair count and tile classification against the oracle's
literal rule (technical report summary 3.1.2)."""
import numpy as np
import pytest

import joint_text_image_b200 as jt
from joint_text_image_b200 import build as jbuild

from test_packed_segments import brute_classes


@pytest.fixture(scope="module", autouse=True)
def built():
    jbuild.build()


def length(sample):
    images, suffix = sample
    return sum(t + h * w for t, h, w in images) + suffix


def random_batch(rng, B, big=False):
    out = []
    for _ in range(B):
        m = int(rng.integers(0, 4))
        if big:
            images = [(int(rng.integers(0, 200)), int(rng.integers(1, 17)), int(rng.integers(1, 17))) for _ in range(m)]
            suffix = int(rng.integers(0, 50))
        else:
            images = [(int(rng.integers(0, 5)), int(rng.integers(1, 5)), int(rng.integers(1, 5))) for _ in range(m)]
            suffix = int(rng.integers(0, 5))
        out.append((images, suffix))
    return out


@pytest.mark.parametrize("seed", range(6))
def test_multi_mask_and_pairs_bit_exact(oracle_mod, seed):
    rng = np.random.default_rng(40 + seed)
    samples = random_batch(rng, 4, big=seed >= 3)
    S = max(length(x) for x in samples) + int(rng.integers(0, 40))
    seg = jt.hia_segments_build_multi(samples, S, upload=False)
    ref = oracle_mod.mask(samples, S)
    assert np.array_equal(seg.mask(), ref)
    assert seg.info().visible_pairs == int(ref.sum())


@pytest.mark.parametrize("seed", range(4))
def test_multi_tile_classes(oracle_mod, seed):
    rng = np.random.default_rng(50 + seed)
    samples = random_batch(rng, 3, big=True)
    for packed in (False, True):
        S = max(length(x) for x in samples) + (0 if packed else 37)
        seg = jt.hia_segments_build_multi(samples, S, packed=packed, upload=False)
        inf = seg.info()
        m = oracle_mod.mask(samples, inf.S).astype(bool)
        cls = seg.tile_classes()
        for b, x in enumerate(samples):
            rows = length(x) if packed else inf.S
            want = brute_classes(m[b], rows, inf.S, inf.fwd_q_tiles, inf.fwd_kv_tiles)
            got = cls[b].copy()
            got[(got == 0) | (got == 3)] = 0
            assert np.array_equal(got, want), (packed, b)
        if packed:
            assert inf.visible_pairs == sum(int(m[b, :length(x)].sum()) for b, x in enumerate(samples))


def test_one_image_multi_form_matches_builder():
    canon = [(100, 10, 13, 7), (0, 0, 0, 0), (250, 0, 0, 0), (0, 16, 16, 2)]
    multi = [([(100, 10, 13)], 7), ([], 0), ([], 250), ([(0, 16, 16)], 2)]
    a = jt.hia_segments_build(canon, 600, upload=False)
    b = jt.hia_segments_build_multi(multi, 600, upload=False)
    assert np.array_equal(a.mask(), b.mask()) and np.array_equal(a.tile_classes(), b.tile_classes())
    ia, ib = a.info(), b.info()
    for f in ("visible_pairs", "fwd_tiles_full", "fwd_tiles_partial", "fwd_tiles_skipped"):
        assert getattr(ia, f) == getattr(ib, f), f


def test_context_image_tiles_are_skipped():
    """Query tiles after a 16x16 context image skip its key tiles."""
    seg = jt.hia_segments_build_multi([([(0, 16, 16), (128, 8, 8)], 64)], 512, upload=False)
    cls = seg.tile_classes()[0]
    # rows 256..383 (the text after the first image): its two key tiles are hidden
    assert list(cls[2, :2]) == [0, 0] and cls[2, 2] in (1, 2)


def test_multi_refuses_bad_images():
    with pytest.raises(jt.HiaError):
        jt.hia_segments_build_multi([([(1, 0, 2)], 1)], 16, upload=False)
    with pytest.raises(jt.HiaError):
        jt.hia_segments_build_multi([([(1, 2, 2)], 1)], 5, upload=False)
