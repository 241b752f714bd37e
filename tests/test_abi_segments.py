"""CPU tests of the C ABI: the library loads and exports every declared symbol;
the host segment builder is bit-exact against the oracle's literal mask."""
import os
import re

import numpy as np
import pytest

import joint_text_image_b200 as jt
from joint_text_image_b200 import build as jbuild
from joint_text_image_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    jbuild.build()


HEADERS = ("jointattn.h", "jointmoe.h")


def declared_symbols():
    names = set()
    for h in HEADERS:
        txt = open(os.path.join(ROOT, "include", h)).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        names.update(re.findall(r"\b(hia_\w+)\s*\(", txt))
    return sorted(names)


def test_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 14
    L = jt.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(jt.EXPORTED_SYMBOLS)


def test_nm_shows_symbols():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", jt.LIB_PATH], capture_output=True, text=True).stdout
    for n in declared_symbols():
        assert re.search(rf"\bT {n}\b", out), n


EDGE = [
    [(3, 2, 2, 1)], [(0, 0, 0, 0)], [(5, 0, 0, 0)], [(0, 3, 3, 0)], [(1, 1, 7, 0)], [(2, 7, 1, 3)],
    [(100, 10, 13, 7), (0, 0, 0, 0), (250, 0, 0, 0), (0, 16, 16, 2)],
]


@pytest.mark.parametrize("samples", EDGE)
def test_mask_bit_exact_edge_cases(oracle_mod, samples):
    S = max(p + h * w + s for p, h, w, s in samples) + 3
    seg = jt.hia_segments_build(samples, S, upload=False)
    assert np.array_equal(seg.mask(), oracle_mod.mask(samples, S))


@pytest.mark.parametrize("name", synth.WORKLOADS)
def test_mask_bit_exact_workloads(oracle_mod, name):
    wl = synth.workload(name)
    seg = jt.hia_segments_build(wl.samples, wl.S, upload=False)
    ref = oracle_mod.mask(wl.samples, wl.S)
    # row bound: the last visible key of each row of the literal mask
    S = wl.S
    last = S - 1 - np.argmax(ref[:, :, ::-1], axis=2)
    e_ref = np.where(ref.any(axis=2), last, -1).astype(np.int64)
    assert np.array_equal(seg.row_bound(), e_ref)
    if wl.S <= 3000:
        assert np.array_equal(seg.mask(), ref)
    assert seg.info().visible_pairs == int(ref.sum(dtype=np.int64))


@pytest.mark.parametrize("name", ["tiny", "256px", "mixed"])
def test_tile_classes_consistent_with_mask(oracle_mod, name):
    wl = synth.workload(name)
    seg = jt.hia_segments_build(wl.samples, wl.S, upload=False)
    cls = seg.tile_classes()
    m = oracle_mod.mask(wl.samples, wl.S)
    S = wl.S
    for b in range(wl.B):
        P, h, w, sfx = wl.samples[b]
        L = P + h * w + sfx
        for qt in range(cls.shape[1]):
            for kt in range(cls.shape[2]):
                blk = m[b, qt * 128:min(S, qt * 128 + 128), kt * 128:min(S, kt * 128 + 128)]
                c = cls[b, qt, kt]
                if c == 1:
                    assert blk.all() and kt * 128 + 128 <= S
                elif c in (0, 3):
                    assert not blk.any()
                    assert (c == 3) == (kt * 128 >= L)
                else:
                    assert c == 2
                    assert blk.any() and (not blk.all() or kt * 128 + 128 > S)
    inf = seg.info()
    assert inf.fwd_tiles_full + inf.fwd_tiles_partial + inf.fwd_tiles_skipped == wl.B * inf.fwd_q_tiles ** 2


@pytest.mark.parametrize("bad", [
    ([(-1, 0, 0, 0)], 4), ([(2, 3, 0, 0)], 8), ([(2, 2, 2, 0)], 5), ([(0, 0, 0, 1)], -1),
])
def test_bad_geometry_rejected(bad):
    samples, S = bad
    with pytest.raises(jt.HiaError) as ei:
        jt.hia_segments_build(samples, S, upload=False)
    assert ei.value.code == 1


def test_fwd_rejects_unsupported_without_launch():
    """Argument checks run on the host before any CUDA call."""
    import ctypes
    seg = jt.hia_segments_build([(4, 2, 2, 1)], 9, upload=False)
    L = jt.lib()
    T = jt._Tensor
    z = T(None, 0, 0, 0, 0)
    # head_dim 96 unsupported; Hq % Hkv != 0 unsupported; segments not on device
    assert L.hia_attn_fwd(seg.handle, 4, 1, 96, z, z, z, None, None, 1.0, z, None, None, 0, None) == 2
    assert L.hia_attn_fwd(seg.handle, 3, 2, 128, z, z, z, None, None, 1.0, z, None, None, 0, None) == 2
    buf = ctypes.create_string_buffer(64)
    p = ctypes.addressof(buf) + (-ctypes.addressof(buf)) % 16
    assert L.hia_attn_fwd(seg.handle, 4, 1, 64, z, z, z, p, p, 1.0, z, None, None, 0, None) == 5
    assert L.hia_rope2d_tables(seg.handle, 63, 10000.0, p, p, None) == 1
    assert L.hia_debug_wait_timeout(0, None) == 1


@pytest.mark.parametrize("dims", [
    (100, 300, 128, 8, 2),     # H not a multiple of 256
    (100, 256, 100, 8, 2),     # I not a multiple of 128
    (100, 256, 128, 81, 2),    # E above 80
    (100, 256, 128, 8, 9),     # topk above E
    (100, 256, 128, 64, 17),   # topk above 16
    (-1, 256, 128, 8, 2),      # negative T
    (100, 256, 128, 0, 1),     # no routed expert
])
def test_moe_bad_dims_rejected(dims):
    """Host-side validation of the MoE sizes: no workspace size, and the
    forward refuses before anything is launched (null pointers are never
    reached)."""
    import ctypes
    assert jt.hia_moe_workspace_bytes(*dims) == 0
    d = jt._MoeDims(*dims)
    assert jt.lib().hia_moe_fwd(ctypes.byref(d), *([None] * 8), 0, None) == 1


def test_moe_workspace_size_and_empty_batch():
    import ctypes
    assert jt.hia_moe_workspace_bytes(10803, 4096, 3072, 64, 8) > 0
    # T = 0: nothing to do, no pointer needed
    d = jt._MoeDims(0, 256, 128, 8, 2)
    assert jt.lib().hia_moe_fwd(ctypes.byref(d), *([None] * 8), 0, None) == 0


def test_bwd_split_units_and_mode():
    """The descriptor's split schedule: kv tiles within 10% of the longest
    query range; the mode setter refuses unknown modes."""
    seg = jt.hia_segments_build(synth.workload("1024px_bwd").samples, synth.workload("1024px_bwd").S,
                                upload=False)
    assert seg.info().bwd_split_units > 0
    assert seg.info().bwd_split_units < seg.info().bwd_kv_tiles
    for mode in (0, 1, 2):
        seg.set_bwd_split(mode)
    with pytest.raises(jt.HiaError):
        seg.set_bwd_split(3)
    tiny = jt.hia_segments_build(synth.workload("tiny").samples, synth.workload("tiny").S, upload=False)
    assert tiny.info().bwd_split_units == 0  # one query range of 2 tiles: nothing worth splitting
