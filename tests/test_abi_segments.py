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
    """The descriptor's split schedules cut some kv tiles (those within 15% of
    the longest query range), never all; the mode setter takes the six modes
    and refuses others."""
    seg = jt.hia_segments_build(synth.workload("1024px_bwd").samples, synth.workload("1024px_bwd").S,
                                upload=False)
    assert seg.info().bwd_split_units > 0
    assert seg.info().bwd_split_units < seg.info().bwd_kv_tiles
    for mode in range(6):
        seg.set_bwd_split(mode)
    for bad in (-1, 6):
        with pytest.raises(jt.HiaError):
            seg.set_bwd_split(bad)
    tiny = jt.hia_segments_build(synth.workload("tiny").samples, synth.workload("tiny").S, upload=False)
    assert tiny.info().bwd_split_units == 0  # one query range of 2 tiles: nothing worth splitting
    assert len(tiny.bwd_schedules()) == 1


def _schedule_layouts():
    wl = synth.workload("1024px_bwd")
    yield "1024px_bwd", jt.hia_segments_build(wl.samples, wl.S, upload=False)
    wl = synth.workload("mixed")
    yield "mixed", jt.hia_segments_build(wl.samples, wl.S, upload=False)
    yield "mixed packed", jt.hia_segments_build_packed(wl.samples, upload=False)
    wl = synth.workload("multi_image")
    yield "multi_image", jt.hia_segments_build_multi(wl.samples, wl.S, upload=False)


@pytest.mark.parametrize("which", [0, 1, 2, 3])
def test_bwd_schedules_cover_every_query_range_once(which):
    """Every backward schedule covers each (sample, kv tile) query range of
    the whole schedule exactly once: unsplit, or cut into `parts` consecutive
    sub-ranges of at least two query tiles (parts 0 .. parts-1) that share a
    slot; slots are 0 .. n-1; entries run heaviest first; the split tiles are
    exactly those at or above the schedule's threshold."""
    name, seg = list(_schedule_layouts())[which]
    sch = seg.bwd_schedules()
    assert sch[0][0] == 1 and (sch[0][1][:, 4] == -1).all() and (sch[0][1][:, 6] == 1).all()
    whole = {(int(e[0]), int(e[1])): (int(e[2]), int(e[3])) for e in sch[0][1]}
    assert len(whole) == len(sch[0][1])
    longest = max(hi - lo for lo, hi in whole.values())
    seen_parts = set()
    for parts, ent in sch:
        cost = ent[:, 3] - ent[:, 2]
        assert (np.diff(cost) <= 0).all(), name  # heaviest first
        assert (ent[:, 7] == 0).all()
        got = {}
        slots = {}
        for e in ent:
            b, kt, lo, hi, slot, part, p = (int(x) for x in e[:7])
            if slot < 0:
                assert part == 0 and p == 1
                assert (b, kt) not in got
                got[(b, kt)] = [(lo, hi)]
            else:
                assert p == parts and 0 <= part < parts and hi - lo >= 2
                slots.setdefault(slot, set()).add((b, kt))
                got.setdefault((b, kt), []).append((part, lo, hi))
        assert set(got) == set(whole)
        split = set()
        for key, rs in got.items():
            if len(rs) == 1 and len(rs[0]) == 2:
                assert rs[0] == whole[key]
                continue
            split.add(key)
            rs = sorted(rs)
            assert [r[0] for r in rs] == list(range(parts))
            assert rs[0][1] == whole[key][0] and rs[-1][2] == whole[key][1]
            assert all(rs[i][2] == rs[i + 1][1] for i in range(parts - 1))
        assert sorted(slots) == list(range(len(slots))) and all(len(v) == 1 for v in slots.values())
        if parts > 1:
            assert split, name
            # a threshold: every split tile is at least as long as every unsplit tile of 2 * parts or more
            shortest_split = min(whole[k][1] - whole[k][0] for k in split)
            assert all(whole[k][1] - whole[k][0] < shortest_split for k in whole
                       if k not in split and whole[k][1] - whole[k][0] >= 2 * parts)
            assert 100 * shortest_split >= 85 * longest
            seen_parts.add(parts)
    assert seen_parts == {2, 3, 4}


def _makespan(entries, Hkv, g, n_sm):
    """Greedy list scheduling: entries in order, each as Hkv CTAs, each CTA on
    the SM that frees first; a CTA costs its query tiles * g + 9, a part of a
    split kv tile its query tiles * g * 1.2 + 9, and 22.5 more for the last
    part."""
    import heapq
    sms = [0.0] * n_sm
    span = 0.0
    for e in entries:
        it = float(e[3] - e[2]) * g
        c = it * 1.2 + 9.0 + (22.5 if e[5] == e[6] - 1 else 0.0) if e[4] >= 0 else it + 9.0
        for _ in range(Hkv):
            t = heapq.heappop(sms) + c
            heapq.heappush(sms, t)
            span = max(span, t)
    return span


@pytest.mark.parametrize("which", [0, 1, 3])
def test_bwd_choice_follows_the_estimate(which):
    """The schedule a launch takes: AUTO the one whose list-scheduling
    estimate finishes first (ties to the earlier), NEVER the whole one, ALWAYS
    the best split one, PARTS_k the best one with k parts."""
    name, seg = list(_schedule_layouts())[which]
    sch = seg.bwd_schedules()
    for Hkv, g, n_sm in ((8, 4, 148), (2, 16, 132), (1, 1, 8)):
        spans = [_makespan(e, Hkv, g, n_sm) for _, e in sch]
        def best(admit):
            idx = [i for i in range(len(sch)) if admit(sch[i][0])]
            return min(idx, key=lambda i: (spans[i], i)) if idx else 0
        expect = {0: best(lambda p: True), 1: 0, 2: best(lambda p: p > 1),
                  3: best(lambda p: p == 2), 4: best(lambda p: p == 3), 5: best(lambda p: p == 4)}
        for mode, want in expect.items():
            seg.set_bwd_split(mode)
            assert seg.bwd_choice(Hkv, g, n_sm) == want, (name, mode, Hkv, g, n_sm)
    seg.set_bwd_split(0)


def test_bwd_workspace_sized_for_the_chosen_schedule():
    """The backward workspace holds the fp32 dK/dV partials of the schedule a
    launch takes (for every part, kv head and split tile a 128 x D block for
    dK and one for dV, plus a ticket per split tile and kv head), so it grows
    with the forced part count and equals the unsplit size plus that much."""
    wl = synth.workload("1024px_bwd")
    seg = jt.hia_segments_build(wl.samples, wl.S, upload=False)
    Hq, Hkv, D = wl.Hq, wl.Hkv, wl.D
    align = lambda n: (n + 255) // 256 * 256
    seg.set_bwd_split(1)
    base = jt.hia_attn_bwd_workspace_bytes(seg, Hq, Hkv, D)
    sch = seg.bwd_schedules()
    sizes = {}
    for mode in (3, 4, 5):
        seg.set_bwd_split(mode)
        parts, ent = sch[seg.bwd_choice(Hkv, Hq // Hkv, 148)]
        assert parts == mode - 1
        slots = len({int(e[4]) for e in ent if e[4] >= 0})
        got = jt.hia_attn_bwd_workspace_bytes(seg, Hq, Hkv, D)
        assert got == base + align(slots * Hkv * parts * 2 * 128 * D * 4) + align(slots * Hkv * 4)
        sizes[mode] = got
    assert base < sizes[3] and base < sizes[5]
    seg.set_bwd_split(0)
