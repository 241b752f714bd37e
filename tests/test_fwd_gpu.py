"""GPU parity of the RoPE tables and the forward against the fp64 oracle."""
import numpy as np
import pytest
import torch

import joint_text_image_b200 as jt
from joint_text_image_b200 import synth
from helpers import check_fwd, run_fwd, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "needs a GPU"
    jt.lib()


@pytest.mark.parametrize("name", ["tiny", "256px", "mixed"])
def test_rope_tables_within_one_ulp(oracle_mod, name):
    wl = synth.workload(name)
    seg = jt.hia_segments_build(wl.samples, wl.S)
    c, s = jt.hia_rope2d_tables(seg, wl.D, wl.base)
    cr, sr = oracle_mod.rope_tables(wl.samples, wl.S, wl.D, wl.base)
    for got, ref in ((c, cr), (s, sr)):
        got = got.cpu().numpy()
        ref32 = ref.astype(np.float32)
        ulp = np.spacing(np.abs(ref32))
        assert np.all(np.abs(got.astype(np.float64) - ref32.astype(np.float64)) <= ulp)


def test_rope_tables_text_only_bitwise_1d():
    """A text-only sample's tables equal the diagonal (1D) rows bit for bit."""
    S, D = 300, 128
    seg = jt.hia_segments_build([(S, 0, 0, 0), (40, 8, 8, 2)], S)
    c, s = jt.hia_rope2d_tables(seg, D)
    c, s = c.cpu(), s.cpu()
    assert torch.equal(c[1, :40], c[0, :40]) and torch.equal(s[1, 106:], s[0, 106:])
    assert torch.equal(c[1, 106:], c[0, 106:])


@pytest.mark.parametrize("name", ["tiny", "256px"])
def test_fwd_full_parity(oracle_mod, name):
    wl = synth.workload(name)
    (q, k, v), o, lse = run_fwd(wl)
    check_fwd(oracle_mod, wl, q, k, v, o, lse)


@pytest.mark.parametrize("name", ["1024px", "mixed"])
def test_fwd_sampled_parity_full_size(oracle_mod, name):
    wl = synth.workload(name)
    (q, k, v), o, lse = run_fwd(wl)
    rows = sample_rows(wl, 4)
    check_fwd(oracle_mod, wl, q, k, v, o, lse, rows=rows)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))


def test_fwd_text_only_equals_causal_1d():
    """The text-only 2048-token row of the mixed batch: causal attention with 1D RoPE,
    checked against torch SDPA (is_causal) on the library's own rotated inputs."""
    wl = synth.custom([(300, 0, 0, 0)], 4, 2, 128, name="text_only")
    (q, k, v), o, _ = run_fwd(wl)
    seg = jt.hia_segments_build(wl.samples, wl.S)
    c, s = jt.hia_rope2d_tables(seg, wl.D)
    c, s = c.cpu().double()[:, :, None], s.cpu().double()[:, :, None]
    rot = lambda x: x * c + torch.cat([-x[..., 64:], x[..., :64]], -1) * s
    qr, kr = rot(q.double()), rot(k.double())
    ref = torch.nn.functional.scaled_dot_product_attention(
        qr.permute(0, 2, 1, 3), kr.repeat_interleave(2, 2).permute(0, 2, 1, 3),
        v.double().repeat_interleave(2, 2).permute(0, 2, 1, 3), is_causal=True).permute(0, 2, 1, 3)
    assert np.abs(o - ref.numpy()).max() < 2e-2


@pytest.mark.parametrize("samples,S,Hq,Hkv,D", [
    ([(5, 3, 3, 2)], 19, 4, 1, 64),                     # S < one tile
    ([(100, 10, 13, 7), (0, 0, 0, 0), (250, 0, 0, 0), (0, 16, 16, 2)], 261, 6, 2, 128),  # odd g, empty row, ragged
    ([(129, 1, 127, 1), (0, 11, 23, 0)], 300, 2, 2, 128),  # g = 1, image first, ragged tail
    ([(1, 0, 0, 0)], 1, 2, 1, 64),                      # S = 1
    ([(64, 8, 16, 0)], 256, 8, 2, 128),                 # exact tiles
])
def test_fwd_edge_cases(oracle_mod, samples, S, Hq, Hkv, D):
    wl = synth.custom(samples, Hq, Hkv, D, S=S)
    (q, k, v), o, lse = run_fwd(wl, seed=3)
    check_fwd(oracle_mod, wl, q, k, v, o, lse)
    for b, (P, h, w, s) in enumerate(samples):
        if P + h * w + s == 0:
            assert np.all(o[b] == 0) and np.all(np.isneginf(lse[b]))


def test_fwd_fused_qkv_layout(oracle_mod):
    """q, k, v as strided views of one fused [B,S,Hkv,g+2,D] projection output."""
    wl = synth.custom([(40, 6, 6, 3), (10, 4, 9, 0)], 8, 2, 128)
    g = 4
    gen = torch.Generator().manual_seed(5)
    fused = torch.randn(wl.B, wl.S, wl.Hkv, g + 2, wl.D, generator=gen).to(torch.bfloat16)
    q5, k4, v4 = fused[:, :, :, :g], fused[:, :, :, g], fused[:, :, :, g + 1]
    fc = fused.cuda()
    seg = jt.hia_segments_build(wl.samples, wl.S)
    c, s = jt.hia_rope2d_tables(seg, wl.D)
    o, lse = jt.hia_attn_fwd(seg, fc[:, :, :, :g], fc[:, :, :, g], fc[:, :, :, g + 1], c, s)
    torch.cuda.synchronize()
    q = q5.reshape(wl.B, wl.S, wl.Hq, wl.D)
    check_fwd(oracle_mod, wl, q, k4, v4, o.float().cpu().numpy(), lse.cpu().numpy())


def test_bounded_wait_expires_and_reports():
    assert jt.hia_get_device_status() == 0
    jt.hia_debug_wait_timeout(2_000_000)  # 2 ms, nothing ever arrives
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 4
    assert jt.hia_get_device_status() == 0  # read-and-clear
    # the context is still usable
    wl = synth.workload("tiny")
    run_fwd(wl)


def test_fma_exp2_matches_exp2():
    """The FMA-pipe exponential used for part of the softmax: relative error
    <= 1e-4 against 2^x over the range the softmax feeds it (x <= 8 after the
    lazy rescale), and at most 2^-125 (about 2.4e-38) for x <= -125, -inf
    included."""
    x = torch.cat([torch.linspace(-125.0, 8.0, 200001),
                   torch.tensor([-125.5, -126.0, -127.0, -200.0, -float("inf"), -0.0, 1e-8, -1e-8, 7.9999995])])
    xd = x.cuda()
    y = torch.empty_like(xd)
    assert jt.lib().hia_debug_exp2(xd.data_ptr(), y.data_ptr(), x.numel(), jt._stream()) == 0
    torch.cuda.synchronize()
    ref = torch.exp2(x.double())
    got = y.cpu().double()
    assert torch.isfinite(got).all()
    fin = x >= -125.0
    rel = ((got[fin] - ref[fin]) / ref[fin]).abs()
    assert rel.max() <= 1e-4, rel.max()
    low = got[~fin]
    assert ((low >= 0) & (low <= 2.0 ** -125 * 1.0001)).all(), low
