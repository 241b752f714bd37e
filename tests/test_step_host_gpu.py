"""GPU: one training step from host buffers (hia_attn_step_host) against the
device-pointer entry points and the fp64 oracle."""
import numpy as np
import pytest
import torch

import joint_text_image_b200 as jt
from joint_text_image_b200 import synth
from helpers import check_bwd, check_fwd, gpu_tables

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "needs a GPU"
    jt.lib()


def host_outputs(wl, pin):
    B, S, Hq, Hkv, D = wl.B, wl.S, wl.Hq, wl.Hkv, wl.D
    mk = lambda shape, dt: torch.empty(shape, dtype=dt, pin_memory=pin)
    return (mk((B, S, Hq, D), torch.bfloat16), mk((B, Hq, S), torch.float32), mk((B, S, Hq, D), torch.bfloat16),
            mk((B, S, Hkv, D), torch.bfloat16), mk((B, S, Hkv, D), torch.bfloat16))


def device_reference(wl, seg, q, k, v, do):
    c, s = gpu_tables(seg, wl.D, wl.base)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = jt.hia_attn_fwd(seg, qd, kd, vd, c, s, wl.scale)
    dq, dk, dv = jt.hia_attn_bwd(seg, qd, kd, vd, c, s, o, lse, dod, wl.scale)
    torch.cuda.synchronize()
    return [t.cpu() for t in (o, lse, dq, dk, dv)]


@pytest.mark.parametrize("name,pin", [("tiny", True), ("tiny", False), ("256px", True)])
def test_step_host_matches_device_api(oracle_mod, name, pin):
    wl = synth.workload(name)
    q, k, v, do = synth.tensors(wl, 0, grad=True)
    if pin:
        q, k, v, do = (t.pin_memory() for t in (q, k, v, do))
    seg = jt.hia_segments_build(wl.samples, wl.S)
    step = jt.hia_step_create(seg, wl.Hq, wl.Hkv, wl.D, wl.base)
    o, lse, dq, dk, dv = host_outputs(wl, pin)
    jt.hia_attn_step_host(step, q, k, v, do, o, lse, dq, dk, dv, scale=wl.scale)
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 0
    ro, rlse, rdq, rdk, rdv = device_reference(wl, seg, q, k, v, do)
    # same kernels on the same inputs: o, lse, dk, dv are bitwise equal; dq
    # differs only by the order of its fp32 reductions across CTAs
    assert torch.equal(o, ro) and torch.equal(lse, rlse)
    assert torch.equal(dk, rdk) and torch.equal(dv, rdv)
    rel = (dq.float() - rdq.float()).norm() / rdq.float().norm()
    assert rel <= 1e-3, rel
    check_fwd(oracle_mod, wl, q, k, v, o.float().numpy(), lse.numpy())
    check_bwd(oracle_mod, wl, (q, k, v, do), (dq.float().numpy(), dk.float().numpy(), dv.float().numpy()))


def test_step_host_two_streams_overlap():
    """Two steps on two streams (one step's copies under the other's kernels)
    give the same outputs as one step at a time."""
    wl = synth.workload("256px")
    seg = jt.hia_segments_build(wl.samples, wl.S)
    ins = [tuple(t.pin_memory() for t in synth.tensors(wl, seed, grad=True)) for seed in (0, 1)]
    steps = [jt.hia_step_create(seg, wl.Hq, wl.Hkv, wl.D, wl.base) for _ in range(2)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [host_outputs(wl, True) for _ in range(2)]
    for _ in range(3):
        for i in range(2):
            jt.hia_attn_step_host(steps[i], *ins[i], *outs[i], scale=wl.scale, stream=streams[i])
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 0
    for i in range(2):
        ref = host_outputs(wl, False)
        jt.hia_attn_step_host(steps[0], *ins[i], *ref, scale=wl.scale)
        torch.cuda.synchronize()
        for j, (a, b) in enumerate(zip(outs[i], ref)):
            if j == 2:  # dq: reduction order
                assert (a.float() - b.float()).norm() <= 1e-3 * b.float().norm()
            else:
                assert torch.equal(a, b)


def test_step_host_rejects_bad_buffers():
    wl = synth.workload("tiny")
    seg = jt.hia_segments_build(wl.samples, wl.S)
    step = jt.hia_step_create(seg, wl.Hq, wl.Hkv, wl.D, wl.base)
    q, k, v, do = synth.tensors(wl, 0, grad=True)
    o, lse, dq, dk, dv = host_outputs(wl, False)
    with pytest.raises(ValueError):
        jt.hia_attn_step_host(step, q[:, :-1].contiguous(), k, v, do, o, lse, dq, dk, dv)
    with pytest.raises(ValueError):
        jt.hia_attn_step_host(step, q.cuda(), k, v, do, o, lse, dq, dk, dv)
    with pytest.raises(jt.HiaError):
        jt.hia_step_create(seg, wl.Hq, wl.Hkv, 96, wl.base)
    # the C entry point refuses null host pointers
    rc = jt.lib().hia_attn_step_host(step.handle, None, k.data_ptr(), v.data_ptr(), do.data_ptr(), 0.125,
                                     o.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                     jt._stream())
    assert rc == 1  # HIA_ERR_INVALID_ARG
