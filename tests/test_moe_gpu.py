"""GPU parity of the MoE feed-forward (hia_moe_fwd) against the fp64 oracle
(oracle/moe.py) on the same seeded inputs.

Routing.  The kernels compute the router logits to fp32 precision (the pages
keep the router in fp32) and the oracle in fp64, so a token whose k-th and
(k+1)-th logits are closer than the fp32 error may be routed either way; both
are correct.  The chosen sets must therefore agree, except between experts
whose oracle logits lie within TIE_TOL of the k-th largest; such tokens are
rare (checked), and the output is then compared with the oracle evaluated on
the GPU's own (valid) choice.  The fp32 logits carry an error of about
sqrt(H) * 2^-24 * |x| |w| (tensor-core fp32 accumulation of exact products):
~1e-6 here; TIE_TOL = 1e-3 leaves a wide margin for the accumulation order.

Weights are the renormalized probabilities of the chosen experts: fp32
softmax against fp64, within 1e-5.

Output.  bf16 operands, fp32 accumulation; the SwiGLU product is rounded to
bf16 between the projections, each expert's output and the final sum are
rounded to bf16: each rounding is 2^-9 relative at most, about 1e-3 relative
in the Frobenius norm of a row.  Bound: relative Frobenius error 1e-2 per
token row and over the whole output (the same bound the attention gradients
use).
"""
import numpy as np
import pytest
import torch

import joint_text_image_b200 as jt
from joint_text_image_b200 import synth
from oracle import moe

pytestmark = pytest.mark.gpu

TIE_TOL, W_TOL, ROW_REL, ALL_REL = 1e-3, 1e-5, 1e-2, 1e-2


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    assert torch.cuda.is_available(), "needs a GPU"
    jt.lib()


def run(x, wg, w13, w2, topk, workspace=None):
    out, ids, w = jt.hia_moe_fwd(x.cuda(), wg.cuda(), w13.cuda(), w2.cuda(), topk, workspace=workspace)
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 0
    return out.float().cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()


def check(x, wg, w13, w2, topk, out, ids, w, tokens=None):
    """Routing, weights and output of the given token rows against the oracle.
    w13, w2: bf16 torch tensors, or objects giving one expert's fp64 weights
    per index."""
    rows = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens)
    xs = x.double().numpy()[rows]
    wgd = wg.double().numpy()
    ref_ids, _, probs, logits = moe.router(xs, wgd, topk)
    gi, gw = ids[rows], w[rows]
    E = wgd.shape[0]
    assert gi.min() >= 0 and gi.max() < E
    n_tie = 0
    for t in range(len(rows)):
        assert len(set(gi[t].tolist())) == topk, "an expert chosen twice"
        if set(gi[t].tolist()) != set(ref_ids[t].tolist()):
            kth = np.sort(logits[t])[::-1][topk - 1]
            for e in set(gi[t].tolist()) ^ set(ref_ids[t].tolist()):
                assert abs(logits[t, e] - kth) <= TIE_TOL, f"token {rows[t]}: expert {e} is not a near-tie"
            n_tie += 1
        # chosen in descending order (up to near-ties)
        assert np.all(np.diff(logits[t, gi[t]]) <= TIE_TOL)
    assert n_tie <= max(2, len(rows) // 500), f"{n_tie} near-tie tokens"
    p = np.take_along_axis(probs, gi, axis=1)
    np.testing.assert_allclose(gw, p / p.sum(axis=1, keepdims=True), rtol=0, atol=W_TOL)
    if isinstance(w13, torch.Tensor):
        w13, w2 = w13.double().numpy(), w2.double().numpy()
    ref, _, _ = moe.moe_fwd(x.double().numpy(), wgd, w13, w2, topk, ids=ids, tokens=rows)
    got = out[rows]
    assert np.all(np.isfinite(got))
    rel_rows = np.linalg.norm(got - ref, axis=1) / np.linalg.norm(ref, axis=1)
    rel_all = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel_rows.max() <= ROW_REL, f"worst row {rows[rel_rows.argmax()]}: {rel_rows.max():.3e}"
    assert rel_all <= ALL_REL, f"{rel_all:.3e}"
    print(f"[parity-moe] {len(rows)} tokens: rel {rel_all:.3e}, worst row {rel_rows.max():.3e}, "
          f"near-ties {n_tie}")
    return rel_all


def _weights_np(w13, w2):
    """The oracle reads weights expert by expert; keep bf16 torch tensors and
    convert one expert at a time to bound host memory."""
    class Lazy:
        def __init__(self, t):
            self.t = t

        def __getitem__(self, e):
            return self.t[e].double().numpy()
    return Lazy(w13), Lazy(w2)


@pytest.mark.parametrize("name", ["moe_tiny", "moe_mid"])
def test_moe_full_parity(name):
    mw = synth.moe_workload(name)
    x, wg, w13, w2 = synth.moe_tensors(mw, 0)
    out, ids, w = run(x, wg, w13, w2, mw.topk)
    check(x, wg, w13, w2, mw.topk, out, ids, w)


@pytest.mark.parametrize("T,H,I,E,topk", [
    (1, 256, 128, 8, 2),       # one token
    (5, 512, 256, 64, 8),      # most experts get no token
    (130, 256, 128, 4, 4),     # every expert chosen by every token
    (257, 256, 384, 5, 3),     # E not a multiple of 16, I three tiles
    (129, 768, 128, 16, 1),    # top-1: weight exactly 1
])
def test_moe_edge_shapes(T, H, I, E, topk):
    mw = synth.MoeWorkload("edge", T, H, I, E, topk)
    x, wg, w13, w2 = synth.moe_tensors(mw, 3)
    out, ids, w = run(x, wg, w13, w2, topk)
    check(x, wg, w13, w2, topk, out, ids, w)
    if topk == 1:
        assert np.all(w == 1.0)


@pytest.mark.parametrize("case", range(6))
def test_moe_random_shapes(case):
    """Seeded random sizes inside the supported range (H a multiple of 256, I
    of 128, 1 <= E <= 80, top-k up to min(E, 16), ragged token counts): routing,
    weights and output against the oracle."""
    rng = np.random.default_rng(300 + case)
    E = int(rng.integers(1, 81))
    topk = int(rng.integers(1, min(E, 16) + 1))
    mw = synth.MoeWorkload("random", int(rng.integers(1, 700)), 256 * int(rng.integers(1, 4)),
                           128 * int(rng.integers(1, 4)), E, topk)
    x, wg, w13, w2 = synth.moe_tensors(mw, 10 + case)
    out, ids, w = run(x, wg, w13, w2, mw.topk)
    check(x, wg, w13, w2, mw.topk, out, ids, w)


def test_moe_all_tokens_to_one_expert():
    """A router that sends every token to expert 3 (imbalance: one group of T
    rows, the others nearly empty)."""
    mw = synth.MoeWorkload("skew", 700, 256, 128, 16, 2)
    x, wg, w13, w2 = synth.moe_tensors(mw, 5)
    x = (x.float() + 2.0).to(torch.bfloat16)  # a component shared by every token
    wg = wg.clone()
    wg[3] = 4.0 / mw.H                        # logit_3 ~ 8 for every token
    out, ids, w = run(x, wg, w13, w2, mw.topk)
    assert np.all(ids[:, 0] == 3)
    check(x, wg, w13, w2, mw.topk, out, ids, w)


def test_moe_deterministic_and_workspace_garbage():
    """Two calls (the second with a workspace full of NaN bytes) give the same
    bits: the counters and padding rows are cleared by the call itself, and a
    row's result does not depend on its slot in the sorted buffers."""
    mw = synth.moe_workload("moe_mid")
    x, wg, w13, w2 = synth.moe_tensors(mw, 1)
    a = run(x, wg, w13, w2, mw.topk)
    ws = torch.full((jt.hia_moe_workspace_bytes(mw.T, mw.H, mw.I, mw.E, mw.topk),), 0xFF, dtype=torch.uint8,
                    device="cuda")
    b = run(x, wg, w13, w2, mw.topk, workspace=ws)
    c = run(x, wg, w13, w2, mw.topk, workspace=ws)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    for u, v in zip(a, c):
        assert np.array_equal(u, v)


def test_moe_full_size_sampled_tokens():
    """The benchmark's workload (the 1024px batch's 10,803 tokens, H = 4096,
    I = 3072, 64 experts, top-8): routing of every token checked against the
    fp64 router, the output on sampled tokens (first, last, random) against
    the oracle."""
    mw = synth.moe_workload("moe_1024px")
    x, wg, w13, w2 = synth.moe_tensors(mw, 0)
    out, ids, w = run(x, wg, w13, w2, mw.topk)
    rng = np.random.default_rng(0)
    rows = sorted({0, 1, 127, 128, mw.T - 1} | set(rng.integers(0, mw.T, 59).tolist()))
    L13, L2 = _weights_np(w13, w2)
    check(x, wg, L13, L2, mw.topk, out, ids, w, tokens=rows)
    # routing of every token (router only; cheap in fp64)
    ref_ids, _, _, logits = moe.router(x.double().numpy(), wg.double().numpy(), mw.topk)
    diff = np.nonzero(np.any(np.sort(ids, 1) != np.sort(ref_ids, 1), axis=1))[0]
    assert len(diff) <= mw.T // 500, f"{len(diff)} tokens routed differently"
    for t in diff:
        kth = np.sort(logits[t])[::-1][mw.topk - 1]
        for e in set(ids[t].tolist()) ^ set(ref_ids[t].tolist()):
            assert abs(logits[t, e] - kth) <= TIE_TOL
    # every expert's load: the tokens the GPU sent to it
    load = np.bincount(ids.ravel(), minlength=mw.E)
    assert load.sum() == mw.T * mw.topk
