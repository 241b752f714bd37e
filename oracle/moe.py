"""fp64 CPU oracle for the MoE feed-forward of a HunyuanImage-3.0 decoder block:
the router (softmax over all experts, top-k, renormalized), the routed SwiGLU
experts with fused [up; gate] projections, and the shared expert.

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` and the CPU legs of
``bench.py``.  The product path (``joint_text_image_b200``) never imports it,
and it shares no code, table or constant with the CUDA path.

Sources (page title, section / API item):
  - HunyuanImage 3.0 Technical Report summary, 3.1.1 Architecture: 64
    experts, 8 activated per token, plus one shared MLP.
  - nemo_automodel ... hunyuan_image3.model, build_moe_config: softmax over
    all experts, top-k, renormalized, one shared expert; HunyuanImage3Block:
    routed experts (MoE) plus the fused shared expert, added;
    ``_keep_in_fp32_modules_strict = ['mlp.gate']`` (the router weight is
    fp32).
  - "HunyuanImage-3.0" model-coverage page, Train: the router is kept in fp32
    (gate_precision: float32); the state-dict adapter converts fused
    [up; gate] expert projections to grouped experts.
  - nemo_automodel ... hunyuan_image3.layers, HunyuanSharedMLP: a SwiGLU MLP
    whose gate_and_up_proj holds [up; gate], up first; forward maps
    [tokens, hidden] to [tokens, hidden].

Readings where the pages are silent (each is listed in the design notes):
  - SwiGLU: a = silu(gate) * up with silu(z) = z / (1 + exp(-z)), then the
    down projection; routed experts use the same fused [up; gate] layout as
    the shared one (the coverage page's adapter turns the release's fused
    up/gate expert weights into grouped experts);
  - top-k ties: the lower expert index is taken first;
  - the routing weights multiply each selected expert's output and the
    shared expert's output is added with weight 1;
  - no bias anywhere (the pages' layers give none for these projections);
  - everything here is fp64: x, the weights and every intermediate (the
    kernels' bf16 roundings are covered by the parity tolerances, and their
    fp32 router is compared allowing near-ties to break either way).

Weight layout used by both sides: w13 [E + 1, 2I, H] (rows [0, I) up, rows
[I, 2I) gate), w2 [E + 1, H, I]; index E is the shared expert.  wg [E, H].
"""
from __future__ import annotations

import numpy as np


def silu(z):
    """silu(z) = z * sigmoid(z) (HunyuanSharedMLP: SwiGLU)."""
    return z / (1.0 + np.exp(-z))


def router(x, wg, topk):
    """Routing of every token (build_moe_config: softmax over all experts,
    top-k, renormalized; the router in fp32 per the coverage page -- here in
    fp64).  x [T, H], wg [E, H].  Returns ids [T, topk] (descending weight,
    ties to the lower expert index), weights [T, topk] summing to 1 per token,
    probs [T, E] and logits [T, E]."""
    x = np.asarray(x, dtype=np.float64)
    wg = np.asarray(wg, dtype=np.float64)
    logits = x @ wg.T
    z = logits - logits.max(axis=1, keepdims=True)
    e = np.exp(z)
    probs = e / e.sum(axis=1, keepdims=True)
    # stable sort of -probs: equal probabilities keep increasing expert index
    order = np.argsort(-probs, axis=1, kind="stable")
    ids = order[:, :topk]
    top = np.take_along_axis(probs, ids, axis=1)
    weights = top / top.sum(axis=1, keepdims=True)
    return ids, weights, probs, logits


def expert(x, w13, w2):
    """One SwiGLU expert on rows x [n, H]: [up; gate] = x W13^T (up first),
    a = silu(gate) * up, y = a W2^T (HunyuanSharedMLP)."""
    x = np.asarray(x, dtype=np.float64)
    w13 = np.asarray(w13, dtype=np.float64)
    w2 = np.asarray(w2, dtype=np.float64)
    I = w13.shape[0] // 2
    h = x @ w13.T
    up, gate = h[:, :I], h[:, I:]
    return (silu(gate) * up) @ w2.T


def moe_fwd(x, wg, w13, w2, topk, ids=None, tokens=None):
    """The MoE feed-forward of one block: out = sum_k weight_k * expert_{e_k}(x)
    + shared(x) (HunyuanImage3Block: routed experts plus the shared expert).

    x [T, H]; wg [E, H]; w13 [E + 1, 2I, H], w2 [E + 1, H, I] (index E = the
    shared expert).  ids: an optional [T, topk] selection to use instead of
    this oracle's own top-k (a selection that differs only by breaking a
    near-tie the other way); the weights are then the oracle's probabilities of
    those experts, renormalized.  tokens: optional row subset (indices into
    T); the result has one row per selected token.
    Returns (out [n, H], ids [n, topk], weights [n, topk])."""
    x = np.asarray(x, dtype=np.float64)
    rows = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens)
    xs = x[rows]
    E = np.asarray(wg).shape[0]
    own_ids, _, probs, _ = router(xs, wg, topk)
    if ids is None:
        sel = own_ids
    else:
        sel = np.asarray(ids)[rows] if tokens is not None else np.asarray(ids)
    top = np.take_along_axis(probs, sel, axis=1)
    weights = top / top.sum(axis=1, keepdims=True)
    out = expert(xs, w13[E], w2[E])  # the shared expert, weight 1
    for e in range(E):
        t_idx, k_idx = np.nonzero(sel == e)
        if t_idx.size == 0:
            continue
        y = expert(xs[t_idx], w13[e], w2[e])
        np.add.at(out, t_idx, weights[t_idx, k_idx][:, None] * y)
    return out, sel, weights
