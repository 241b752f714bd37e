"""Shared test plumbing: run the CUDA path and the oracle on the same seeded inputs."""
import numpy as np
import torch

import joint_text_image_b200 as jt
from joint_text_image_b200 import synth

# Tolerances against the fp64 oracle on identical bf16 inputs: O max-abs 2e-2
# and mean-abs 2e-3, dQ/dK/dV relative Frobenius 1e-2 (the stated targets).
# LSE has no stated target; its bound comes from the arithmetic: the MMA
# operands are the RoPE-rotated q, k rounded to bf16 (relative error <= 2^-9
# each), so a scaled score s = scale * q_r . k_r carries an error of about
# scale * 2^-9 * sqrt(2 * sum_i (q_i k_i)^2) (independent roundings), i.e.
# std ~1.6e-3 for N(0,1) inputs at D = 128, and LSE, a softmax-weighted mean
# of the score errors, stays within max_k |ds_k|: ~4.5 std over the 10^6-10^7
# rows checked gives 7e-3, so max-abs 1e-2 and mean-abs 1e-3.
O_MAX, O_MEAN, LSE_MAX, LSE_MEAN, GRAD_REL = 2e-2, 2e-3, 1e-2, 1e-3, 1e-2
# The relative Frobenius bound above is over whole tensors, where an error
# confined to one tile (a tail tile, a partial image edge) adds only a small
# share of the norm.  Every block is therefore also checked on its own: each
# 128-row block of dq (per sample and kv-head group of g heads) and each
# 128-key block of dk and dv (per sample and kv head), bound 2e-2.  The
# measured whole-tensor error is ~3.6e-3 and the bf16 rounding of the
# operands is uniform over blocks, so a block-local bug is what breaks it.
# A block whose reference is exactly zero (padded keys; a one-token sample,
# whose dq cancels exactly) takes the absolute form of the whole-tensor rule:
# its norm must stay within the bound.
GRAD_BLOCK_REL, GRAD_BLOCK = 2e-2, 128


def gpu_tables(seg, D, base=10000.0):
    return jt.hia_rope2d_tables(seg, D, base)


def run_fwd(wl, seed=0, q=None, k=None, v=None):
    if q is None:
        q, k, v = synth.tensors(wl, seed)
    seg = jt.hia_segments_build(wl.samples, wl.S)
    c, s = gpu_tables(seg, wl.D, wl.base)
    o, lse = jt.hia_attn_fwd(seg, q.cuda(), k.cuda(), v.cuda(), c, s, wl.scale)
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 0
    return (q, k, v), o.float().cpu().numpy(), lse.cpu().numpy()


def sample_rows(wl, n_per_segment=6, seed=0):
    """Query rows covering every segment: text, image, suffix, padding, tile edges."""
    rng = np.random.default_rng(seed)
    rows = {0, wl.S - 1, min(127, wl.S - 1), min(128, wl.S - 1)}
    for (P, h, w, s) in wl.samples:
        I1 = P + h * w
        L = I1 + s
        for lo, hi in ((0, P), (P, I1), (I1, L), (L, wl.S)):
            if hi > lo:
                rows.update({lo, hi - 1})
                rows.update(int(x) for x in rng.integers(lo, hi, size=n_per_segment))
    return sorted(r for r in rows if 0 <= r < wl.S)


def check_fwd(oracle_mod, wl, q, k, v, o, lse, rows=None, groups=None, qk_norm=None):
    o_ref, lse_ref, _ = oracle_mod.attn_fwd(wl.samples, q.double().numpy(), k.double().numpy(),
                                            v.double().numpy(), wl.scale, wl.base, rows=rows, groups=groups,
                                            qk_norm=qk_norm)
    sel_r = slice(None) if rows is None else np.asarray(rows)
    g = wl.Hq // wl.Hkv
    if groups is None:
        hsel = np.ones((wl.B, wl.Hq), dtype=bool)
    else:
        hsel = np.repeat(np.asarray(groups, dtype=bool), g, axis=1)
    errs, lerrs = [], []
    for b in range(wl.B):
        for h in range(wl.Hq):
            if not hsel[b, h]:
                continue
            a = o[b, sel_r, h]
            r = o_ref[b, sel_r, h]
            errs.append(np.abs(a - r))
            la, lr = lse[b, h, sel_r], lse_ref[b, h, sel_r]
            fin = np.isfinite(lr)
            assert np.array_equal(np.isfinite(la), fin)
            lerrs.append(np.abs(la[fin] - lr[fin]))
    e = np.concatenate([x.ravel() for x in errs])
    le = np.concatenate([x.ravel() for x in lerrs]) if lerrs else np.zeros(1)
    assert np.all(np.isfinite(e)), "non-finite output"
    assert e.max() <= O_MAX, f"O max-abs {e.max():.3e}"
    assert e.mean() <= O_MEAN, f"O mean-abs {e.mean():.3e}"
    assert le.max() <= LSE_MAX, f"LSE max-abs {le.max():.3e}"
    assert le.mean() <= LSE_MEAN, f"LSE mean-abs {le.mean():.3e}"
    print(f"[parity] {wl.name}: O max {e.max():.3e} mean {e.mean():.3e}; LSE max {le.max():.3e} "
          f"mean {le.mean():.3e}")
    return e.max(), e.mean(), le.max()


def run_fwd_bwd(wl, seed=0):
    q, k, v, do = synth.tensors(wl, seed, grad=True)
    seg = jt.hia_segments_build(wl.samples, wl.S)
    c, s = gpu_tables(seg, wl.D, wl.base)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = jt.hia_attn_fwd(seg, qd, kd, vd, c, s, wl.scale)
    dq, dk, dv = jt.hia_attn_bwd(seg, qd, kd, vd, c, s, o, lse, dod, wl.scale)
    torch.cuda.synchronize()
    assert jt.hia_get_device_status() == 0
    f = lambda t: t.float().cpu().numpy()
    return (q, k, v, do), (f(dq), f(dk), f(dv))


def check_bwd(oracle_mod, wl, inputs, grads, groups=None, qk_norm=None, dw=None):
    """dq, dk, dv against the oracle by relative Frobenius norm; with qk_norm
    also the weight gradients dw = (dwq, dwk) (full problems only)."""
    q, k, v, do = inputs
    f64 = lambda t: t.double().numpy()
    if qk_norm is None:
        ref = oracle_mod.attn_bwd(wl.samples, f64(q), f64(k), f64(v), f64(do), wl.scale, wl.base,
                                  groups=groups)[:3]
    else:
        full = oracle_mod.attn_bwd_qknorm(wl.samples, f64(q), f64(k), f64(v), f64(do), qk_norm, wl.scale,
                                          wl.base, groups=groups)
        ref = full[:3]
        if dw is not None:
            for name, got, r in zip(("dwq", "dwk"), dw, full[3:5]):
                rel = np.linalg.norm(np.asarray(got, dtype=np.float64) - r) / np.linalg.norm(r)
                assert rel <= GRAD_REL, f"{name} relative Frobenius {rel:.3e}"
                print(f"[parity-bwd] {wl.name}: {name} {rel:.3e}")
    g = wl.Hq // wl.Hkv
    gsel = np.ones((wl.B, wl.Hkv), dtype=bool) if groups is None else np.asarray(groups, dtype=bool)
    out = {}
    for name, got, r in zip(("dq", "dk", "dv"), grads, ref):
        per = g if name == "dq" else 1
        a, bref = [], []
        for b in range(wl.B):
            for hk in range(wl.Hkv):
                if gsel[b, hk]:
                    a.append(got[b, :, hk * per:(hk + 1) * per])
                    bref.append(r[b, :, hk * per:(hk + 1) * per])
        worst = check_blocks(name, a, bref)
        a = np.concatenate([x.ravel() for x in a])
        bref = np.concatenate([x.ravel() for x in bref])
        assert np.all(np.isfinite(a)), f"{name} non-finite"
        nr = np.linalg.norm(bref)
        rel = np.linalg.norm(a - bref) / nr if nr > 0 else np.linalg.norm(a)
        out[name] = rel
        out[name + "_worst_block"] = worst
        assert rel <= GRAD_REL, f"{name} relative Frobenius {rel:.3e}"
    print(f"[parity-bwd] {wl.name}: " + " ".join(f"{k} {v:.3e}" for k, v in out.items()))
    return out


def check_blocks(name, got, ref, block=GRAD_BLOCK, bound=GRAD_BLOCK_REL):
    """Relative Frobenius error of every `block`-row slice of each [S, heads, D]
    array pair in got / ref (lists); returns the worst one."""
    worst = 0.0
    for i, (a, r) in enumerate(zip(got, ref)):
        S = r.shape[0]
        for r0 in range(0, S, block):
            ab = np.asarray(a[r0:r0 + block], dtype=np.float64)
            rb = r[r0:r0 + block]
            nr = np.linalg.norm(rb)
            if nr == 0:
                assert np.linalg.norm(ab) <= bound, f"{name}: block {i}/{r0} should be zero"
                continue
            rel = np.linalg.norm(ab - rb) / nr
            assert rel <= bound, f"{name}: block {i} rows [{r0}, {r0 + block}) relative Frobenius {rel:.3e}"
            worst = max(worst, rel)
    return worst
