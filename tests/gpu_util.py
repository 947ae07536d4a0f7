"""Helpers shared by the GPU parity tests (no attention arithmetic of their own:
the weights come from the oracle).

Two checks per comparison:

1. The stated tolerance: max|dO| <= 1e-2 * max|V| and |dlse| <= 2e-3.
2. A per-element bound from the GPU path's own roundings, which is much
   tighter where the output is small (long sequences average many values, so
   O is far below max|V|).  The path rounds P to the element type (unit
   roundoff u = 2^-8 for bf16, 2^-11 for fp16) before the value product and
   sums the same rounded P for the denominator, so
       dO_i = sum_j w_j (d_j - sum_k w_k d_k) V_ji ~= sum_j w_j d_j (V_ji - O_i)
   with |d_j| <= u.  Rounding errors of different keys are independent, each
   of variance u^2 / 3, so dO_i has standard deviation
       sigma_i = u / sqrt(3) * sqrt(sum_j w_j^2 (V_ji - O_i)^2).
   The fp32 scores add an error of the same shape, orders of magnitude
   smaller, folded in below.  Output rounding adds at most u * |O_i|.  The
   bound is 8 sigma_i + u |O_i| + 2^-20 max|V|.  For n <= 21 visible keys the
   worst case of the sum is at most sqrt(3 n) <= 8 sigma_i, so short rows are
   covered without the statistical argument; for long rows the sum is close
   to Gaussian and 8 sigma is far beyond the largest of millions of samples.
   Merging split pieces re-forms the same sums (each piece's O and lse carry
   its own rounded denominator), so splits add only fp32-level error.  fp16
   P below 2^-14 is subnormal (absolute error up to 2^-25); that term is
   added for fp16.
   A relative Frobenius check, ||dO|| <= 2^-6 ||O||, catches an error of the
   size of the output even on a few rows.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import mla_oracle as mo

O_TOL_REL = 1e-2     # max|dO| <= 1e-2 * max|V|
LSE_TOL = 2e-3       # |dlse| <= 2e-3
SIGMAS = 8.0
FRO_REL = 2.0 ** -6
UNIT_ROUNDOFF = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}


def to_gpu(w):
    return (w.q.cuda(), w.k_cache.cuda(), w.block_table.cuda(), w.seqlens.cuda())


def max_abs_v(w, batches=None) -> float:
    """Largest |V| over the valid tokens of the given sequences."""
    k = w.k_cache.float()
    bt = w.block_table
    m = 0.0
    for b in (range(w.batch) if batches is None else batches):
        L = int(w.seqlens[b])
        if L == 0:
            continue
        j = torch.arange(L)
        rows = k[bt[b, j // 64].long(), j % 64, :, :512]
        m = max(m, float(rows.abs().max()))
    return m


def rounding_bound(w, out_ref: np.ndarray, sel, u: float, vmax: float) -> np.ndarray:
    """Per-element bound on |O_gpu - O_exact| for the sequences in `sel` (see the module
    docstring); NaN elsewhere."""
    q = mo.as_f64(w.q)
    k = mo.as_f64(w.k_cache)
    bt = mo.as_i64(w.block_table)
    hg = w.h_q // w.h_kv
    bound = np.full(out_ref.shape, np.nan)
    for b in sel:
        L = int(w.seqlens[b])
        for g in range(w.h_kv):
            K = mo.gather_keys(k, bt[b], L, g)
            heads = slice(g * hg, (g + 1) * hg)
            kn = np.sqrt((K * K).sum(axis=1)).max(initial=0.0)
            for s in range(w.s_q):
                n = mo.visible_keys(L, s, w.s_q, w.causal)
                o = out_ref[b, s, heads]
                if n == 0:
                    bound[b, s, heads] = 2.0 ** -20 * vmax
                    continue
                W = mo.attention_weights(q[b, s, heads], K[:n], w.scale)    # [hg, n]
                V = K[:n, :512]
                W2 = W * W
                var = W2 @ (V * V) - 2.0 * o * (W2 @ V) + o * o * W2.sum(axis=1, keepdims=True)
                # fp32 score error: at most |scale| 2^-24 sqrt(576) |q| max|K_j| in standard deviation
                qn = np.sqrt((q[b, s, heads] ** 2).sum(axis=1, keepdims=True))
                sx = abs(w.scale) * 2.0 ** -24 * 24.0 * qn * kn
                sig2 = (u * u / 3.0 + sx * sx) * np.maximum(var, 0.0)
                if u < 2.0 ** -8:
                    # fp16 P below 2^-14 is subnormal: absolute error up to 2^-25 against a
                    # denominator >= 1 (the key that set the running max has P = 1)
                    dev2 = (V * V).sum(axis=0) - 2.0 * o * V.sum(axis=0) + n * o * o
                    sig2 = sig2 + 2.0 ** -50 / 3.0 * np.maximum(dev2, 0.0)
                sig = np.sqrt(sig2)
                bound[b, s, heads] = SIGMAS * sig + u * np.abs(o) + 2.0 ** -20 * vmax
    return bound


def compare(w, out_gpu, lse_gpu, out_ref, lse_ref, batches=None, what=""):
    """Assert parity on the selected sequences: the stated tolerances, then the rounding bound
    and the relative Frobenius error.  Returns the errors for reporting."""
    u = UNIT_ROUNDOFF[out_gpu.dtype]
    out_gpu = out_gpu.float().cpu().numpy()
    lse_gpu = lse_gpu.float().cpu().numpy()
    sel = list(range(w.batch)) if batches is None else list(batches)
    vmax = max(max_abs_v(w, sel), 1e-30)
    diff = np.abs(out_gpu[sel] - out_ref[sel])
    o_err = diff.max()
    ref_l = lse_ref[sel]
    gpu_l = lse_gpu[sel]
    fin = np.isfinite(ref_l)
    assert np.array_equal(np.isfinite(gpu_l), fin), f"{what}: -inf pattern of lse differs"
    assert np.all(np.isneginf(gpu_l[~fin]))
    l_err = np.abs(gpu_l[fin] - ref_l[fin]).max(initial=0.0)
    # 1. the stated tolerances
    assert o_err <= O_TOL_REL * vmax, f"{what}: max|dO| = {o_err:.3e} > {O_TOL_REL} * {vmax:.3f}"
    assert l_err <= LSE_TOL, f"{what}: max|dlse| = {l_err:.3e}"
    # 2. the rounding bound, element by element, and the relative Frobenius error
    bound = rounding_bound(w, out_ref, sel, u, vmax)[sel]
    ratio = float((diff / bound).max())
    worst = np.unravel_index(int(np.argmax(diff / bound)), diff.shape)
    assert ratio <= 1.0, (f"{what}: |dO| {diff[worst]:.3e} exceeds the rounding bound {bound[worst]:.3e} "
                          f"at {worst} (ref {out_ref[sel][worst]:.4e})")
    ref_norm = float(np.sqrt((out_ref[sel] ** 2).sum()))
    fro = float(np.sqrt((diff ** 2).sum())) / ref_norm if ref_norm > 0 else 0.0
    assert fro <= FRO_REL, f"{what}: ||dO|| / ||O|| = {fro:.3e} > {FRO_REL:.3e}"
    rel_max = float(o_err / max(np.abs(out_ref[sel]).max(), 1e-30))
    print(f"{what}: max|dO| {o_err:.2e} ({o_err / vmax:.2e} of max|V|, {rel_max:.2e} of max|O|), "
          f"||dO||/||O|| {fro:.2e}, worst |dO|/bound {ratio:.2f}, max|dlse| {l_err:.2e}")
    return o_err / vmax, l_err
