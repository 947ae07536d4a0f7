"""Helpers shared by the GPU parity tests (no attention arithmetic here)."""

from __future__ import annotations

import numpy as np
import torch

O_TOL_REL = 1e-2     # max|dO| <= 1e-2 * max|V|
LSE_TOL = 2e-3       # |dlse| <= 2e-3


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


def compare(w, out_gpu, lse_gpu, out_ref, lse_ref, batches=None, what=""):
    """Assert parity within the stated tolerances on the selected sequences."""
    out_gpu = out_gpu.float().cpu().numpy()
    lse_gpu = lse_gpu.float().cpu().numpy()
    sel = list(range(w.batch)) if batches is None else list(batches)
    vmax = max(max_abs_v(w, sel), 1e-30)
    o_err = np.abs(out_gpu[sel] - out_ref[sel]).max()
    ref_l = lse_ref[sel]
    gpu_l = lse_gpu[sel]
    fin = np.isfinite(ref_l)
    assert np.array_equal(np.isfinite(gpu_l), fin), f"{what}: -inf pattern of lse differs"
    assert np.all(np.isneginf(gpu_l[~fin]))
    l_err = np.abs(gpu_l[fin] - ref_l[fin]).max(initial=0.0)
    assert o_err <= O_TOL_REL * vmax, f"{what}: max|dO| = {o_err:.3e} > {O_TOL_REL} * {vmax:.3f}"
    assert l_err <= LSE_TOL, f"{what}: max|dlse| = {l_err:.3e}"
    return o_err / vmax, l_err
