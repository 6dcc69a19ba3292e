"""Comparison helpers shared by the parity tests (no method arithmetic here)."""
import math

import numpy as np
import torch


def cuda(t):
    return t.contiguous().cuda()


def rel_rowwise(gpu, ref):
    """max over rows of ||gpu - ref||_inf / ||ref||_inf (rows = last dim); finite parts only."""
    g = np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    g = g.reshape(-1, g.shape[-1])
    r = r.reshape(-1, r.shape[-1])
    fin = np.isfinite(r)
    assert np.array_equal(fin, np.isfinite(g)), "finite/-inf pattern differs"
    g = np.where(fin, g, 0.0)
    r = np.where(fin, r, 0.0)
    num = np.abs(g - r).max(1)
    den = np.abs(r).max(1)
    den = np.where(den > 0, den, 1.0)
    return float((num / den).max()) if len(num) else 0.0


def bf16_ulp(x):
    """Spacing of bf16 values at |x| (8 significant bits)."""
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 2.0 ** -126)))
    return 2.0 ** (np.maximum(e, -126) - 7)


def bf16_out_ratio(gpu, ref, rel=1e-3):
    """Worst ratio of |gpu - ref| to the bf16-output allowance: the fp32 score tolerance
    (rel, norm-wise per row) plus one bf16 ulp of ref for the output rounding.
    <= 1 passes.  -inf entries must match exactly."""
    g = np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    g = g.reshape(-1, g.shape[-1])
    r = r.reshape(-1, r.shape[-1])
    fin = np.isfinite(r)
    if not np.array_equal(fin, np.isfinite(g)):
        return float("inf")
    rz = np.where(fin, r, 0.0)
    gz = np.where(fin, g, 0.0)
    allow = bf16_ulp(rz) + rel * np.abs(rz).max(1, keepdims=True)
    return float((np.abs(gz - rz) / allow).max()) if rz.size else 0.0


def within_bf16_ulp(gpu, ref, n_ulp=1.0):
    g = np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    fin = np.isfinite(r)
    if not np.array_equal(fin, np.isfinite(g)):
        return False
    return bool(np.all(np.abs(g[fin] - r[fin]) <= n_ulp * bf16_ulp(r[fin]) + 1e-300))


def check_topk_band(gpu_idx, ref_scores, nvis, k, bf16_scores):
    """Top-k set parity with the ambiguity band: an entry is ambiguous when its oracle score is
    within max(1e-3 |s_k|, 1 bf16 ulp of s_k in bf16-score mode) of the oracle's k-th score.
    The GPU set minus ambiguous entries must equal the oracle set minus ambiguous entries, the
    sizes must agree, and the indices must be unique, visible and ascending.  Returns the number
    of entries on which the sets differ (all of them inside the band)."""
    g = np.asarray(gpu_idx)
    s = np.asarray(ref_scores, np.float64)[:nvis]
    take = min(k, nvis)
    sel_g = g[g >= 0]
    assert len(sel_g) == take, f"selected {len(sel_g)} entries, expected {take}"
    assert np.all(g[take:] == -1)
    assert np.all(np.diff(sel_g) > 0), "indices not strictly ascending"
    assert np.all(sel_g < nvis), "invisible entry selected"
    order = np.lexsort((np.arange(nvis), -s))
    ref_set = set(order[:take].tolist())
    if take == nvis:
        assert set(sel_g.tolist()) == ref_set
        return 0
    sk = s[order[take - 1]]
    band = max(1e-3 * abs(sk), bf16_ulp(sk) if bf16_scores else 0.0)
    amb = set(np.nonzero(np.abs(s - sk) <= band)[0].tolist())
    gs = set(sel_g.tolist())
    assert gs - amb == ref_set - amb, f"sets differ outside the band: {sorted((gs ^ ref_set) - amb)[:10]}"
    return len(gs ^ ref_set)


def as_f64(t):
    return t.detach().cpu().to(torch.float64).numpy()


def sqrt_d(d):
    return 1.0 / math.sqrt(d)
