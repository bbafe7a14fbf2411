"""Comparison metrics for the CUDA path against the fp64 oracle.

Tolerances (stated for this method): forward max |dO| <= 1e-2 and mean |dO| <= 1e-3,
|dL| <= 1e-3; backward max |dG| / max |G_ref| <= 2e-2 for each of dQ, dK, dV (absolute 2e-2
where the exact gradient is identically zero).
Reading for the forward max: O is stored in bfloat16, so storage alone can cost half a bf16 ulp
of |O| (0.0156 for |O| in [4, 8)); each element is allowed 1e-2 + half an ulp of its reference
value.  The strict maximum is reported beside it.
"""
import numpy as np

FWD_MAX = 1e-2
FWD_MEAN = 1e-3
LSE_MAX = 1e-3
BWD_REL = 2e-2


def bf16_half_ulp(x):
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    e = np.floor(np.log2(ax))
    return 2.0 ** (e - 8)


def to_np(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy().astype(np.float64)


def fwd_report(o, o_ref, lse, lse_ref):
    d = np.abs(o - o_ref)
    excess = d - (FWD_MAX + bf16_half_ulp(o_ref))
    return {
        "max_abs": float(d.max()) if d.size else 0.0,
        "mean_abs": float(d.mean()) if d.size else 0.0,
        "max_excess": float(excess.max()) if d.size else -1.0,
        "n_strict_over": int((d > FWD_MAX).sum()),
        "lse_max": float(np.abs(lse - lse_ref).max()) if lse.size else 0.0,
    }


def assert_fwd(o, o_ref, lse, lse_ref, what=""):
    r = fwd_report(o, o_ref, lse, lse_ref)
    assert np.isfinite(o).all() and np.isfinite(lse).all(), f"{what}: non-finite output"
    assert r["max_excess"] <= 0.0, f"{what}: forward max error {r}"
    assert r["mean_abs"] <= FWD_MEAN, f"{what}: forward mean error {r}"
    assert r["lse_max"] <= LSE_MAX, f"{what}: logsumexp error {r}"
    return r


def bwd_report(g, g_ref):
    """max |g - g_ref| / max |g_ref|.  Where the exact gradient is identically zero (N = 1:
    one key gives P = 1 and dS = 0, so dQ = dK = 0) the ratio has no denominator; the error is
    then measured in absolute terms (denominator 1)."""
    den = float(np.abs(g_ref).max()) if g_ref.size else 0.0
    if den == 0.0:
        den = 1.0
    return float(np.abs(g - g_ref).max() / den) if g.size else 0.0


def assert_bwd(grads, refs, what=""):
    out = {}
    for name, g, r in zip(("dq", "dk", "dv"), grads, refs):
        assert np.isfinite(g).all(), f"{what}: non-finite {name}"
        e = bwd_report(g, r)
        out[name] = e
        assert e <= BWD_REL, f"{what}: {name} relative max error {e:.3e} > {BWD_REL} ({out})"
    return out
