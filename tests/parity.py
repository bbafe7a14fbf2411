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


# ------------------------------------------------------------------------------------------------
# FP8 forward.  Reading of the tolerance (the pages give none for FP8): the kernel computes the
# scores exactly (products of e4m3 values are exact in fp32, sums are fp32) and L from the fp32
# exponentials, so |dL| <= 1e-3 as for bf16.  The one rounding step the definition does not have
# is the softmax weights' rounding to e4m3 before they multiply V: weight p (relative to the row
# maximum, which the kernel keeps exact at 2^8) has error at most e(p) = max(2^-4 p, min(p, 2^-18))
# (3 mantissa bits while normal, spacing 2^-17 of the maximum below 2^-14).  Hence, per element,
#   |dO_ic| <= sum_j e(p_ij) |v_jc| / l_i + 1/2 ulp_bf16(O_ic) + 1e-3   (worst case), and
#   E[dO_ic^2] <= sum_j e(p_ij)^2 v_jc^2 / (3 l_i^2) + ulp^2 / 12       (uniform rounding errors),
# checked as: every element within its worst-case bound, and the mean squared error at most 1.5x
# the mean of the variance bound (which a systematic error -- a bias in P, a wrong scale -- fails).
FP8_REL = 2.0 ** -4
FP8_FLOOR = 2.0 ** -18


def fp8_error_bounds(q, k, v, causal, scale, block=512):
    """Worst-case bound and variance bound of the FP8 forward's error for ONE head (fp64 [N, d]
    dequantised arrays), from the exact weights; returns (bound [N, d], var [N, d]) without the
    bf16 storage terms."""
    N = q.shape[0]
    bound = np.empty((N, v.shape[1]))
    var = np.empty((N, v.shape[1]))
    for r0 in range(0, N, block):
        rows = np.arange(r0, min(N, r0 + block))
        s = scale * (q[rows] @ k.T)
        if causal:
            s = np.where(np.arange(k.shape[0])[None, :] > rows[:, None], -np.inf, s)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        l = p.sum(axis=1, keepdims=True)
        e = np.maximum(FP8_REL * p, np.minimum(p, FP8_FLOOR))
        bound[rows] = (e @ np.abs(v)) / l
        var[rows] = ((e * e) @ (v * v)) / (3.0 * l * l)
    return bound, var


def assert_fwd_fp8(o, o_ref, lse, lse_ref, bound, var, what=""):
    """FP8 forward against the fp64 oracle on the dequantised inputs (reading above)."""
    assert np.isfinite(o).all() and np.isfinite(lse).all(), f"{what}: non-finite output"
    d = np.abs(o - o_ref)
    ulp = 2.0 * bf16_half_ulp(o_ref)
    excess = d - (bound + ulp / 2 + 1e-3)
    r = {"max_abs": float(d.max()), "max_excess": float(excess.max()),
         "mse": float((d * d).mean()), "var_bound": float((var + ulp * ulp / 12).mean()),
         "lse_max": float(np.abs(lse - lse_ref).max())}
    assert r["max_excess"] <= 0.0, f"{what}: FP8 forward element outside its bound {r}"
    assert r["mse"] <= 1.5 * r["var_bound"], f"{what}: FP8 forward mean squared error {r}"
    assert r["lse_max"] <= LSE_MAX, f"{what}: logsumexp error {r}"
    return r
