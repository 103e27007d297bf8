"""Shared helpers of the tests: device transfer of the seeded 16-bit inputs and
the parity bars (bf16 or f16 inputs/outputs with fp32 accumulation):
max |dO| <= 2e-2, mean |dO| <= 2e-3, |dLSE| <= 1e-3 absolute, and for each
gradient max |dg| / max |g_oracle| <= 5e-2.  A per-row relative bar
||dO_i|| / ||O_i|| <= 2e-2 is added because O rows of long causal rows are
small enough that the absolute bar alone could miss a wrong row."""
import numpy as np

from synth import bits_to_f32

O_MAX = 2e-2
O_MEAN = 2e-3
LSE_ABS = 1e-3
GRAD_REL = 5e-2
O_ROW_REL = 2e-2


def to_device(bits, fmt="bf16"):
    import torch
    dtype = torch.float16 if fmt == "f16" else torch.bfloat16
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dtype)
    return t.cuda()


def to_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def f64(bits, fmt="bf16"):
    return bits_to_f32(bits, fmt).astype(np.float64)


def check_fwd(o, lse, o_ref, lse_ref, what=""):
    """o, o_ref: (..., D) rows; lse, lse_ref matching rows."""
    o, lse, o_ref, lse_ref = map(np.asarray, (o, lse, o_ref, lse_ref))
    dead = np.isinf(lse_ref)
    assert np.array_equal(np.isneginf(lse), dead), f"{what}: -inf LSE rows differ"
    assert np.all(np.isfinite(o)), f"{what}: non-finite O"
    d = np.abs(o - o_ref)
    assert d.max() <= O_MAX, f"{what}: max|dO| = {d.max():.3e}"
    assert d.mean() <= O_MEAN, f"{what}: mean|dO| = {d.mean():.3e}"
    if (~dead).any():
        dl = np.abs(lse[~dead] - lse_ref[~dead])
        assert dl.max() <= LSE_ABS, f"{what}: max|dLSE| = {dl.max():.3e}"
    o2 = o.reshape(-1, o.shape[-1])
    r2 = o_ref.reshape(-1, o_ref.shape[-1])
    nrm = np.linalg.norm(r2, axis=1)
    live = nrm > 1e-6
    if live.any():
        rel = np.linalg.norm(o2 - r2, axis=1)[live] / nrm[live]
        assert rel.max() <= O_ROW_REL, f"{what}: max row-relative |dO| = {rel.max():.3e}"
    return float(d.max()), float(d.mean())


def check_grad(g, g_ref, what="", floor=0.0):
    """max |g - g_ref| / max |g_ref| <= 5e-2.  ``floor`` (an absolute magnitude)
    bounds the normaliser from below for gradients the mathematics makes
    identically zero (e.g. dQ when each query sees exactly one key: dS = 0),
    where the oracle's max |g| is rounding noise."""
    g, g_ref = np.asarray(g), np.asarray(g_ref)
    assert np.all(np.isfinite(g)), f"{what}: non-finite gradient"
    scale = max(np.abs(g_ref).max(), floor)
    err = np.abs(g - g_ref).max() / max(scale, 1e-30)
    assert err <= GRAD_REL, f"{what}: max|dg|/max|g| = {err:.3e}"
    return float(err)
