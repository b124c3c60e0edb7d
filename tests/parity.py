"""Shared helpers for the GPU parity tests: tolerances and sampled oracle slices.

Tolerances (from the acceptance bar for this path):
* fp32 path: max |x - ref| <= 1e-4 * max |ref| for every output;
* bf16-input / fp32-state path: ||x - ref||_2 / ||ref||_2 <= 2e-2 for every output.
"""
import numpy as np
import torch

F32_TOL = 1e-4
BF16_TOL = 2e-2


def f64(t):
    return t.detach().to("cpu").double().numpy() if hasattr(t, "detach") else np.asarray(t, dtype=np.float64)


def maxabs_rel(x, ref):
    x, ref = f64(x), f64(ref)
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


def l2_rel(x, ref):
    x, ref = f64(x), f64(ref)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-30))


def assert_close(x, ref, dtype, name=""):
    if dtype == "f32":
        err = maxabs_rel(x, ref)
        assert err <= F32_TOL, f"{name}: max-abs rel error {err:.3e} > {F32_TOL}"
    else:
        err = l2_rel(x, ref)
        assert err <= BF16_TOL, f"{name}: rel L2 error {err:.3e} > {BF16_TOL}"
    assert np.all(np.isfinite(f64(x))), f"{name}: non-finite values"
    return err


def to_dev(x, dev="cuda"):
    return {n: t.to(dev) for n, t in x.items()}


def bh_slice(x, pairs):
    """Cut the (b, h) pairs out of a [B,T,H,D] / [B,H,Dk,Dv] input dict (CPU tensors)."""
    out = {}
    for n, t in x.items():
        if n == "S0":
            out[n] = torch.stack([t[b, h] for b, h in pairs])[:, None]          # [P,1,Dk,Dv]
        else:
            out[n] = torch.stack([t[b, :, h] for b, h in pairs])[:, :, None]    # [P,T,1,D]
    return out


def assert_chains_close(got, ref, dtype, name, head_axis=1):
    """Every (batch, head) chain of one batch row: `got` (device or host tensor) and `ref` (fp64)
    are [T, H, D] (head_axis=1) or [H, Dk, Dv] (head_axis=0); each head's chain must meet the
    tolerance on its own.  Returns the worst error."""
    g, r = f64(got), f64(ref)
    worst = 0.0
    for h in range(g.shape[head_axis]):
        gh, rh = np.take(g, h, axis=head_axis), np.take(r, h, axis=head_axis)
        worst = max(worst, assert_close(gh, rh, dtype, f"{name} head {h}"))
    return worst


def sample_pairs(B, H, n, seed=0):
    rng = np.random.default_rng(seed)
    idx = rng.choice(B * H, size=min(n, B * H), replace=False)
    pairs = sorted({(int(i) // H, int(i) % H) for i in idx})
    # always include the first and the last (b, h) of the launch
    pairs = sorted(set(pairs) | {(0, 0), (B - 1, H - 1)})
    return pairs
