"""Seeded synthetic inputs for the GDN-2 chunkwise recurrence.

This module is shared by the CPU oracle tests, the GPU parity tests and the
benchmark.  It holds the input *distributions* only and none of the
recurrence's arithmetic: every tensor is drawn from a CPU ``torch.Generator``
and returned on the CPU, so both sides consume bit-identical values.

Recipe (per the workload description of the Gated DeltaNet-2 write-ups:
16 heads, d_k = d_v = 128, L2-normalised q/k, log-decay kept in fp32):

* draw order is fixed: q, k, v, x (decay logits), b-logit, w-logit, S0, do;
* q, k ~ N(0, 1), then L2-normalised per (token, head) over the channel axis
  in fp32, then cast to the compute dtype;
* v ~ N(0, 1);
* log alpha = -softplus(x), x ~ N(-3, 1), per channel, computed and kept in
  fp32 (never cast to bf16);
* b, w = sigmoid(N(0, 1)) computed in fp32 then cast;
* S0 ~ N(0, std 0.02) in fp32 (or zeros);
* do ~ N(0, 1) cast to the compute dtype.

Decode steps draw q, k, v, x, b-logit, w-logit for one token per sequence in
the same order from one generator, step after step.
"""
from __future__ import annotations

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    return x / torch.sqrt((x * x).sum(-1, keepdim=True) + 1e-12)


def make_inputs(B: int, T: int, H: int, Dk: int, Dv: int, *, dtype: str = "bf16",
                seed: int = 0, s0: str = "normal", with_do: bool = False,
                b_scale: float = 1.0, x_mean: float = -3.0, device: str = "cpu", raw: bool = False) -> dict:
    """Draw one forward (or forward+backward) problem.

    Layouts: q, k, b, log_alpha are [B, T, H, Dk]; v, w, do are [B, T, H, Dv];
    S0 is [B, H, Dk, Dv] fp32.  ``b_scale`` stretches the erase gate range
    (2.0 gives b in [0, 2]); ``x_mean`` moves the decay logits (a larger
    value gives stronger decay).  ``device="cuda"`` draws the same
    distributions with a seeded CUDA generator (a different stream of numbers,
    used for timing only, never for parity).  ``raw=True`` returns the same draws
    before the input prologue: q, k unnormalised (N(0, 1) per channel) and b, w as
    their N(0, 1) logits.
    """
    dt = DTYPES[dtype]
    gen = torch.Generator(device=device).manual_seed(seed)
    kw = dict(generator=gen, dtype=torch.float32, device=device)
    q = torch.randn(B, T, H, Dk, **kw)
    k = torch.randn(B, T, H, Dk, **kw)
    if not raw:
        q, k = _l2norm(q), _l2norm(k)
    v = torch.randn(B, T, H, Dv, **kw)
    x = torch.randn(B, T, H, Dk, **kw) + x_mean
    bl = torch.randn(B, T, H, Dk, **kw)
    wl = torch.randn(B, T, H, Dv, **kw)
    S0 = torch.randn(B, H, Dk, Dv, **kw) * 0.02
    if s0 == "zeros":
        S0 = torch.zeros_like(S0)
    out = {
        "q": q.to(dt), "k": k.to(dt), "v": v.to(dt),
        "log_alpha": -torch.nn.functional.softplus(x),
        "b": (bl if raw else torch.sigmoid(bl) * b_scale).to(dt),
        "w": (wl if raw else torch.sigmoid(wl)).to(dt),
        "S0": S0,
    }
    if with_do:
        out["do"] = torch.randn(B, T, H, Dv, **kw).to(dt)
    return out


class DecodeStream:
    """Per-step single-token inputs for ``N`` sequences, drawn in order."""

    def __init__(self, N: int, H: int, Dk: int, Dv: int, *, dtype: str = "bf16", seed: int = 0,
                 device: str = "cpu"):
        self.N, self.H, self.Dk, self.Dv = N, H, Dk, Dv
        self.dt = DTYPES[dtype]
        self.gen = torch.Generator(device=device).manual_seed(seed)
        self.kw = dict(generator=self.gen, dtype=torch.float32, device=device)
        # initial state first, so that erase acts from step one
        self.S0 = torch.randn(N, H, Dk, Dv, **self.kw) * 0.02

    def step(self, raw: bool = False) -> dict:
        """One step's inputs; ``raw=True``: q, k unnormalised and b, w as logits."""
        N, H, Dk, Dv, kw = self.N, self.H, self.Dk, self.Dv, self.kw
        q = torch.randn(N, H, Dk, **kw)
        k = torch.randn(N, H, Dk, **kw)
        if not raw:
            q, k = _l2norm(q), _l2norm(k)
        v = torch.randn(N, H, Dv, **kw)
        x = torch.randn(N, H, Dk, **kw) - 3.0
        bl = torch.randn(N, H, Dk, **kw)
        wl = torch.randn(N, H, Dv, **kw)
        return {
            "q": q.to(self.dt), "k": k.to(self.dt), "v": v.to(self.dt),
            "log_alpha": -torch.nn.functional.softplus(x),
            "b": (bl if raw else torch.sigmoid(bl)).to(self.dt), "w": (wl if raw else torch.sigmoid(wl)).to(self.dt),
        }


# Named workloads: (B, T, H, Dk, Dv, dtype, S0 kind)
WORKLOADS = {
    "tiny_f32": dict(B=1, T=256, H=2, Dk=64, Dv=64, dtype="f32", s0="zeros"),
    "layer_4k": dict(B=8, T=4096, H=16, Dk=128, Dv=128, dtype="bf16", s0="normal"),
    # the layer shape at batch 2: profiler captures of one launch (still larger than L2)
    "layer_4k_b2": dict(B=2, T=4096, H=16, Dk=128, Dv=128, dtype="bf16", s0="normal"),
    "sweep_2k": dict(B=32, T=2048, H=16, Dk=128, Dv=128, dtype="bf16", s0="normal"),
    "sweep_4k": dict(B=16, T=4096, H=16, Dk=128, Dv=128, dtype="bf16", s0="normal"),
    "sweep_8k": dict(B=8, T=8192, H=16, Dk=128, Dv=128, dtype="bf16", s0="normal"),
    "sweep_16k": dict(B=4, T=16384, H=16, Dk=128, Dv=128, dtype="bf16", s0="normal"),
    "sweep_32k": dict(B=2, T=32768, H=16, Dk=128, Dv=128, dtype="bf16", s0="normal"),
}
DECODE_WORKLOAD = dict(N=256, H=16, Dk=128, Dv=128, steps=1024, dtype="bf16")
