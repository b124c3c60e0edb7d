"""The input prologue (GDN2_QK_L2NORM: raw q, k normalised in the call; GDN2_BW_LOGITS: b, w
given as logits) against the oracle's ref_fwd_prologue / ref_bwd_prologue.

* the bf16 forward with per-channel gates runs the prologue inside the tensor-core kernel,
  for every flag combination, both head sizes, a ragged tail and a scalar decay;
* the fp32 forward, the bf16 forward with a scalar gate, the backward and the decode step
  run it as a separate pass;
* at the layer_4k size (B=8, T=4096, H=16, d=128), every (batch, head) sequence of the fused
  forward against the oracle.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_78_b200 as g
import oracle
from parity import assert_chains_close, assert_close
from synthetic_inputs import DecodeStream, make_inputs

pytestmark = pytest.mark.gpu

PRO = g.QK_L2NORM | g.BW_LOGITS


def dev(t):
    return None if t is None else t.cuda()


def raw_inputs(B, T, H, D, dtype, seed):
    x = make_inputs(B, T, H, D, D, dtype=dtype, seed=seed, with_do=True, raw=True)
    if dtype == "bf16":
        # q, k far from unit length, as projections give them (bf16 has the range)
        x["q"] = (x["q"].float() * 4.0).to(torch.bfloat16)
        x["k"] = (x["k"].float() * 0.5).to(torch.bfloat16)
    return x


def oracle_fwd(x, flags):
    return oracle.ref_fwd_prologue(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"],
                                   norm=bool(flags & g.QK_L2NORM), sigmoid=bool(flags & g.BW_LOGITS))


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("flags", [PRO, g.QK_L2NORM, g.BW_LOGITS])
def test_fused_forward_matches_oracle(cuda_lib, D, flags):
    x = raw_inputs(2, 200, 2, D, "bf16", seed=31)  # 3 chunks and a tail of 8
    if not flags & g.BW_LOGITS:  # gates given as values
        x["b"] = torch.sigmoid(x["b"].float()).to(torch.bfloat16)
        x["w"] = torch.sigmoid(x["w"].float()).to(torch.bfloat16)
    if not flags & g.QK_L2NORM:  # unit q, k given (raw ones would make the delta rule diverge)
        for n in ("q", "k"):
            t = x[n].float()
            x[n] = (t / t.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    o, ST = g.gdn2_chunk_fwd_gated(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]), dev(x["b"]),
                                   dev(x["w"]), dev(x["S0"]), flags=flags)
    assert g.gdn2_sync_status() == 0
    ro, rS = oracle_fwd(x, flags)
    assert_close(o, ro, "bf16", "o")
    assert_close(ST, rS, "bf16", "S_T")


def test_fused_forward_with_scalar_decay(cuda_lib):
    B, T, H, D = 2, 192, 2, 128
    x = raw_inputs(B, T, H, D, "bf16", seed=33)
    gs = -torch.nn.functional.softplus(torch.randn(B, T, H, generator=torch.Generator().manual_seed(7)) - 3.0)
    o, ST = g.gdn2_chunk_fwd_gated(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(gs), dev(x["b"]), dev(x["w"]),
                                   dev(x["S0"]), flags=PRO | g.DECAY_SCALAR)
    assert g.gdn2_sync_status() == 0
    ro, rS = oracle.ref_fwd_prologue(x["q"], x["k"], x["v"], gs[..., None].expand(B, T, H, D), x["b"], x["w"],
                                     x["S0"])
    assert_close(o, ro, "bf16", "o")
    assert_close(ST, rS, "bf16", "S_T")


def test_fp32_forward_prologue_pass(cuda_lib):
    x = raw_inputs(1, 130, 2, 64, "f32", seed=35)
    o, ST = g.gdn2_chunk_fwd_gated(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]), dev(x["b"]),
                                   dev(x["w"]), dev(x["S0"]), flags=PRO)
    assert g.gdn2_sync_status() == 0
    ro, rS = oracle_fwd(x, PRO)
    assert_close(o, ro, "f32", "o")
    assert_close(ST, rS, "f32", "S_T")


def test_scalar_gate_logits_prologue_pass(cuda_lib):
    """A scalar erase-gate logit goes through the separate pass, then the broadcast."""
    B, T, H, D = 2, 130, 2, 128
    x = raw_inputs(B, T, H, D, "bf16", seed=37)
    bl = torch.randn(B, T, H, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    o, ST = g.gdn2_chunk_fwd_gated(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]), dev(bl), dev(x["w"]),
                                   dev(x["S0"]), flags=PRO | g.ERASE_SCALAR)
    assert g.gdn2_sync_status() == 0
    ro, rS = oracle.ref_fwd_prologue(x["q"], x["k"], x["v"], x["log_alpha"], bl[..., None].expand(B, T, H, D),
                                     x["w"], x["S0"])
    assert_close(o, ro, "bf16", "o")
    assert_close(ST, rS, "bf16", "S_T")


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f32", 64), ("bf16", 64)])
def test_backward_matches_oracle(cuda_lib, dtype, D):
    x = raw_inputs(2, 150, 2, D, dtype, seed=39)
    gr = g.gdn2_chunk_bwd_gated(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]), dev(x["b"]), dev(x["w"]),
                                dev(x["S0"]), dev(x["do"]), flags=PRO)
    assert g.gdn2_sync_status() == 0
    ref = oracle.ref_bwd_prologue(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], x["do"])
    for gk, rk in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dlog_alpha", "dg"), ("db", "db"), ("dw", "dw"),
                   ("dS0", "dS0")):
        assert_close(gr[gk], ref[rk], dtype, gk)


def test_backward_scalar_gate_logits(cuda_lib):
    B, T, H, D = 1, 130, 2, 128
    x = raw_inputs(B, T, H, D, "bf16", seed=41)
    wl = torch.randn(B, T, H, generator=torch.Generator().manual_seed(11)).to(torch.bfloat16)
    gr = g.gdn2_chunk_bwd_gated(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]), dev(x["b"]), dev(wl),
                                dev(x["S0"]), dev(x["do"]), flags=PRO | g.WRITE_SCALAR)
    assert g.gdn2_sync_status() == 0
    ref = oracle.ref_bwd_prologue(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], wl[..., None].expand(B, T, H, D),
                                  x["S0"], x["do"])
    assert_close(gr["dw"], ref["dw"].sum(-1), "bf16", "dw (scalar)")
    assert_close(gr["dq"], ref["dq"], "bf16", "dq")
    assert_close(gr["db"], ref["db"], "bf16", "db")


def test_decode_prologue_matches_oracle(cuda_lib):
    N, H, D, steps = 8, 2, 128, 12
    ds = DecodeStream(N, H, D, D, dtype="bf16", seed=43)
    S = ds.S0.clone().cuda()
    Sr = ds.S0.double().numpy().copy()
    for _ in range(steps):
        s = ds.step(raw=True)
        o = g.gdn2_decode_step_gated(dev(s["q"]), dev(s["k"]), dev(s["v"]), dev(s["log_alpha"]), dev(s["b"]),
                                     dev(s["w"]), S, flags=PRO)
        qn, kn, bs, ws = oracle.ref_prologue(s["q"], s["k"], s["b"], s["w"])
        ro, Sr = oracle.ref_decode(qn, kn, s["v"], s["log_alpha"], bs, ws, Sr)
        assert_close(o, ro, "bf16", "o")
    assert g.gdn2_sync_status() == 0
    assert_close(S, Sr, "bf16", "S")


def test_fused_forward_layer_4k_all_chains(cuda_lib):
    """The bench's fused-prologue launch at full size; every (b, h) chain against the oracle."""
    B, T, H, D = 8, 4096, 16, 128
    x = raw_inputs(B, T, H, D, "bf16", seed=45)
    o, ST = g.gdn2_chunk_fwd_gated(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(x["log_alpha"]), dev(x["b"]),
                                   dev(x["w"]), dev(x["S0"]), flags=PRO)
    assert g.gdn2_sync_status() == 0
    oc, Sc = o.cpu(), ST.cpu()
    for b in range(B):
        ro, rS = oracle_fwd({n: x[n][b:b + 1] for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")}, PRO)
        assert_chains_close(oc[b], ro[0], "bf16", f"o[{b}]")
        assert_chains_close(Sc[b], rS[0], "bf16", f"S_T[{b}]", head_axis=0)


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f32", 64)])
def test_standalone_prologue_matches_oracle(cuda_lib, dtype, D):
    B, T, H = 2, 70, 3
    x = raw_inputs(B, T, H, D, dtype, seed=47)
    out = g.gdn2_prologue(dev(x["q"]), dev(x["k"]), dev(x["b"]), dev(x["w"]), flags=PRO)
    ref = oracle.ref_prologue(x["q"], x["k"], x["b"], x["w"])
    for got, r, n in zip((out["q"], out["k"], out["b"], out["w"]), ref, "qkbw"):
        assert_close(got, r, dtype, n)
    # a per-token erase-gate logit and an absent write gate
    bl = torch.randn(B, T, H, generator=torch.Generator().manual_seed(13)).to(x["q"].dtype)
    out = g.gdn2_prologue(dev(x["q"]), dev(x["k"]), dev(bl), None, flags=PRO | g.ERASE_SCALAR | g.WRITE_NONE)
    assert out["w"] is None
    assert_close(out["b"], oracle.ref_prologue(x["q"], x["k"], bl, None)[2], dtype, "b (per token)")
    assert g.gdn2_sync_status() == 0


@pytest.mark.parametrize("dtype,flags", [("f32", PRO), ("bf16", g.QK_L2NORM), ("bf16", g.BW_LOGITS),
                                         ("bf16", PRO | g.ERASE_SCALAR)])
def test_decode_prologue_variants(cuda_lib, dtype, flags):
    """Fused into the decode kernel for per-channel b and w (every flag combination, both dtypes);
    a per-token erase-gate logit goes through the prologue pass."""
    N, H, D, steps = 4, 2, 64 if dtype == "f32" else 128, 6
    ds = DecodeStream(N, H, D, D, dtype=dtype, seed=47)
    S = ds.S0.clone().cuda()
    Sr = ds.S0.double().numpy().copy()
    gen = torch.Generator().manual_seed(3)
    for _ in range(steps):
        s = ds.step(raw=True)
        if not flags & g.BW_LOGITS:
            s["b"] = torch.sigmoid(s["b"].float()).to(s["q"].dtype)
            s["w"] = torch.sigmoid(s["w"].float()).to(s["q"].dtype)
        if not flags & g.QK_L2NORM:
            for n in ("q", "k"):
                t = s[n].float()
                s[n] = (t / t.norm(dim=-1, keepdim=True)).to(s["q"].dtype)
        b_in, b_ref = s["b"], s["b"]
        if flags & g.ERASE_SCALAR:
            b_in = torch.randn(N, H, generator=gen).to(s["q"].dtype)
            b_ref = b_in[..., None].expand(N, H, D)
        o = g.gdn2_decode_step_gated(dev(s["q"]), dev(s["k"]), dev(s["v"]), dev(s["log_alpha"]), dev(b_in),
                                     dev(s["w"]), S, flags=flags)
        qn, kn, bs, ws = oracle.ref_prologue(s["q"], s["k"], b_ref, s["w"], norm=bool(flags & g.QK_L2NORM),
                                             sigmoid=bool(flags & g.BW_LOGITS))
        ro, Sr = oracle.ref_decode(qn, kn, s["v"], s["log_alpha"], bs, ws, Sr)
        assert_close(o, ro, dtype, "o")
    assert g.gdn2_sync_status() == 0
    assert_close(S, Sr, dtype, "S")


def test_backward_scalar_decay_with_prologue(cuda_lib):
    """Raw q, k and gate logits with a scalar decay: the prologue runs as a pass, the kernels read
    log alpha per token, and dlog alpha is the per-channel gradient summed over the channels."""
    B, T, H, D = 1, 130, 2, 128
    x = raw_inputs(B, T, H, D, "bf16", seed=43)
    la = -torch.nn.functional.softplus(torch.randn(B, T, H, generator=torch.Generator().manual_seed(13)) - 3.0)
    gr = g.gdn2_chunk_bwd_gated(dev(x["q"]), dev(x["k"]), dev(x["v"]), dev(la), dev(x["b"]), dev(x["w"]),
                                dev(x["S0"]), dev(x["do"]), flags=PRO | g.DECAY_SCALAR)
    assert g.gdn2_sync_status() == 0
    ref = oracle.ref_bwd_prologue(x["q"], x["k"], x["v"], la[..., None].expand(B, T, H, D), x["b"], x["w"],
                                  x["S0"], x["do"])
    for gk, rk in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("db", "db"), ("dw", "dw"), ("dS0", "dS0")):
        assert_close(gr[gk], ref[rk], "bf16", gk)
    assert gr["dlog_alpha"].shape == (B, T, H)
    assert_close(gr["dlog_alpha"], ref["dg"].sum(-1), "bf16", "dlog_alpha (scalar)")
