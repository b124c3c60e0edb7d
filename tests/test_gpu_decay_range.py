"""Decay of any strength.  The chunkwise tensor-core kernels form e^{-G} (G the cumulative
log-decay inside a 64-token chunk), which leaves the fp32 range once G falls below about -88,
and the chunkwise backward's dlog alpha loses accuracy as the chunk's decay grows.  The pages
bound the decay only by alpha in (0, 1] (the aiexpert.news gate paragraph), so the library must
stay exact past those points: the forward runs chunks whose log-decay falls below -80 on some
channel token by token, the backward does so below -16, and the fp32 path is token-level
throughout.  Every case here is checked against the oracle's token recurrence, with the status
word clear.

* a sweep of uniform decay strengths, chunk log-decay 6 ... 96, on both sides of both limits;
* x ~ N(+2, 1) (log alpha about -2.1 per token, about -135 per chunk): every chunk token by token;
* one channel at log alpha = -10 per token (-640 per chunk), the others from the recipe;
* strong decay in some chunks only, so that the two forms alternate along a sequence;
* alpha underflowing to zero (log alpha = -100) on whole tokens;
* the fused input prologue, a scalar decay, the chunk-parallel scan, packed variable-length
  sequences and the training pair, each with strong decay.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_78_b200 as g
import oracle
from parity import assert_close
from synthetic_inputs import make_inputs

pytestmark = pytest.mark.gpu

GRADS = (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dlog_alpha", "dg"), ("db", "db"), ("dw", "dw"),
         ("dS0", "dS0"))


def dev(t):
    return None if t is None else t.cuda()


def fwd_bwd_check(x, dtype, dST=None):
    d = {n: dev(t) for n, t in x.items()}
    args = (d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    o, ST = g.gdn2_chunk_fwd(*args)
    gr = g.gdn2_chunk_bwd(*args, d["do"], dev(dST))
    assert g.gdn2_sync_status() == 0
    ro, rS = oracle.ref_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"])
    assert_close(o, ro, dtype, "o")
    assert_close(ST, rS, dtype, "S_T")
    r = oracle.ref_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], x["do"], dST)
    for gk, rk in GRADS:
        assert_close(gr[gk], r[rk], dtype, gk)


@pytest.mark.parametrize("chunk_decay", [6, 12, 20, 40, 70, 96])
def test_uniform_decay_sweep(cuda_lib, chunk_decay):
    """log alpha = -(chunk_decay / 64) (0.5 + U(0, 1)) on every channel: below and above the
    backward's limit (16) and the forward's (80)."""
    x = make_inputs(1, 256, 2, 128, 128, dtype="bf16", seed=5, with_do=True)
    u = torch.rand(x["log_alpha"].shape, generator=torch.Generator().manual_seed(2))
    x["log_alpha"] = -(chunk_decay / 64.0) * (0.5 + u)
    fwd_bwd_check(x, "bf16")


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("bf16", 64), ("f32", 128), ("f32", 64)])
def test_strong_decay_everywhere(cuda_lib, dtype, D):
    """x_mean = +2: about -135 per chunk on every channel; T = 200 has a ragged last chunk."""
    x = make_inputs(2, 200, 2, D, D, dtype=dtype, seed=71, x_mean=2.0, with_do=True)
    assert float(x["log_alpha"][0, :64].sum(0).min()) < -100.0
    dST = torch.randn(2, 2, D, D, generator=torch.Generator().manual_seed(3))
    fwd_bwd_check(x, dtype, dST)


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("bf16", 64), ("f32", 128), ("f32", 64)])
def test_one_channel_at_minus_ten_per_token(cuda_lib, dtype, D):
    x = make_inputs(2, 256, 2, D, D, dtype=dtype, seed=73, with_do=True)
    x["log_alpha"][..., 5] = -10.0
    fwd_bwd_check(x, dtype)


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("bf16", 64), ("f32", 128)])
def test_strong_decay_in_some_chunks(cuda_lib, dtype, D):
    """Chunks 1 and 4 of 7 (tokens 64-127, 256-319) decay at -4 per token on a quarter of the
    channels; the others follow the recipe.  The two forms alternate along each sequence, in the
    forward, the dS chain and the gradients."""
    x = make_inputs(3, 400, 2, D, D, dtype=dtype, seed=75, with_do=True)
    for a, b in ((64, 128), (256, 320)):
        x["log_alpha"][:, a:b, :, : D // 4] = -4.0
    dST = torch.randn(3, 2, D, D, generator=torch.Generator().manual_seed(5))
    fwd_bwd_check(x, dtype, dST)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_alpha_zero_tokens(cuda_lib, dtype):
    """log alpha = -100 on every channel of a few tokens: alpha underflows to 0 and the state is
    wiped there (the oracle's exp(-100) is 3.7e-44; both are negligible)."""
    D = 128
    x = make_inputs(1, 192, 2, D, D, dtype=dtype, seed=77, with_do=True)
    x["log_alpha"][:, [0, 70, 71, 150]] = -100.0
    fwd_bwd_check(x, dtype)


def test_fused_prologue_with_strong_decay(cuda_lib):
    """The fused input prologue (raw q, k normalised in the kernel; b, w as logits) in chunks that
    run token by token."""
    B, T, H, D = 2, 200, 2, 128
    x = make_inputs(B, T, H, D, D, dtype="bf16", seed=79, raw=True, x_mean=2.0)
    x["q"] = (x["q"].float() * 3.0).to(torch.bfloat16)
    for flags in (g.QK_L2NORM | g.BW_LOGITS, g.QK_L2NORM, g.BW_LOGITS):
        xi = dict(x)
        if not flags & g.BW_LOGITS:
            xi["b"] = torch.sigmoid(x["b"].float()).to(torch.bfloat16)
            xi["w"] = torch.sigmoid(x["w"].float()).to(torch.bfloat16)
        if not flags & g.QK_L2NORM:
            for n in ("q", "k"):
                t = x[n].float()
                xi[n] = (t / t.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
        o, ST = g.gdn2_chunk_fwd_gated(*(dev(xi[n]) for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")),
                                       flags=flags)
        assert g.gdn2_sync_status() == 0
        ro, rS = oracle.ref_fwd_prologue(xi["q"], xi["k"], xi["v"], xi["log_alpha"], xi["b"], xi["w"], xi["S0"],
                                         norm=bool(flags & g.QK_L2NORM), sigmoid=bool(flags & g.BW_LOGITS))
        assert_close(o, ro, "bf16", f"o flags={flags}")
        assert_close(ST, rS, "bf16", f"S_T flags={flags}")


@pytest.mark.parametrize("D", [128, 64])
def test_scalar_decay_strong(cuda_lib, D):
    """One log alpha per (token, head), -3 per token in the second half of the sequence: the
    tensor-core forward's scalar-decay instance, and the backward on the broadcast decay."""
    B, T, H = 2, 260, 2
    x = make_inputs(B, T, H, D, D, dtype="bf16", seed=81, with_do=True)
    gs = -torch.nn.functional.softplus(torch.randn(B, T, H, generator=torch.Generator().manual_seed(2)) - 3.0)
    gs[:, 130:] = -3.0
    o, ST = g.gdn2_chunk_fwd_gated(*(dev(x[n]) for n in ("q", "k", "v")), dev(gs), dev(x["b"]), dev(x["w"]),
                                   dev(x["S0"]), flags=g.DECAY_SCALAR)
    gr = g.gdn2_chunk_bwd_gated(*(dev(x[n]) for n in ("q", "k", "v")), dev(gs), dev(x["b"]), dev(x["w"]),
                                dev(x["S0"]), dev(x["do"]), flags=g.DECAY_SCALAR)
    assert g.gdn2_sync_status() == 0
    gfull = gs[..., None].expand(B, T, H, D).contiguous()
    ro, rS = oracle.ref_fwd(x["q"], x["k"], x["v"], gfull, x["b"], x["w"], x["S0"])
    assert_close(o, ro, "bf16", "o")
    assert_close(ST, rS, "bf16", "S_T")
    r = oracle.ref_bwd(x["q"], x["k"], x["v"], gfull, x["b"], x["w"], x["S0"], x["do"])
    assert_close(gr["dlog_alpha"], r["dg"].sum(-1), "bf16", "dlog_alpha (scalar)")
    for gk, rk in GRADS:
        if gk != "dlog_alpha":
            assert_close(gr[gk], r[rk], "bf16", gk)


def test_scan_with_strong_decay(cuda_lib):
    """The chunk-parallel scan (2 chains of 51 chunks, 3 segments): the middle segment's
    transition and the start states pass through chunks that run token by token."""
    B, T, H, D = 1, 3237, 2, 128
    assert g.gdn2_workspace_size(0, torch.bfloat16, B, T, H, D, D) > 0
    x = make_inputs(B, T, H, D, D, dtype="bf16", seed=83)
    x["log_alpha"][:, 1000:1300, :, :16] = -3.0
    x["log_alpha"][:, 2200:2400] = -2.5
    o, ST = g.gdn2_chunk_fwd(*(dev(x[n]) for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")))
    assert g.gdn2_sync_status() == 0
    ro, rS = oracle.ref_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"])
    assert_close(o, ro, "bf16", "o")
    assert_close(ST, rS, "bf16", "S_T")


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f32", 64)])
def test_varlen_with_strong_decay(cuda_lib, dtype, D):
    lens = [70, 1, 200, 64, 0, 129]
    H = 2
    x = make_inputs(1, sum(lens), H, D, D, dtype=dtype, seed=85, with_do=True, x_mean=1.5)
    S0 = torch.randn(len(lens), H, D, D, generator=torch.Generator().manual_seed(6)) * 0.02
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    d = {k: x[k].cuda() for k in ("q", "k", "v", "log_alpha", "b", "w", "do")}
    o, ST = g.gdn2_chunk_fwd_varlen(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], cu.cuda(), S0.cuda())
    gr = g.gdn2_chunk_bwd_varlen(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], cu.cuda(), S0.cuda(),
                                 d["do"])
    assert g.gdn2_sync_status() == 0
    o, ST = o.cpu(), ST.cpu()
    for n, L in enumerate(lens):
        a, b = int(cu[n]), int(cu[n + 1])
        if L == 0:
            continue
        s = {k: x[k][:, a:b] for k in ("q", "k", "v", "log_alpha", "b", "w", "do")}
        ro, rS = oracle.ref_fwd(s["q"], s["k"], s["v"], s["log_alpha"], s["b"], s["w"], S0[n:n + 1])
        assert_close(o[a:b], ro[0], dtype, f"o seq {n}")
        assert_close(ST[n], rS[0], dtype, f"S_T seq {n}")
        r = oracle.ref_bwd(s["q"], s["k"], s["v"], s["log_alpha"], s["b"], s["w"], S0[n:n + 1], s["do"])
        for gk, rk in GRADS:
            if gk == "dS0":
                assert_close(gr[gk][n], r[rk][0], dtype, f"{gk} seq {n}")
            else:
                assert_close(gr[gk][a:b], r[rk][0], dtype, f"{gk} seq {n}")


def test_training_pair_with_strong_decay(cuda_lib):
    """The forward that records the chunk-boundary states for the backward, with chunks that
    run token by token, gives the plain calls' results bit for bit."""
    x = make_inputs(2, 300, 2, 128, 128, dtype="bf16", seed=87, with_do=True)
    x["log_alpha"][:, 100:200] = -1.5
    d = {n: dev(t) for n, t in x.items()}
    args = (d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    o1, S1, ws = g.gdn2_chunk_fwd_save(*args)
    gr1 = g.gdn2_chunk_bwd_saved(*args, d["do"], workspace=ws)
    o2, S2 = g.gdn2_chunk_fwd(*args)
    gr2 = g.gdn2_chunk_bwd(*args, d["do"])
    assert g.gdn2_sync_status() == 0
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    for k in gr1:
        assert torch.equal(gr1[k], gr2[k]), k
    r = oracle.ref_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], x["do"])
    for gk, rk in GRADS:
        assert_close(gr1[gk], r[rk], "bf16", gk)
