"""The seeded input recipe both sides consume (CPU): layouts and dtypes, the stated
distributions, the draw order, and determinism.  Distribution checks use enough samples that
the tolerances are several standard errors wide."""
import math

import pytest
import torch

from synthetic_inputs import WORKLOADS, DecodeStream, make_inputs


def test_layouts_and_dtypes():
    x = make_inputs(2, 50, 3, 64, 32, dtype="bf16", seed=1, with_do=True)
    for n in ("q", "k", "b", "log_alpha"):
        assert x[n].shape == (2, 50, 3, 64), n
    for n in ("v", "w", "do"):
        assert x[n].shape == (2, 50, 3, 32), n
    assert x["S0"].shape == (2, 3, 64, 32)
    for n in ("q", "k", "v", "b", "w", "do"):
        assert x[n].dtype == torch.bfloat16, n
    assert x["log_alpha"].dtype == torch.float32 and x["S0"].dtype == torch.float32
    y = make_inputs(1, 8, 2, 16, 16, dtype="f32", seed=1)
    for n in ("q", "k", "v", "b", "w"):
        assert y[n].dtype == torch.float32, n
    assert "do" not in y


def test_q_and_k_are_unit_rows_before_the_cast():
    x = make_inputs(1, 400, 4, 128, 128, dtype="f32", seed=2)
    for n in ("q", "k"):
        norms = x[n].double().norm(dim=-1)
        assert torch.allclose(norms, torch.ones_like(norms), atol=1e-6), n
    xb = make_inputs(1, 400, 4, 128, 128, dtype="bf16", seed=2)
    for n in ("q", "k"):  # the bf16 cast of unit rows: within bf16 rounding of 1, not exactly 1
        norms = xb[n].double().norm(dim=-1)
        assert (norms - 1).abs().max() < 1e-2, n
        assert torch.equal(xb[n], x[n].to(torch.bfloat16)), n


def test_decay_logits_gates_and_initial_state_follow_the_recipe():
    x = make_inputs(4, 512, 4, 128, 128, dtype="f32", seed=3)
    la = x["log_alpha"].double()
    assert (la < 0).all()
    logits = torch.log(torch.expm1(-la))  # softplus^-1 of -log alpha recovers x ~ N(-3, 1)
    n = logits.numel()
    assert abs(logits.mean().item() + 3.0) < 6 / math.sqrt(n)
    assert abs(logits.std().item() - 1.0) < 0.01
    for g in ("b", "w"):  # sigmoid of N(0, 1): inside (0, 1), symmetric about 1/2
        v = x[g].double()
        assert (v > 0).all() and (v < 1).all()
        assert abs(v.mean().item() - 0.5) < 0.005
        z = torch.logit(v)
        assert abs(z.std().item() - 1.0) < 0.01
    s = x["S0"].double()
    assert abs(s.std().item() - 0.02) < 5e-4 and abs(s.mean().item()) < 2e-4
    assert torch.equal(make_inputs(1, 4, 2, 8, 8, seed=0, s0="zeros")["S0"], torch.zeros(1, 2, 8, 8))


def test_knobs_and_raw_draws():
    x = make_inputs(2, 64, 2, 32, 32, dtype="f32", seed=4, b_scale=2.0)
    assert x["b"].max() > 1.0 and x["b"].max() < 2.0
    hi = make_inputs(2, 64, 2, 32, 32, dtype="f32", seed=4, x_mean=0.0)
    assert hi["log_alpha"].mean() < x["log_alpha"].mean()  # larger logits: stronger decay
    raw = make_inputs(2, 64, 2, 32, 32, dtype="f32", seed=4, raw=True)
    cooked = make_inputs(2, 64, 2, 32, 32, dtype="f32", seed=4)
    # the same draws before the prologue: normalising raw q gives the cooked q, sigmoid(raw b)
    # gives the cooked b, and v, log alpha, S0 are untouched
    qn = raw["q"] / torch.sqrt((raw["q"] ** 2).sum(-1, keepdim=True) + 1e-12)
    assert torch.allclose(qn, cooked["q"], atol=1e-7)
    assert torch.allclose(torch.sigmoid(raw["b"]), cooked["b"], atol=1e-7)
    for n in ("v", "log_alpha", "S0"):
        assert torch.equal(raw[n], cooked[n]), n
    assert (raw["b"] < 0).any()  # logits, not gates


def test_seeds_are_deterministic_and_distinct():
    a = make_inputs(1, 32, 2, 16, 16, seed=7, with_do=True)
    b = make_inputs(1, 32, 2, 16, 16, seed=7, with_do=True)
    c = make_inputs(1, 32, 2, 16, 16, seed=8, with_do=True)
    for n in a:
        assert torch.equal(a[n], b[n]), n
        assert not torch.equal(a[n], c[n]), n


def test_decode_stream_draws_steps_in_order():
    s1 = DecodeStream(3, 2, 16, 16, dtype="bf16", seed=5)
    s2 = DecodeStream(3, 2, 16, 16, dtype="bf16", seed=5)
    assert s1.S0.shape == (3, 2, 16, 16) and abs(s1.S0.std().item() - 0.02) < 0.01
    first = s1.step()
    assert first["q"].shape == (3, 2, 16) and first["w"].shape == (3, 2, 16)
    assert first["log_alpha"].dtype == torch.float32 and first["q"].dtype == torch.bfloat16
    second = s1.step()
    assert not torch.equal(first["q"], second["q"])
    again = s2.step()
    for n in first:
        assert torch.equal(first[n], again[n]), n


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_named_workloads_are_well_formed(name):
    w = WORKLOADS[name]
    assert w["Dk"] in (64, 128) and w["Dv"] == w["Dk"] and w["H"] >= 1 and w["B"] >= 1
    assert w["dtype"] in ("f32", "bf16") and w["s0"] in ("normal", "zeros")
    if name.startswith("sweep_"):
        assert w["B"] * w["T"] == 65536  # a fixed 65,536 tokens per call
