"""GPU parity of gdn2_chunk_fwd against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import checks
from synthetic_inputs import WORKLOADS, make_inputs
from parity import assert_chains_close, assert_close, to_dev

pytestmark = pytest.mark.gpu


def run_fwd(g, x, S0=True, want_state=True):
    d = to_dev(x)
    o, ST = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"],
                             d["S0"] if S0 else None, want_state=want_state)
    assert g.gdn2_sync_status() == 0
    return o, ST


def ref(x, S0=True):
    return oracle.ref_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"] if S0 else None)


def test_tiny_f32_workload(cuda_lib):
    """fp32, B=1, H=2, T=256, d=64, S0 = 0."""
    x = make_inputs(**WORKLOADS["tiny_f32"], seed=0)
    o, ST = run_fwd(cuda_lib, x)
    ro, rS = ref(x)
    assert_close(o, ro, "f32", "o")
    assert_close(ST, rS, "f32", "S_T")


def test_tiny_f32_gate_collapse_and_b_zero(cuda_lib):
    """GPU path with b = w = beta 1 equals KDA; with b = 0 equals the closed form."""
    x = make_inputs(**WORKLOADS["tiny_f32"], seed=0)
    beta = torch.sigmoid(torch.randn(1, 256, 2, generator=torch.Generator().manual_seed(1)))
    xk = dict(x, b=beta[..., None].expand(1, 256, 2, 64).contiguous(),
              w=beta[..., None].expand(1, 256, 2, 64).contiguous())
    o, ST = run_fwd(cuda_lib, xk)
    ro, rS = checks.kda_recurrence(x["q"], x["k"], x["v"], x["log_alpha"], beta, x["S0"])
    assert_close(o, ro, "f32", "o (KDA)")
    assert_close(ST, rS, "f32", "S_T (KDA)")
    xg = dict(x, b=torch.zeros_like(x["b"]))
    o, ST = run_fwd(cuda_lib, xg)
    ro, rS = checks.gla_closed_form(x["q"], x["k"], x["v"], x["log_alpha"], x["w"], x["S0"])
    assert_close(o, ro, "f32", "o (b=0)")
    assert_close(ST, rS, "f32", "S_T (b=0)")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("T", [1, 37, 64, 200, 320])
def test_shapes_and_ragged_lengths(cuda_lib, dtype, D, T):
    x = make_inputs(2, T, 3, D, D, dtype=dtype, seed=T + D)
    o, ST = run_fwd(cuda_lib, x)
    ro, rS = ref(x)
    assert_close(o, ro, dtype, "o")
    assert_close(ST, rS, dtype, "S_T")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_strong_decay_and_wide_erase(cuda_lib, dtype):
    x = make_inputs(2, 256, 2, 128, 128, dtype=dtype, seed=5, x_mean=-1.0, b_scale=2.0)
    o, ST = run_fwd(cuda_lib, x)
    ro, rS = ref(x)
    assert_close(o, ro, dtype, "o")
    assert_close(ST, rS, dtype, "S_T")


def test_zero_length_and_optional_state(cuda_lib):
    g = cuda_lib
    x = make_inputs(2, 0, 2, 64, 64, dtype="bf16", seed=1)
    o, ST = run_fwd(g, x)
    assert o.shape[1] == 0
    assert torch.equal(ST.cpu(), x["S0"])
    o, ST = run_fwd(g, x, S0=False)
    assert torch.count_nonzero(ST) == 0
    x = make_inputs(1, 128, 2, 128, 128, dtype="bf16", seed=2)
    o1, _ = run_fwd(g, x, want_state=False)
    o2, ST = run_fwd(g, x)
    assert torch.equal(o1, o2)
    # zero initial state passed as NULL
    o, ST = run_fwd(g, x, S0=False)
    ro, rS = ref(x, S0=False)
    assert_close(o, ro, "bf16", "o")
    assert_close(ST, rS, "bf16", "S_T")


def test_state_in_place_and_resume(cuda_lib):
    """S_T may alias S0; two halves with the state carried equal one call."""
    g = cuda_lib
    x = make_inputs(2, 256, 2, 128, 128, dtype="bf16", seed=3)
    d = to_dev(x)
    o_full, S_full = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    S = d["S0"].clone()
    halves = []
    for sl in (slice(0, 128), slice(128, 256)):
        part = {n: d[n][:, sl].contiguous() for n in ("q", "k", "v", "log_alpha", "b", "w")}
        o, _ = g.gdn2_chunk_fwd(part["q"], part["k"], part["v"], part["log_alpha"], part["b"],
                                part["w"], S, S_T=S)
        halves.append(o)
    torch.cuda.synchronize()
    o_cat = torch.cat(halves, dim=1)
    assert torch.allclose(o_cat.float(), o_full.float(), rtol=0, atol=1e-2)
    assert torch.allclose(S, S_full, rtol=0, atol=1e-4)


def test_side_stream(cuda_lib):
    g = cuda_lib
    x = make_inputs(1, 192, 2, 128, 128, dtype="bf16", seed=4)
    d = to_dev(x)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o, ST = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], stream=s)
    s.synchronize()
    ro, rS = ref(x)
    assert_close(o, ro, "bf16", "o")


def _full_size(g, name):
    """Every (batch, head) chain of a full-size workload against the oracle, one batch row at a
    time (the oracle's inputs for a whole workload do not need to be in host memory at once)."""
    x = make_inputs(**WORKLOADS[name], seed=0)
    o, ST = run_fwd(g, x)
    assert torch.isfinite(o).all() and torch.isfinite(ST).all()
    oc, Sc = o.cpu(), ST.cpu()
    for b in range(x["q"].shape[0]):
        ro, rS = ref({n: t[b:b + 1] for n, t in x.items()})
        assert_chains_close(oc[b], ro[0], "bf16", f"{name} o[{b}]")
        assert_chains_close(Sc[b], rS[0], "bf16", f"{name} S_T[{b}]", head_axis=0)


def test_full_size_layer_4k(cuda_lib):
    """B=8, H=16, T=4096, d=128, bf16: all 128 (b, h) chains against the oracle."""
    _full_size(cuda_lib, "layer_4k")


@pytest.mark.parametrize("name", ["sweep_2k", "sweep_4k", "sweep_8k", "sweep_16k", "sweep_32k"])
def test_full_size_length_sweep(cuda_lib, name):
    _full_size(cuda_lib, name)
