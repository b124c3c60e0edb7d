"""GPU parity of gdn2_chunk_bwd against the oracle's reverse-mode recurrence.

The oracle's backward is itself pinned by finite differences (CPU tests)."""
import numpy as np
import pytest
import torch

import oracle
from synthetic_inputs import WORKLOADS, make_inputs
from parity import assert_chains_close, assert_close, to_dev

pytestmark = pytest.mark.gpu

GRADS = (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dlog_alpha", "dg"), ("db", "db"),
         ("dw", "dw"), ("dS0", "dS0"))


def run_bwd(g, x, dST=None, S0=True):
    d = to_dev(x)
    out = g.gdn2_chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"],
                           d["S0"] if S0 else None, d["do"], None if dST is None else dST.cuda())
    assert g.gdn2_sync_status() == 0
    return out


def ref_bwd(x, dST=None, S0=True):
    return oracle.ref_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"],
                         x["S0"] if S0 else None, x["do"], dST)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("D,T", [(64, 64), (64, 200), (128, 128), (128, 37)])
def test_bwd_small(cuda_lib, dtype, D, T):
    x = make_inputs(2, T, 2, D, D, dtype=dtype, seed=T + D, with_do=True)
    dST = torch.randn(2, 2, D, D, generator=torch.Generator().manual_seed(7))
    out = run_bwd(cuda_lib, x, dST)
    r = ref_bwd(x, dST)
    for gk, rk in GRADS:
        assert_close(out[gk], r[rk], dtype, gk)


@pytest.mark.parametrize("D", [128, 64])
def test_bwd_several_chunks_per_block(cuda_lib, D):
    """B=3, T=2000 (31 full chunks and a ragged one of 16 tokens), H=4: 384 chunk tasks, so
    every block of the persistent gradient kernel runs two or three of them, full and ragged
    ones mixed, and the chain runs 32 chunks through its three-stage ring; dS_T is nonzero."""
    x = make_inputs(3, 2000, 4, D, D, dtype="bf16", seed=401 + D, with_do=True)
    dST = torch.randn(3, 4, D, D, generator=torch.Generator().manual_seed(11))
    out = run_bwd(cuda_lib, x, dST)
    r = ref_bwd(x, dST)
    for gk, rk in GRADS:
        assert_close(out[gk], r[rk], "bf16", gk)


def test_bwd_tiny_f32_workload_no_state_grad(cuda_lib):
    x = make_inputs(**WORKLOADS["tiny_f32"], seed=0, with_do=True)
    out = run_bwd(cuda_lib, x)
    r = ref_bwd(x)
    for gk, rk in GRADS:
        assert_close(out[gk], r[rk], "f32", gk)


def test_bwd_zero_length(cuda_lib):
    g = cuda_lib
    x = make_inputs(1, 0, 2, 64, 64, dtype="bf16", seed=0, with_do=True)
    dST = torch.randn(1, 2, 64, 64)
    out = run_bwd(g, x, dST)
    assert torch.equal(out["dS0"].cpu(), dST)


def test_bwd_full_size_layer_4k(cuda_lib):
    """B=8, H=16, T=4096, d=128, bf16, do ~ N(0,1), dS_T = 0: every gradient of all 128 (b, h)
    chains against the oracle, one batch row at a time."""
    x = make_inputs(**WORKLOADS["layer_4k"], seed=0, with_do=True)
    out = run_bwd(cuda_lib, x)
    host = {gk: out[gk].cpu() for gk, _ in GRADS}
    for gk, _ in GRADS:
        assert torch.isfinite(host[gk]).all(), gk
    for b in range(8):
        r = ref_bwd({n: t[b:b + 1] for n, t in x.items()})
        for gk, rk in GRADS:
            assert_chains_close(host[gk][b], r[rk][0], "bf16", f"{gk}[{b}]", head_axis=0 if gk == "dS0" else 1)


@pytest.mark.parametrize("dtype,D,T", [("bf16", 128, 200), ("bf16", 64, 130), ("f32", 64, 100)])
def test_training_pair_equals_plain_calls(cuda_lib, dtype, D, T):
    """gdn2_chunk_fwd_save / gdn2_chunk_bwd_saved give the plain calls' results bit for bit."""
    g = cuda_lib
    x = make_inputs(2, T, 2, D, D, dtype=dtype, seed=61, with_do=True)
    d = to_dev(x)
    args = (d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    o1, S1, ws = g.gdn2_chunk_fwd_save(*args)
    gr1 = g.gdn2_chunk_bwd_saved(*args, d["do"], workspace=ws)
    o2, S2 = g.gdn2_chunk_fwd(*args)
    gr2 = g.gdn2_chunk_bwd(*args, d["do"])
    assert g.gdn2_sync_status() == 0
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    for k in gr1:
        assert torch.equal(gr1[k], gr2[k]), k
    ref = ref_bwd(x)
    for gk, rk in GRADS:
        assert_close(gr1[gk], ref[rk], dtype, gk)
