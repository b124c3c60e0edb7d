"""GPU parity of the variable-length entry points: N sequences packed along the token
axis, each checked against the oracle run on that sequence alone (from its own S0)."""
import numpy as np
import pytest
import torch

import oracle
from synthetic_inputs import make_inputs
from parity import assert_close

pytestmark = pytest.mark.gpu

LENS = [1, 63, 64, 65, 200, 0, 130, 37]


def packed_inputs(lens, H, D, dtype, seed):
    """One packed [1, total_T, H, D] draw (the recipe of make_inputs) and per-sequence S0."""
    x = make_inputs(1, sum(lens), H, D, D, dtype=dtype, seed=seed, with_do=True)
    gen = torch.Generator().manual_seed(seed + 1)
    S0 = torch.randn(len(lens), H, D, D, generator=gen) * 0.02
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    return x, S0, cu


def seq_slice(x, S0, cu, n):
    a, b = int(cu[n]), int(cu[n + 1])
    s = {k: x[k][:, a:b] for k in ("q", "k", "v", "log_alpha", "b", "w", "do")}
    s["S0"] = S0[n:n + 1]
    return s


def run_varlen_fwd(g, x, S0, cu):
    d = {k: x[k].cuda() for k in ("q", "k", "v", "log_alpha", "b", "w")}
    o, ST = g.gdn2_chunk_fwd_varlen(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], cu.cuda(), S0.cuda())
    assert g.gdn2_sync_status() == 0
    return o.cpu(), ST.cpu()


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f32", 64), ("bf16", 64)])
def test_varlen_forward_matches_each_sequence(cuda_lib, dtype, D):
    x, S0, cu = packed_inputs(LENS, 2, D, dtype, seed=31)
    o, ST = run_varlen_fwd(cuda_lib, x, S0, cu)
    for n, L in enumerate(LENS):
        s = seq_slice(x, S0, cu, n)
        if L == 0:
            assert torch.equal(ST[n], S0[n])
            continue
        ro, rS = oracle.ref_fwd(s["q"], s["k"], s["v"], s["log_alpha"], s["b"], s["w"], s["S0"])
        a, b = int(cu[n]), int(cu[n + 1])
        assert_close(o[a:b], ro[0], dtype, f"o seq {n} (T={L})")
        assert_close(ST[n], rS[0], dtype, f"S_T seq {n} (T={L})")


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f32", 64), ("bf16", 64)])
def test_varlen_backward_matches_each_sequence(cuda_lib, dtype, D):
    g = cuda_lib
    x, S0, cu = packed_inputs(LENS, 2, D, dtype, seed=37)
    dST = torch.randn(len(LENS), 2, D, D, generator=torch.Generator().manual_seed(5))
    d = {k: x[k].cuda() for k in ("q", "k", "v", "log_alpha", "b", "w", "do")}
    out = g.gdn2_chunk_bwd_varlen(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], cu.cuda(), S0.cuda(),
                                  d["do"], dST.cuda())
    assert g.gdn2_sync_status() == 0
    out = {k: t.cpu() for k, t in out.items()}
    pairs = (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dlog_alpha", "dg"), ("db", "db"), ("dw", "dw"))
    for n, L in enumerate(LENS):
        if L == 0:
            assert torch.equal(out["dS0"][n], dST[n])
            continue
        s = seq_slice(x, S0, cu, n)
        r = oracle.ref_bwd(s["q"], s["k"], s["v"], s["log_alpha"], s["b"], s["w"], s["S0"], s["do"], dST[n:n + 1])
        a, b = int(cu[n]), int(cu[n + 1])
        for gk, rk in pairs:
            assert_close(out[gk][a:b], r[rk][0], dtype, f"{gk} seq {n} (T={L})")
        assert_close(out["dS0"][n], r["dS0"][0], dtype, f"dS0 seq {n} (T={L})")


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f32", 64)])
def test_equal_lengths_reproduce_the_fixed_length_call(cuda_lib, dtype, D):
    g = cuda_lib
    N, T, H = 3, 128, 2
    x = make_inputs(N, T, H, D, D, dtype=dtype, seed=41, with_do=True)
    d = {k: t.cuda() for k, t in x.items()}
    o_f, S_f = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    cu = torch.arange(0, (N + 1) * T, T, dtype=torch.int32, device="cuda")
    flat = {k: d[k].reshape(1, N * T, H, D) for k in ("q", "k", "v", "log_alpha", "b", "w", "do")}
    o_v, S_v = g.gdn2_chunk_fwd_varlen(flat["q"], flat["k"], flat["v"], flat["log_alpha"], flat["b"], flat["w"], cu,
                                       d["S0"])
    assert g.gdn2_sync_status() == 0
    assert torch.equal(o_v.reshape(N, T, H, D), o_f)
    assert torch.equal(S_v, S_f)
    gf = g.gdn2_chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"], d["do"])
    gv = g.gdn2_chunk_bwd_varlen(flat["q"], flat["k"], flat["v"], flat["log_alpha"], flat["b"], flat["w"], cu,
                                 d["S0"], flat["do"])
    assert g.gdn2_sync_status() == 0
    for k in ("dq", "dk", "dv", "dlog_alpha", "db", "dw"):
        assert torch.equal(gv[k].reshape(gf[k].shape), gf[k]), k
    assert torch.equal(gv["dS0"], gf["dS0"])


def test_invalid_cu_seqlens_is_reported(cuda_lib):
    """A decreasing cu_seqlens is skipped on the device and reported by gdn2_sync_status."""
    g = cuda_lib
    x, S0, _ = packed_inputs([100, 50], 2, 128, "bf16", seed=3)
    cu = torch.tensor([0, 100, 50, 150], dtype=torch.int32, device="cuda")  # sequence 1 runs backwards
    d = {k: x[k].cuda() for k in ("q", "k", "v", "log_alpha", "b", "w")}
    S0 = torch.zeros(3, 2, 128, 128, device="cuda")
    g.gdn2_chunk_fwd_varlen(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], cu, S0)
    assert g.gdn2_sync_status() == -10  # GDN2_ERR_SEQLENS
    assert g.gdn2_sync_status() == 0    # the status word was cleared
