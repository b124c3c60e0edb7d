"""The chunk-parallel scan of the forward (few long chains: at most 48 (batch, head) pairs and
at least 48 chunks).  Over a segment the state map is affine; pass 0 runs segment 0 and, for the
middle segment, its zero-start end state and its transition; a combine gives the later segments
their start states; pass 1 runs them.  The result must match the oracle's token recurrence, and
the serial chunk chain the same call takes when it is given no workspace."""
import pytest
import torch

import gated_delta_rule_78_b200 as g
import oracle
from parity import assert_chains_close, assert_close, bh_slice, l2_rel, sample_pairs
from synthetic_inputs import make_inputs

pytestmark = pytest.mark.gpu


def dev(t):
    return None if t is None else t.cuda()


@pytest.mark.parametrize("D,T,nseg", [(128, 3237, 3), (64, 3237, 3), (128, 8215, 8)])
def test_scan_matches_oracle(cuda_lib, D, T, nseg):
    # T = 3237: 51 chunks, 3 segments of 17 with a ragged last one; T = 8215: 129 chunks, 8 segments
    B, H = 1, 2
    st = 4 * D * D * B * H
    assert g.gdn2_workspace_size(0, torch.bfloat16, B, T, H, D, D) == st * (3 * nseg - 4)  # the scan, nseg segments
    x = make_inputs(B, T, H, D, D, dtype="bf16", seed=51, s0="zeros" if D == 64 else "normal")
    S0 = None if D == 64 else x["S0"]  # d = 64 also covers a missing S0
    o, ST = g.gdn2_chunk_fwd(*(dev(x[n]) for n in ("q", "k", "v", "log_alpha", "b", "w")), dev(S0))
    assert g.gdn2_sync_status() == 0
    ro, rS = oracle.ref_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], S0)
    assert_close(o, ro, "bf16", "o")
    assert_close(ST, rS, "bf16", "S_T")


def test_scan_equals_serial_chain(cuda_lib):
    B, T, H, D = 2, 8192, 8, 128
    x = make_inputs(B, T, H, D, D, dtype="bf16", seed=53)
    args = [dev(x[n]) for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")]
    o1, S1 = g.gdn2_chunk_fwd(*args)                                             # scan
    o2, S2 = g.gdn2_chunk_fwd(*args, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))  # serial
    assert g.gdn2_sync_status() == 0
    assert l2_rel(o1, o2) < 1e-2 and l2_rel(S1, S2) < 1e-2
    pairs = sample_pairs(B, H, 1, seed=5)
    xs = bh_slice({n: x[n] for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")}, pairs)
    ro, rS = oracle.ref_fwd(*(xs[n] for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")))
    oc, Sc = o1.cpu(), S1.cpu()
    for i, (b, h) in enumerate(pairs):
        assert_close(oc[b, :, h], ro[i, :, 0], "bf16", f"o[{b},{h}]")
        assert_close(Sc[b, h], rS[i, 0], "bf16", f"S_T[{b},{h}]")


def test_scan_sweep_32k_all_chains(cuda_lib):
    """The sweep's longest shape (B=2, T=32768, H=16: 32 chains through the scan), every chain
    against the oracle."""
    B, T, H, D = 2, 32768, 16, 128
    assert g.gdn2_workspace_size(0, torch.bfloat16, B, T, H, D, D) > 0
    x = make_inputs(B, T, H, D, D, dtype="bf16", seed=55)
    o, ST = g.gdn2_chunk_fwd(*(dev(x[n]) for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")))
    assert g.gdn2_sync_status() == 0
    oc, Sc = o.cpu(), ST.cpu()
    for b in range(B):
        xs = {n: x[n][b:b + 1] for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")}
        ro, rS = oracle.ref_fwd(*(xs[n] for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")))
        assert_chains_close(oc[b], ro[0], "bf16", f"o[{b}]")
        assert_chains_close(Sc[b], rS[0], "bf16", f"S_T[{b}]", head_axis=0)


def test_scan_long_first_segment(cuda_lib):
    """64 chains (49 to 74): segment 0 twice as long as the two after it."""
    B, T, H, D = 4, 4200, 16, 128  # 66 chunks: 32, 17, 17
    assert g.gdn2_workspace_size(0, torch.bfloat16, B, T, H, D, D) == B * H * D * D * 4 * 5
    x = make_inputs(B, T, H, D, D, dtype="bf16", seed=57)
    args = [dev(x[n]) for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")]
    o1, S1 = g.gdn2_chunk_fwd(*args)                                             # scan
    o2, S2 = g.gdn2_chunk_fwd(*args, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))  # serial
    assert g.gdn2_sync_status() == 0
    assert l2_rel(o1, o2) < 1e-2 and l2_rel(S1, S2) < 1e-2
    pairs = sample_pairs(B, H, 1, seed=7)
    xs = bh_slice({n: x[n] for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")}, pairs)
    ro, rS = oracle.ref_fwd(*(xs[n] for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")))
    oc, Sc = o1.cpu(), S1.cpu()
    for i, (b, h) in enumerate(pairs):
        assert_close(oc[b, :, h], ro[i, :, 0], "bf16", f"o[{b},{h}]")
        assert_close(Sc[b, h], rS[i, 0], "bf16", f"S_T[{b},{h}]")
