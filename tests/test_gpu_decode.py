"""GPU parity of gdn2_decode_step against the oracle's token recurrence."""
import numpy as np
import pytest
import torch

import oracle
from synthetic_inputs import DECODE_WORKLOAD, DecodeStream
from parity import assert_close, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,D", [("f32", 64), ("f32", 128), ("bf16", 64)])
def test_decode_small(cuda_lib, dtype, D):
    g = cuda_lib
    ds = DecodeStream(3, 4, D, D, dtype=dtype, seed=D)
    S = ds.S0.cuda()
    Sref = ds.S0.double().numpy()
    for _ in range(20):
        x = ds.step()
        d = to_dev(x)
        o = g.gdn2_decode_step(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S)
        ro, Sref = oracle.ref_decode(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], Sref)
        assert_close(o, ro, dtype, "o")
    assert g.gdn2_sync_status() == 0
    assert_close(S, Sref, dtype, "S")


def test_decode_1024_steps_full_size(cuda_lib):
    """256 sequences, H=16, d=128, fp32 state in place, 1024 steps.  Every step's o
    and the final S are compared on a sample of sequences (all heads)."""
    g = cuda_lib
    w = DECODE_WORKLOAD
    ds = DecodeStream(w["N"], w["H"], w["Dk"], w["Dv"], dtype=w["dtype"], seed=0)
    seqs = [0, 97, 201, w["N"] - 1]
    S = ds.S0.cuda()
    Sref = ds.S0[seqs].double().numpy()
    worst = 0.0
    for step in range(w["steps"]):
        x = ds.step()
        d = to_dev(x)
        o = g.gdn2_decode_step(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S)
        xs = {n: t[seqs] for n, t in x.items()}
        ro, Sref = oracle.ref_decode(xs["q"], xs["k"], xs["v"], xs["log_alpha"], xs["b"], xs["w"], Sref)
        worst = max(worst, assert_close(o[seqs], ro, "bf16", f"o step {step}"))
    assert g.gdn2_sync_status() == 0
    assert_close(S[seqs], Sref, "bf16", "final S")
    assert torch.isfinite(S).all()
