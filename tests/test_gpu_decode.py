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
    """256 sequences, H=16, d=128, fp32 state in place, 1024 steps.  The oracle advances every
    sequence; o of every sequence is compared at every 64th step and at the last, and the final
    state of every sequence."""
    g = cuda_lib
    w = DECODE_WORKLOAD
    ds = DecodeStream(w["N"], w["H"], w["Dk"], w["Dv"], dtype=w["dtype"], seed=0)
    S = ds.S0.cuda()
    Sref = np.ascontiguousarray(ds.S0.double().numpy())
    checked = 0
    for step in range(w["steps"]):
        x = ds.step()
        d = to_dev(x)
        o = g.gdn2_decode_step(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], S)
        ro, Sref = oracle.ref_decode(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], Sref, inplace=True)
        if step % 64 == 0 or step == w["steps"] - 1:
            oc = o.cpu()
            for n in range(w["N"]):
                assert_close(oc[n], ro[n], "bf16", f"o step {step} seq {n}")
            checked += 1
    assert checked == w["steps"] // 64 + 1
    assert g.gdn2_sync_status() == 0
    Sc = S.cpu()
    assert torch.isfinite(Sc).all()
    for n in range(w["N"]):
        assert_close(Sc[n], Sref[n], "bf16", f"final S seq {n}")
