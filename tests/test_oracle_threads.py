"""The oracle threads over (batch, head) pairs only, so its results do not depend on the thread
count (CPU, bit for bit)."""
import numpy as np

import oracle
from synthetic_inputs import DecodeStream, make_inputs


def test_forward_and_backward_do_not_depend_on_threads():
    x = make_inputs(3, 70, 3, 16, 8, dtype="bf16", seed=12, with_do=True)
    arg = (x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"])
    f1, f4 = oracle.ref_fwd(*arg, nthreads=1), oracle.ref_fwd(*arg, nthreads=4)
    for a, b in zip(f1, f4):
        assert np.array_equal(np.asarray(a), np.asarray(b))
    b1 = oracle.ref_bwd(*arg, x["do"], nthreads=1)
    b4 = oracle.ref_bwd(*arg, x["do"], nthreads=4)
    assert b1.keys() == b4.keys()
    for n in b1:
        assert np.array_equal(np.asarray(b1[n]), np.asarray(b4[n])), n


def test_decode_does_not_depend_on_threads():
    ds = DecodeStream(5, 3, 16, 8, dtype="bf16", seed=13)
    s = ds.step()
    arg = (s["q"], s["k"], s["v"], s["log_alpha"], s["b"], s["w"])
    r1 = oracle.ref_decode(*arg, ds.S0, nthreads=1)
    r4 = oracle.ref_decode(*arg, ds.S0, nthreads=4)
    for a, b in zip(r1, r4):
        assert np.array_equal(np.asarray(a), np.asarray(b))
