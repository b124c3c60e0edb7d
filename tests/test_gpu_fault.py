"""Failure detection on the GPU without a fault: a bounded wait on an mbarrier phase that
nothing completes gives up, the kernel records a timeout in the status word and returns, the
host reads GDN2_ERR_TIMEOUT, and the context keeps running kernels correctly."""
import pytest
import torch

import oracle
from parity import assert_close, to_dev
from synthetic_inputs import make_inputs

pytestmark = pytest.mark.gpu

GDN2_ERR_TIMEOUT = -7


def test_forced_timeout_is_reported_then_cleared_and_the_context_stays_usable(cuda_lib):
    g = cuda_lib
    assert g.gdn2_sync_status() == 0
    g.gdn2_selftest_timeout(2000)  # one wait of at most 2 ms on a phase nothing completes
    assert g.gdn2_sync_status() == GDN2_ERR_TIMEOUT
    assert g.gdn2_sync_status() == 0  # read and cleared
    x = make_inputs(1, 200, 2, 128, 128, dtype="bf16", seed=91)
    d = to_dev(x)
    o, S_T = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d["S0"])
    assert g.gdn2_sync_status() == 0
    ro, rS = oracle.ref_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"])
    assert_close(o, ro, "bf16", "o")
    assert_close(S_T, rS, "bf16", "S_T")
