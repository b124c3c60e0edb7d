"""gdn2_chunk_bwd_noalloc: the backward that takes its scratch from the
library's static device array instead of a caller workspace.

Its gradients must match gdn2_chunk_bwd's on the same inputs, call after call:
the array keeps what the previous call left, so consecutive calls use
different shapes, dtypes and seeds.  Collected last so that it also runs after
every other test in one process."""
import ctypes

import pytest
import torch

import gated_delta_rule_78_b200 as g
from synthetic_inputs import make_inputs
from parity import assert_close, to_dev

GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0")
P = ctypes.c_void_p(0x7F0000000000)         # aligned stand-in address, never dereferenced
NUL = ctypes.c_void_p(0)


def noalloc_raw(lib, dt, B, T, H, D, dq=P):
    return lib.gdn2_chunk_bwd_noalloc(dt, B, T, H, D, D, P, P, P, P, P, P, NUL, P, NUL,
                                      dq, P, P, P, P, P, P, NUL)


def test_noalloc_rejects_before_any_cuda_call():
    """Size and argument errors come back before the library touches a device."""
    lib = g.load()
    assert g.NOALLOC_MAX_SCRATCH_BYTES == 32 << 20
    # fp32, B*H = 1, T = 4096, d = 128 needs 37.25 MiB of scratch: over the limit
    assert lib.gdn2_workspace_size(1, 0, 1, 4096, 1, 128, 128) > g.NOALLOC_MAX_SCRATCH_BYTES
    assert noalloc_raw(lib, 0, 1, 4096, 1, 128) == -9
    # bf16, B*H = 4, T = 4096, d = 128 needs 36.25 MiB
    assert lib.gdn2_workspace_size(1, 1, 1, 4096, 4, 128, 128) > g.NOALLOC_MAX_SCRATCH_BYTES
    assert noalloc_raw(lib, 1, 1, 4096, 4, 128) == -9
    assert b"static" in lib.gdn2_strerror(-9)
    assert noalloc_raw(lib, 1, 1, 64, 1, 96) == -8
    assert noalloc_raw(lib, 7, 1, 64, 1, 128) == -3
    assert noalloc_raw(lib, 1, 0, 64, 1, 128) == -2
    assert noalloc_raw(lib, 1, 1, 64, 1, 128, dq=NUL) == -1


def _grads_like(x):
    d = {n: torch.empty_like(x[n]) for n in ("q", "k", "v", "b", "w")}
    B, T, H, D = x["q"].shape
    return {"dq": d["q"], "dk": d["k"], "dv": d["v"], "db": d["b"], "dw": d["w"],
            "dlog_alpha": torch.empty_like(x["log_alpha"]),
            "dS0": torch.empty(B, H, D, D, dtype=torch.float32, device=x["q"].device)}


# consecutive calls: bf16 d=128 with a ragged tail, then fp32 d=64 with a state
# gradient, then a bf16 case again on new inputs (after the fp32 call's leftovers)
CALLS = [("bf16", 1, 200, 2, 128, 11, False),
         ("f32", 2, 130, 3, 64, 12, True),
         ("bf16", 2, 96, 1, 128, 13, True)]


@pytest.mark.gpu
def test_noalloc_matches_workspace_backward(cuda_lib):
    for dtype, B, T, H, D, seed, with_dst in CALLS:
        tdt = torch.float32 if dtype == "f32" else torch.bfloat16
        assert g.gdn2_workspace_size(1, tdt, B, T, H, D, D) <= g.NOALLOC_MAX_SCRATCH_BYTES
        x = to_dev(make_inputs(B, T, H, D, D, dtype=dtype, seed=seed, with_do=True))
        dST = (torch.randn(B, H, D, D, generator=torch.Generator().manual_seed(seed)).cuda()
               if with_dst else None)
        args = (x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], x["do"], dST)
        # fill the outputs with garbage first: every element must be written
        out = _grads_like(x)
        for t in out.values():
            t.fill_(float("nan"))
        got = cuda_lib.gdn2_chunk_bwd_noalloc(*args, out=out)
        assert cuda_lib.gdn2_sync_status() == 0
        ref = cuda_lib.gdn2_chunk_bwd(*args)
        assert cuda_lib.gdn2_sync_status() == 0
        for n in GRADS:
            assert_close(got[n], ref[n], dtype, f"{n} ({dtype}, T={T}, D={D})")


@pytest.mark.gpu
def test_noalloc_over_limit_writes_nothing(cuda_lib):
    x = to_dev(make_inputs(1, 4096, 4, 128, 128, dtype="bf16", seed=5, with_do=True))
    out = _grads_like(x)
    for t in out.values():
        t.fill_(7.0)
    with pytest.raises(g.Gdn2Error, match="GDN2_ERR_TOO_LARGE"):
        cuda_lib.gdn2_chunk_bwd_noalloc(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"],
                                        x["S0"], x["do"], out=out)
    torch.cuda.synchronize()
    for n in GRADS:
        assert bool((out[n] == 7.0).all()), n
