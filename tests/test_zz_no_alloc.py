"""gdn2_chunk_bwd_noalloc: the backward that takes its scratch from the
library's static device array instead of a caller workspace, for callers that
cannot allocate device memory when they run it (code inside a memory pool or
allocator, runtimes with a fixed device-memory budget, plain C hosts).

It runs the same kernels on the same workspace layout as gdn2_chunk_bwd, so
its gradients must equal gdn2_chunk_bwd's bit for bit, call after call: the
array keeps what the previous call left, so consecutive calls use different
shapes, dtypes and seeds.  Collected last so that it also runs after every
other test in one process; it passes alone in a fresh process too."""
import ctypes

import pytest
import torch

import gated_delta_rule_78_b200 as g
import oracle
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
    # fp32, B*H = 4, T = 4096, d = 128 needs 48.25 MiB of scratch: over the limit
    assert lib.gdn2_workspace_size(1, 0, 1, 4096, 4, 128, 128) > g.NOALLOC_MAX_SCRATCH_BYTES
    assert noalloc_raw(lib, 0, 1, 4096, 4, 128) == -9
    # bf16, B*H = 4, T = 4096, d = 128 needs 36.25 MiB
    assert lib.gdn2_workspace_size(1, 1, 1, 4096, 4, 128, 128) > g.NOALLOC_MAX_SCRATCH_BYTES
    assert noalloc_raw(lib, 1, 1, 4096, 4, 128) == -9
    assert b"static" in lib.gdn2_strerror(-9)
    assert noalloc_raw(lib, 1, 1, 64, 1, 96) == -8
    assert noalloc_raw(lib, 7, 1, 64, 1, 128) == -3
    assert noalloc_raw(lib, 1, 0, 64, 1, 128) == -2
    assert noalloc_raw(lib, 1, 1, 64, 1, 128, dq=NUL) == -1
    # the same size rules as gdn2_chunk_bwd: more than 65535 heads is outside the contract
    assert noalloc_raw(lib, 1, 1, 64, 70000, 64) == -8
    assert noalloc_raw(lib, 1, 1, 64, 1, 128, dq=ctypes.c_void_p(0x7F0000000004)) == -4


def _grads_like(x):
    d = {n: torch.empty_like(x[n]) for n in ("q", "k", "v", "b", "w")}
    B, T, H, D = x["q"].shape
    return {"dq": d["q"], "dk": d["k"], "dv": d["v"], "db": d["b"], "dw": d["w"],
            "dlog_alpha": torch.empty_like(x["log_alpha"]),
            "dS0": torch.empty(B, H, D, D, dtype=torch.float32, device=x["q"].device)}


# Consecutive calls on the one shared array, each after another's leftovers: bf16 d=128 with a
# ragged tail; bf16 d=64 right after it (the head size that runs zero-padded to 128, where stale
# padded columns would show); fp32 d=64 with a state gradient; bf16 d=128 with decay strong
# enough (x ~ N(+2, 1)) that every chunk takes the token-level gradients and their scratch; and
# bf16 d=128 on new inputs again.  (dtype, B, T, H, D, seed, with dS_T, decay logit mean)
CALLS = [("bf16", 1, 200, 2, 128, 11, False, -3.0),
         ("bf16", 2, 150, 2, 64, 14, True, -3.0),
         ("f32", 2, 130, 3, 64, 12, True, -3.0),
         ("bf16", 1, 160, 2, 128, 15, True, 2.0),
         ("bf16", 2, 96, 1, 128, 13, True, -3.0)]


def _inputs(dtype, B, T, H, D, seed, with_dst, x_mean):
    x = to_dev(make_inputs(B, T, H, D, D, dtype=dtype, seed=seed, with_do=True, x_mean=x_mean))
    dST = (torch.randn(B, H, D, D, generator=torch.Generator().manual_seed(seed)).cuda() if with_dst else None)
    return x, dST


@pytest.mark.gpu
def test_noalloc_matches_workspace_backward(cuda_lib):
    """The same kernels on the same workspace layout: the gradients equal gdn2_chunk_bwd's bit for
    bit, call after call; one call is also checked against the oracle."""
    for dtype, B, T, H, D, seed, with_dst, x_mean in CALLS:
        tdt = torch.float32 if dtype == "f32" else torch.bfloat16
        assert g.gdn2_workspace_size(1, tdt, B, T, H, D, D) <= g.NOALLOC_MAX_SCRATCH_BYTES
        x, dST = _inputs(dtype, B, T, H, D, seed, with_dst, x_mean)
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
            assert torch.equal(got[n], ref[n]), f"{n} ({dtype}, T={T}, D={D}, x_mean={x_mean})"
        if x_mean > 0:  # the token-level gradients ran in the static array: against the oracle too
            xc = {n: t.cpu() for n, t in x.items()}
            r = oracle.ref_bwd(xc["q"], xc["k"], xc["v"], xc["log_alpha"], xc["b"], xc["w"], xc["S0"], xc["do"],
                               None if dST is None else dST.cpu())
            for n, rn in zip(GRADS, ("dq", "dk", "dv", "dg", "db", "dw", "dS0")):
                assert_close(got[n], r[rn], dtype, f"{n} against the oracle")


@pytest.mark.gpu
def test_noalloc_second_call_takes_no_device_memory(cuda_lib):
    """Once a first call has loaded the library's code and committed the array on this device,
    a further call of the same shape leaves the device's free memory where it was."""
    dtype, B, T, H, D, seed, with_dst, x_mean = CALLS[0]
    x, dST = _inputs(dtype, B, T, H, D, seed, with_dst, x_mean)
    out = _grads_like(x)
    args = (x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], x["do"], dST)
    cuda_lib.gdn2_chunk_bwd_noalloc(*args, out=out)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    cuda_lib.gdn2_chunk_bwd_noalloc(*args, out=out)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert cuda_lib.gdn2_sync_status() == 0


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
