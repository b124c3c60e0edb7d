"""gdn2_chunk_fwd_host: the forward on host buffers (copies pipelined with the kernels by batch
rows) gives gdn2_chunk_fwd's results bit for bit."""
import pytest
import torch

import gated_delta_rule_78_b200 as g
from synthetic_inputs import make_inputs

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "log_alpha", "b", "w", "S0")


@pytest.mark.parametrize("dtype,B,T,D,pinned,with_s0", [
    ("bf16", 7, 200, 128, True, True),     # one batch row per slice, ragged tail
    ("bf16", 2, 130, 64, True, False),     # two slices, no S0
    ("bf16", 1, 64, 128, False, True),     # one slice, pageable memory
    ("f32", 4, 100, 64, True, True),       # two rows per slice, fp32 path
])
def test_host_forward_equals_device_forward(cuda_lib, dtype, B, T, D, pinned, with_s0):
    H = 2
    x = make_inputs(B, T, H, D, D, dtype=dtype, seed=71)
    hx = {n: (t.pin_memory() if pinned else t.contiguous()) for n, t in x.items()}
    s0 = hx["S0"] if with_s0 else None
    o_h, S_h = g.gdn2_chunk_fwd_host(*(hx[n] for n in NAMES[:6]), s0)
    torch.cuda.synchronize()
    d = {n: t.cuda() for n, t in x.items()}
    o_d, S_d = g.gdn2_chunk_fwd(*(d[n] for n in NAMES[:6]), d["S0"] if with_s0 else None)
    assert g.gdn2_sync_status() == 0
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(S_h, S_d.cpu())


def test_host_forward_zero_length(cuda_lib):
    B, H, D = 3, 2, 64
    x = make_inputs(B, 1, H, D, D, dtype="bf16", seed=73)
    empty = {n: t[:, :0].contiguous() if n != "S0" else t for n, t in x.items()}
    o, S_T = g.gdn2_chunk_fwd_host(*(empty[n] for n in NAMES[:6]), x["S0"])
    torch.cuda.synchronize()
    assert o.shape[1] == 0 and torch.equal(S_T, x["S0"])
    o, S_T = g.gdn2_chunk_fwd_host(*(empty[n] for n in NAMES[:6]), None)
    torch.cuda.synchronize()
    assert torch.count_nonzero(S_T) == 0
