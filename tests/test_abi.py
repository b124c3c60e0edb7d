"""The C-ABI library loads, exports every declared symbol, and rejects invalid
arguments with the documented status codes before touching the GPU (CPU only)."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_78_b200 as g

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]

F32, BF16 = 0, 1
P = ctypes.c_void_p(0x7F0000000000)         # aligned stand-in address, never dereferenced
MIS = ctypes.c_void_p(0x7F0000000004)       # 4-byte aligned only
NUL = ctypes.c_void_p(0)
S = ctypes.c_void_p(0)                      # stream


def declared_symbols():
    names = []
    for h in HEADERS:
        text = open(h).read()
        names += re.findall(r"GDN2_API\s+[\w\s\*]+?\b(gdn2_\w+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    return g.load()


def test_library_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert set(g.EXPORTS) <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_strerror_covers_all_codes(lib):
    for code in g.STATUS_NAMES:
        assert len(lib.gdn2_strerror(code)) > 0
    assert lib.gdn2_strerror(12345) == b"unknown status"


def fwd(lib, dt=BF16, B=1, T=64, H=1, Dk=128, Dv=128, q=P, o=P, S0=NUL, ST=NUL):
    return lib.gdn2_chunk_fwd(dt, B, T, H, Dk, Dv, q, P, P, P, P, P, S0, o, ST, NUL, 0, S)


def bwd(lib, dt=BF16, B=1, T=64, H=1, Dk=128, Dv=128, ws=P, ws_bytes=1 << 40, dq=P):
    return lib.gdn2_chunk_bwd(dt, B, T, H, Dk, Dv, P, P, P, P, P, P, NUL, P, NUL,
                              dq, P, P, P, P, P, P, ws, ws_bytes, S)


def dec(lib, dt=BF16, N=1, H=1, Dk=128, Dv=128, S_=P):
    return lib.gdn2_decode_step(dt, N, H, Dk, Dv, P, P, P, P, P, P, S_, P, S)


def test_invalid_arguments_return_status(lib):
    assert fwd(lib, dt=7) == -3
    assert fwd(lib, B=0) == -2
    assert fwd(lib, H=-1) == -2
    assert fwd(lib, T=-5) == -2
    assert fwd(lib, Dk=96, Dv=96) == -8
    assert fwd(lib, Dk=128, Dv=64) == -8
    assert fwd(lib, q=NUL) == -1
    assert fwd(lib, o=NUL) == -1
    assert fwd(lib, q=MIS) == -4
    assert fwd(lib, S0=MIS) == -4
    assert fwd(lib, ST=MIS) == -4
    assert dec(lib, N=0) == -2
    assert dec(lib, S_=NUL) == -1
    assert dec(lib, S_=MIS) == -4
    assert dec(lib, Dk=32, Dv=32) == -8
    assert bwd(lib, dq=NUL) == -1
    assert bwd(lib, ws=NUL) == -5
    assert bwd(lib, ws_bytes=16) == -5
    assert bwd(lib, ws=MIS) == -4


def fwd_v(lib, dt=BF16, N=2, T=64, H=1, Dk=128, cu=P, q=P):
    return lib.gdn2_chunk_fwd_varlen(dt, N, T, H, Dk, Dk, cu, q, P, P, P, P, P, NUL, P, NUL, NUL, 0, S)


def bwd_v(lib, dt=BF16, N=2, T=64, H=1, Dk=128, cu=P, ws=P, ws_bytes=1 << 40):
    return lib.gdn2_chunk_bwd_varlen(dt, N, T, H, Dk, Dk, cu, P, P, P, P, P, P, NUL, P, NUL,
                                     P, P, P, P, P, P, P, ws, ws_bytes, S)


def test_varlen_invalid_arguments_return_status(lib):
    assert fwd_v(lib, cu=NUL) == -1
    assert fwd_v(lib, cu=ctypes.c_void_p(0x7F0000000002)) == -4
    assert fwd_v(lib, q=NUL) == -1
    assert fwd_v(lib, N=0) == -2
    assert fwd_v(lib, Dk=96) == -8
    assert fwd_v(lib, H=70000) == -8
    assert bwd_v(lib, cu=NUL) == -1
    assert bwd_v(lib, ws=NUL) == -5
    assert bwd_v(lib, ws_bytes=16) == -5


def test_varlen_workspace_size(lib):
    assert lib.gdn2_workspace_size(2, BF16, 4, 1000, 16, 128, 128) == 0
    fixed = lib.gdn2_workspace_size(1, BF16, 4, 1024, 16, 128, 128)
    packed = lib.gdn2_workspace_size(3, BF16, 4, 4096, 16, 128, 128)
    # four sequences in 4096 packed rows: room for 64 + 4 chunks per head instead of 4 x 16
    assert fixed < packed < fixed * 1.1
    assert lib.gdn2_workspace_size(3, F32, 4, 4096, 16, 64, 64) > 0
    assert lib.gdn2_workspace_size(3, BF16, 4, 0, 16, 128, 128) == 0


def fwd_g(lib, flags, g=P, b=P, w=P, ws=P, ws_bytes=1 << 40):
    return lib.gdn2_chunk_fwd_gated(flags, BF16, 1, 64, 1, 128, 128, P, P, P, g, b, w, NUL, P, NUL, ws, ws_bytes, S)


def dec_g(lib, flags, g=P, b=P, w=P, ws=NUL, ws_bytes=0):
    return lib.gdn2_decode_step_gated(flags, BF16, 1, 1, 128, 128, P, P, P, g, b, w, P, P, ws, ws_bytes, S)


def test_gated_decode_invalid_arguments_return_status(lib):
    """Every case returns before a launch (the pointers are stand-ins)."""
    assert dec_g(lib, 256) == -8                              # unknown flag bit
    assert dec_g(lib, g.DECAY_SCALAR | g.DECAY_NONE) == -8    # scalar and absent for one gate
    assert dec_g(lib, g.ERASE_SCALAR, b=NUL) == -1            # a scalar gate needs its tensor
    assert dec_g(lib, g.DECAY_SCALAR, g=MIS) == -4
    assert dec_g(lib, 0, w=NUL) == -1                         # so does a per-channel one
    # the prologue as a pass (scalar b logits) needs a workspace; per-channel b, w fuse it
    assert dec_g(lib, g.BW_LOGITS | g.ERASE_SCALAR) == -5
    assert dec_g(lib, g.BW_LOGITS | g.ERASE_SCALAR, ws=MIS, ws_bytes=1 << 20) == -4


def test_gated_flags_and_workspace(lib):
    assert fwd_g(lib, 256) == -8                      # unknown flag bit
    assert fwd_g(lib, g.ERASE_SCALAR | g.ERASE_NONE) == -8  # scalar and absent for one gate
    assert fwd_g(lib, g.ERASE_SCALAR, b=NUL) == -1     # a scalar gate needs its tensor
    assert fwd_g(lib, g.ERASE_SCALAR, ws=NUL) == -5    # and a workspace to broadcast it into
    # per-channel gates need no workspace in the forward
    assert lib.gdn2_workspace_size_gated(0, 0, BF16, 2, 128, 4, 128, 128) == 0
    one = 2 * 128 * 4 * 128 * 2                        # one broadcast bf16 gate
    assert lib.gdn2_workspace_size_gated(0, g.ERASE_SCALAR, BF16, 2, 128, 4, 128, 128) == one
    assert lib.gdn2_workspace_size_gated(0, g.DECAY_NONE, BF16, 2, 128, 4, 128, 128) == 2 * one
    plain = lib.gdn2_workspace_size(1, BF16, 2, 128, 4, 128, 128)
    # scalar b and w together, and a scalar decay, run natively in the bf16 backward (no broadcast
    # gates, no full-size gate gradients); a scalar b alone, or fp32, is broadcast and its
    # gradient summed back
    assert lib.gdn2_workspace_size_gated(1, g.ERASE_SCALAR | g.WRITE_SCALAR, BF16, 2, 128, 4, 128, 128) == plain
    assert lib.gdn2_workspace_size_gated(1, g.ERASE_SCALAR, BF16, 2, 128, 4, 128, 128) == plain + 2 * one
    assert lib.gdn2_workspace_size_gated(1, g.DECAY_SCALAR, BF16, 2, 128, 4, 128, 128) == plain
    gdn = g.DECAY_SCALAR | g.ERASE_SCALAR | g.WRITE_SCALAR
    assert lib.gdn2_workspace_size_gated(1, gdn, BF16, 2, 128, 4, 128, 128) == plain
    assert lib.gdn2_workspace_size_gated(1, g.DECAY_SCALAR, F32, 2, 128, 4, 128, 128) == \
        lib.gdn2_workspace_size(1, F32, 2, 128, 4, 128, 128) + 2 * 2 * one  # fp32: g and dg, 4 bytes each
    plain32 = lib.gdn2_workspace_size(1, F32, 2, 128, 4, 128, 128)
    assert (lib.gdn2_workspace_size_gated(1, g.ERASE_SCALAR | g.WRITE_SCALAR, F32, 2, 128, 4, 128, 128)
            == plain32 + 4 * 2 * one)
    # the decode kernel reads every gate layout as it is: no workspace without the prologue
    for fl in (g.ERASE_SCALAR, g.DECAY_SCALAR | g.ERASE_SCALAR | g.WRITE_SCALAR, g.DECAY_NONE | g.WRITE_NONE):
        assert lib.gdn2_workspace_size_gated(2, fl, BF16, 8, 0, 4, 128, 128) == 0
    # input prologue: fused in the bf16 forward with per-channel gates (no workspace); a pass
    # into the workspace (q_n, k_n, b_s, w_s) everywhere else
    pro = g.QK_L2NORM | g.BW_LOGITS
    assert lib.gdn2_workspace_size_gated(0, pro, BF16, 2, 128, 4, 128, 128) == 0
    assert lib.gdn2_workspace_size_gated(0, g.QK_L2NORM, BF16, 2, 128, 4, 128, 128) == 0
    assert lib.gdn2_workspace_size_gated(0, pro, F32, 2, 128, 4, 64, 64) == 4 * (2 * 128 * 4 * 64 * 4)
    assert lib.gdn2_workspace_size_gated(1, pro, BF16, 2, 128, 4, 128, 128) == plain + 4 * one
    # scalar b logits: q_n, k_n, per-token b_s, w_s, then the broadcast b
    assert lib.gdn2_workspace_size_gated(0, pro | g.ERASE_SCALAR, BF16, 2, 128, 4, 128, 128) == 4 * one + 2 * 128 * 4 * 2
    # decode: fused for per-channel b and w; a scalar b logit goes through the pass
    # (q_n, k_n, w_s per channel, b_s per token, which the kernel then reads as it is)
    assert lib.gdn2_workspace_size_gated(2, g.QK_L2NORM, BF16, 8, 0, 4, 128, 128) == 0
    assert lib.gdn2_workspace_size_gated(2, pro | g.ERASE_SCALAR, BF16, 8, 0, 4, 128, 128) == \
        3 * 8 * 4 * 128 * 2 + 256


def test_workspace_size(lib):
    assert lib.gdn2_workspace_size(0, BF16, 8, 4096, 16, 128, 128) == 0
    need = lib.gdn2_workspace_size(1, BF16, 8, 4096, 16, 128, 128)
    states = 8 * 16 * 64 * 128 * 128 * 4
    assert need >= states
    assert lib.gdn2_workspace_size(1, BF16, 8, 4096, 16, 96, 96) == 0
    assert lib.gdn2_workspace_size(1, 9, 8, 4096, 16, 128, 128) == 0
    assert lib.gdn2_workspace_size(5, BF16, 8, 4096, 16, 128, 128) == 0


def test_missing_library_fails_loudly(tmp_path):
    import importlib
    mod = importlib.import_module("gated_delta_rule_78_b200._lib")
    saved = mod._lib
    try:
        mod._lib = None
        with pytest.raises(OSError):
            mod.load(str(tmp_path / "nope.so"))
    finally:
        mod._lib = saved


def pro(lib, flags=g.QK_L2NORM | g.BW_LOGITS, dt=BF16, N=4, H=2, D=128, q=P, b=P, qn=P):
    return lib.gdn2_prologue(flags, dt, N, H, D, q, P, b, P, qn, P, P, P, S)


def test_prologue_arguments(lib):
    assert pro(lib, flags=256) == -8                  # unknown flag bit
    assert pro(lib, dt=9) == -3
    assert pro(lib, N=-1) == -2
    assert pro(lib, H=0) == -2
    assert pro(lib, D=96) == -8
    assert pro(lib, q=NUL) == -1                      # normalisation needs q
    assert pro(lib, qn=MIS) == -4
    assert pro(lib, b=NUL) == -1                      # logits need b
    assert pro(lib, flags=g.BW_LOGITS | g.ERASE_NONE, b=NUL, q=NUL, qn=NUL, N=0) == 0  # only w is needed
    assert pro(lib, N=0) == 0                         # nothing to do, no launch
    assert pro(lib, flags=g.QK_L2NORM, b=NUL, N=0) == 0  # b unused without BW_LOGITS


def test_forward_workspace_for_the_scan(lib):
    # few long chains: the chunk-parallel scan, (3 nseg - 4) states per chain for nseg segments,
    # the plan chosen by the wave model of the 148 SMs
    st = 128 * 128 * 4
    # 32 chains: segment 0 of twice the length, then four more (5 segments, 11 states)
    assert lib.gdn2_workspace_size(0, BF16, 2, 32768, 16, 128, 128) == 32 * st * 11
    # 2 chains of 48 chunks: 3 equal segments (the minimum of 16 chunks each)
    assert lib.gdn2_workspace_size(0, BF16, 1, 3072, 2, 64, 64) == 2 * 64 * 64 * 4 * 5
    assert lib.gdn2_workspace_size(0, BF16, 1, 3008, 2, 128, 128) == 0   # 47 chunks: serial
    # 64 chains: 3 segments, the first twice as long (a short last one at 63 chunks)
    assert lib.gdn2_workspace_size(0, BF16, 4, 16384, 16, 128, 128) == 64 * st * 5
    assert lib.gdn2_workspace_size(0, BF16, 4, 4032, 16, 128, 128) == 64 * st * 5
    assert lib.gdn2_workspace_size(0, BF16, 5, 16384, 15, 128, 128) == 0  # 75 chains: serial
    assert lib.gdn2_workspace_size(0, BF16, 8, 4096, 16, 128, 128) == 0   # 128 chains: serial
    assert lib.gdn2_workspace_size(0, F32, 2, 32768, 16, 128, 128) == 0   # fp32 path: serial
    # fewer chains get more segments: 16 chains, segment 0 of twice the length and seven more
    # (8 segments; the model gives 171 chunk steps against 172 for six equal ones and 512 serial)
    assert lib.gdn2_workspace_size(0, BF16, 1, 32768, 16, 128, 128) == 16 * st * (3 * 8 - 4)


def test_training_pair_arguments(lib):
    def fsave(ws=P, ws_bytes=1 << 40, T=64, dt=BF16):
        return lib.gdn2_chunk_fwd_save(dt, 1, T, 1, 128, 128, P, P, P, P, P, P, NUL, P, NUL, ws, ws_bytes, S)
    assert fsave(ws=NUL) == -5                        # the states go into the backward's workspace
    assert fsave(ws_bytes=16) == -5
    assert fsave(ws=MIS) == -4
    assert fsave(T=-1) == -2
    assert fsave(dt=7) == -3
    assert lib.gdn2_chunk_bwd_saved(BF16, 1, 64, 1, 128, 128, P, P, P, P, P, P, NUL, P, NUL,
                                    P, P, P, P, P, P, P, NUL, 0, S) == -5


def test_host_forward_arguments(lib):
    def fh(ws=P, ws_bytes=1 << 40, q=P):
        return lib.gdn2_chunk_fwd_host(BF16, 2, 64, 1, 128, 128, q, P, P, P, P, P, NUL, P, NUL, ws, ws_bytes, S)
    assert fh(ws=NUL) == -5
    assert fh(ws_bytes=16) == -5
    assert fh(q=NUL) == -1
    assert fh(ws=MIS) == -4
    # three staging slots of one batch row each (B >= 6): q, k, v, b, w, o bf16, log alpha fp32, S0, S_T
    B, T, H, D = 8, 4096, 16, 128
    tok = T * H * D
    slot = 6 * tok * 2 + tok * 4 + 2 * H * D * D * 4
    assert lib.gdn2_workspace_size(4, BF16, B, T, H, D, D) == 3 * slot
    assert lib.gdn2_workspace_size(4, BF16, B, 0, H, D, D) == 0


def test_selftest_timeout_arguments(lib):
    """The failure-detection self-test validates its limit before it launches anything."""
    assert lib.gdn2_selftest_timeout(0, S) == -2
    assert lib.gdn2_selftest_timeout(-5, S) == -2
    assert lib.gdn2_selftest_timeout(100001, S) == -2
