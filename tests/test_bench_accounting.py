"""bench.py's roofline accounting on CPU: the algorithmic bytes of each call equal the bytes of
the tensors the call reads and writes (counted here from tensors of the recipe's shapes and
dtypes), the peak fallback, and the roofline arithmetic."""
import importlib.util
import json
import os

import pytest
import torch

from synthetic_inputs import DecodeStream, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_acct", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def nbytes(*ts):
    return sum(t.numel() * t.element_size() for t in ts)


@pytest.mark.parametrize("B,T,H,D", [(2, 100, 3, 128), (1, 64, 2, 64)])
def test_forward_bytes_are_the_tensors_read_and_written(bench, B, T, H, D):
    x = make_inputs(B, T, H, D, D, dtype="bf16", seed=0)
    o = torch.empty_like(x["v"])
    S_T = torch.empty_like(x["S0"])
    read = nbytes(*(x[n] for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")))
    assert bench.fwd_bytes(B, T, H, D) == read + nbytes(o, S_T)


def test_forward_bytes_at_the_headline_shape(bench):
    # 2048 B per token-head at d = 128, plus S0 read and S_T written (fp32)
    assert bench.fwd_bytes(8, 4096, 16, 128) == 8 * 4096 * 16 * 2048 + 8 * 16 * 2 * 128 * 128 * 4 == 1090519040


@pytest.mark.parametrize("B,T,H,D", [(2, 100, 3, 128), (1, 64, 2, 64)])
def test_backward_bytes_are_the_tensors_read_and_written(bench, B, T, H, D):
    x = make_inputs(B, T, H, D, D, dtype="bf16", seed=0, with_do=True)
    read = nbytes(*(x[n] for n in ("q", "k", "v", "log_alpha", "b", "w", "S0", "do")))
    grads = [torch.empty_like(x[n]) for n in ("q", "k", "v", "log_alpha", "b", "w", "S0")]
    assert bench.bwd_bytes(B, T, H, D) == read + nbytes(*grads)  # dS_T = 0 is not read


def test_decode_bytes_are_the_state_and_token_vectors(bench):
    N, H, D = 5, 3, 128
    ds = DecodeStream(N, H, D, D, dtype="bf16", seed=0)
    s = ds.step()
    o = torch.empty_like(s["v"])
    tokens = nbytes(*(s[n] for n in ("q", "k", "v", "log_alpha", "b", "w")), o)
    assert bench.decode_bytes(N, H, D) == 2 * nbytes(ds.S0) + tokens


def test_peak_fallback_and_roofline_arithmetic(bench, tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    pk = bench.peaks()  # no MEASURED_PEAKS.json: the recipe's fallback
    assert pk["source"] == "fallback" and pk["hbm_gbs"] == 6650.0 and pk["bf16_tflops"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6000.0, "bf16_tflops": 1500.0}))
    pk = bench.peaks()
    assert pk["source"] == "measured" and pk["hbm_gbs"] == 6000.0
    r = bench.roofline(3_000_000_000, 1.0, pk)  # 3 GB in 1 ms
    assert r["achieved"] == 3000.0 and r["frac"] == 0.5 and r["unit"] == "GB/s" and r["bound"] == "hbm"
    assert r["traffic"] is None and r["algorithmic_bytes"] == 3_000_000_000
