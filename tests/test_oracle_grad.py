"""Pins for the oracle's reverse-mode backward (CPU only).

* central finite differences of the forward at B=1, H=1, T=32, d=8 (fp64,
  h = 1e-6) for every input and S0, with a nonzero dS_T;
* the token-form backward equals the hand-derived chunkwise backward;
* a backward that applies the gates as post-scaling (instead of inside the
  products) fails the finite-difference check, which shows the check is
  sensitive to where the gates enter.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import checks
from synthetic_inputs import make_inputs

NAMES = ("q", "k", "v", "log_alpha", "b", "w", "S0")


def _setup(T=32, D=8, seed=0):
    x = make_inputs(1, T, 1, D, D, dtype="f32", seed=seed, with_do=True)
    x = {n: t.double().numpy().copy() for n, t in x.items()}
    dST = np.random.default_rng(seed).normal(size=(1, 1, D, D))
    return x, dST


def _loss(x, dST):
    o, ST = oracle.ref_fwd(*(x[n] for n in NAMES))
    return float(np.sum(o * x["do"]) + np.sum(ST * dST))


def _fd(x, dST, h=1e-6):
    grads = {}
    for n in NAMES:
        gr = np.zeros_like(x[n])
        flat = x[n].reshape(-1)
        for i in range(flat.size):
            old = flat[i]
            flat[i] = old + h
            lp = _loss(x, dST)
            flat[i] = old - h
            lm = _loss(x, dST)
            flat[i] = old
            gr.reshape(-1)[i] = (lp - lm) / (2 * h)
        grads[n] = gr
    return grads


_KEY = {"q": "dq", "k": "dk", "v": "dv", "log_alpha": "dg", "b": "db", "w": "dw", "S0": "dS0"}


@pytest.fixture(scope="module")
def fd_case():
    x, dST = _setup()
    return x, dST, _fd(x, dST)


def _relerr(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def test_backward_matches_finite_differences(fd_case):
    x, dST, fd = fd_case
    an = oracle.ref_bwd(*(x[n] for n in NAMES), x["do"], dST)
    for n in NAMES:
        assert _relerr(an[_KEY[n]], fd[n]) < 1e-6, n


@pytest.mark.parametrize("C,T", [(8, 32), (16, 40), (64, 64)])
def test_token_backward_equals_chunked_backward(C, T):
    x, dST = _setup(T=T, seed=3)
    a = oracle.ref_bwd(*(x[n] for n in NAMES), x["do"], dST)
    b = checks.chunked_bwd(*(x[n] for n in NAMES), x["do"], dST, C=C)
    for n in a:
        assert _relerr(a[n], b[n]) < 1e-10, n


def test_post_scaled_gates_fail_the_check(fd_case):
    """Surrogate: gradients of the ungated delta rule, then multiplied by the gates."""
    x, dST, fd = fd_case
    ones_k, ones_v = np.ones_like(x["b"]), np.ones_like(x["w"])
    un = oracle.ref_bwd(x["q"], x["k"], x["v"], x["log_alpha"], ones_k, ones_v, x["S0"], x["do"], dST)
    surrogate = {"dk": un["dk"] * x["b"], "dv": un["dv"] * x["w"], "dq": un["dq"]}
    assert _relerr(surrogate["dk"], fd["k"]) > 1e-2
    assert _relerr(surrogate["dv"], fd["v"]) > 1e-2


def test_backward_ragged_and_multi_head():
    """Several heads and a length that is not a multiple of the checkpoint block."""
    x = make_inputs(2, 70, 3, 6, 5, dtype="f32", seed=4, with_do=True)
    x = {n: t.double().numpy() for n, t in x.items()}
    a = oracle.ref_bwd(*(x[n] for n in NAMES), x["do"])
    b = checks.chunked_bwd(*(x[n] for n in NAMES), x["do"], None, C=16)
    for n in a:
        assert _relerr(a[n], b[n]) < 1e-10, n
