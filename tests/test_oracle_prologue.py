"""Pins for the oracle's input prologue (CPU only).

The aixai.ru post's architecture paragraph L2-normalises queries and keys before the
recurrent update and takes the erase and write gates from their own projections
(read here as logits through the logistic sigmoid).  What pins ``oracle.ref_prologue``,
``ref_fwd_prologue`` and ``ref_bwd_prologue``:

* every normalised row has unit length (up to the 1e-6 guard);
* the forward is invariant to a positive rescaling of each token's q and k;
* the sigmoid's closed-form values: logit 0 gives a gate of 1/2 and logit ln 3 gives
  3/4, so the prologue forward equals the plain forward at those gates;
* a logit of -40 closes the erase gate: the forward equals the b = 0 closed form
  (gated additive linear attention) of ``oracle.checks``;
* central finite differences of the composite forward (prologue, then recurrence)
  in the raw q, k and the gate logits at B=1, T=16, H=1, d=8 (fp64);
* a backward that skips the projection term of the normalisation's derivative
  fails that finite-difference check.
"""
import numpy as np
import pytest

import oracle
from oracle import checks
from synthetic_inputs import make_inputs


def _raw(T=16, D=8, seed=0, scale=3.0):
    x = make_inputs(1, T, 1, D, D, dtype="f32", seed=seed, with_do=True, raw=True)
    x = {n: t.double().numpy().copy() for n, t in x.items()}
    x["q"] *= scale  # well away from unit length, so that the normalisation matters
    x["k"] *= scale
    return x


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def test_rows_have_unit_length():
    x = _raw()
    qn, kn, _, _ = oracle.ref_prologue(x["q"], x["k"], x["b"], x["w"])
    for y in (qn, kn):
        n = np.sqrt((y * y).sum(-1))
        assert np.allclose(n, 1.0, atol=1e-6)


def test_rescaling_q_and_k_changes_nothing():
    x = _raw()
    o1, S1 = oracle.ref_fwd_prologue(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"])
    rng = np.random.default_rng(5)
    cq = rng.uniform(0.3, 4.0, size=x["q"].shape[:-1] + (1,))
    ck = rng.uniform(0.3, 4.0, size=x["k"].shape[:-1] + (1,))
    o2, S2 = oracle.ref_fwd_prologue(x["q"] * cq, x["k"] * ck, x["v"], x["log_alpha"], x["b"], x["w"], x["S0"])
    assert _rel(o2, o1) < 1e-6 and _rel(S2, S1) < 1e-6
    # while the recurrence itself is not scale invariant
    o3, _ = oracle.ref_fwd(x["q"] * cq, x["k"] * ck, x["v"], x["log_alpha"], x["b"], x["w"], x["S0"])
    o4, _ = oracle.ref_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"])
    assert _rel(o3, o4) > 1e-2


@pytest.mark.parametrize("logit,gate", [(0.0, 0.5), (np.log(3.0), 0.75)])
def test_sigmoid_closed_form_values(logit, gate):
    x = _raw()
    bl = np.full_like(x["b"], logit)
    wl = np.full_like(x["w"], logit)
    o1, S1 = oracle.ref_fwd_prologue(x["q"], x["k"], x["v"], x["log_alpha"], bl, wl, x["S0"], norm=False)
    o2, S2 = oracle.ref_fwd(x["q"], x["k"], x["v"], x["log_alpha"], np.full_like(bl, gate),
                            np.full_like(wl, gate), x["S0"])
    assert _rel(o1, o2) < 1e-14 and _rel(S1, S2) < 1e-14


def test_closed_erase_gate_is_linear_attention():
    x = _raw()
    bl = np.full_like(x["b"], -40.0)  # sigmoid(-40) ~ 4e-18
    o1, S1 = oracle.ref_fwd_prologue(x["q"], x["k"], x["v"], x["log_alpha"], bl, x["w"], x["S0"])
    qn, kn, _, ws = oracle.ref_prologue(x["q"], x["k"], None, x["w"])
    o2, S2 = checks.gla_closed_form(qn, kn, x["v"], x["log_alpha"], ws, x["S0"])
    assert _rel(o1, o2) < 1e-12 and _rel(S1, S2) < 1e-12


RAW = ("q", "k", "b", "w")
KEY = {"q": "dq", "k": "dk", "b": "db", "w": "dw"}


def _loss(x, dST):
    o, ST = oracle.ref_fwd_prologue(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"])
    return float(np.sum(o * x["do"]) + np.sum(ST * dST))


@pytest.fixture(scope="module")
def fd_case():
    x = _raw()
    dST = np.random.default_rng(1).normal(size=x["S0"].shape)
    h = 1e-6
    grads = {}
    for n in RAW:
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
    return x, dST, grads


def test_backward_matches_finite_differences(fd_case):
    x, dST, fd = fd_case
    g = oracle.ref_bwd_prologue(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], x["do"], dST)
    for n in RAW:
        assert _rel(g[KEY[n]], fd[n]) < 1e-6, n


def test_dropped_projection_term_is_caught(fd_case):
    x, dST, fd = fd_case
    qn, kn, bs, ws = oracle.ref_prologue(x["q"], x["k"], x["b"], x["w"])
    g = oracle.ref_bwd(qn, kn, x["v"], x["log_alpha"], bs, ws, x["S0"], x["do"], dST)
    # dq scaled by r only, without the - q_n (q_n . dq_n) term
    r = 1.0 / np.sqrt((x["q"] * x["q"]).sum(-1, keepdims=True) + oracle.NORM_EPS)
    assert _rel(g["dq"] * r, fd["q"]) > 1e-2
