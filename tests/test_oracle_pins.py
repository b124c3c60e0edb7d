"""Pins for the fp64 CPU oracle's forward and decode (CPU only).

Each check ties the C token recurrence to something other than itself:
separately written recurrences it must reduce to, a closed form, hand-derived
values, exact algebraic properties, and its own chunkwise second form.  The
planted-mistake tests at the end show that plausible slips in the recurrence
fail at least one of these pins.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import checks
from synthetic_inputs import make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _inp(B=2, T=37, H=2, Dk=8, Dv=6, seed=0, **kw):
    return make_inputs(B, T, H, Dk, Dv, dtype="f32", seed=seed, **kw)


def _rel(a, b):
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


def _fwd(x, **over):
    d = dict(x)
    d.update(over)
    return oracle.ref_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], d.get("S0"))


# ---------------------------------------------------------------- hand cases
def test_hand_derived_cases():
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        arr = {n: np.array(c[n], dtype=np.float64)[None, :, None, :] for n in ("q", "k", "v", "g", "b", "w")}
        S0 = np.array(c["S0"], dtype=np.float64)[None, None]
        o, ST = oracle.ref_fwd(arr["q"], arr["k"], arr["v"], arr["g"], arr["b"], arr["w"], S0)
        np.testing.assert_allclose(o[0, :, 0, :], np.array(c["o"]), rtol=1e-14, atol=1e-14, err_msg=c["name"])
        np.testing.assert_allclose(ST[0, 0], np.array(c["ST"]), rtol=1e-14, atol=1e-14, err_msg=c["name"])


# ---------------------------------------------------------------- I1 / I2
def test_collapse_to_kda():
    """b_t = w_t = beta_t 1 must give KDA exactly."""
    x = _inp(seed=1)
    beta = torch.sigmoid(torch.randn(2, 37, 2, generator=torch.Generator().manual_seed(5)))
    bb = beta[..., None].expand(2, 37, 2, 8).double()
    ww = beta[..., None].expand(2, 37, 2, 6).double()
    o1, S1 = _fwd(x, b=bb, w=ww)
    o2, S2 = checks.kda_recurrence(x["q"], x["k"], x["v"], x["log_alpha"], beta, x["S0"])
    assert _rel(o1, o2) < 1e-12 and _rel(S1, S2) < 1e-12


def test_collapse_to_gated_deltanet_and_deltanet():
    """Scalar decay + collapsed gates = Gated DeltaNet; zero decay = DeltaNet."""
    x = _inp(seed=2)
    gen = torch.Generator().manual_seed(6)
    beta = torch.sigmoid(torch.randn(2, 37, 2, generator=gen))
    gs = -torch.nn.functional.softplus(torch.randn(2, 37, 2, generator=gen) - 3)
    bb = beta[..., None].expand(2, 37, 2, 8).double()
    ww = beta[..., None].expand(2, 37, 2, 6).double()
    o1, S1 = _fwd(x, b=bb, w=ww, log_alpha=gs[..., None].expand(2, 37, 2, 8).double())
    o2, S2 = checks.gated_deltanet_recurrence(x["q"], x["k"], x["v"], gs, beta, x["S0"])
    assert _rel(o1, o2) < 1e-12 and _rel(S1, S2) < 1e-12
    o1, S1 = _fwd(x, b=bb, w=ww, log_alpha=torch.zeros(2, 37, 2, 8, dtype=torch.float64))
    o2, S2 = checks.deltanet_recurrence(x["q"], x["k"], x["v"], beta, x["S0"])
    assert _rel(o1, o2) < 1e-12 and _rel(S1, S2) < 1e-12


# ---------------------------------------------------------------- I3
def test_b_zero_is_gated_linear_attention():
    x = _inp(seed=3)
    o1, S1 = _fwd(x, b=torch.zeros_like(x["b"]))
    o2, S2 = checks.gla_closed_form(x["q"], x["k"], x["v"], x["log_alpha"], x["w"], x["S0"])
    assert _rel(o1, o2) < 1e-12 and _rel(S1, S2) < 1e-12


def test_plain_causal_linear_attention():
    """alpha = 1, b = 0, w = 1: o_t = S0^T q_t + sum_{i<=t} (q_t . k_i) v_i."""
    x = _inp(seed=4)
    q, k, v, S0 = (x[n].double().numpy() for n in ("q", "k", "v", "S0"))
    o1, _ = _fwd(x, b=torch.zeros_like(x["b"]), w=torch.ones_like(x["w"]),
                 log_alpha=torch.zeros_like(x["log_alpha"]))
    scores = np.einsum("bthc,bihc->bhti", q, k)
    mask = np.tril(np.ones((q.shape[1], q.shape[1])))
    o2 = np.einsum("bhti,bihd->bthd", scores * mask, v) + np.einsum("bhcd,bthc->bthd", S0, q)
    assert _rel(o1, o2) < 1e-12


# ---------------------------------------------------------------- I4
@pytest.mark.parametrize("C,T", [(16, 64), (16, 37), (64, 200), (8, 8)])
def test_chunked_form_equals_token_form(C, T):
    x = _inp(T=T, seed=10 + C)
    o1, S1 = _fwd(x)
    o2, S2 = checks.chunked_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], C=C)
    assert _rel(o1, o2) < 1e-10 and _rel(S1, S2) < 1e-10


def test_chunked_form_strong_decay_and_wide_erase():
    """Strong decay (large e^{-G} factors) and the b in [0,2] erase range."""
    x = _inp(T=128, seed=11, x_mean=1.0, b_scale=2.0)
    o1, S1 = _fwd(x)
    o2, S2 = checks.chunked_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"], C=64)
    assert _rel(o1, o2) < 1e-9 and _rel(S1, S2) < 1e-9


# ---------------------------------------------------------------- I5
def test_one_hot_keys_update_one_row():
    """k_t = e_j: S[j,:] <- (1-b_j) alpha_j S[j,:] + w.v ; other rows only decay."""
    Dk, Dv = 5, 4
    rng = np.random.default_rng(7)
    S = rng.normal(size=(Dk, Dv))
    for j in range(Dk):
        k = np.zeros(Dk); k[j] = 1.0
        q = rng.normal(size=Dk); v = rng.normal(size=Dv)
        g = -rng.uniform(0, 1, size=Dk); b = rng.uniform(0, 2, size=Dk); w = rng.uniform(0, 1, size=Dv)
        expect = np.exp(g)[:, None] * S
        expect[j] = (1 - b[j]) * np.exp(g[j]) * S[j] + w * v
        args = [a[None, None, None, :] for a in (q, k, v, g, b, w)]
        o, ST = oracle.ref_fwd(*args, S[None, None])
        np.testing.assert_allclose(ST[0, 0], expect, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(o[0, 0, 0], expect.T @ q, rtol=1e-12, atol=1e-12)
        S = expect


def test_orthonormal_keys_exact_retrieval():
    """alpha = 1, b = w = 1, orthonormal keys: after the writes S^T k_j = v of the last write to k_j."""
    D, T = 8, 20
    rng = np.random.default_rng(8)
    Qm, _ = np.linalg.qr(rng.normal(size=(D, D)))
    keys = Qm.T  # rows orthonormal
    idx = rng.integers(0, D, size=T)
    k = keys[idx]
    v = rng.normal(size=(T, D))
    one = np.ones((T, D))
    _, ST = oracle.ref_fwd(rng.normal(size=(1, T, 1, D)), k[None, :, None], v[None, :, None],
                           np.zeros((1, T, 1, D)), one[None, :, None], one[None, :, None],
                           rng.normal(size=(1, 1, D, D)))
    for j in set(idx.tolist()):
        last = max(t for t in range(T) if idx[t] == j)
        np.testing.assert_allclose(ST[0, 0].T @ keys[j], v[last], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- I6 / I7 / I8
def test_linear_in_value_and_initial_state():
    x1, x2 = _inp(seed=20), _inp(seed=21)
    a, c = 0.7, -1.3
    o1, S1 = _fwd(x1)
    o2, S2 = _fwd(x1, v=x2["v"], S0=x2["S0"])
    o3, S3 = _fwd(x1, v=a * x1["v"].double() + c * x2["v"].double(),
                  S0=a * x1["S0"].double() + c * x2["S0"].double())
    assert _rel(o3, a * o1 + c * o2) < 1e-11 and _rel(S3, a * S1 + c * S2) < 1e-11


def test_value_columns_are_separable():
    x = _inp(seed=22)
    perm = torch.randperm(6, generator=torch.Generator().manual_seed(3))
    o1, S1 = _fwd(x)
    o2, S2 = _fwd(x, v=x["v"][..., perm], w=x["w"][..., perm], S0=x["S0"][..., perm])
    np.testing.assert_array_equal(o2, o1[..., perm.numpy()])
    np.testing.assert_array_equal(S2, S1[..., perm.numpy()])


def test_split_sequence_resume():
    x = _inp(T=64, seed=23)
    o, S = _fwd(x)
    h = {n: (t[:, :32] if t.dim() == 4 and n != "S0" else t) for n, t in x.items()}
    o1, S1 = _fwd(h)
    h2 = {n: (t[:, 32:] if t.dim() == 4 and n != "S0" else t) for n, t in x.items()}
    o2, S2 = _fwd(h2, S0=S1)
    assert _rel(np.concatenate([o1, o2], axis=1), o) < 1e-12 and _rel(S2, S) < 1e-12


def test_decode_step_equals_one_token_forward():
    x = _inp(B=3, T=1, seed=24)
    o, S = _fwd(x)
    od, Sd = oracle.ref_decode(x["q"][:, 0], x["k"][:, 0], x["v"][:, 0], x["log_alpha"][:, 0],
                               x["b"][:, 0], x["w"][:, 0], x["S0"])
    np.testing.assert_array_equal(od, o[:, 0])
    np.testing.assert_array_equal(Sd, S)


def test_empty_sequence_returns_initial_state():
    x = _inp(T=0, seed=25)
    o, S = _fwd(x)
    assert o.shape[1] == 0
    np.testing.assert_array_equal(S, x["S0"].double().numpy())


# ---------------------------------------------------------------- planted mistakes
def _token_mutant(x, mistake):
    """NumPy token recurrence with one planted mistake (CPU only)."""
    q, k, v, g, b, w = (x[n].double().numpy() for n in ("q", "k", "v", "log_alpha", "b", "w"))
    S0 = x["S0"].double().numpy()
    B, T, H, Dk = q.shape
    o = np.zeros(v.shape)
    ST = np.zeros(S0.shape)
    for bb in range(B):
        for hh in range(H):
            S = S0[bb, hh].copy()
            for t in range(T):
                a = np.exp(g[bb, t, hh])
                kt, bt, wt, vt, qt = k[bb, t, hh], b[bb, t, hh], w[bb, t, hh], v[bb, t, hh], q[bb, t, hh]
                Sprev = S
                Sp = S if mistake in ("no_decay", "decay_after_write") else a[:, None] * S
                e = kt if mistake == "erase_ignores_b" else bt * kt
                if mistake == "write_gate_on_delta":
                    u = wt * (vt - Sp.T @ e)
                elif mistake == "erase_sign":
                    u = wt * vt + Sp.T @ e
                else:
                    u = wt * vt - Sp.T @ e
                S = Sp + np.outer(kt, u)
                if mistake == "decay_after_write":
                    S = a[:, None] * S
                o[bb, t, hh] = (Sprev if mistake == "output_before_update" else S).T @ qt
            ST[bb, hh] = S
    return o, ST


def _pins_hold(fwd):
    """Run the KDA-collapse, b=0 closed-form and one-hot pins on a forward function."""
    x = _inp(B=1, T=12, H=1, Dk=5, Dv=5, seed=30)
    beta = torch.sigmoid(torch.randn(1, 12, 1, generator=torch.Generator().manual_seed(9)))
    xk = dict(x, b=beta[..., None].expand(1, 12, 1, 5).double(), w=beta[..., None].expand(1, 12, 1, 5).double())
    o1, S1 = fwd(xk)
    o2, S2 = checks.kda_recurrence(x["q"], x["k"], x["v"], x["log_alpha"], beta, x["S0"])
    ok_kda = _rel(o1, o2) < 1e-10 and _rel(S1, S2) < 1e-10
    xg = dict(x, b=torch.zeros_like(x["b"]))
    o1, S1 = fwd(xg)
    o2, S2 = checks.gla_closed_form(x["q"], x["k"], x["v"], x["log_alpha"], x["w"], x["S0"])
    ok_gla = _rel(o1, o2) < 1e-10 and _rel(S1, S2) < 1e-10
    eye = torch.eye(5, dtype=torch.float64)
    xo = dict(x, k=eye[torch.arange(12) % 5][None, :, None, :])
    _, S1 = fwd(xo)
    S = x["S0"].double().numpy()[0, 0].copy()
    bb, ww, vv, gg = (x[n].double().numpy()[0, :, 0] for n in ("b", "w", "v", "log_alpha"))
    for t in range(12):
        j = t % 5
        S = np.exp(gg[t])[:, None] * S
        S[j] = (1 - bb[t, j]) * S[j] + ww[t] * vv[t]
    ok_hot = _rel(S1[0, 0], S) < 1e-10
    return ok_kda and ok_gla and ok_hot


def test_pins_accept_the_oracle():
    assert _pins_hold(lambda d: _fwd(d))
    assert _pins_hold(lambda d: _token_mutant(d, None))


@pytest.mark.parametrize("mistake", ["no_decay", "decay_after_write", "erase_ignores_b",
                                     "write_gate_on_delta", "erase_sign", "output_before_update"])
def test_pins_reject_planted_mistakes(mistake):
    assert not _pins_hold(lambda d: _token_mutant(d, mistake))
