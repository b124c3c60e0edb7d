"""The algebra the tensor-core kernels are built on, checked in fp64 against the oracle (CPU).

The kernels do not follow the chunked form step by step. They
* fold Diag(gamma) into the state gradient that the dS chain hands to the gradient kernel,
* form the chain from M = Q~ - P W (dS_c = Gm dS_n - W^T K~ (Gm dS_n) + M^T dO),
* split gamma dgamma into a part from the chunk-start state and a part from the update,
* fold the prologue's norms into the solve as row scales (I + R A R)^-1 = R^-1 (I + R^2 A)^-1 R,
* and compose runs of chunks as affine maps of the start state (the chunk-parallel scan).
Each test below writes one of these forms out in NumPy, in the order the kernels use it, and
compares it with the token-recurrence oracle, so that a mistake in the restructured algebra
shows up without a GPU.  (Test code: the forms here share nothing with the CUDA sources.)"""
import numpy as np
import pytest

import oracle


def softplus(x):
    return np.logaddexp(0.0, x)


def chunk_inputs(L, d, seed, decay_mean=-1.0):
    """One head's inputs for L tokens ([L, d] each), a start state, dO and an end-state gradient."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((L, d))
    k = rng.standard_normal((L, d))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    return dict(q=q, k=k, v=rng.standard_normal((L, d)), g=-softplus(rng.standard_normal((L, d)) + decay_mean),
                b=rng.uniform(0.0, 1.0, (L, d)), w=rng.uniform(0.0, 1.0, (L, d)),
                S=0.3 * rng.standard_normal((d, d)), dO=rng.standard_normal((L, d)),
                dSn=rng.standard_normal((d, d)))


def as_bthd(x):
    return x[None, :, None, :]


def factors(q, k, g, b):
    """Decay folding and the state-independent factors of one chunk."""
    G = np.cumsum(g, axis=0)
    Qt, Et, Kt = q * np.exp(G), b * k * np.exp(G), k * np.exp(-G)
    gam = np.exp(G[-1])
    A = np.tril(Et @ Kt.T, -1)
    T = np.linalg.inv(np.eye(len(q)) + A)
    P = np.tril(Qt @ Kt.T)
    return G, Qt, Et, Kt, gam, T, P


def kernel_chunk_fwd(q, k, v, g, b, w, S):
    """The forward kernel's chunk step: U = T (X - E~ S), O = Q~ S + P U, S' = Gm (S + K~^T U)."""
    _, Qt, Et, Kt, gam, T, P = factors(q, k, g, b)
    U = T @ (w * v - Et @ S)
    return Qt @ S + P @ U, gam[:, None] * (S + Kt.T @ U)


def kernel_chunk_bwd(q, k, v, g, b, w, S, dO, dSn):
    """The backward kernels' chunk step, in the gradient kernel's product order, with the
    chain's state gradient.  dSn is the gradient of the chunk-end state; Gm dSn is what the
    chain stores for the gradient kernel."""
    G, Qt, Et, Kt, gam, T, P = factors(q, k, g, b)
    X = w * v
    U = T @ (X - Et @ S)
    GdS = gam[:, None] * dSn
    dU = P.T @ dO + Kt @ GdS
    dY = T.T @ dU
    dv, dw = dY * w, dY * v
    dP = np.tril(dO @ U.T)
    dA = np.tril(-dY @ U.T, -1)
    dQt = dO @ S.T + dP @ Kt
    dEt = -dY @ S.T + dA @ Kt
    dKt_upd = U @ GdS.T
    dKt = dKt_upd + dP.T @ Qt + dA.T @ Et
    e, em = np.exp(G), np.exp(-G)
    de = dEt * e
    grads = dict(dq=dQt * e, db=de * k, dk=de * b + dKt * em, dv=dv, dw=dw)
    dG = dQt * Qt + dEt * Et - dKt * Kt
    # gamma dgamma = gamma rowsum(dS_n . S) + gamma rowsum(dS_n . K~^T U): the second part as the
    # sum over tokens of K~ . dK~'s update part
    dG[-1] += (GdS * S).sum(axis=1) + (Kt * dKt_upd).sum(axis=0)
    grads["dg"] = np.cumsum(dG[::-1], axis=0)[::-1]
    W = T @ Et
    M = Qt - P @ W
    grads["dS0"] = GdS - W.T @ (Kt @ GdS) + M.T @ dO
    return grads


@pytest.mark.parametrize("L", [16, 11, 1])
def test_chunk_forward_equals_token_recurrence(L):
    x = chunk_inputs(L, 8, seed=L)
    O, Sn = kernel_chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["b"], x["w"], x["S"])
    ro, rS = oracle.ref_fwd(*(as_bthd(x[n]) for n in "qkvgbw"), x["S"][None, None])
    np.testing.assert_allclose(O, ro[0, :, 0], rtol=0, atol=1e-12 * np.abs(ro).max())
    np.testing.assert_allclose(Sn, rS[0, 0], rtol=0, atol=1e-12 * np.abs(rS).max())


@pytest.mark.parametrize("L", [16, 11, 1])
def test_chunk_backward_equals_oracle(L):
    """One chunk: the gradient kernel's products, the factor chain with the gamma dgamma split,
    and the chain's dS_c = Gm dS_n - W^T K~ (Gm dS_n) + M^T dO."""
    x = chunk_inputs(L, 8, seed=100 + L)
    got = kernel_chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["b"], x["w"], x["S"], x["dO"], x["dSn"])
    ref = oracle.ref_bwd(*(as_bthd(x[n]) for n in "qkvgbw"), x["S"][None, None], as_bthd(x["dO"]),
                         x["dSn"][None, None])
    for key in ("dq", "dk", "dv", "dg", "db", "dw"):
        r = ref[key][0, :, 0]
        np.testing.assert_allclose(got[key], r, rtol=0, atol=1e-10 * np.abs(r).max(), err_msg=key)
    np.testing.assert_allclose(got["dS0"], ref["dS0"][0, 0], rtol=0, atol=1e-10 * np.abs(ref["dS0"]).max())


def test_chunked_backward_over_a_sequence():
    """Several chunks and a ragged tail: chunk-start states from the forward step, the state
    gradient carried newest first through the chain, each chunk's gradients from its own start
    state and end-state gradient, as the three backward launches do."""
    C, T, d = 16, 53, 8
    x = chunk_inputs(T, d, seed=7)
    starts = list(range(0, T, C))
    states, S = [], x["S"]
    for t0 in starts:
        sl = slice(t0, min(T, t0 + C))
        states.append(S)
        _, S = kernel_chunk_fwd(*(x[n][sl] for n in "qkvgbw"), S)
    got = {n: np.zeros_like(x[n[1:]]) for n in ("dq", "dk", "dv", "dg", "db", "dw")}
    dS = x["dSn"]
    for i in reversed(range(len(starts))):
        sl = slice(starts[i], min(T, starts[i] + C))
        gr = kernel_chunk_bwd(*(x[n][sl] for n in "qkvgbw"), states[i], x["dO"][sl], dS)
        for n in got:
            got[n][sl] = gr[n]
        dS = gr["dS0"]
    ref = oracle.ref_bwd(*(as_bthd(x[n]) for n in "qkvgbw"), x["S"][None, None], as_bthd(x["dO"]),
                         x["dSn"][None, None])
    for key in got:
        r = ref[key][0, :, 0]
        np.testing.assert_allclose(got[key], r, rtol=0, atol=1e-10 * np.abs(r).max(), err_msg=key)
    np.testing.assert_allclose(dS, ref["dS0"][0, 0], rtol=0, atol=1e-10 * np.abs(ref["dS0"]).max())


def test_prologue_norms_as_row_scales_of_the_solve():
    """Raw q, k: with R = Diag(1/|k_t|) the normalised problem's A is R A R.  The forward kernel
    solves T'' = (I + R^2 A)^-1 instead, forms U' = T'' (R X - R^2 E~ S), and takes U' where the
    normalised problem takes R U (state update K~^T U', output rows scaled by 1/|q_t|)."""
    L, d = 16, 8
    x = chunk_inputs(L, d, seed=21)
    rng = np.random.default_rng(22)
    q, k = x["q"] * rng.uniform(0.3, 3.0, (L, 1)), x["k"] * rng.uniform(0.3, 3.0, (L, 1))  # raw lengths
    eps = oracle.NORM_EPS
    rk = 1.0 / np.sqrt((k * k).sum(1) + eps)
    rq = 1.0 / np.sqrt((q * q).sum(1) + eps)
    _, Qt, Et, Kt, gam, _, P = factors(q, k, x["g"], x["b"])  # raw-key factors, as the kernel keeps them
    A = np.tril(Et @ Kt.T, -1)
    R = np.diag(rk)
    T2 = np.linalg.inv(np.eye(L) + R @ R @ A)
    np.testing.assert_allclose(np.linalg.inv(np.eye(L) + R @ A @ R), np.linalg.inv(R) @ T2 @ R, rtol=1e-12)
    S = x["S"]
    U2 = T2 @ (rk[:, None] * (x["w"] * x["v"]) - (rk * rk)[:, None] * (Et @ S))
    O = rq[:, None] * (Qt @ S + P @ U2)
    Sn = gam[:, None] * (S + Kt.T @ U2)
    ro, rS = oracle.ref_fwd_prologue(*(as_bthd(a) for a in (q, k, x["v"], x["g"], x["b"], x["w"])), S[None, None],
                                     norm=True, sigmoid=False)
    np.testing.assert_allclose(O, ro[0, :, 0], rtol=0, atol=1e-12 * np.abs(ro).max())
    np.testing.assert_allclose(Sn, rS[0, 0], rtol=0, atol=1e-12 * np.abs(rS).max())


def run_map(x, sl_chunks, S0):
    S = S0
    for sl in sl_chunks:
        _, S = kernel_chunk_fwd(*(x[n][sl] for n in "qkvgbw"), S)
    return S


def test_runs_of_chunks_compose_as_affine_maps():
    """The scan: a run's end state is Phi S_start + S^, where S^ is its end state from a zero start
    and Phi its chain with X = 0 from S = I; the maps of consecutive runs compose."""
    C, T, d = 16, 96, 8
    x = chunk_inputs(T, d, seed=31)
    chunks = [slice(t, t + C) for t in range(0, T, C)]
    runs = [chunks[:2], chunks[2:5], chunks[5:]]
    zero_w = dict(x, w=np.zeros_like(x["w"]))
    maps = [(run_map(zero_w, r, np.eye(d)), run_map(x, r, np.zeros((d, d)))) for r in runs]
    S = x["S"]
    for Phi, Shat in maps:
        S = Phi @ S + Shat
    _, rS = oracle.ref_fwd(*(as_bthd(x[n]) for n in "qkvgbw"), x["S"][None, None])
    np.testing.assert_allclose(S, rS[0, 0], rtol=0, atol=1e-11 * np.abs(rS).max())
    # composing two maps first gives the same end state
    (P0, H0), (P1, H1) = maps[0], maps[1]
    S01 = (P1 @ P0) @ x["S"] + (P1 @ H0 + H1)
    np.testing.assert_allclose(S01, run_map(x, runs[0] + runs[1], x["S"]), rtol=0, atol=1e-12)


def test_a_planted_mistake_in_the_chain_is_caught():
    """Dropping Diag(gamma) from the chain's carried term (dS_c = dS_n - ...) must fail the
    comparison, so the chunk backward test above can see a mistake of that kind."""
    x = chunk_inputs(16, 8, seed=41)
    got = kernel_chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["b"], x["w"], x["S"], x["dO"], x["dSn"])
    _, _, Et, Kt, gam, T, P = factors(x["q"], x["k"], x["g"], x["b"])
    W = T @ Et
    wrong = got["dS0"] - (gam[:, None] * x["dSn"] - W.T @ (Kt @ (gam[:, None] * x["dSn"]))) \
        + (x["dSn"] - W.T @ (Kt @ x["dSn"]))
    ref = oracle.ref_bwd(*(as_bthd(x[n]) for n in "qkvgbw"), x["S"][None, None], as_bthd(x["dO"]),
                         x["dSn"][None, None])["dS0"][0, 0]
    assert np.abs(wrong - ref).max() > 1e-3 * np.abs(ref).max()
