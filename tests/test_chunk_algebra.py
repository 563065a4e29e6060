"""The chunk-level algebra the tensor-core kernels are built on, checked in fp64 against the
oracle's per-token rule (field guide §02, steps 1-6) on small random streams.

Per chunk of L tokens with in-chunk decay prefix gamma (gamma_t = g_1 + ... + g_t), with
D_t = e^{gamma_L - gamma_t} and Gamma_ts = e^{gamma_t - gamma_s}:
  A = strictly lower (diag(beta) Gamma o K K^T),  T = (I + A)^-1,
  P = (M o Gamma o Q K^T) T  (M: s <= t),
  R = diag(beta) (V - diag(e^gamma) K S^T),
  y = diag(e^gamma) Q S^T + P R,    S^T <- e^{gamma_L} S^T + K^T diag(D) T R.
Two regroupings of the same update are checked as well: the state update through
W2^T = K^T diag(D) T (no U = T R), and the whole chunk as one affine map of the state,
  S^T <- (e^{gamma_L} I - W2^T diag(beta e^gamma) K) S^T + W2^T diag(beta) V,
  y   = (diag(e^gamma) Q - P diag(beta e^gamma) K) S^T + P diag(beta) V,
which leaves one product with the state per chunk on the sequential path.  A fourth form
software-pipelines the three-round chain: the next chunk's first product splits as
  [K;Q]_{c+1} S_{c+1}^T = e^{gamma_L} [K;Q]_{c+1} S_c^T + X_{c+1} U~_c,
  X_{c+1} = [K;Q]_{c+1} K_c^T,  U~_c = diag(D) T R,
so its state part can run a chunk early, off the chain."""
import numpy as np
import pytest


def _stream(rng, T, dk, dv):
    q = rng.standard_normal((T, dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    g = -rng.uniform(0.0, 3.0, T)
    beta = rng.uniform(0.05, 1.0, T)
    return q, k, v, g, beta


def _chunk_terms(q, k, v, g, beta):
    L = len(g)
    gam = np.cumsum(g)
    Gam = np.exp(np.minimum(gam[:, None] - gam[None, :], 0.0))  # e^{gamma_t - gamma_s}, s <= t
    lower = np.tril(np.ones((L, L)), -1)
    A = lower * (beta[:, None] * Gam * (k @ k.T))
    T = np.linalg.inv(np.eye(L) + A)
    P = (np.tril(np.ones((L, L))) * Gam * (q @ k.T)) @ T
    D = np.exp(gam[-1] - gam)
    return gam, T, P, D


def _run(q, k, v, g, beta, S0, C, form):
    S = S0.T.copy()  # S^T: [d_k, d_v]
    ys = []
    if form == "pipelined":
        return _run_pipelined(q, k, v, g, beta, S0, C)
    for c0 in range(0, len(g), C):
        sl = slice(c0, c0 + C)
        qc, kc, vc, gc, bc = q[sl], k[sl], v[sl], g[sl], beta[sl]
        gam, T, P, D = _chunk_terms(qc, kc, vc, gc, bc)
        eg, eL = np.exp(gam), np.exp(gam[-1])
        if form == "affine":
            W2t = kc.T @ (D[:, None] * T)
            Mc = eL * np.eye(len(S)) - W2t @ ((bc * eg)[:, None] * kc)
            Bc = W2t @ (bc[:, None] * vc)
            Qt = eg[:, None] * qc - P @ ((bc * eg)[:, None] * kc)
            ys.append(Qt @ S + P @ (bc[:, None] * vc))
            S = Mc @ S + Bc
            continue
        R = bc[:, None] * (vc - eg[:, None] * (kc @ S))
        ys.append(eg[:, None] * (qc @ S) + P @ R)
        if form == "w2":
            S = eL * S + (kc.T @ (D[:, None] * T)) @ R
        else:
            S = eL * S + kc.T @ (D[:, None] * (T @ R))
    return np.concatenate(ys), S.T


def _run_pipelined(q, k, v, g, beta, S0, C):
    """Three rounds, with [K S^T ; Q S^T] of each chunk after the first formed from the previous
    chunk's state and its U~ only: e^{gamma_L} (early product) + X U~."""
    S = S0.T.copy()
    ys = []
    carry = None  # (e^{gamma_L} [K;Q]_{c} S_{c-1}^T, X_c U~_{c-1}) for the next chunk
    starts = list(range(0, len(g), C))
    for ci, c0 in enumerate(starts):
        sl = slice(c0, c0 + C)
        qc, kc, vc, gc, bc = q[sl], k[sl], v[sl], g[sl], beta[sl]
        gam, T, P, D = _chunk_terms(qc, kc, vc, gc, bc)
        eg, eL = np.exp(gam), np.exp(gam[-1])
        KQ = np.concatenate([kc, qc])
        first = KQ @ S if carry is None else carry[0] + carry[1]
        KS, QS = first[:len(gc)], first[len(gc):]
        R = bc[:, None] * (vc - eg[:, None] * KS)
        ys.append(eg[:, None] * QS + P @ R)
        Ut = D[:, None] * (T @ R)
        if ci + 1 < len(starts):
            nsl = slice(starts[ci + 1], starts[ci + 1] + C)
            KQn = np.concatenate([k[nsl], q[nsl]])
            carry = (eL * (KQn @ S), (KQn @ kc.T) @ Ut)  # early product; X_{c+1} U~_c
        S = eL * S + kc.T @ Ut
    return np.concatenate(ys), S.T


@pytest.mark.parametrize("form", ["three_rounds", "w2", "affine", "pipelined"])
@pytest.mark.parametrize("T,C", [(1, 64), (63, 64), (64, 64), (65, 64), (200, 64), (37, 16)])
def test_chunk_forms_equal_token_form(oracle_mod, form, T, C):
    rng = np.random.default_rng(7 + T + C)
    dk, dv = 24, 20
    q, k, v, g, beta = _stream(rng, T, dk, dv)
    S0 = rng.standard_normal((dv, dk)) * 0.3
    y_ref, S_ref = oracle_mod.recurrence(q, k, v, g, beta, S0)
    y, S = _run(q, k, v, g, beta, S0, C, form)
    assert np.abs(y - y_ref).max() <= 1e-11 * max(1.0, np.abs(y_ref).max())
    assert np.linalg.norm(S - S_ref) <= 1e-11 * np.linalg.norm(S_ref)


def test_a_dropped_decay_factor_is_caught(oracle_mod):
    """The check above has teeth: the affine form without D in W2^T disagrees."""
    rng = np.random.default_rng(3)
    q, k, v, g, beta = _stream(rng, 100, 16, 12)
    S0 = rng.standard_normal((12, 16)) * 0.3
    y_ref, _ = oracle_mod.recurrence(q, k, v, g, beta, S0)
    orig = _chunk_terms

    def no_decay(*a):
        gam, T, P, D = orig(*a)
        return gam, T, P, np.ones_like(D)

    globals()["_chunk_terms"] = no_decay
    try:
        y, _ = _run(q, k, v, g, beta, S0, 32, "affine")
    finally:
        globals()["_chunk_terms"] = orig
    assert np.abs(y - y_ref).max() > 1e-3
