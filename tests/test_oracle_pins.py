"""Pins for the fp64 oracle: checks of oracle/ against facts that do not come from it.

Each check uses a formula or fact other than the oracle's own loop:
  * the equivalent update form S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T
    (joezjh.github.io notes, "Gated DeltaNet 核心机制", second display), with explicit
    d_k x d_k matrices;
  * brute-force unrolled matrix products for T <= 8;
  * invariants that follow from the update rule: no-op gates, exact retrieval with
    orthonormal keys, the one-step read-back identity, linearity in (V, S0), and
    split-sequence invariance;
  * a hand-worked example in exact rational arithmetic (tests/golden/hand_example.json);
  * closed forms of the sigmoid-gate zero-centred RMSNorm epilogue.
Shapes use d_k != d_v so that a transposed state fails.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def rand_case(rng, lengths, H, dk, dv, s0=True, unit_k=True):
    N = int(sum(lengths))
    q = rng.standard_normal((N, H, dk))
    k = rng.standard_normal((N, H, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((N, H, dv))
    la = -np.exp(rng.uniform(-1, 1, size=(1, H))) * np.logaddexp(0, rng.standard_normal((N, H)))
    b = 1 / (1 + np.exp(-rng.standard_normal((N, H))))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    S0 = rng.standard_normal((len(lengths), H, dk, dv)) * 0.3 if s0 else None
    return q, k, v, la, b, cu, S0


def alt_form(q, k, v, la, b, cu, S0, scale):
    """The pages' equivalent form with explicit (I - beta k k^T) matrices."""
    N, H, dk = q.shape
    dv = v.shape[2]
    n_seq = len(cu) - 1
    y = np.zeros((N, H, dv))
    ST = np.zeros((n_seq, H, dk, dv))
    I = np.eye(dk)
    for i in range(n_seq):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[i, h].copy()
            for t in range(cu[i], cu[i + 1]):
                kk = k[t, h][:, None]
                A = np.exp(la[t, h]) * (I - b[t, h] * (kk @ kk.T))
                S = A @ S + b[t, h] * kk @ v[t, h][None, :]
                y[t, h] = S.T @ (scale * q[t, h])
            ST[i, h] = S
    return y, ST


def rel(a, b):
    return np.max(np.abs(a - b)) / max(np.sqrt(np.mean(b * b)), 1e-300)


@pytest.mark.parametrize("dk,dv,lengths,H", [(5, 3, (7, 1, 0, 12), 2), (16, 8, (33,), 3),
                                             (4, 6, (3, 9), 1)])
def test_equivalent_form(oracle_mod, dk, dv, lengths, H):
    rng = np.random.default_rng(dk * 100 + dv)
    q, k, v, la, b, cu, S0 = rand_case(rng, lengths, H, dk, dv, unit_k=False)
    for s0 in (None, S0):
        y, ST, _ = oracle_mod.recurrent(q, k, v, la, b, cu, S0=s0, scale=0.7)
        y2, ST2 = alt_form(q, k, v, la, b, cu, s0, 0.7)
        assert rel(y, y2) < 1e-12
        assert rel(ST, ST2) < 1e-12


@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_brute_force_products(oracle_mod, T):
    """S_T = M_T..M_1 S0 + sum_s M_T..M_{s+1} beta_s k_s v_s^T, M_t = alpha_t (I - beta_t k_t k_t^T)."""
    rng = np.random.default_rng(T)
    dk, dv, H = 6, 4, 2
    q, k, v, la, b, cu, S0 = rand_case(rng, (T,), H, dk, dv)
    y, ST, _ = oracle_mod.recurrent(q, k, v, la, b, cu, S0=S0)
    for h in range(H):
        M = [np.exp(la[t, h]) * (np.eye(dk) - b[t, h] * np.outer(k[t, h], k[t, h]))
             for t in range(T)]

        def prod(lo, hi):  # M_{hi-1} ... M_lo  (identity when empty)
            P = np.eye(dk)
            for t in range(lo, hi):
                P = M[t] @ P
            return P

        for t in range(T):
            St = prod(0, t + 1) @ S0[0, h]
            for s in range(t + 1):
                St = St + prod(s + 1, t + 1) @ (b[s, h] * np.outer(k[s, h], v[s, h]))
            assert rel(y[t, h], St.T @ q[t, h]) < 1e-12
        assert rel(ST[0, h], St) < 1e-12


def test_noop_gates(oracle_mod):
    """alpha = 1, beta = 0 leaves S = S0 and reads y_t = S0^T q_t."""
    rng = np.random.default_rng(11)
    q, k, v, la, b, cu, S0 = rand_case(rng, (9, 4), 2, 5, 7)
    la[:] = 0.0
    b[:] = 0.0
    y, ST, _ = oracle_mod.recurrent(q, k, v, la, b, cu, S0=S0)
    assert np.array_equal(ST, S0)
    for i in range(2):
        for t in range(cu[i], cu[i + 1]):
            for h in range(2):
                assert rel(y[t, h], S0[i, h].T @ q[t, h]) < 1e-14


def test_orthonormal_retrieval(oracle_mod):
    """alpha = beta = 1, S0 = 0, orthonormal keys: S_t^T k_s = v_s exactly for s <= t."""
    rng = np.random.default_rng(5)
    dk, dv, T = 12, 5, 12
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm.T[:T][:, None, :]                      # rows are orthonormal keys
    v = rng.standard_normal((T, 1, dv))
    src = [int(rng.integers(0, t + 1)) for t in range(T)]
    q = np.stack([k[s] for s in src])             # query an earlier key
    la = np.zeros((T, 1))
    b = np.ones((T, 1))
    cu = np.array([0, T])
    y, ST, _ = oracle_mod.recurrent(q, k, v, la, b, cu)
    for t in range(T):
        assert np.max(np.abs(y[t, 0] - v[src[t], 0])) < 1e-12
    for s in range(T):
        assert np.max(np.abs(ST[0, 0].T @ k[s, 0] - v[s, 0])) < 1e-12


def test_readback_identity(oracle_mod):
    """For unit k_t: S_t^T k_t = (1 - beta_t) alpha_t S_{t-1}^T k_t + beta_t v_t."""
    rng = np.random.default_rng(21)
    T, H, dk, dv = 10, 2, 8, 3
    q, k, v, la, b, cu, S0 = rand_case(rng, (T,), H, dk, dv)
    q = k.copy()                                  # read back along the key just written
    y, _, _ = oracle_mod.recurrent(q, k, v, la, b, cu, S0=S0)
    for t in range(T):
        if t == 0:
            Sprev = S0[0]
        else:
            _, Sp, _ = oracle_mod.recurrent(q[:t], k[:t], v[:t], la[:t], b[:t],
                                            np.array([0, t]), S0=S0)
            Sprev = Sp[0]
        for h in range(H):
            a, bb = np.exp(la[t, h]), b[t, h]
            want = (1 - bb) * a * (Sprev[h].T @ k[t, h]) + bb * v[t, h]
            assert rel(y[t, h], want) < 1e-12


def test_linearity_in_values_and_state(oracle_mod):
    rng = np.random.default_rng(3)
    q, k, v1, la, b, cu, S01 = rand_case(rng, (6, 11), 2, 7, 4)
    v2 = rng.standard_normal(v1.shape)
    S02 = rng.standard_normal(S01.shape)
    c = -1.7
    ya, Sa, _ = oracle_mod.recurrent(q, k, v1 + c * v2, la, b, cu, S0=S01 + c * S02)
    y1, S1, _ = oracle_mod.recurrent(q, k, v1, la, b, cu, S0=S01)
    y2, S2, _ = oracle_mod.recurrent(q, k, v2, la, b, cu, S0=S02)
    assert rel(ya, y1 + c * y2) < 1e-12
    assert rel(Sa, S1 + c * S2) < 1e-12


def test_split_sequence(oracle_mod):
    """run(T) equals run(T1) followed by run(T - T1) from S_T1, bit for bit."""
    rng = np.random.default_rng(8)
    T, T1 = 23, 9
    q, k, v, la, b, cu, S0 = rand_case(rng, (T,), 3, 6, 5)
    y, ST, _ = oracle_mod.recurrent(q, k, v, la, b, cu, S0=S0)
    ya, Sa, _ = oracle_mod.recurrent(q[:T1], k[:T1], v[:T1], la[:T1], b[:T1],
                                     np.array([0, T1]), S0=S0)
    yb, Sb, _ = oracle_mod.recurrent(q[T1:], k[T1:], v[T1:], la[T1:], b[T1:],
                                     np.array([0, T - T1]), S0=Sa)
    assert np.array_equal(np.concatenate([ya, yb]), y)
    assert np.array_equal(Sb, ST)


def test_threads_do_not_change_results(oracle_mod):
    rng = np.random.default_rng(9)
    q, k, v, la, b, cu, S0 = rand_case(rng, (5, 17, 3), 4, 6, 6)
    y1, S1, n1 = oracle_mod.recurrent(q, k, v, la, b, cu, S0=S0, n_threads=1)
    y4, S4, n4 = oracle_mod.recurrent(q, k, v, la, b, cu, S0=S0, n_threads=4)
    assert n1 == 1 and n4 == 4
    assert np.array_equal(y1, y4) and np.array_equal(S1, S4)


def test_hand_example(oracle_mod):
    g = json.load(open(os.path.join(HERE, "golden", "hand_example.json")))
    r = g["recurrence"]
    # exact rational replay of the worked example: confirms the stored numbers
    S = [[Fraction(0)] * 2 for _ in range(2)]
    for t in range(3):
        a, bb = Fraction(r["alpha"][t]), Fraction(r["beta"][t])
        kt = [Fraction(x) for x in r["k"][t]]
        S = [[a * x for x in row] for row in S]
        e = [Fraction(r["v"][t][j]) - sum(S[i][j] * kt[i] for i in range(2)) for j in range(2)]
        S = [[S[i][j] + bb * kt[i] * e[j] for j in range(2)] for i in range(2)]
        yt = [sum(S[i][j] * r["q"][t][i] for i in range(2)) for j in range(2)]
        assert yt == [Fraction(x) for x in r["y"][t]]
    assert S == [[Fraction(x) for x in row] for row in r["S_T"]]
    q = np.array(r["q"], float)[:, None, :]
    k = np.array(r["k"], float)[:, None, :]
    v = np.array(r["v"], float)[:, None, :]
    la = np.log(np.array(r["alpha"]))[:, None]
    b = np.array(r["beta"])[:, None]
    y, ST, _ = oracle_mod.recurrent(q, k, v, la, b, np.array([0, 3]))
    assert np.max(np.abs(y[:, 0] - np.array(r["y"], float))) < 1e-14
    assert np.max(np.abs(ST[0, 0] - np.array(r["S_T"], float))) < 1e-14
    gn = g["gate_norm"]
    o = oracle_mod.gate_norm(np.array([gn["y"]], float), np.array([gn["z"]], float),
                             np.array(gn["w"], float), eps=gn["eps"])
    assert np.max(np.abs(o[0] - np.array(gn["o"]))) < 1e-15


def test_decode_step_matches_one_token_recurrence(oracle_mod):
    rng = np.random.default_rng(13)
    n, H, dk, dv = 3, 2, 5, 4
    q = rng.standard_normal((n, H, dk))
    k = rng.standard_normal((n, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((n, H, dv))
    alpha = rng.uniform(0.05, 1.0, (n, H))
    beta = rng.uniform(0.0, 1.0, (n, H))
    S = rng.standard_normal((n, H, dk, dv))
    y, Sn = oracle_mod.decode_step(q, k, v, alpha, beta, S, scale=0.5)
    # as a prefill of one token per sequence
    y2, Sn2, _ = oracle_mod.recurrent(q.reshape(n, H, dk), k, v, np.log(alpha), beta,
                                      np.arange(n + 1), S0=S, scale=0.5)
    assert rel(y, y2) < 1e-13 and rel(Sn, Sn2) < 1e-13
    # single-pass identity: y = alpha S^T q + beta (k.q) e with e = v - alpha S^T k
    for i in range(n):
        for h in range(H):
            a, bb = alpha[i, h], beta[i, h]
            e = v[i, h] - a * S[i, h].T @ k[i, h]
            want = 0.5 * (a * S[i, h].T @ q[i, h] + bb * (k[i, h] @ q[i, h]) * e)
            assert rel(y[i, h], want) < 1e-13


def test_gate_norm_closed_forms(oracle_mod):
    rng = np.random.default_rng(17)
    y = rng.standard_normal((40, 16)) * 3.0
    eps = 1e-6
    # sigmoid(z) = 1 exactly in fp64 for z >= 40; w = 0  =>  rms(o) = rms(y)/sqrt(rms(y)^2+eps)
    o = oracle_mod.gate_norm(y, np.full_like(y, 40.0), np.zeros(16), eps=eps)
    ms = np.mean(y * y, axis=1)
    assert np.allclose(np.sqrt(np.mean(o * o, axis=1)), np.sqrt(ms / (ms + eps)), rtol=1e-14)
    # z = 0 => gate 1/2 ; scale invariance with eps = 0
    w = rng.standard_normal(16) * 0.02
    o1 = oracle_mod.gate_norm(y, np.zeros_like(y), w, eps=0.0)
    o2 = oracle_mod.gate_norm(7.5 * y, np.zeros_like(y), w, eps=0.0)
    assert np.allclose(o1, o2, rtol=1e-13, atol=0)
    want = 0.5 * y / np.sqrt(ms)[:, None] * (1 + w)
    assert np.allclose(o1, want, rtol=1e-13, atol=0)
    # a row of zeros stays zero (eps > 0)
    o0 = oracle_mod.gate_norm(np.zeros((1, 16)), np.zeros((1, 16)), w, eps=eps)
    assert np.all(o0 == 0)
