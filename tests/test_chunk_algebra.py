"""The chunkwise-parallel form, restated in fp64 numpy, against the token recurrence.

The pages give only the token recurrence; the chunked form the CUDA kernels use is
derived from it (by induction over the update rule of the joezjh.github.io notes,
"Gated DeltaNet 核心机制"). With u~_t = beta_t e_t and, inside one chunk of C tokens,
g_t = sum_{r<=t} log alpha_r, gamma_t = exp(g_t), Gamma_ts = exp(g_t - g_s) (s <= t):

    S_t = gamma_t S0 + sum_{s<=t} Gamma_ts k_s u~_s^T
    (I + L) U~ = diag(beta) V - diag(beta gamma) K S0,  L_ts = beta_t Gamma_ts k_t.k_s (s < t)
    T = (I + L)^-1,  U = T diag(beta) V,  W = T diag(beta gamma) K,  U~ = U - W S0
    Y = diag(gamma) Q S0 + tril(Q K^T o Gamma) U~          (diagonal kept: y reads S_t)
    S_C = gamma_C S0 + (diag(gamma_C / gamma) K)^T U~

Every exponent above is <= 0. This test pins that algebra (which the kernels follow)
to the oracle before any kernel is trusted with it, for chunk sizes 1..64, partial
last chunks and packed sequences.
"""
import numpy as np
import pytest


def chunk_form(q, k, v, la, b, cu, S0, C, scale=1.0):
    N, H, dk = q.shape
    dv = v.shape[2]
    y = np.zeros((N, H, dv))
    ST = np.zeros((len(cu) - 1, H, dk, dv))
    for i in range(len(cu) - 1):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[i, h].copy()
            for c0 in range(cu[i], cu[i + 1], C):
                c1 = min(c0 + C, cu[i + 1])
                K, Q, V = k[c0:c1, h], scale * q[c0:c1, h], v[c0:c1, h]
                bb = b[c0:c1, h]
                g = np.cumsum(la[c0:c1, h])
                gam = np.exp(g)
                D = g[:, None] - g[None, :]
                Gam = np.where(np.tril(np.ones_like(D)) > 0, np.exp(np.minimum(D, 0.0)), 0.0)
                L = np.tril(bb[:, None] * (K @ K.T) * Gam, -1)
                T = np.linalg.inv(np.eye(c1 - c0) + L)
                U = T @ (bb[:, None] * V)
                W = T @ ((bb * gam)[:, None] * K)
                Ut = U - W @ S
                P = (Q @ K.T) * Gam
                y[c0:c1, h] = gam[:, None] * (Q @ S) + P @ Ut
                S = gam[-1] * S + (np.exp(g[-1] - g)[:, None] * K).T @ Ut
            ST[i, h] = S
    return y, ST


@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_chunk_form_matches_recurrence(oracle_mod, C):
    rng = np.random.default_rng(C)
    lengths = (70, 3, 129, 0, 64)
    H, dk, dv = 2, 8, 6
    N = sum(lengths)
    q = rng.standard_normal((N, H, dk))
    k = rng.standard_normal((N, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((N, H, dv))
    # strong decay: in-chunk cumulative log decay reaches far below -88 (exp(-g) would overflow fp32)
    la = -np.exp(rng.uniform(-3, 1.5, (1, H))) * np.logaddexp(0, rng.standard_normal((N, H)))
    b = 1 / (1 + np.exp(-rng.standard_normal((N, H))))
    cu = np.concatenate([[0], np.cumsum(lengths)])
    S0 = rng.standard_normal((len(lengths), H, dk, dv)) * 0.1
    y_ref, S_ref, _ = oracle_mod.recurrent(q, k, v, la, b, cu, S0=S0, scale=0.9)
    y, S = chunk_form(q, k, v, la, b, cu, S0, C, scale=0.9)
    scale_y = np.sqrt(np.mean(y_ref ** 2))
    assert np.max(np.abs(y - y_ref)) / scale_y < 1e-10
    assert np.max(np.abs(S - S_ref)) / np.sqrt(np.mean(S_ref ** 2)) < 1e-10
