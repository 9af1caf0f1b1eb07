"""The chunkwise backward, restated in fp64 numpy, against the oracle's token adjoint.

The forward inside one chunk (start state S; see test_chunk_algebra.py) is
    L = strict_tril(diag(beta) (K K^T o Gamma)),  T = (I + L)^-1
    U = T diag(beta) V,  W = T diag(beta gamma) K,  U~ = U - W S
    Y = diag(gamma) Q S + (Q K^T o Gamma) U~,       S' = gamma_C S + (diag(D) K)^T U~
with D_s = exp(g_C - g_s). Its reverse, given dY and dS', is the chain rule through these
matrix products, in reverse order:
    dU~ = (Q K^T o Gamma)^T dY + diag(D) K dS';     dS = gamma_C dS' + (diag(gamma) Q)^T dY - W^T dU~
    dT = dU~ (diag(beta) V)^T - dU~ S^T (diag(beta gamma) K)^T;   dL = -T^T dT T^T (strictly lower)
    (and T^T dT T^T = (T^T dU~) U~^T, because U~ = T (diag(beta) V - diag(beta gamma) K S))
plus the terms of Q, K, V, beta and of gamma, Gamma and D, which become gradients of the
in-chunk cumulative log decay g and, by a reverse cumulative sum, of log alpha. This is
the algebra a chunked (tensor-core) backward would follow; the test pins it to the
oracle's token-by-token adjoint for chunk sizes 1..64, partial chunks and packed sequences.
"""
import numpy as np
import pytest


def chunk_backward(q, k, v, la, b, cu, S0, dy, dS_T, C, scale=1.0):
    N, H, dk = q.shape
    dv = v.shape[2]
    out = dict(q=np.zeros_like(q), k=np.zeros_like(k), v=np.zeros_like(v), la=np.zeros_like(la),
               b=np.zeros_like(b), S0=np.zeros((len(cu) - 1, H, dk, dv)))
    for i in range(len(cu) - 1):
        for h in range(H):
            # forward, keeping each chunk's start state
            S = S0[i, h].copy()
            starts = list(range(cu[i], cu[i + 1], C))
            S_in = []
            for c0 in starts:
                c1 = min(c0 + C, cu[i + 1])
                S_in.append(S.copy())
                K, V, bb = k[c0:c1, h], v[c0:c1, h], b[c0:c1, h]
                g = np.cumsum(la[c0:c1, h])
                gam = np.exp(g)
                Dm = g[:, None] - g[None, :]
                Gam = np.where(np.tril(np.ones_like(Dm)) > 0, np.exp(np.minimum(Dm, 0.0)), 0.0)
                T = np.linalg.inv(np.eye(c1 - c0) + np.tril(bb[:, None] * (K @ K.T) * Gam, -1))
                Ut = T @ (bb[:, None] * V) - T @ ((bb * gam)[:, None] * K) @ S
                S = gam[-1] * S + (np.exp(g[-1] - g)[:, None] * K).T @ Ut
            # backward over the chunks in reverse
            dS = dS_T[i, h].copy()
            for c0, S in zip(reversed(starts), reversed(S_in)):
                c1 = min(c0 + C, cu[i + 1])
                n = c1 - c0
                K, V, bb = k[c0:c1, h], v[c0:c1, h], b[c0:c1, h]
                Q = scale * q[c0:c1, h]
                dY = dy[c0:c1, h]
                g = np.cumsum(la[c0:c1, h])
                gam = np.exp(g)
                Dm = g[:, None] - g[None, :]
                mask = np.tril(np.ones((n, n)))
                Gam = np.where(mask > 0, np.exp(np.minimum(Dm, 0.0)), 0.0)
                A = K @ K.T
                L = np.tril(bb[:, None] * A * Gam, -1)
                T = np.linalg.inv(np.eye(n) + L)
                bV, bgK = bb[:, None] * V, (bb * gam)[:, None] * K
                U, W = T @ bV, T @ bgK
                Ut = U - W @ S
                QK = Q @ K.T
                P = QK * Gam
                D = np.exp(g[-1] - g)
                Kd = D[:, None] * K
                dSp = dS                                   # dL/dS' of this chunk
                # S' = gamma_C S + Kd^T Ut
                dS_new = gam[-1] * dSp
                dKd = Ut @ dSp.T
                dUt = Kd @ dSp
                dgamC = np.sum(dSp * S)
                # Y = diag(gam) Q S + P Ut
                dUt += P.T @ dY
                dP = dY @ Ut.T
                dQ = gam[:, None] * (dY @ S.T)
                dS_new += Q.T @ (gam[:, None] * dY)
                dgam = np.sum((Q @ S) * dY, axis=1)
                # P = QK o Gam
                dQ += (dP * Gam) @ K
                dK = (dP * Gam).T @ Q
                dGam = dP * QK * mask
                # Ut = U - W S
                dU, dW = dUt, -dUt @ S.T
                dS_new += -W.T @ dUt
                # U = T bV, W = T bgK
                dT = dU @ bV.T + dW @ bgK.T
                TdU, TdW = T.T @ dU, T.T @ dW
                dV = bb[:, None] * TdU
                db = np.sum(V * TdU, axis=1) + gam * np.sum(K * TdW, axis=1)
                dK += (bb * gam)[:, None] * TdW
                dgam += bb * np.sum(K * TdW, axis=1)
                # T = (I + L)^-1; since U~ = T Z with Z = bV - bgK S and dT = dU~ Z^T, the
                # product T^T dT T^T is (T^T dU~) U~^T, the form the kernels take
                dL = np.tril(-TdU @ Ut.T, -1)
                dL_full = np.tril(-T.T @ dT @ T.T, -1)
                assert np.max(np.abs(dL - dL_full)) <= 1e-12 * max(1.0, np.max(np.abs(dL_full)))
                # L = strict_tril(diag(b) (A o Gam))
                db += np.sum(dL * A * Gam, axis=1)
                dA = bb[:, None] * dL * Gam
                dK += (dA + dA.T) @ K
                dGam += dL * bb[:, None] * A
                # Kd = diag(D) K
                dK += D[:, None] * dKd
                dD = np.sum(K * dKd, axis=1)
                # decays -> g -> log alpha
                dg = gam * dgam
                GG = dGam * Gam
                dg += GG.sum(axis=1) - GG.sum(axis=0)
                dg -= dD * D
                dg[-1] += np.sum(dD * D) + gam[-1] * dgamC
                out["la"][c0:c1, h] = np.cumsum(dg[::-1])[::-1]
                out["q"][c0:c1, h] = scale * dQ
                out["k"][c0:c1, h] = dK
                out["v"][c0:c1, h] = dV
                out["b"][c0:c1, h] = db
                dS = dS_new
            out["S0"][i, h] = dS
    return out


@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_chunk_backward_matches_token_adjoint(oracle_mod, C):
    rng = np.random.default_rng(100 + C)
    lengths = (70, 3, 0, 37)
    H, dk, dv = 2, 5, 4
    N = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    q = rng.standard_normal((N, H, dk))
    k = rng.standard_normal((N, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((N, H, dv))
    la = -np.exp(rng.uniform(-3, 0.5, (1, H))) * np.logaddexp(0, rng.standard_normal((N, H)))
    b = 1 / (1 + np.exp(-rng.standard_normal((N, H))))
    S0 = rng.standard_normal((len(lengths), H, dk, dv)) * 0.2
    dy = rng.standard_normal((N, H, dv))
    dS_T = rng.standard_normal((len(lengths), H, dk, dv))
    ref = dict(zip(("q", "k", "v", "la", "b", "S0"),
                   oracle_mod.backward(q, k, v, la, b, cu, dy, S0=S0, dS_T=dS_T, scale=0.8)))
    got = chunk_backward(q, k, v, la, b, cu, S0, dy, dS_T, C, scale=0.8)
    for name in ref:
        err = np.max(np.abs(got[name] - ref[name])) / np.sqrt(np.mean(ref[name] ** 2))
        assert err < 1e-9, (name, err)
