"""Pins of the oracle's gradients (oracle.backward) against things fixed outside it.

The gradients are those of L = sum_t <dy_t, y_t> + <dS_T, S_T> for the token recurrence of
the joezjh.github.io notes page "Qwen3.8-Flash-Next" (section "Gated DeltaNet 核心机制").
- central finite differences of the forward oracle, along random directions, for every
  input (q, k, v, log alpha, beta, S0), on packed sequences including one longer than the
  oracle's 64-token recomputation segments and an empty one;
- torch autograd of an independent fp64 restatement of the recurrence (written here);
- closed forms with the gates switched off (alpha = 1, beta = 0: the state never changes).
Every pin takes the oracle module (or a mutant of it) as its first argument.
"""
import numpy as np
import pytest
import torch


def _problem(seed, lens=(3, 0, 70, 6), H=2, dk=3, dv=4, gates_off=False):
    rng = np.random.default_rng(seed)
    N = int(sum(lens))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    q = rng.standard_normal((N, H, dk)) * 0.5
    k = rng.standard_normal((N, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((N, H, dv))
    la = -rng.uniform(0.01, 0.5, (N, H))
    b = rng.uniform(0.1, 0.9, (N, H))
    if gates_off:
        la, b = np.zeros((N, H)), np.zeros((N, H))
    S0 = rng.standard_normal((len(lens), H, dk, dv)) * 0.3
    dy = rng.standard_normal((N, H, dv))
    dS_T = rng.standard_normal((len(lens), H, dk, dv))
    return dict(q=q, k=k, v=v, log_alpha=la, beta=b, S0=S0, dy=dy, dS_T=dS_T, cu=cu, scale=0.7)


def _loss(m, P, **over):
    x = dict(P, **over)
    y, S_T, _ = m.recurrent(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["cu"], S0=x["S0"],
                            scale=x["scale"])
    return float(np.sum(y * x["dy"]) + np.sum(S_T * x["dS_T"]))


def _grads(m, P):
    return dict(zip(("q", "k", "v", "log_alpha", "beta", "S0"),
                    m.backward(P["q"], P["k"], P["v"], P["log_alpha"], P["beta"], P["cu"], P["dy"],
                               S0=P["S0"], dS_T=P["dS_T"], scale=P["scale"])))


def pin_finite_differences(m, seed=0):
    P = _problem(seed)
    g = _grads(m, P)
    rng = np.random.default_rng(seed + 100)
    eps = 1e-6
    for name in ("q", "k", "v", "log_alpha", "beta", "S0"):
        d = rng.standard_normal(P[name].shape)
        fd = (_loss(m, P, **{name: P[name] + eps * d}) - _loss(m, P, **{name: P[name] - eps * d})) / (2 * eps)
        an = float(np.sum(g[name] * d))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def _torch_grads(P):
    """Independent fp64 restatement of the recurrence, differentiated by torch autograd."""
    T = {n: torch.tensor(P[n], dtype=torch.float64, requires_grad=True)
         for n in ("q", "k", "v", "log_alpha", "beta", "S0")}
    cu = P["cu"]
    H = P["q"].shape[1]
    loss = torch.zeros((), dtype=torch.float64)
    for i in range(len(cu) - 1):
        for h in range(H):
            S = T["S0"][i, h]
            for t in range(int(cu[i]), int(cu[i + 1])):
                kt, vt, qt = T["k"][t, h], T["v"][t, h], T["q"][t, h]
                S = torch.exp(T["log_alpha"][t, h]) * S
                S = S + T["beta"][t, h] * torch.outer(kt, vt - S.T @ kt)
                loss = loss + torch.dot(torch.from_numpy(P["dy"][t, h]), S.T @ (P["scale"] * qt))
            loss = loss + torch.sum(S * torch.from_numpy(P["dS_T"][i, h]))
    grads = torch.autograd.grad(loss, [T[n] for n in ("q", "k", "v", "log_alpha", "beta", "S0")])
    return dict(zip(("q", "k", "v", "log_alpha", "beta", "S0"), [x.numpy() for x in grads]))


def pin_autograd(m, seed=1):
    P = _problem(seed, lens=(5, 2, 0, 9), dk=4, dv=3)
    g, ref = _grads(m, P), _torch_grads(P)
    for name in ref:
        err = np.max(np.abs(g[name] - ref[name])) / max(1e-300, np.max(np.abs(ref[name])))
        assert err <= 1e-12, (name, err)


def pin_gates_off(m, seed=2):
    """alpha = 1, beta = 0: S_t = S0 for every t, so with G_t = dS_T + sum_{s >= t} scale q_s dy_s^T
    the gradients are dq_t = scale S0 dy_t, dv_t = dk_t = 0, dbeta_t = k_t^T G_t (v_t - S0^T k_t),
    dlog_alpha_t = <G_t, S0> and dS0 = G_1."""
    P = _problem(seed, lens=(6, 4), gates_off=True)
    g = _grads(m, P)
    cu, H, s = P["cu"], P["q"].shape[1], P["scale"]
    for i in range(len(cu) - 1):
        for h in range(H):
            S0 = P["S0"][i, h]
            G = P["dS_T"][i, h].copy()
            for t in range(int(cu[i + 1]) - 1, int(cu[i]) - 1, -1):
                G = G + s * np.outer(P["q"][t, h], P["dy"][t, h])
                kt, vt = P["k"][t, h], P["v"][t, h]
                assert np.allclose(g["q"][t, h], s * S0 @ P["dy"][t, h], rtol=0, atol=1e-13)
                assert np.all(g["v"][t, h] == 0.0) and np.all(g["k"][t, h] == 0.0)
                assert abs(g["beta"][t, h] - kt @ G @ (vt - S0.T @ kt)) <= 1e-12
                assert abs(g["log_alpha"][t, h] - np.sum(G * S0)) <= 1e-12
            assert np.allclose(g["S0"][i, h], G, rtol=0, atol=1e-12)


PINS = [pin_finite_differences, pin_autograd, pin_gates_off]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_backward_pin(oracle_mod, pin):
    pin(oracle_mod)
