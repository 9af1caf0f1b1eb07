"""Pins of the oracle's featurisation step (oracle.featurize) against things fixed
outside it.

The step is the feature and gate computation in front of the recurrence (joezjh.github.io
notes page "Qwen3.8-Flash-Next", section "GDN 参数化细节"; pwwt.cn translation, section
2.1.1, Figure 2 caption). Each pin below reduces it to a library routine or a closed form:
- the short causal convolution equals torch's depthwise conv1d padded by W-1 and cut to
  its first T outputs, SiLU equals torch's silu and the L2 norm (eps = 0) torch's
  normalize, sequence by sequence;
- a unit impulse reproduces the taps, newest tap first;
- sequences packed together give what each gives alone (nothing crosses cu_seqlens);
- with eps = 0 every q and k row has unit norm, and v rows are not normalised;
- the gates take their closed-form values at chosen logits.
Every pin takes the oracle module (or a mutant of it) as its first argument, so that
test_oracle_mutants.py can run them against planted mistakes.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F


def _inputs(rng, lens, H, dk, dv, W):
    N = int(sum(lens))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    x = [rng.standard_normal((N, H, d)) for d in (dk, dk, dv)]
    cw = [rng.standard_normal((H * d, W)) / math.sqrt(W) for d in (dk, dk, dv)]
    gates = [rng.standard_normal((N, H)), rng.standard_normal((N, H)), rng.uniform(-1, 1, H),
             rng.standard_normal(H)]
    return x, cw, gates, cu


def _library_features(x, cw, cu, l2):
    """torch's depthwise conv1d (+ silu, + normalize) per sequence, fp64."""
    N, H, d = x.shape
    W = cw.shape[1]
    out = np.zeros_like(x)
    wt = torch.from_numpy(cw).reshape(H * d, 1, W)
    for i in range(len(cu) - 1):
        a, b = int(cu[i]), int(cu[i + 1])
        if b == a:
            continue
        seq = torch.from_numpy(np.ascontiguousarray(x[a:b].reshape(b - a, H * d).T))[None]
        c = F.conv1d(seq, wt, padding=W - 1, groups=H * d)[0, :, : b - a]   # [H*d, T]
        f = F.silu(c).T.reshape(b - a, H, d)
        if l2:
            f = F.normalize(f, dim=-1, eps=1e-300)
        out[a:b] = f.numpy()
    return out


def pin_library(m, lens=(5, 1, 9, 3), H=2, dk=8, dv=16, W=4, seed=0):
    rng = np.random.default_rng(seed)
    x, cw, g, cu = _inputs(rng, lens, H, dk, dv, W)
    q, k, v, beta, log_alpha = m.featurize(*x, *cw, *g, cu, eps=0.0)
    for got, xs, c, l2 in ((q, x[0], cw[0], True), (k, x[1], cw[1], True), (v, x[2], cw[2], False)):
        ref = _library_features(xs, c, cu, l2)
        assert np.max(np.abs(got - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))
    bl, al, A, b = g
    assert np.max(np.abs(beta - torch.sigmoid(torch.from_numpy(bl)).numpy())) <= 1e-15
    sp = F.softplus(torch.from_numpy(al + b[None, :]), beta=1.0, threshold=1000.0).numpy()
    assert np.max(np.abs(log_alpha - (-np.exp(A)[None, :] * sp))) <= 1e-12


def pin_impulse(m, W=4, d=4):
    """A unit impulse at token t0 of channel c (v stream): the outputs at t0 + i are
    SiLU of the tap that multiplies the token i places back, i.e. tap W-1-i."""
    N, H, t0, c = 9, 1, 3, 2
    x = [np.zeros((N, H, d)) for _ in range(3)]
    x[2][t0, 0, c] = 1.0
    taps = np.arange(1, W + 1, dtype=np.float64) * 0.25        # distinct: 0.25, 0.5, ...
    cw = [np.zeros((d, W)), np.zeros((d, W)), np.zeros((d, W))]
    cw[2][c] = taps
    zeros = np.zeros((N, H))
    _, _, v, _, _ = m.featurize(*x, *cw, zeros, zeros, np.zeros(H), np.zeros(H), [0, N])
    expect = np.zeros(N)
    for i in range(W):
        expect[t0 + i] = F.silu(torch.tensor(taps[W - 1 - i], dtype=torch.float64)).item()
    assert np.max(np.abs(v[:, 0, c] - expect)) <= 1e-15
    others = np.delete(v[:, 0, :], c, axis=1)
    assert np.all(others == 0.0)


def pin_isolation(m, lens=(6, 2, 7), H=2, dk=8, dv=8, W=4, seed=1):
    rng = np.random.default_rng(seed)
    x, cw, g, cu = _inputs(rng, lens, H, dk, dv, W)
    packed = m.featurize(*x, *cw, *g, cu, eps=1e-6)
    for i in range(len(lens)):
        a, b = int(cu[i]), int(cu[i + 1])
        alone = m.featurize(*[t[a:b] for t in x], *cw, g[0][a:b], g[1][a:b], g[2], g[3], [0, b - a],
                            eps=1e-6)
        for p, s in zip(packed, alone):
            assert np.array_equal(p[a:b], s)


def pin_norms(m, seed=2):
    rng = np.random.default_rng(seed)
    x, cw, g, cu = _inputs(rng, (7, 4), 3, 16, 16, 3)
    q, k, v, _, _ = m.featurize(*x, *cw, *g, cu, eps=0.0)
    for t in (q, k):
        assert np.max(np.abs(np.linalg.norm(t, axis=-1) - 1.0)) <= 1e-13
    assert np.max(np.abs(np.linalg.norm(v, axis=-1) - 1.0)) > 0.1


def pin_gate_values(m):
    N, H, d = 3, 2, 4
    x = [np.zeros((N, H, d)) for _ in range(3)]
    cw = [np.zeros((H * d, 1)) for _ in range(3)]
    bl = np.zeros((N, H))
    b = np.array([0.7, -2.0])
    al = np.stack([-b, -b, np.array([40.0, 40.0]) - b])     # logit + b = 0, 0, 40
    A = np.array([0.0, math.log(3.0)])
    _, _, _, beta, la = m.featurize(*x, *cw, bl, al, A, b, [0, N])
    assert np.all(beta == 0.5)
    assert abs(la[0, 0] + math.log(2.0)) <= 1e-15               # -1 * softplus(0) = -ln 2
    assert abs(la[1, 1] + 3.0 * math.log(2.0)) <= 1e-14         # -3 * ln 2
    assert abs(la[2, 1] + 3.0 * (40.0 + math.log1p(math.exp(-40.0)))) <= 1e-12
    q, _, v, _, _ = m.featurize(*x, *cw, bl, al, A, b, [0, N])
    assert np.all(q == 0.0) and np.all(v == 0.0)                # zero input: SiLU(0) = 0


def pin_width_one(m, seed=3):
    """W = 1: the convolution is a per-channel scale of the current token."""
    rng = np.random.default_rng(seed)
    x, cw, g, cu = _inputs(rng, (5, 3), 2, 8, 8, 1)
    _, _, v, _, _ = m.featurize(*x, *cw, *g, cu)
    ref = F.silu(torch.from_numpy(x[2] * cw[2][:, 0].reshape(1, 2, 8))).numpy()
    assert np.max(np.abs(v - ref)) <= 1e-15


PINS = [pin_library, pin_impulse, pin_isolation, pin_norms, pin_gate_values, pin_width_one]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_featurize_pin(oracle_mod, pin):
    pin(oracle_mod)


@pytest.mark.parametrize("W", [1, 2, 3, 4])
def test_featurize_library_all_widths(oracle_mod, W):
    pin_library(oracle_mod, lens=(1, 2, 11), W=W, seed=10 + W)
    pin_impulse(oracle_mod, W=W)
