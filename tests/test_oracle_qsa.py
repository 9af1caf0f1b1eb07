"""Pins of the QSA indexer oracle (oracle/qsa_indexer.py) against things fixed outside it.

- Partial RoPE: position 0 is the identity, norms are kept, the last d - rot dimensions
  pass through, a unit vector turns by exactly the angle the reading fixes, and scores
  depend only on the position difference; an independent complex-number rotation agrees.
- Key compression equals numpy's reshape-and-mean followed by the closed-form RMSNorm.
- Block causality: exactly floor((i + 1) / r) blocks are visible to token i.
- Scores equal an independent einsum restatement (complex rotation, maximum for ReLU);
  keys opposite to every query give zero scores.
- Top-K equals numpy's lexsort on (-score, index); the token set has r |B_i| + ((i+1) mod r)
  tokens, none after i.
Every pin takes the module under test as its first argument; test_qsa_pins_catch_mutant
below runs them against copies of the oracle with planted mistakes.
"""
import importlib.util
import math
import os

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "qsa_indexer.py")


def load(path=SRC, name="qsa_indexer_under_test"):
    spec = importlib.util.spec_from_file_location(name, path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _rot_complex(x, pos, rot=64, base=10000.0):
    """Independent rotation: pair j with j + rot/2 as the complex number x_j + i x_{j+rot/2}."""
    x = np.array(x, dtype=np.float64, copy=True)
    half = rot // 2
    z = x[..., :half] + 1j * x[..., half:rot]
    th = np.asarray(pos, dtype=np.float64)[..., None] * base ** (-2.0 * np.arange(half) / rot)
    z = z * np.exp(1j * th)
    x[..., :half], x[..., half:rot] = z.real, z.imag
    return x


def pin_rope(m, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((5, 128))
    assert np.array_equal(m.prope(x, 0), x)
    y = m.prope(x, 37)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13, atol=0)
    assert np.array_equal(y[:, 64:], x[:, 64:])
    e0 = np.zeros(128)
    e0[0] = 1.0
    p = 0.75
    want = np.zeros(128)
    want[0], want[32] = math.cos(p), math.sin(p)
    assert np.allclose(m.prope(e0, p), want, rtol=0, atol=1e-15)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    for i, j, s in ((9, 4, 13), (100, 0, 7), (3, 3, 1000)):
        a = np.dot(m.prope(q, i), m.prope(k, j))
        b = np.dot(m.prope(q, i + s), m.prope(k, j + s))
        assert abs(a - b) <= 1e-10 * max(1.0, abs(a))
    assert np.allclose(m.prope(x, 12.0), _rot_complex(x, 12.0), rtol=0, atol=1e-12)


def pin_compression(m, seed=1):
    rng = np.random.default_rng(seed)
    n, d, r = 23, 128, 4
    kx = rng.standard_normal((n, d))
    wk = rng.standard_normal(d) * 0.1
    nb = n // r
    pooled = kx[:nb * r].reshape(nb, r, d).mean(axis=1)
    want = pooled / np.sqrt(np.mean(pooled ** 2, axis=1, keepdims=True) + 1e-6) * (1 + wk)
    got = m.compress_keys(kx, r, wk, rot=0)
    assert got.shape == (nb, d)
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def _inputs(seed, n=37, Hq=4, d=128):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((n, Hq, d)), rng.standard_normal((n, d)), rng.standard_normal(d) * 0.1,
            rng.standard_normal(d) * 0.1)


def pin_block_causal(m, seed=2):
    qx, kx, wq, wk = _inputs(seed)
    for r in (1, 4, 5):
        I = m.scores(qx, kx, r, wq, wk)
        n, nb = I.shape
        assert nb == n // r
        for i in range(n):
            vis = np.isfinite(I[i])
            assert vis.sum() == min((i + 1) // r, nb)
            assert all(vis[b] == (b * r + r - 1 <= i) for b in range(nb))


def pin_scores_independent(m, seed=3):
    qx, kx, wq, wk = _inputs(seed, n=21)
    r = 4
    n, Hq, d = qx.shape
    qn = qx / np.sqrt(np.mean(qx ** 2, axis=-1, keepdims=True) + 1e-6) * (1 + wq)
    q = _rot_complex(qn, np.arange(n)[:, None])
    nb = n // r
    kp = kx[:nb * r].reshape(nb, r, d).mean(axis=1)
    kn = kp / np.sqrt(np.mean(kp ** 2, axis=-1, keepdims=True) + 1e-6) * (1 + wk)
    k = _rot_complex(kn, np.arange(nb) * r)
    dots = np.einsum("ihd,bd->ihb", q, k)
    want = np.maximum(dots, 0.0).sum(axis=1)
    causal = (np.arange(nb)[None, :] * r + r - 1) <= np.arange(n)[:, None]
    want = np.where(causal, want, -np.inf)
    got = m.scores(qx, kx, r, wq, wk)
    fin = np.isfinite(want)
    assert np.array_equal(np.isfinite(got), fin)
    assert np.allclose(got[fin], want[fin], rtol=1e-12, atol=1e-12)


def pin_relu(m, seed=4):
    rng = np.random.default_rng(seed)
    n, Hq, d = 16, 4, 128
    qx = np.abs(rng.standard_normal((n, Hq, d))) + 0.1
    kx = -(np.abs(rng.standard_normal((n, d))) + 0.1)
    I = m.scores(qx, kx, 4, np.zeros(d), np.zeros(d), rot=0)
    assert np.all(I[np.isfinite(I)] == 0.0)
    assert np.isfinite(I).sum() > 0


def pin_topk(m, seed=5):
    rng = np.random.default_rng(seed)
    n, nb, r, K = 12, 10, 4, 16              # K_B = 4
    I = np.round(rng.standard_normal((n, nb)), 1)   # plenty of ties
    I[np.arange(n) % 3 == 0, 0] = -np.inf
    I[2, :] = -np.inf
    I[3, 5:] = -np.inf
    got = m.select_blocks(I, K, r)
    assert got.shape == (n, 4)
    for i in range(n):
        fin = np.where(np.isfinite(I[i]))[0]
        order = fin[np.lexsort((fin, -I[i, fin]))][:4]
        want = np.full(4, -1)
        want[:len(order)] = order
        assert np.array_equal(got[i], want), (i, got[i], want)


def pin_token_set(m, seed=6):
    qx, kx, wq, wk = _inputs(seed, n=45)
    r, K = 4, 16
    I, B = m.indexer(qx, kx, wq, wk, K=K, r=r)
    for i in range(qx.shape[0]):
        S = m.token_set(B[i], i, r)
        n_sel = int((B[i] >= 0).sum())
        assert len(S) == r * n_sel + (i + 1) % r
        assert max(S, default=-1) <= i and S == sorted(set(S))


PINS = [pin_rope, pin_compression, pin_block_causal, pin_scores_independent, pin_relu, pin_topk,
        pin_token_set]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_qsa_pin(pin):
    pin(load())


MUTANTS = {
    "rope_not_a_rotation": [("x[..., :half] = a * c - b * s", "x[..., :half] = a * c + b * s")],
    "rope_wrong_pairing": [("a, b = x[..., :half].copy(), x[..., half:rot].copy()",
                            "a, b = x[..., 0:rot:2].copy(), x[..., 1:rot:2].copy()")],
    "causal_off_by_one": [("if b * r + r - 1 <= i:", "if b * r <= i:")],
    "relu_dropped": [("max(0.0, float(np.dot(q[i, h], kb[b])))", "float(np.dot(q[i, h], kb[b]))")],
    "pool_sum_not_mean": [("kb[b] = kx[b * r:(b + 1) * r].mean(axis=0)", "kb[b] = kx[b * r:(b + 1) * r].sum(axis=0)")],
    "key_positions_not_block_starts": [("return prope(kb, np.arange(nb) * r, rot, base)",
                                           "return prope(kb, np.arange(nb), rot, base)")],
    "ties_to_high_index": [("cand = [(-I[i, b], b) for b", "cand = [(-I[i, b], -b) for b"),
                           ("for j, (_, b) in enumerate(cand[:kb]):\n            out[i, j] = b",
                            "for j, (_, b) in enumerate(cand[:kb]):\n            out[i, j] = -b")],
    "tail_from_current_block": [("toks.update(range(r * ((i + 1) // r), i + 1))",
                                 "toks.update(range(r * (i // r), i + 1))")],
    "norm_weight_not_centred": [("* (1.0 + np.asarray(w, np.float64))", "* np.asarray(w, np.float64)")],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_qsa_pins_catch_mutant(tmp_path, name):
    src = open(SRC).read()
    for old, new in MUTANTS[name]:
        assert src.count(old) == 1, (name, old)
        src = src.replace(old, new)
    path = tmp_path / f"{name}.py"
    path.write_text(src)
    mod = load(str(path), f"qsa_mutant_{name}")
    failed = 0
    for pin in PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError, IndexError):
            failed += 1
    assert failed >= 1, f"no pin caught mutant {name}"
