"""GPU parity of the QSA compressed indexer (gdn_qsa_indexer, gdn_qsa_token_sets) against
the fp64 oracle in oracle/qsa_indexer.py, through the C ABI.

- Scores, on every visible (token, block): max|got - ref| / rms(ref) <= 1e-4 for fp32
  inputs (fp32 CUDA-core scores) and <= 2e-2 for bf16 inputs (bf16 tensor-core products of
  the normalised, rotated vectors, fp32 accumulation).
- Selected blocks: bit-exact against the oracle's selection applied to the kernel's own
  scores (the selection is an integer decision taken in the kernel's precision).
- Token sets: bit-exact against the oracle's token set of the kernel's selection.
Cases: ragged packed sequences (empty, shorter than r, partial tail blocks), r in {1, 4, 5},
Hq in {1, 2, 4}, budgets below and above the visible block count, exact ties (identical
blocks with the rotation off; all-zero scores), and sampled rows of the benchmark shape
(16,384 tokens, Hq = 4, r = 4, K = 2048).
"""
import math

import numpy as np
import pytest
import torch

import workloads as W
from oracle import qsa_indexer as Q

gdn = pytest.importorskip("gated_deltanet_05_b200")

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert gdn.device_error() == "GDN_OK"


def _run(inp, r, K, rot=64, base=10000.0, eps=1e-6):
    d = {k: inp[k].cuda() for k in ("qx", "kx", "wq", "wk", "cu_seqlens")}
    I, B = gdn.qsa_indexer(d["qx"], d["kx"], d["wq"], d["wk"], d["cu_seqlens"], r=r, K=K, rot=rot, base=base,
                           eps=eps, cu_seqlens_host=inp["cu_seqlens"])
    T, cnt = gdn.qsa_token_sets(B, d["cu_seqlens"], r=r, cu_seqlens_host=inp["cu_seqlens"])
    torch.cuda.synchronize()
    return I.cpu().numpy().astype(np.float64), B.cpu().numpy(), T.cpu().numpy(), cnt.cpu().numpy()


def _check(inp, r, K, rot=64, base=10000.0, eps=1e-6, check_scores=True):
    I, B, T, cnt = _run(inp, r, K, rot, base, eps)
    cu = inp["cu_seqlens"].tolist()
    qx = inp["qx"].double().numpy()
    kx = inp["kx"].double().numpy()
    wq, wk = inp["wq"].double().numpy(), inp["wk"].double().numpy()
    kb = -(-K // r)
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if a == b:
            continue
        nb = (b - a) // r
        vis = np.array([[bb * r + r - 1 <= i for bb in range(nb)] for i in range(b - a)], dtype=bool)
        got = np.where(vis, I[a:b, :nb], -np.inf) if nb > 0 else np.zeros((b - a, 0))
        if check_scores and nb > 0:
            ref = Q.scores(qx[a:b], kx[a:b], r, wq, wk, eps, rot, base)
            assert np.array_equal(np.isfinite(ref), vis)
            if vis.any():
                rms = math.sqrt(float(np.mean(ref[vis] ** 2)))
                err = float(np.max(np.abs(got[vis] - ref[vis])))
                assert err <= TOL[inp["dtype"]] * max(rms, 1e-30), (err, rms)
        # the selection, decided on the kernel's own scores
        want = Q.select_blocks(got, K, r) if nb > 0 else np.full((b - a, kb), -1)
        assert np.array_equal(B[a:b], want)
        for i in range(b - a):
            ts = Q.token_set(B[a + i], i, r)
            assert cnt[a + i] == len(ts)
            assert np.array_equal(T[a + i, :len(ts)], ts)
            assert (T[a + i, len(ts):] == -1).all()
    return I, B


@pytest.mark.parametrize("lengths,Hq,r,K,dtype", [
    ((37,), 4, 4, 16, "f32"), ((130, 5, 61), 4, 4, 64, "f32"), ((200,), 2, 1, 7, "f32"),
    ((90, 0, 77), 3, 5, 40, "f32"),
    ((37,), 4, 4, 16, "bf16"), ((130, 5, 61), 4, 4, 64, "bf16"), ((300, 2, 129), 1, 4, 40, "bf16"),
    ((257,), 2, 1, 500, "bf16"), ((90, 0, 77), 2, 5, 40, "bf16"),
])
def test_qsa_indexer_parity(lengths, Hq, r, K, dtype):
    inp = W.make_qsa_inputs(lengths, Hq, dtype, seed=sum(lengths) + Hq + r)
    _check(inp, r, K)


@pytest.mark.parametrize("n,dtype", [(4100, "f32"), (4100, "bf16"), (9000, "bf16")])
def test_qsa_many_key_steps_split_over_ctas(n, dtype):
    """A 4,100-token sequence at r = 1: up to 4,100 visible blocks per token, i.e. 33 key
    steps of 128 blocks, split over several CTAs per query tile; sampled rows. 9,000 tokens:
    72 key steps, and score rows of up to 9,000 blocks for the selection."""
    inp = W.make_qsa_inputs((n,), 2, dtype, seed=9)
    r, K = 1, 300
    I, B, T, cnt = _run(inp, r, K)
    qx = inp["qx"].double().numpy()
    kx = inp["kx"].double().numpy()
    wq, wk = inp["wq"].double().numpy(), inp["wk"].double().numpy()
    kbv = Q.compress_keys(kx, r, wk)
    rows = [0, 1, 127, 128, 1023, 2049, n - 1] + ([8500] if n > 8500 else [])
    got, ref = [], []
    for i in rows:
        q = Q.prope(Q.rmsnorm(qx[i], wq), np.full((qx.shape[1],), i))
        ref.append(np.maximum(kbv[:i + 1] @ q.T, 0.0).sum(axis=1))
        got.append(I[i, :i + 1])
        row = np.full((1, n), -np.inf)
        row[0, :i + 1] = I[i, :i + 1]
        assert np.array_equal(B[i], Q.select_blocks(row, K, r)[0])
    # max |error| over the sampled scores, relative to their rms (a single row can be tiny)
    got, ref = np.concatenate(got), np.concatenate(ref)
    assert float(np.max(np.abs(got - ref))) <= TOL[dtype] * math.sqrt(float(np.mean(ref ** 2)))


def test_qsa_ties_go_to_the_lower_block():
    """Exact ties: with the rotation off, identical key blocks give identical scores; with
    queries opposite to most blocks, most scores are exactly 0. The lower block index wins."""
    n, Hq, r, K = 160, 1, 4, 24
    rng = np.random.default_rng(3)
    q = np.ones((n, Hq, 128))
    k = -np.ones((n, 128))
    for bb in (3, 7, 8, 20, 31):                     # a few blocks score 128-ish, all equal
        k[bb * r:(bb + 1) * r] = 1.0
    k[17 * r:18 * r] = rng.standard_normal(128)      # one block with its own score
    for dtype in ("f32", "bf16"):
        cast = (lambda a: torch.from_numpy(a).to(torch.bfloat16)) if dtype == "bf16" else \
            (lambda a: torch.from_numpy(a.astype(np.float32)))
        inp = {"qx": cast(q), "kx": cast(k), "wq": torch.zeros(128), "wk": torch.zeros(128),
               "cu_seqlens": torch.tensor([0, n], dtype=torch.int32), "dtype": dtype}
        I, B = _check(inp, r, K, rot=0)
        i = n - 1
        equal = [b for b in B[i] if b in (3, 7, 8, 20, 31)]
        assert equal == [3, 7, 8, 20, 31]                      # one score, in index order
        zeros = [b for b in B[i] if b >= 0 and I[i, b] == 0.0]
        assert len(zeros) > 0 and zeros == sorted(zeros)


def test_qsa_benchmark_shape_sampled_rows():
    """16,384 tokens, Hq = 4, r = 4, K = 2048 (the benchmark shape), bf16: scores of sampled
    rows against the oracle's vectors, the selection on the kernel's scores."""
    cfg = W.QSA_WORKLOAD
    inp = W.make_qsa_inputs(cfg["lengths"], cfg["Hq"], cfg["dtype"], seed=cfg["seed"])
    r, K = cfg["r"], cfg["K"]
    I, B, T, cnt = _run(inp, r, K)
    qx = inp["qx"].double().numpy()
    kx = inp["kx"].double().numpy()
    wq, wk = inp["wq"].double().numpy(), inp["wk"].double().numpy()
    kbv = Q.compress_keys(kx, r, wk)
    n = qx.shape[0]
    got, ref = [], []
    for i in [3, 4, 2047, 2048, 8191, 12000, n - 1]:
        nvis = (i + 1) // r
        q = Q.prope(Q.rmsnorm(qx[i], wq), np.full((qx.shape[1],), i))
        ref.append(np.maximum(kbv[:nvis] @ q.T, 0.0).sum(axis=1))
        got.append(I[i, :nvis])
        row = np.full((1, n // r), -np.inf)
        row[0, :nvis] = I[i, :nvis]
        assert np.array_equal(B[i], Q.select_blocks(row, K, r)[0])
        ts = Q.token_set(B[i], i, r)
        assert cnt[i] == len(ts) and np.array_equal(T[i, :len(ts)], ts)
    got, ref = np.concatenate(got), np.concatenate(ref)
    assert float(np.max(np.abs(got - ref))) <= TOL["bf16"] * math.sqrt(float(np.mean(ref ** 2)))
