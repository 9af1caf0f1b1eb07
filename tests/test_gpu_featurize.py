"""GPU parity of the featurisation step (gdn_featurize) against the fp64 oracle.

Bar: fp32 outputs max|got - ref| / rms(ref) <= 1e-4; bf16 outputs within one rounding to
bf16 of the exact value (|got - ref| <= 2^-8 |ref| + 1e-5 rms(ref) per element). Cases
cover every supported width d (16..128) and convolution width W (1..4), head counts that
leave a warp's head group partly empty,
sequences shorter than the window, an empty sequence, runs cut by sequence starts and
ragged totals, the full prefill workload shape, the hand-off into chunk_fwd, and the
device-side check of a cu_seqlens that does not cover the tokens.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.helpers import TOL, f64, rel_err

gdn = pytest.importorskip("gated_deltanet_05_b200")

pytestmark = pytest.mark.gpu

KEYS = ("xq", "xk", "xv", "conv_q", "conv_k", "conv_v", "beta_logit", "alpha_logit", "A", "b_alpha",
        "cu_seqlens")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert gdn.device_error() == "GDN_OK"


def _inputs(dtype, lengths, H, dk, dv, width, seed):
    w = dataclasses.replace(W.WORKLOADS["prefill"], dtype=dtype, H=H, d_k=dk, d_v=dv, seed=seed)
    return W.make_featurize_inputs(w, lengths=lengths, width=width)


def _run(inp, eps=1e-6):
    d = {k: inp[k].cuda() for k in KEYS}
    out = gdn.featurize(*[d[k] for k in KEYS], eps=eps, cu_seqlens_host=inp["cu_seqlens"])
    torch.cuda.synchronize()
    return [t.cpu() for t in out]


def _oracle(inp, eps=1e-6):
    return oracle.featurize(*[inp[k] for k in KEYS[:-1]], inp["cu_seqlens"].numpy(), eps=eps)


def _check(got, ref, dtype):
    """fp32 outputs (every output for fp32 streams; the gates always): max|d| / rms(ref) <=
    1e-4. bf16 outputs (q, k, v for bf16 streams) are the fp32 result rounded to nearest:
    each element within one bf16 rounding of the exact value, |d| <= 2^-8 |ref|, plus the
    fp32 error, 1e-5 rms(ref). (A max|d| / rms bound would mostly measure how large the
    largest SiLU outputs are relative to the rms.)"""
    for i, (name, g, r) in enumerate(zip(("q", "k", "v", "beta", "log_alpha"), got, ref)):
        g = f64(g)
        if dtype == "bf16" and i < 3:
            rms = float(np.sqrt(np.mean(r * r)))
            excess = np.abs(g - r) - (2.0 ** -8 * np.abs(r) + 1e-5 * rms)
            assert float(excess.max(initial=-1.0)) <= 0.0, f"{name}: beyond bf16 rounding by {excess.max():.3e}"
        else:
            err = rel_err(g, r)
            assert err <= TOL["f32"], f"{name}: {err:.3e} > {TOL['f32']}"


CASES = [
    # dtype, lengths, H, d_k, d_v, W
    ("f32", (37, 1, 2, 0, 70), 3, 16, 16, 4),
    ("f32", (64, 33), 1, 32, 32, 3),
    ("f32", (5, 91), 3, 64, 64, 2),
    ("f32", (100, 3, 29), 2, 128, 128, 1),
    ("f32", (45, 19), 3, 32, 64, 4),
    ("bf16", (37, 1, 2, 0, 70), 3, 16, 16, 4),
    ("bf16", (64, 33), 5, 64, 64, 4),
    ("bf16", (129, 3, 250), 2, 128, 128, 4),
    ("bf16", (17,), 4, 128, 64, 3),
]


@pytest.mark.parametrize("dtype,lengths,H,dk,dv,width", CASES)
def test_featurize_parity(dtype, lengths, H, dk, dv, width):
    inp = _inputs(dtype, lengths, H, dk, dv, width, seed=hash((lengths, H, dk, width)) % 1000)
    _check(_run(inp), _oracle(inp), dtype)


def test_featurize_full_prefill_shape():
    """The prefill workload's shape (4 x 4096 tokens, H = 16, d = 128, bf16), every element."""
    inp = W.make_featurize_inputs(W.WORKLOADS["prefill"])
    _check(_run(inp), _oracle(inp), "bf16")


def test_featurize_zero_eps_unit_rows():
    inp = _inputs("f32", (40, 24), 2, 64, 64, 4, seed=7)
    q, k, v, _, _ = _run(inp, eps=0.0)
    for t in (q, k):
        assert float((t.norm(dim=-1) - 1.0).abs().max()) <= 1e-5
    assert float((v.norm(dim=-1) - 1.0).abs().max()) > 0.1


def test_featurize_empty_batch():
    inp = _inputs("bf16", (0, 0), 2, 128, 128, 4, seed=8)
    q, k, v, beta, la = _run(inp)
    assert q.shape == (0, 2, 128) and beta.shape == (0, 2)


def test_featurize_feeds_chunk_fwd():
    """featurize -> chunk_fwd on the device against oracle.featurize -> oracle.recurrent."""
    inp = _inputs("f32", (50, 30), 2, 16, 16, 4, seed=9)
    q, k, v, beta, la = _run(inp)
    d = [t.cuda() for t in (q, k, v, la, beta)]
    y, S_T = gdn.chunk_fwd(*d, inp["cu_seqlens"].cuda(), chunk=16, cu_seqlens_host=inp["cu_seqlens"])
    rq, rk, rv, rb, rla = _oracle(inp)
    y_ref, S_ref, _ = oracle.recurrent(rq, rk, rv, rla, rb, inp["cu_seqlens"].numpy())
    assert rel_err(f64(y), y_ref) <= TOL["f32"]
    assert rel_err(f64(S_T), oracle.state_to_lib(S_ref)) <= TOL["f32"]


def test_featurize_device_check_on_short_cu_seqlens():
    """cu_seqlens on the device ends before n_tok and no host copy is given: the kernel
    records GDN_ERR_DEVICE_CHECK instead of reading past the array."""
    inp = _inputs("f32", (5, 6), 2, 32, 32, 4, seed=10)
    n_tok = 12                                        # one token more than cu_seqlens covers
    dev = {k: inp[k].cuda() for k in KEYS}
    xs = [torch.zeros((n_tok, 2, 32), device="cuda") for _ in range(3)]
    gates = [torch.zeros((n_tok, 2), device="cuda") for _ in range(2)]
    outs = [torch.empty((n_tok, 2, 32), device="cuda") for _ in range(3)] + \
           [torch.empty((n_tok, 2), device="cuda") for _ in range(2)]
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = gdn.lib().gdn_featurize(p(xs[0]), p(xs[1]), p(xs[2]), 0, p(dev["conv_q"]), p(dev["conv_k"]),
                                 p(dev["conv_v"]), 4, p(gates[0]), p(gates[1]), p(dev["A"]),
                                 p(dev["b_alpha"]), p(dev["cu_seqlens"]), None, 2, n_tok, 2, 32, 32,
                                 1e-6, *[p(t) for t in outs],
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    assert gdn.device_error() == "GDN_ERR_DEVICE_CHECK"
    assert gdn.device_error() == "GDN_OK"
