"""GPU parity of the multi-token decode (gdn_decode_tokens) against the fp64 oracle.

n tokens per chain and call are n steps of the recurrence started from the current state,
so the oracle is the token-by-token recurrence over sequences of n tokens with S0 = the
state. Bar: max|got - ref| / rms(ref) on every fp32 y and on the final state, fp32 inputs
<= 1e-4, bf16 inputs <= 2e-2; a bf16 y must be the round-to-nearest-even of the fp32 y
of the same call (the two calls start from the same state). Cases: every d (16..128), d_k != d_v,
1..8 tokens, odd head counts, more chains than SMs, a 400-token run of 100 calls of 4
tokens, agreement with n calls of gdn_decode_step, and at d = 128 the pipelined kernel
against the one-CTA-per-chain kernel (taken when v is not 16-byte aligned).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.helpers import TOL, assert_is_rounding, f64, rel_err

gdn = pytest.importorskip("gated_deltanet_05_b200")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert gdn.device_error() == "GDN_OK"


def _tokens(n_seq, n, H, dk, dv, dtype, seed):
    """Inputs of n decode steps: [n_seq, n, H, .] (steps drawn with the decode generator)."""
    w = W.WORKLOADS["decode"]
    steps = [W.make_decode_inputs(w, seed * 100 + i, n_seq=n_seq, H=H, d=dk) for i in range(n)]
    vs = [W.make_decode_inputs(w, seed * 100 + 50 + i, n_seq=n_seq, H=H, d=dv)["v"] for i in range(n)]
    cast = (lambda t: t.to(torch.bfloat16)) if dtype == "bf16" else (lambda t: t)
    q = cast(torch.stack([s["q"] for s in steps], 1))
    k = cast(torch.stack([s["k"] for s in steps], 1))
    v = cast(torch.stack(vs, 1))
    alpha = torch.stack([s["alpha"] for s in steps], 1)
    beta = torch.stack([s["beta"] for s in steps], 1)
    return q, k, v, alpha, beta


def _oracle(q, k, v, alpha, beta, S_lib):
    """y [n_seq, n, H, dv] and the final state (library layout) from the fp64 recurrence."""
    n_seq, n, H, dk = q.shape
    dv = v.shape[3]
    flat = lambda t, d: t.reshape(n_seq * n, H, d)
    cu = np.arange(0, n_seq * n + 1, n, dtype=np.int64)
    la = np.log(f64(alpha).reshape(n_seq * n, H))
    y, S_T, _ = oracle.recurrent(flat(q, dk), flat(k, dk), flat(v, dv), la, beta.reshape(n_seq * n, H),
                                 cu, S0=oracle.state_from_lib(S_lib))
    return y.reshape(n_seq, n, H, dv), oracle.state_to_lib(S_T)


@pytest.mark.parametrize("n_seq,n,H,dk,dv,dtype", [
    (3, 4, 2, 128, 128, "f32"), (2, 1, 3, 64, 64, "f32"), (5, 8, 1, 32, 32, "f32"),
    (2, 3, 3, 16, 16, "f32"), (2, 5, 2, 32, 64, "f32"), (2, 2, 2, 128, 64, "f32"),
    (4, 4, 2, 128, 128, "bf16"), (3, 7, 5, 64, 64, "bf16"),
    # more chains than SMs
    (40, 4, 8, 128, 128, "f32"), (30, 3, 10, 128, 128, "bf16"), (97, 8, 5, 128, 128, "f32"),
])
def test_decode_tokens_parity(n_seq, n, H, dk, dv, dtype):
    q, k, v, alpha, beta = _tokens(n_seq, n, H, dk, dv, dtype, seed=n_seq * 10 + n)
    g = torch.Generator().manual_seed(n)
    S0 = (torch.randn(n_seq, H, dv, dk, generator=g) * 0.05).float()
    S = S0.cuda()
    args = (q.cuda(), k.cuda(), v.cuda(), alpha.cuda(), beta.cuda())
    y = gdn.decode_tokens(*args, S)
    S16 = S0.cuda()
    y16 = gdn.decode_tokens(*args, S16, y_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    y_ref, S_ref = _oracle(q, k, v, alpha, beta, S0.numpy().astype(np.float64))
    tol = TOL[dtype]
    assert y.dtype == torch.float32
    assert rel_err(f64(y), y_ref) <= tol
    assert rel_err(f64(S), S_ref) <= tol
    # the bf16 output of the same call is the rounding of the fp32 one; the state is the same
    assert_is_rounding(y16.cpu(), y.cpu())
    assert torch.equal(S16, S)


def test_decode_tokens_long_run():
    """100 calls of 4 tokens (400 steps) from a zero state, fp32, against one oracle run."""
    n_seq, n, H, d, calls = 4, 4, 2, 128, 100
    q, k, v, alpha, beta = _tokens(n_seq, n * calls, H, d, d, "f32", seed=7)
    S = torch.zeros(n_seq, H, d, d, device="cuda")
    ys = []
    for c in range(calls):
        sl = slice(c * n, (c + 1) * n)
        ys.append(gdn.decode_tokens(q[:, sl].contiguous().cuda(), k[:, sl].contiguous().cuda(),
                                    v[:, sl].contiguous().cuda(), alpha[:, sl].contiguous().cuda(),
                                    beta[:, sl].contiguous().cuda(), S).cpu())
    y = torch.cat(ys, 1)
    y_ref, S_ref = _oracle(q, k, v, alpha, beta, np.zeros((n_seq, H, d, d)))
    assert rel_err(f64(y), y_ref) <= TOL["f32"]
    assert rel_err(f64(S), S_ref) <= TOL["f32"]


def test_decode_tokens_matches_single_steps():
    n_seq, n, H, d = 8, 4, 4, 128
    q, k, v, alpha, beta = _tokens(n_seq, n, H, d, d, "f32", seed=3)
    S0 = torch.randn(n_seq, H, d, d) * 0.05
    S_a, S_b = S0.cuda(), S0.cuda()
    y_a = gdn.decode_tokens(q.cuda(), k.cuda(), v.cuda(), alpha.cuda(), beta.cuda(), S_a)
    y_b = torch.stack([gdn.decode_step(q[:, i].contiguous().cuda(), k[:, i].contiguous().cuda(),
                                       v[:, i].contiguous().cuda(), alpha[:, i].contiguous().cuda(),
                                       beta[:, i].contiguous().cuda(), S_b) for i in range(n)], 1)
    torch.cuda.synchronize()
    assert rel_err(f64(y_a), f64(y_b)) <= 1e-5
    assert rel_err(f64(S_a), f64(S_b)) <= 1e-5


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_tokens_both_kernels_agree(dtype):
    """d = 128 runs the pipelined kernel when v is 16-byte aligned and the one-CTA-per-chain
    kernel otherwise (v only needs 4-byte alignment); both against the oracle, and against
    each other."""
    n_seq, n, H, d = 6, 4, 3, 128
    q, k, v, alpha, beta = _tokens(n_seq, n, H, d, d, dtype, seed=11)
    S0 = (torch.randn(n_seq, H, d, d, generator=torch.Generator().manual_seed(2)) * 0.05).float()
    args = [q.cuda(), k.cuda(), v.cuda(), alpha.cuda(), beta.cuda()]
    S_a = S0.cuda()
    y_a = gdn.decode_tokens(*args, S_a)
    # the same v 4 bytes into a larger buffer: 4-byte aligned (what the call requires of v),
    # not 16-byte aligned
    off = 4 // v.element_size()
    big = torch.empty(v.numel() + 16, dtype=v.dtype, device="cuda")
    v_off = big[off:off + v.numel()].view(v.shape)
    v_off.copy_(args[2])
    assert v_off.data_ptr() % 16 != 0 and v_off.data_ptr() % 4 == 0
    S_b = S0.cuda()
    y_b = gdn.decode_tokens(args[0], args[1], v_off, args[3], args[4], S_b)
    torch.cuda.synchronize()
    y_ref, S_ref = _oracle(q, k, v, alpha, beta, S0.numpy().astype(np.float64))
    for y, S in ((y_a, S_a), (y_b, S_b)):
        assert rel_err(f64(y), y_ref) <= TOL[dtype]
        assert rel_err(f64(S), S_ref) <= TOL[dtype]
    assert rel_err(f64(y_a), f64(y_b)) <= 1e-5
    assert rel_err(f64(S_a), f64(S_b)) <= 1e-5
