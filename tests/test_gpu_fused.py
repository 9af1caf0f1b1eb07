"""GPU parity of the prefill with the output epilogue in one call (gdn_chunk_fwd_gated: the
prefill writes y into o, then the gate-norm rewrites o in place).

o = sigmoid(z) * RMSNorm(y) * (1 + w) is checked two ways:
- against the fp64 oracle (oracle.recurrent, then oracle.gate_norm on its y): fp32 o at the
  bf16-input bar max|d| / rms <= 2e-2. A bf16 o is computed from y rounded to bf16 and is
  itself rounded, so it is held per element to three bf16 unit roundoffs (2^-8 each, 8
  significant bits) of the fp32 o: y's rounding, its effect on the row's rms (at most one
  unit, as o is invariant to the scale of y) and o's rounding;
- against the two separate library calls (gdn_chunk_fwd with y in o's dtype, then
  gdn_gate_norm on that y) on the device: bit-identical, for fp32 and bf16 o.
Lengths cover full chunks, partial last chunks whose second half is empty (n <= 32), an
empty sequence and S0 != 0; the full prefill workload is checked on sampled chains.
"""
import pytest
import torch

import oracle
import workloads as W
from tests.helpers import TOL, f64, oracle_prefill, rel_err, subset, to_dev

gdn = pytest.importorskip("gated_deltanet_05_b200")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert gdn.device_error() == "GDN_OK"


def _inputs(lengths, H=2, seed=5, s0_std=0.0):
    w = W.Workload("fused", "bf16", tuple(lengths), H, 128, 128, 64, seed=seed, s0_std=s0_std)
    return W.make_prefill_inputs(w)


def _fused(inp, o_dtype):
    d = to_dev(inp)
    o, S_T = gdn.chunk_fwd_gated(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                                 d["z"], d["w_norm"], S0=d.get("S0"), cu_seqlens_host=inp["cu_seqlens"],
                                 o_dtype=o_dtype)
    torch.cuda.synchronize()
    return o, S_T


@pytest.mark.parametrize("lengths,s0", [((64,), 0.0), ((1,), 0.0), ((65,), 0.0), ((63, 129, 2), 0.02),
                                        ((300, 0, 77), 0.0), ((96, 33, 31), 0.02)])
def test_fused_matches_oracle(lengths, s0):
    inp = _inputs(lengths, s0_std=s0, seed=len(lengths) * 7 + lengths[0])
    o32, S_T = _fused(inp, torch.float32)
    y_ref, S_ref = oracle_prefill(inp)
    o_ref = oracle.gate_norm(y_ref, inp["z"], inp["w_norm"])
    assert rel_err(f64(o32), o_ref) <= TOL["bf16"]
    assert rel_err(f64(S_T), S_ref) <= TOL["bf16"]
    o16, _ = _fused(inp, torch.bfloat16)
    assert bool(((o16.float() - o32).abs() <= o32.abs() * (3 * 2.0 ** -8 + 2.0 ** -14) + 1e-30).all())


@pytest.mark.parametrize("lengths", [(128, 64), (200, 1, 70)])
@pytest.mark.parametrize("o_dtype", [torch.float32, torch.bfloat16])
def test_fused_matches_unfused_library_path(lengths, o_dtype):
    inp = _inputs(lengths, H=3, seed=11)
    d = to_dev(inp)
    o_f, S_f = _fused(inp, o_dtype)
    y, S_u = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                           cu_seqlens_host=inp["cu_seqlens"], y_dtype=o_dtype)
    o_u = gdn.gate_norm(y, d["z"], d["w_norm"], out_dtype=o_dtype)
    torch.cuda.synchronize()
    assert torch.equal(o_f, o_u)
    assert torch.equal(S_f, S_u)


def test_fused_full_prefill_workload_sampled():
    """4 x 4096 tokens, H = 16 (the bench step): every token of sampled chains against the
    oracle with fp32 o, and the bf16 o of every chain within three bf16 roundings of it."""
    inp = W.make_prefill_inputs(W.WORKLOADS["prefill"])
    o16, _ = _fused(inp, torch.bfloat16)
    o, S_T = _fused(inp, torch.float32)
    assert bool(((o16.float() - o).abs() <= o.abs() * (3 * 2.0 ** -8 + 2.0 ** -14) + 1e-30).all())
    o, S_T = o.cpu(), S_T.cpu()
    for seq, head in ((0, 0), (3, 15), (2, 7)):
        sub, idx, hs = subset(inp, [seq], [head])
        y_ref, S_ref = oracle_prefill(sub)
        o_ref = oracle.gate_norm(y_ref, sub["z"], inp["w_norm"])
        got = o.index_select(0, idx).index_select(1, hs)
        assert rel_err(f64(got), o_ref) <= TOL["bf16"]
        assert rel_err(f64(S_T[seq:seq + 1, head:head + 1]), S_ref) <= TOL["bf16"]
