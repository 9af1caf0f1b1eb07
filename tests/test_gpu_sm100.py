"""GPU parity of the sm_100a tensor-core prefill kernel (bf16 q/k/v, d_k = d_v = 128,
chunk 64, fp32 state) against the fp64 oracle, through the C ABI.

Bar: max|got - ref| / rms(ref) <= 2e-2 on y and on the final states (bf16 inputs, fp32
state). Ragged lengths cover partial chunks, empty and one-token sequences; the full
workloads compare sampled chains (every token of the chain and its final state).
"""
import numpy as np
import pytest
import torch

import workloads as W
from tests.helpers import TOL, f64, oracle_prefill, rel_err, subset
from tests.test_gpu_parity import assert_is_rounding, check_prefill, custom, run_prefill

gdn = pytest.importorskip("gated_deltanet_05_b200")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert gdn.device_error() == "GDN_OK"


@pytest.mark.parametrize("lengths", [(64,), (1,), (65,), (63, 129, 2), (300, 0, 77)])
def test_bf16_tensor_core_kernel_ragged(lengths):
    inp = custom("bf16", lengths, 2, 128, 64, seed=sum(lengths), s0_std=0.02)
    check_prefill(inp)


def test_bf16_tensor_core_kernel_zero_state_and_scale():
    inp = custom("bf16", (500, 260), 3, 128, 64, seed=11)
    check_prefill(inp, scale=0.5)


def test_bf16_strong_decay():
    inp = custom("bf16", (1000,), 2, 128, 64, seed=12, A_range=(1.0, 2.5))
    check_prefill(inp)


def test_bf16_without_final_state():
    inp = custom("bf16", (130,), 2, 128, 64, seed=13)
    y, S_T = run_prefill(inp, final_state=False)
    assert S_T is None
    y_ref, _ = oracle_prefill(inp)
    assert rel_err(f64(y), y_ref) <= TOL["bf16"]


def test_bf16_output_is_rounding_of_fp32_output():
    inp = custom("bf16", (200, 64), 2, 128, 64, seed=15)
    y32, S32 = run_prefill(inp)
    y16, S16 = run_prefill(inp, y_dtype=torch.bfloat16)
    assert_is_rounding(y16, y32)
    assert torch.equal(S16, S32)                         # the state does not depend on y's dtype


def test_bf16_split_sequence_matches_whole():
    """chunk_fwd over T tokens == chunk_fwd over T1 then over the rest from S_T1."""
    inp = custom("bf16", (640,), 2, 128, 64, seed=14, s0_std=0.02)
    y, S = run_prefill(inp)
    T1 = 192
    a = dict(inp)
    b = dict(inp)
    for key in ("q", "k", "v", "log_alpha", "beta"):
        a[key] = inp[key][:T1]
        b[key] = inp[key][T1:]
    a["cu_seqlens"] = torch.tensor([0, T1], dtype=torch.int32)
    b["cu_seqlens"] = torch.tensor([0, 640 - T1], dtype=torch.int32)
    ya, Sa = run_prefill(a)
    b["S0"] = Sa
    yb, Sb = run_prefill(b)
    assert rel_err(f64(torch.cat([ya, yb])), f64(y)) <= TOL["bf16"]
    assert rel_err(f64(Sb), f64(S)) <= TOL["bf16"]


def _check_sampled(name, seqs, heads, tol=None):
    inp = W.make_prefill_inputs(W.WORKLOADS[name])
    y, S_T = run_prefill(inp)
    sub, idx, hs = subset(inp, seqs, heads)
    y_ref, S_ref = oracle_prefill(sub)
    y_got = y.index_select(0, idx).index_select(1, hs)
    S_got = S_T[list(seqs)][:, list(heads)]
    tol = TOL[inp["dtype"]] if tol is None else tol
    ey, es = rel_err(f64(y_got), y_ref), rel_err(f64(S_got), S_ref)
    assert ey <= tol and es <= tol, (ey, es)
    # every output is finite
    assert torch.isfinite(y.float()).all() and torch.isfinite(S_T).all()


def test_prefill_workload_sampled():
    _check_sampled("prefill", seqs=[0, 3], heads=[0, 15])


def test_varlen_workload_sampled():
    lens = W.WORKLOADS["varlen"].lengths
    seqs = [int(np.argmin(lens)), int(np.argmax(lens))]
    _check_sampled("varlen", seqs=seqs, heads=[0, 7])


def test_long_workload_sampled():
    _check_sampled("long", seqs=[0], heads=[5])


