"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, element by element.

Bar (max|got - ref| / rms(ref), on y, the final states and the gate-norm output):
fp32 inputs <= 1e-4; bf16 inputs with fp32 state <= 2e-2. Workloads come from the seeded
generators in workloads/; full-size cases compare sampled chains (all their tokens and
final states), which the oracle computes chain by chain.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.helpers import TOL, assert_is_rounding, f64, oracle_prefill, rel_err, to_dev

gdn = pytest.importorskip("gated_deltanet_05_b200")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert gdn.device_error() == "GDN_OK"


def run_prefill(inp, scale=1.0, final_state=True, y_dtype=torch.float32):
    d = to_dev(inp)
    y, S_T = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                           S0=d.get("S0"), chunk=inp["chunk"], scale=scale,
                           cu_seqlens_host=inp["cu_seqlens"], final_state=final_state,
                           y_dtype=y_dtype)
    torch.cuda.synchronize()
    return y.cpu(), (None if S_T is None else S_T.cpu())


def check_prefill(inp, scale=1.0, tol=None):
    tol = TOL[inp["dtype"]] if tol is None else tol
    y, S_T = run_prefill(inp, scale)
    y_ref, S_ref = oracle_prefill(inp, scale)
    ey, es = rel_err(f64(y), y_ref), rel_err(f64(S_T), S_ref)
    assert ey <= tol and es <= tol, (ey, es)
    return ey, es


def custom(dtype, lengths, H, d, chunk, seed, s0_std=0.0, A_range=(-1.0, 1.0)):
    w = W.Workload("custom", dtype, tuple(lengths), H, d, d, chunk, seed, A_range=A_range,
                   s0_std=s0_std)
    return W.make_prefill_inputs(w)


# ----------------------------------------------------------------------------- prefill
def test_tiny_workload_fp32():
    inp = W.make_prefill_inputs(W.WORKLOADS["tiny"])
    check_prefill(inp)


@pytest.mark.parametrize("d,chunk", [(16, 16), (32, 32), (64, 64), (128, 64), (128, 16)])
def test_fp32_chunk_kernel_ragged(d, chunk):
    inp = custom("f32", (1, 37, 130, 64), 2, d, chunk, seed=d + chunk, s0_std=0.05)
    check_prefill(inp, scale=0.8)


def test_fp32_chunk_kernel_bf16_output_is_rounding():
    inp = custom("f32", (70, 3), 2, 32, 32, seed=3)
    y32, _ = run_prefill(inp)
    y16, _ = run_prefill(inp, y_dtype=torch.bfloat16)
    assert_is_rounding(y16, y32)


def test_fp32_strong_decay_no_overflow():
    inp = custom("f32", (200,), 2, 32, 64, seed=5, A_range=(2.0, 3.0))
    check_prefill(inp)


# ----------------------------------------------------------------------------- decode
@pytest.mark.parametrize("d", [16, 32, 64, 128])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_small(d, dtype):
    w = W.WORKLOADS["decode"]
    n, H = 5, 3
    S = torch.randn(n, H, d, d, generator=torch.Generator().manual_seed(d)) * 0.1
    Sd = S.cuda()
    S_ref = oracle.state_from_lib(S)
    for step in range(3):
        x = W.make_decode_inputs(w, step, n_seq=n, H=H, d=d)
        cast = (lambda t: t.to(torch.bfloat16)) if dtype == "bf16" else (lambda t: t)
        q, k, v = cast(x["q"]), cast(x["k"]), cast(x["v"])
        S_before = Sd.clone()
        y = gdn.decode_step(q.cuda(), k.cuda(), v.cuda(), x["alpha"].cuda(), x["beta"].cuda(),
                            Sd, scale=0.9)
        y16 = gdn.decode_step(q.cuda(), k.cuda(), v.cuda(), x["alpha"].cuda(), x["beta"].cuda(),
                              S_before, scale=0.9, y_dtype=torch.bfloat16)
        y_ref, S_ref = oracle.decode_step(q, k, v, x["alpha"], x["beta"], S_ref, scale=0.9)
        assert y.dtype == torch.float32
        assert rel_err(f64(y.cpu()), y_ref) <= TOL[dtype]
        assert_is_rounding(y16.cpu(), y.cpu())        # bf16 y: the rounding of the fp32 y
        assert torch.equal(S_before, Sd)
    assert rel_err(f64(Sd.cpu()), oracle.state_to_lib(S_ref)) <= TOL[dtype]


def test_decode_workload_full_size():
    """256 x 32 chains, d = 128: all chains for the first steps, then a sampled subset of
    sequences for every one of the 1000 steps; the state after the last step on the subset."""
    w = W.WORKLOADS["decode"]
    n, H, d = w.n_seq_decode, w.H, w.d_k
    S = torch.zeros(n, H, d, d, device="cuda")
    sub = [0, 101, 255]
    S_ref_sub = np.zeros((len(sub), H, d, d))
    for step in range(w.decode_steps):
        x = W.make_decode_inputs(w, step)
        y = gdn.decode_step(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), x["alpha"].cuda(),
                            x["beta"].cuda(), S)
        if step < 2:
            S_prev = S_full_ref if step else np.zeros((n, H, d, d))
            y_ref, S_full_ref = oracle.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"],
                                                   S_prev)
            assert rel_err(f64(y.cpu()), y_ref) <= TOL["f32"]
        y_sub_ref, S_ref_sub = oracle.decode_step(x["q"][sub], x["k"][sub], x["v"][sub],
                                                  x["alpha"][sub], x["beta"][sub], S_ref_sub)
        if step % 50 == 0 or step == w.decode_steps - 1:
            assert rel_err(f64(y[sub].cpu()), y_sub_ref) <= TOL["f32"], step
    S_got = S[sub].cpu()
    assert rel_err(f64(S_got), oracle.state_to_lib(S_ref_sub)) <= TOL["f32"]


def test_prefill_then_decode_matches_recurrence():
    """Prefill state handed to the decode step continues the same recurrence."""
    inp = custom("f32", (70, 33), 2, 64, 32, seed=21)
    y, S_T = run_prefill(inp)
    x = W.make_decode_inputs(W.WORKLOADS["decode"], 7, n_seq=2, H=2, d=64)
    Sd = S_T.cuda().contiguous()
    yd = gdn.decode_step(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), x["alpha"].cuda(),
                         x["beta"].cuda(), Sd)
    _, S_ref = oracle_prefill(inp)
    y_ref, S_new = oracle.decode_step(x["q"], x["k"], x["v"], x["alpha"], x["beta"],
                                      oracle.state_from_lib(S_ref))
    assert rel_err(f64(yd.cpu()), y_ref) <= TOL["f32"]
    assert rel_err(f64(Sd.cpu()), oracle.state_to_lib(S_new)) <= TOL["f32"]


# ----------------------------------------------------------------------------- gate-norm
@pytest.mark.parametrize("dv", [16, 32, 64, 128, 256])
@pytest.mark.parametrize("ydt,zdt", [("f32", "f32"), ("bf16", "bf16"), ("f32", "bf16"),
                                     ("bf16", "f32")])
def test_gate_norm_small(dv, ydt, zdt):
    g = torch.Generator().manual_seed(dv)
    tdt = {"bf16": torch.bfloat16, "f32": torch.float32}
    rows = 1000 + 3
    y = (torch.randn(rows, dv, generator=g) * 2).to(tdt[ydt])
    z = torch.randn(rows, dv, generator=g).to(tdt[zdt])
    w = torch.randn(dv, generator=g) * 0.02
    y[5] = 0                                             # an all-zero row stays finite
    o = gdn.gate_norm(y.cuda(), z.cuda(), w.cuda(), eps=1e-6, out_dtype=torch.float32).cpu()
    o_ref = oracle.gate_norm(y, z, w, eps=1e-6)
    assert rel_err(f64(o), o_ref) <= TOL["f32"]          # inputs are exact; fp32 math
    assert torch.isfinite(o).all()
    o16 = gdn.gate_norm(y.cuda(), z.cuda(), w.cuda(), eps=1e-6, out_dtype=torch.bfloat16).cpu()
    assert_is_rounding(o16, o)
    assert rel_err(f64(o16), o_ref) <= TOL["bf16"]       # a bf16 o still meets the bf16 bar


@pytest.mark.parametrize("dv", [64, 128, 256])
@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_gate_norm_in_place(dv, dt):
    """o may be y itself (the header's in-place form, which gdn_chunk_fwd_gated uses): the
    result is bit-identical to the out-of-place call, including a ragged last pass of rows."""
    g = torch.Generator().manual_seed(7 + dv)
    rows = 4096 + 37
    y = (torch.randn(rows, dv, generator=g) * 2).to(dt).cuda()
    z = torch.randn(rows, dv, generator=g).to(torch.bfloat16).cuda()
    w = (torch.randn(dv, generator=g) * 0.02).cuda()
    want = gdn.gate_norm(y, z, w, out_dtype=dt)
    yy = y.clone()
    got = gdn.gate_norm(yy, z, w, out=yy)
    torch.cuda.synchronize()
    assert got.data_ptr() == yy.data_ptr()
    assert torch.equal(got, want)


def test_gate_norm_prefill_workload():
    inp = W.make_prefill_inputs(W.WORKLOADS["prefill"])
    y = inp["v"].float() * 0.7                           # an fp32 y of the workload's shape
    o = gdn.gate_norm(y.cuda(), inp["z"].cuda(), inp["w_norm"].cuda(),
                      out_dtype=torch.float32).cpu()
    rows = torch.arange(0, y.shape[0], 97)
    o_ref = oracle.gate_norm(y[rows], inp["z"][rows], inp["w_norm"])
    assert rel_err(f64(o[rows]), o_ref) <= TOL["f32"]
