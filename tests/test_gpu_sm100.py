"""GPU parity of the sm_100a tensor-core prefill kernel (bf16 q/k/v, d_k = d_v = 128,
chunk 64, fp32 state) against the fp64 oracle, through the C ABI.

Bar: max|got - ref| / rms(ref) <= 2e-2 on y and on the final states (bf16 inputs, fp32
state). Ragged lengths cover partial chunks, empty and one-token sequences; the full
workloads (4 x 4096 tokens H = 16; 65,536 tokens H = 32 with S0 != 0; the packed varlen
batch, H = 16) compare every chain element by element, y and final state, with y
pre-filled with NaN so that an unwritten output fails. The pages' invariants run on the
tensor-core path too: gates off (alpha = 1, beta = 0) leave S_T = S0 and give
y_t = S0^T q_t; alpha = beta = 1 with orthonormal keys (exact in bf16) retrieves v_s when
q_t = k_s. Inputs beyond the fp16 range of the kernel's operands raise
GDN_ERR_DEVICE_CHECK.
"""
import numpy as np
import pytest
import torch

import workloads as W
from tests.helpers import TOL, check_all_chains, f64, oracle_prefill, rel_err, to_dev
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


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_degenerate_gates(dtype):
    """beta in {0, 1} and log alpha in {0, -30} per token (no decay, and a decay whose
    cumulative sum underflows exp within a chunk), S0 != 0: the tensor-core path (bf16) and
    the fp32 chunk kernel against the oracle."""
    inp = custom(dtype, (200, 64, 5), 2, 128, 64, seed=21, s0_std=0.02)
    rng = np.random.default_rng(22)
    shape = tuple(inp["beta"].shape)
    inp["beta"] = torch.from_numpy(rng.choice([0.0, 1.0], size=shape).astype(np.float32))
    inp["log_alpha"] = torch.from_numpy(rng.choice([0.0, -30.0], size=shape, p=[0.9, 0.1]).astype(np.float32))
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


def _check_full(name):
    inp = W.make_prefill_inputs(W.WORKLOADS[name])
    d = to_dev(inp)
    y = torch.full(inp["v"].shape, float("nan"), dtype=torch.float32, device="cuda")
    y, S_T = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                           S0=d.get("S0"), cu_seqlens_host=inp["cu_seqlens"], out=y)
    torch.cuda.synchronize()
    assert torch.isfinite(y).all() and torch.isfinite(S_T).all()
    check_all_chains(inp, y, S_T, TOL[inp["dtype"]])


def test_prefill_workload_every_chain():
    _check_full("prefill")


def test_varlen_workload_every_chain():
    _check_full("varlen")


def test_long_workload_every_chain():
    _check_full("long")


def _orthonormal_bf16_keys(n, d, seed):
    """n <= d orthonormal vectors that bf16 holds exactly: rows of a block-diagonal
    16 x 16 Sylvester-Hadamard matrix / 4 (entries +-1/4), coordinates permuted and signs
    flipped at random."""
    h = np.array([[1.0]])
    while h.shape[0] < 16:
        h = np.block([[h, h], [h, -h]])
    basis = np.kron(np.eye(d // 16), h / 4.0)
    rng = np.random.default_rng(seed)
    basis = basis[rng.permutation(d)][:, rng.permutation(d)] * rng.choice([-1.0, 1.0], size=d)
    return basis[:n]


def _invariant_inputs(T, H, seed, s0_std):
    inp = custom("bf16", (T,), H, 128, 64, seed=seed, s0_std=s0_std)
    return inp


def test_tensor_core_gates_off_keep_the_state():
    """alpha = 1, beta = 0: S_T = S0 and y_t = S0^T q_t (the state never changes)."""
    inp = _invariant_inputs(200, 2, seed=31, s0_std=0.05)
    inp["log_alpha"] = torch.zeros_like(inp["log_alpha"])
    inp["beta"] = torch.zeros_like(inp["beta"])
    y, S_T = run_prefill(inp)
    S0 = inp["S0"].double()                                  # [1, H, dv, dk]
    y_ref = torch.einsum("hvk,thk->thv", S0[0], inp["q"].double())
    assert rel_err(f64(y), y_ref.numpy()) <= TOL["bf16"]
    assert rel_err(f64(S_T), S0.numpy()) <= TOL["bf16"]


@pytest.mark.parametrize("T", [64, 100, 128])
def test_tensor_core_orthonormal_keys_retrieve_values(T):
    """alpha = beta = 1, S0 = 0, orthonormal keys: S_t^T k_s = v_s for every s <= t, so
    the query q_t = k_{s(t)} with s(t) <= t reads back v_{s(t)} exactly."""
    H, d = 2, 128
    inp = _invariant_inputs(T, H, seed=32 + T, s0_std=0.0)
    rng = np.random.default_rng(T)
    k = np.stack([_orthonormal_bf16_keys(T, d, seed=100 * T + h) for h in range(H)], 1)
    src = np.stack([rng.integers(0, np.arange(T) + 1) for _ in range(H)], 1)   # s(t) <= t
    q = np.stack([k[src[:, h], h] for h in range(H)], 1)
    inp["k"] = torch.from_numpy(np.ascontiguousarray(k)).to(torch.bfloat16)
    inp["q"] = torch.from_numpy(np.ascontiguousarray(q)).to(torch.bfloat16)
    inp["log_alpha"] = torch.zeros_like(inp["log_alpha"])
    inp["beta"] = torch.ones_like(inp["beta"])
    assert torch.equal(inp["k"].double(), torch.from_numpy(k))    # exact in bf16
    y, _ = run_prefill(inp)
    v = inp["v"].double().numpy()           # [T, H, d]
    want = np.stack([v[src[:, h], h] for h in range(H)], 1)
    assert rel_err(f64(y), want) <= TOL["bf16"]


@pytest.mark.parametrize("which", ["q", "k", "v", "S0"])
def test_tensor_core_rejects_values_beyond_fp16(which):
    """The kernel's fp16 operands hold |x| < 65520; an input beyond that is reported as
    GDN_ERR_DEVICE_CHECK instead of turning into inf silently."""
    inp = _invariant_inputs(130, 2, seed=40, s0_std=0.02)
    inp["log_alpha"] = torch.zeros_like(inp["log_alpha"])     # q is converted as gamma * q
    t = inp[which]
    flat = t.view(-1)
    flat[flat.numel() // 3] = 70000.0 if which != "S0" else 1e6
    run_prefill(inp)
    assert gdn.device_error() == "GDN_ERR_DEVICE_CHECK"
    # the library stays usable
    good = _invariant_inputs(130, 2, seed=41, s0_std=0.02)
    check_prefill(good)
    assert gdn.device_error() == "GDN_OK"
