"""gdn_chunk_fwd_noalloc: the allocation-free variant of gdn_chunk_fwd (its scratch is a
fixed device array of the library). Two calls in a row must reproduce gdn_chunk_fwd with
a caller workspace bit for bit, on the tensor-core path (which uses the scratch) and on
a ragged batch; the call must not change how much device memory torch has allocated."""
import pytest
import torch

from tests.test_gpu_parity import custom

gdn = pytest.importorskip("gated_deltanet_05_b200")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)
    yield
    assert gdn.device_error() == "GDN_OK"


def _dev(inp):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


@pytest.mark.parametrize("lengths", [(4096,), (300, 0, 77, 1000)])
def test_noalloc_matches_workspace_entry_point_twice(lengths):
    inp = custom("bf16", lengths, 2, 128, 64, seed=41 + len(lengths), s0_std=0.02)
    d = _dev(inp)
    args = (d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"])
    kw = dict(S0=d["S0"], cu_seqlens_host=inp["cu_seqlens"])
    y_ref, S_ref = gdn.chunk_fwd(*args, **kw)
    y_out = torch.empty_like(y_ref)
    S_out = torch.empty_like(S_ref)
    torch.cuda.synchronize()
    for _ in range(2):
        y_out.fill_(float("nan"))
        S_out.fill_(float("nan"))
        before = torch.cuda.memory_allocated()
        y, S = gdn.chunk_fwd_noalloc(*args, out=y_out, state_out=S_out, **kw)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == before
        assert y is y_out and S is S_out
        assert torch.equal(y, y_ref)
        assert torch.equal(S, S_ref)
