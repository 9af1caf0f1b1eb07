"""Shared helpers for the parity tests: error metric, oracle runs on chain subsets."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Tolerances: max|y - y_ref| / rms(y_ref) (same for states), from the library's contract:
# fp32 inputs 1e-4; bf16 inputs with fp32 state 2e-2.
TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    if rms == 0.0:
        return float(np.max(np.abs(got - ref)))
    return float(np.max(np.abs(got - ref)) / rms)


def assert_is_rounding(lo: torch.Tensor, hi: torch.Tensor):
    """lo (bf16) is the round-to-nearest-even of hi (fp32), to within one bf16 ulp where
    two launches' fp32 values could differ in the last bit."""
    want = hi.to(torch.bfloat16)
    same = lo.view(torch.int16) == want.view(torch.int16)
    ulp = (lo.float() - want.float()).abs() <= want.float().abs() * 2.0 ** -7 + 1e-30
    assert bool(same.float().mean() > 0.999) and bool(ulp.all())


def f64(t) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def subset(inp: dict, seqs, heads) -> dict:
    """Inputs restricted to the given sequences and heads (CPU tensors, same values)."""
    cu = inp["cu_seqlens"].tolist()
    idx = np.concatenate([np.arange(cu[s], cu[s + 1]) for s in seqs]) if seqs else np.zeros(0, int)
    idx_t = torch.from_numpy(idx.astype(np.int64))
    hs = torch.tensor(list(heads), dtype=torch.int64)
    lens = [cu[s + 1] - cu[s] for s in seqs]
    out = dict(inp)
    for key in ("q", "k", "v", "z"):
        if key in inp:
            out[key] = inp[key].index_select(0, idx_t).index_select(1, hs)
    for key in ("log_alpha", "beta"):
        out[key] = inp[key].index_select(0, idx_t).index_select(1, hs)
    if inp.get("S0") is not None:
        out["S0"] = inp["S0"][list(seqs)][:, list(heads)]
    out["cu_seqlens"] = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    out["H"] = len(heads)
    out["lengths"] = tuple(lens)
    return out, idx_t, hs


def oracle_prefill(inp: dict, scale: float = 1.0):
    """fp64 oracle on CPU inputs. Returns (y [N,H,dv], S_T in the library layout [n,H,dv,dk])."""
    S0 = inp.get("S0")
    S0m = None if S0 is None else oracle.state_from_lib(S0)
    y, S_T, _ = oracle.recurrent(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                 inp["cu_seqlens"].numpy(), S0=S0m, scale=scale)
    return y, oracle.state_to_lib(S_T)


def to_dev(inp: dict, device="cuda") -> dict:
    out = {}
    for key, val in inp.items():
        out[key] = val.to(device) if isinstance(val, torch.Tensor) else val
    return out


def check_all_chains(inp: dict, y, S_T, tol: float, scale: float = 1.0, head_group: int = 8,
                     out_fn=None):
    """Every (sequence, head) chain of a full workload against the oracle, element by
    element: y (or out_fn(y_ref, heads) when given, e.g. the gated output) and the final
    states. Heads are taken head_group at a time to bound host memory. Returns the worst
    (y error, state error)."""
    H = inp["q"].shape[1]
    seqs = list(range(inp["cu_seqlens"].numel() - 1))
    worst_y = worst_s = 0.0
    y = y.cpu()
    S_T = None if S_T is None else S_T.cpu()
    for h0 in range(0, H, head_group):
        heads = list(range(h0, min(H, h0 + head_group)))
        sub, _, hs = subset(inp, seqs, heads)
        y_ref, S_ref = oracle_prefill(sub, scale)
        if out_fn is not None:
            y_ref = out_fn(y_ref, sub)
        ey = rel_err(f64(y.index_select(1, hs)), y_ref)
        worst_y = max(worst_y, ey)
        assert ey <= tol, (heads, ey)
        if S_T is not None:
            es = rel_err(f64(S_T[:, heads]), S_ref)
            worst_s = max(worst_s, es)
            assert es <= tol, (heads, es)
    return worst_y, worst_s
