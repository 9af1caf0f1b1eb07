"""Seeded synthetic inputs for the gated delta rule workloads.

This module only draws random numbers and casts them; it holds none of the gated
delta rule's arithmetic. Both the fp64 oracle (tests, CPU baseline) and the CUDA
path (tests, bench) take their inputs from here, so that they see identical values.

Distributions follow the GDN parameterisation on the joezjh.github.io notes page
("Qwen3.8-Flash-Next", section "GDN 参数化细节"): q and k are L2-normalised vectors,
beta = sigmoid(logit), alpha = exp(-exp(A) * softplus(u)) with one A per head; the
value vectors, output gate logits z and the zero-centred RMSNorm weight w are
normal draws. The pages fix no numeric shapes; the shapes below are the five
benchmark workloads of this library:

  tiny      fp32, 1 x 64 tokens, H=2,  d=16,  chunk 16
  prefill   bf16, 4 x 4096,      H=16, d=128, chunk 64
  long      bf16, 1 x 65536,     H=32, d=128, chunk 64, S0 ~ N(0, 0.02), A ~ U(-3, 1)
  varlen    bf16, 8 sequences of U[512, 8192] tokens packed, H=16, d=128, chunk 64
  decode    fp32 state, 256 sequences, H=32, d=128, one token per step

Draw order within one workload: q, k, v, beta logits, A, u, S0, z, w.

The QSA compressed indexer (make_qsa_inputs) takes the indexer's projected query and key
streams: qx ~ N(0, 1) [N_tok, Hq, 128] and kx ~ N(0, 1) [N_tok, 128] in the workload dtype
and the zero-centred RMSNorm weights wq, wk ~ N(0, 0.02); draw order qx, kx, wq, wk. Its
benchmark shape is one 16,384-token sequence with Hq = 4, r = 4, K = 2048 (a scaled-down
stand-in for the pages' 1M-token context prefilled in 16K-token chunks).

The featurisation step in front of the recurrence takes the projected streams instead
(make_featurize_inputs): xq, xk, xv ~ N(0, 1) in the workload dtype, depthwise
convolution weights ~ N(0, 1/W) fp32 with W = 4 taps, beta and alpha logits ~ N(0, 1),
A ~ U(A_range) per head and b_alpha ~ N(0, 0.25) per head; draw order xq, xk, xv,
conv_q, conv_k, conv_v, beta logits, A, alpha logits, b_alpha.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

__all__ = [
    "Workload", "WORKLOADS", "make_prefill_inputs", "make_decode_inputs", "make_featurize_inputs",
    "varlen_lengths", "to_f64", "QSA_WORKLOAD", "make_qsa_inputs",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str            # "f32" or "bf16" for q, k, v, y, z, o
    lengths: tuple        # per-sequence token counts (prefill) ; () for decode
    H: int
    d_k: int
    d_v: int
    chunk: int
    seed: int
    A_range: tuple = (-1.0, 1.0)
    s0_std: float = 0.0   # 0 => zero initial state
    n_seq_decode: int = 0
    decode_steps: int = 0


def varlen_lengths(seed: int = 3, n: int = 8, lo: int = 512, hi: int = 8192) -> tuple:
    """Sequence lengths of the packed variable-length workload, drawn first from `seed`."""
    rng = np.random.default_rng(seed)
    return tuple(int(x) for x in rng.integers(lo, hi + 1, size=n))


WORKLOADS = {
    "tiny": Workload("tiny", "f32", (64,), 2, 16, 16, 16, seed=0),
    "prefill": Workload("prefill", "bf16", (4096,) * 4, 16, 128, 128, 64, seed=1),
    "long": Workload("long", "bf16", (65536,), 32, 128, 128, 64, seed=2,
                     A_range=(-3.0, 1.0), s0_std=0.02),
    "varlen": Workload("varlen", "bf16", varlen_lengths(), 16, 128, 128, 64, seed=3),
    "decode": Workload("decode", "f32", (), 32, 128, 128, 0, seed=4,
                       n_seq_decode=256, decode_steps=1000),
}


def _softplus(x: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, x)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def _cast(x64: np.ndarray, dtype: str) -> torch.Tensor:
    """fp64 -> the workload dtype with round-to-nearest-even (torch's CPU casts)."""
    t = torch.from_numpy(np.ascontiguousarray(x64, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


def _unit_rows(rng: np.random.Generator, shape, dtype: str, block: int = 1 << 14) -> torch.Tensor:
    """N(0,1) vectors along the last axis, L2-normalised in fp64, drawn in row blocks."""
    n = shape[0]
    out = torch.empty(shape, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)
    for r0 in range(0, n, block):
        r1 = min(n, r0 + block)
        x = rng.standard_normal((r1 - r0,) + tuple(shape[1:]))
        x /= np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
        out[r0:r1] = _cast(x, dtype)
    return out


def _normal(rng: np.random.Generator, shape, dtype: str, std: float = 1.0,
            block: int = 1 << 14) -> torch.Tensor:
    n = shape[0]
    out = torch.empty(shape, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)
    for r0 in range(0, n, block):
        r1 = min(n, r0 + block)
        x = rng.standard_normal((r1 - r0,) + tuple(shape[1:])) * std
        out[r0:r1] = _cast(x, dtype)
    return out


def make_prefill_inputs(w: Workload, lengths=None, seed=None, with_gate: bool = True,
                        s0_std=None, A_range=None) -> dict:
    """All tensors of one prefill workload, on the CPU, in the layouts the library takes.

    q, k, v : [N_tok, H, d] in w.dtype (k, q unit vectors)
    log_alpha, beta : [N_tok, H] fp32 (log_alpha <= 0, beta in (0, 1))
    S0 : [n_seq, H, d_v, d_k] fp32 (value-major, the library's state layout) or None
    cu_seqlens : [n_seq + 1] int32
    z : [N_tok, H, d_v] in w.dtype ; w_norm : [d_v] fp32 (stored weight; the scale is 1 + w)
    """
    lengths = tuple(w.lengths if lengths is None else lengths)
    seed = w.seed if seed is None else seed
    s0_std = w.s0_std if s0_std is None else s0_std
    A_lo, A_hi = w.A_range if A_range is None else A_range
    rng = np.random.default_rng(seed)
    n_tok = int(sum(lengths))
    H, dk, dv = w.H, w.d_k, w.d_v
    q = _unit_rows(rng, (n_tok, H, dk), w.dtype)
    k = _unit_rows(rng, (n_tok, H, dk), w.dtype)
    v = _normal(rng, (n_tok, H, dv), w.dtype)
    beta = _sigmoid(rng.standard_normal((n_tok, H)))
    A = rng.uniform(A_lo, A_hi, size=(H,))
    u = rng.standard_normal((n_tok, H))
    log_alpha = -np.exp(A)[None, :] * _softplus(u)
    S0 = None
    if s0_std > 0:
        S0 = torch.from_numpy(
            (rng.standard_normal((len(lengths), H, dv, dk)) * s0_std).astype(np.float32))
    out = dict(
        q=q, k=k, v=v,
        log_alpha=torch.from_numpy(log_alpha.astype(np.float32)),
        beta=torch.from_numpy(beta.astype(np.float32)),
        S0=S0,
        cu_seqlens=torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32),
        H=H, d_k=dk, d_v=dv, chunk=w.chunk, dtype=w.dtype, lengths=lengths,
    )
    if with_gate:
        out["z"] = _normal(rng, (n_tok, H, dv), w.dtype)
        out["w_norm"] = torch.from_numpy((rng.standard_normal(dv) * 0.02).astype(np.float32))
    return out


def make_featurize_inputs(w: Workload, lengths=None, seed=None, width: int = 4) -> dict:
    """Projected streams and gate logits of one prefill workload, for the featurisation step.

    xq, xk : [N_tok, H, d_k], xv : [N_tok, H, d_v] in w.dtype
    conv_q, conv_k : [H*d_k, width], conv_v : [H*d_v, width] fp32
    beta_logit, alpha_logit : [N_tok, H] fp32 ; A, b_alpha : [H] fp32 ; cu_seqlens int32
    """
    lengths = tuple(w.lengths if lengths is None else lengths)
    rng = np.random.default_rng(w.seed if seed is None else seed)
    n_tok = int(sum(lengths))
    H, dk, dv = w.H, w.d_k, w.d_v
    xq = _normal(rng, (n_tok, H, dk), w.dtype)
    xk = _normal(rng, (n_tok, H, dk), w.dtype)
    xv = _normal(rng, (n_tok, H, dv), w.dtype)
    conv = [torch.from_numpy((rng.standard_normal((H * d, width)) / np.sqrt(width)).astype(np.float32))
            for d in (dk, dk, dv)]
    beta_logit = rng.standard_normal((n_tok, H)).astype(np.float32)
    A = rng.uniform(w.A_range[0], w.A_range[1], size=(H,)).astype(np.float32)
    alpha_logit = rng.standard_normal((n_tok, H)).astype(np.float32)
    b_alpha = (rng.standard_normal(H) * 0.5).astype(np.float32)
    return dict(xq=xq, xk=xk, xv=xv, conv_q=conv[0], conv_k=conv[1], conv_v=conv[2],
                beta_logit=torch.from_numpy(beta_logit), alpha_logit=torch.from_numpy(alpha_logit),
                A=torch.from_numpy(A), b_alpha=torch.from_numpy(b_alpha),
                cu_seqlens=torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32),
                H=H, d_k=dk, d_v=dv, dtype=w.dtype, lengths=lengths)


def make_decode_inputs(w: Workload, step: int, n_seq=None, H=None, d=None) -> dict:
    """Inputs of decode step `step`: q, k, v [n_seq, H, d] fp32, alpha, beta [n_seq, H] fp32.

    Each step draws from its own generator default_rng([seed, step]), so any step can
    be regenerated on its own.
    """
    n_seq = w.n_seq_decode if n_seq is None else n_seq
    H = w.H if H is None else H
    d = w.d_k if d is None else d
    rng = np.random.default_rng([w.seed, step])
    q = _unit_rows(rng, (n_seq, H, d), "f32")
    k = _unit_rows(rng, (n_seq, H, d), "f32")
    v = _normal(rng, (n_seq, H, d), "f32")
    beta = _sigmoid(rng.standard_normal((n_seq, H)))
    A = rng.uniform(w.A_range[0], w.A_range[1], size=(H,))
    u = rng.standard_normal((n_seq, H))
    alpha = np.exp(-np.exp(A)[None, :] * _softplus(u))
    return dict(q=q, k=k, v=v,
                alpha=torch.from_numpy(alpha.astype(np.float32)),
                beta=torch.from_numpy(beta.astype(np.float32)))


def to_f64(t) -> np.ndarray:
    """Exact upcast of an fp32/bf16 CPU tensor to a float64 numpy array."""
    if t is None:
        return None
    return t.detach().to("cpu").to(torch.float64).numpy()


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


QSA_WORKLOAD = {"lengths": (16384,), "Hq": 4, "r": 4, "K": 2048, "dtype": "bf16", "seed": 5}


def make_qsa_inputs(lengths, Hq: int, dtype: str = "bf16", seed: int = 5, d: int = 128) -> dict:
    """Inputs of the QSA compressed indexer for packed sequences of the given lengths."""
    rng = np.random.default_rng(seed)
    n = int(sum(lengths))
    cast = (lambda a: torch.from_numpy(a).to(torch.bfloat16)) if dtype == "bf16" else \
        (lambda a: torch.from_numpy(a.astype(np.float32)))
    qx = cast(rng.standard_normal((n, Hq, d)))
    kx = cast(rng.standard_normal((n, d)))
    wq = torch.from_numpy(rng.normal(0.0, 0.02, d).astype(np.float32))
    wk = torch.from_numpy(rng.normal(0.0, 0.02, d).astype(np.float32))
    cu = torch.tensor([0] + list(np.cumsum(lengths)), dtype=torch.int32)
    return {"qx": qx, "kx": kx, "wq": wq, "wk": wk, "cu_seqlens": cu, "lengths": tuple(lengths), "Hq": Hq,
            "dtype": dtype}
