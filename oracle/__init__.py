"""fp64 CPU oracle of the gated delta rule (ctypes wrapper around gdn_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by __graft_entry__.smoke() and by the
CPU-baseline leg of bench.py, never by the library package. It shares no code with
the CUDA path. See gdn_oracle.c for the passages of the pages each function follows.

State orientation: the oracle works in the pages' S in R^{d_k x d_v}. The library
stores the transpose ([.., d_v, d_k]); `state_to_lib` / `state_from_lib` convert.

Parity status: every function here is pinned by tests/test_oracle_pins.py (the
equivalent update form, brute-force matrix products, invariants, closed forms and
a hand-worked example) and, for the featurisation, tests/test_oracle_featurize.py
(a library convolution, the impulse response, sequence isolation, unit norms and the
gates' closed forms) and, for the gradients, tests/test_oracle_backward.py (central finite
differences of the forward oracle, torch autograd of an independent fp64 restatement,
and closed forms with the gates switched off).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c with gcc (IEEE fp64: -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c99", "-fno-fast-math", "-ffp-contract=off", "-shared",
               "-fPIC", "-o", _LIB, _SRC, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
    return _LIB


def _configure(lib):
    """Declare the C signatures on a loaded copy of the oracle library."""
    lib.gdn_oracle_recurrent.restype = ctypes.c_int
    lib.gdn_oracle_recurrent.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _i64p, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_double, _dp, _dp, ctypes.c_int]
    lib.gdn_oracle_decode_step.restype = ctypes.c_int
    lib.gdn_oracle_decode_step.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _dp, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                           ctypes.c_int]
    lib.gdn_oracle_gate_norm.restype = ctypes.c_int
    lib.gdn_oracle_gate_norm.argtypes = [_dp, _dp, _dp, ctypes.c_int64, ctypes.c_int,
                                         ctypes.c_double, _dp]
    lib.gdn_oracle_backward.restype = ctypes.c_int
    lib.gdn_oracle_backward.argtypes = ([_dp] * 6 + [_i64p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_double] + [_dp] * 8)
    lib.gdn_oracle_featurize.restype = ctypes.c_int
    lib.gdn_oracle_featurize.argtypes = ([_dp] * 6 + [ctypes.c_int] + [_dp] * 4 +
                                         [_i64p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_double] + [_dp] * 5)
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _configure(ctypes.CDLL(_LIB))
    return _lib


def _f64(x) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (fp32 / bf16 upcast exactly)
        import torch
        x = x.detach().to("cpu").to(torch.float64).numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def state_to_lib(S_math: np.ndarray) -> np.ndarray:
    """[.., d_k, d_v] (pages' orientation) -> [.., d_v, d_k] (library layout)."""
    return np.ascontiguousarray(np.swapaxes(S_math, -1, -2))


def state_from_lib(S_lib) -> np.ndarray:
    """[.., d_v, d_k] (library layout) -> [.., d_k, d_v] (pages' orientation)."""
    return np.ascontiguousarray(np.swapaxes(_f64(S_lib), -1, -2))


def recurrent(q, k, v, log_alpha, beta, cu_seqlens, S0=None, scale=1.0, n_threads=0,
              want_state=True):
    """Token-by-token fp64 gated delta rule over packed sequences.

    q, k: [N, H, dk]; v: [N, H, dv]; log_alpha, beta: [N, H]; cu_seqlens: [n_seq+1];
    S0: [n_seq, H, dk, dv] in the pages' orientation, or None for zeros.
    Returns (y [N, H, dv], S_T [n_seq, H, dk, dv] or None, threads used).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, b = _f64(log_alpha), _f64(beta)
    S0 = _f64(S0)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens if not hasattr(cu_seqlens, "numpy")
                                         else cu_seqlens.numpy(), dtype=np.int64))
    n_seq = cu.shape[0] - 1
    N, H, dk = q.shape
    dv = v.shape[2]
    assert k.shape == (N, H, dk) and v.shape[:2] == (N, H) and la.shape == (N, H)
    assert b.shape == (N, H) and int(cu[-1]) == N
    if S0 is not None:
        assert S0.shape == (n_seq, H, dk, dv)
    y = np.zeros((N, H, dv), dtype=np.float64)
    S_T = np.zeros((n_seq, H, dk, dv), dtype=np.float64) if want_state else None
    used = _load().gdn_oracle_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b),
                                        _ptr(S0), cu.ctypes.data_as(_i64p), n_seq, H, dk, dv,
                                        float(scale), _ptr(y), _ptr(S_T), int(n_threads))
    if used < 0:
        raise ValueError("gdn_oracle_recurrent: bad argument")
    return y, S_T, used


def decode_step(q, k, v, alpha, beta, S, scale=1.0, n_threads=0):
    """One fp64 decode step for every chain. S: [.., dk, dv] (pages' orientation) is
    copied, updated and returned with y: returns (y [.., dv], S_new [.., dk, dv])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    a, b = _f64(alpha), _f64(beta)
    S = np.array(_f64(S), dtype=np.float64, copy=True)
    lead = q.shape[:-1]
    dk, dv = q.shape[-1], v.shape[-1]
    n_chain = int(np.prod(lead)) if lead else 1
    assert S.shape == tuple(lead) + (dk, dv)
    y = np.zeros(tuple(lead) + (dv,), dtype=np.float64)
    if _load().gdn_oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(S),
                                      _ptr(y), n_chain, dk, dv, float(scale),
                                      int(n_threads)) < 0:
        raise ValueError("gdn_oracle_decode_step: bad argument")
    return y, S


def gate_norm(y, z, w, eps=1e-6):
    """o = sigmoid(z) * y / sqrt(mean(y^2) + eps) * (1 + w), rows over the last axis."""
    y, z, w = _f64(y), _f64(z), _f64(w)
    dv = y.shape[-1]
    n_rows = int(np.prod(y.shape[:-1])) if y.ndim > 1 else 1
    assert z.shape == y.shape and w.shape == (dv,)
    o = np.zeros_like(y)
    if _load().gdn_oracle_gate_norm(_ptr(y), _ptr(z), _ptr(w), n_rows, dv, float(eps),
                                    _ptr(o)) < 0:
        raise ValueError("gdn_oracle_gate_norm: bad argument")
    return o


def featurize(xq, xk, xv, conv_q, conv_k, conv_v, beta_logit, alpha_logit, A, b_alpha,
              cu_seqlens, eps=1e-6):
    """Short causal convolution -> SiLU -> L2 norm (q, k) and the two gates, in fp64.

    xq, xk: [N, H, dk]; xv: [N, H, dv]; conv_q, conv_k: [H*dk, W]; conv_v: [H*dv, W]
    (tap j multiplies the token W-1-j places back); beta_logit, alpha_logit: [N, H];
    A, b_alpha: [H]. Returns (q, k, v, beta, log_alpha)."""
    xq, xk, xv = _f64(xq), _f64(xk), _f64(xv)
    cq, ck, cv = _f64(conv_q), _f64(conv_k), _f64(conv_v)
    bl, al, A, ba = _f64(beta_logit), _f64(alpha_logit), _f64(A), _f64(b_alpha)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens if not hasattr(cu_seqlens, "numpy")
                                         else cu_seqlens.numpy(), dtype=np.int64))
    n_seq = cu.shape[0] - 1
    N, H, dk = xq.shape
    dv = xv.shape[2]
    W = cq.shape[1]
    assert xk.shape == (N, H, dk) and xv.shape[:2] == (N, H) and int(cu[-1]) == N
    assert cq.shape == (H * dk, W) and ck.shape == (H * dk, W) and cv.shape == (H * dv, W)
    assert bl.shape == (N, H) and al.shape == (N, H) and A.shape == (H,) and ba.shape == (H,)
    q, k = np.zeros((N, H, dk)), np.zeros((N, H, dk))
    v = np.zeros((N, H, dv))
    beta, log_alpha = np.zeros((N, H)), np.zeros((N, H))
    if _load().gdn_oracle_featurize(_ptr(xq), _ptr(xk), _ptr(xv), _ptr(cq), _ptr(ck), _ptr(cv),
                                    int(W), _ptr(bl), _ptr(al), _ptr(A), _ptr(ba),
                                    cu.ctypes.data_as(_i64p), n_seq, H, dk, dv, float(eps),
                                    _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(log_alpha)) < 0:
        raise ValueError("gdn_oracle_featurize: bad argument")
    return q, k, v, beta, log_alpha


def backward(q, k, v, log_alpha, beta, cu_seqlens, dy, S0=None, dS_T=None, scale=1.0):
    """Gradients of L = sum_t <dy_t, y_t> + <dS_T, S_T> for the token recurrence, in fp64.

    Shapes as recurrent(); dy [N, H, dv]; dS_T, S0 [n_seq, H, dk, dv] (pages' orientation)
    or None. Returns (dq, dk, dv, dlog_alpha, dbeta, dS0)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    la, b, dy = _f64(log_alpha), _f64(beta), _f64(dy)
    S0, dS_T = _f64(S0), _f64(dS_T)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens if not hasattr(cu_seqlens, "numpy")
                                         else cu_seqlens.numpy(), dtype=np.int64))
    n_seq = cu.shape[0] - 1
    N, H, dk = q.shape
    dv = v.shape[2]
    assert dy.shape == (N, H, dv) and int(cu[-1]) == N
    out = [np.zeros((N, H, dk)), np.zeros((N, H, dk)), np.zeros((N, H, dv)), np.zeros((N, H)),
           np.zeros((N, H)), np.zeros((n_seq, H, dk, dv))]
    if _load().gdn_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(S0),
                                   cu.ctypes.data_as(_i64p), n_seq, H, dk, dv, float(scale),
                                   _ptr(dy), _ptr(dS_T), *[_ptr(o) for o in out]) < 0:
        raise ValueError("gdn_oracle_backward: bad argument")
    return tuple(out)
