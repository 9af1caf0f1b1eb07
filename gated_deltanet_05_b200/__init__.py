"""gated_deltanet_05_b200 -- Python binding of libgdn_b200.so, the B200 gated delta rule library.

Argument marshalling only: every computation runs in the library's CUDA kernels
(see include/gdn.h for the C ABI). PyTorch supplies device memory and the current
stream. There is no CPU path: if the shared library is missing or fails to load,
importing works but every call raises RuntimeError.

    y, S_T = chunk_fwd(q, k, v, log_alpha, beta, cu_seqlens, S0=None, chunk=64)
    o, S_T = chunk_fwd_gated(q, k, v, log_alpha, beta, cu_seqlens, z, w)   # fused gate-norm
    y = decode_step(q, k, v, alpha, beta, S)          # S updated in place
    y = decode_tokens(q, k, v, alpha, beta, S)        # [n_seq, n, H, d]: n tokens, one pass
    o = gate_norm(y, z, w, eps=1e-6)
    q, k, v, beta, log_alpha = featurize(xq, xk, xv, conv_q, conv_k, conv_v,
                                         beta_logit, alpha_logit, A, b_alpha, cu_seqlens)

State tensors use the library's value-major layout [.., d_v, d_k] in fp32.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["chunk_fwd", "chunk_fwd_gated", "chunk_fwd_noalloc", "backward", "selftest_bounded_wait", "decode_step", "decode_tokens", "gate_norm", "featurize",
           "qsa_indexer", "qsa_token_sets",
           "device_error", "lib", "LIB_PATH",
           "GdnError", "EXPORTED_SYMBOLS", "STATUS"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgdn_b200.so")

STATUS = {0: "GDN_OK", 1: "GDN_ERR_INVALID_ARG", 2: "GDN_ERR_UNSUPPORTED", 3: "GDN_ERR_CUDA",
          4: "GDN_ERR_TIMEOUT", 5: "GDN_ERR_DEVICE_CHECK"}
GDN_F32, GDN_BF16 = 0, 1

EXPORTED_SYMBOLS = ("gdn_chunk_fwd_workspace_bytes", "gdn_chunk_fwd", "gdn_chunk_fwd_gated",
                    "gdn_chunk_fwd_noalloc", "gdn_backward_workspace_bytes", "gdn_backward",
                    "gdn_selftest_bounded_wait", "gdn_decode_step", "gdn_decode_tokens",
                    "gdn_gate_norm", "gdn_featurize", "gdn_qsa_workspace_bytes", "gdn_qsa_indexer",
                    "gdn_qsa_token_sets", "gdn_status_string", "gdn_device_error", "gdn_version")


class GdnError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


_lib = None
_load_error = None


def lib():
    """The loaded ctypes library (raises RuntimeError if it cannot be loaded)."""
    global _lib, _load_error
    if _lib is None:
        if _load_error is not None:
            raise RuntimeError(_load_error)
        try:
            L = ctypes.CDLL(LIB_PATH)
        except OSError as e:
            _load_error = (f"libgdn_b200.so could not be loaded from {LIB_PATH} ({e}); build it "
                           "with `python -m gated_deltanet_05_b200.build`")
            raise RuntimeError(_load_error) from None
        vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
        L.gdn_chunk_fwd_workspace_bytes.restype = ctypes.c_size_t
        L.gdn_chunk_fwd_workspace_bytes.argtypes = [i32, i64, i32, i32, i32, i32]
        L.gdn_chunk_fwd.restype = i32
        L.gdn_chunk_fwd.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                    f32, vp, i32, vp, vp, ctypes.c_size_t, vp]
        L.gdn_chunk_fwd_gated.restype = i32
        L.gdn_chunk_fwd_gated.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                          f32, vp, vp, f32, vp, i32, vp, vp, ctypes.c_size_t, vp]
        L.gdn_backward_workspace_bytes.restype = ctypes.c_size_t
        L.gdn_backward_workspace_bytes.argtypes = [vp, i32, i32, i32, i32]
        L.gdn_backward.restype = i32
        L.gdn_backward.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, vp, vp,
                                   vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.gdn_chunk_fwd_noalloc.restype = i32
        L.gdn_chunk_fwd_noalloc.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, i32, i32, i32, i32,
                                            i32, f32, vp, i32, vp, vp]
        L.gdn_selftest_bounded_wait.restype = i32
        L.gdn_selftest_bounded_wait.argtypes = [i64, i32, vp]
        L.gdn_decode_step.restype = i32
        L.gdn_decode_step.argtypes = [vp, vp, vp, i32, vp, vp, vp, i32, i32, i32, i32, f32, vp, i32, vp]
        L.gdn_decode_tokens.restype = i32
        L.gdn_decode_tokens.argtypes = [vp, vp, vp, i32, vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, i32, vp]
        L.gdn_gate_norm.restype = i32
        L.gdn_gate_norm.argtypes = [vp, i32, vp, i32, vp, i64, i32, f32, vp, i32, vp]
        L.gdn_featurize.restype = i32
        L.gdn_featurize.argtypes = [vp, vp, vp, i32, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, i32, i64,
                                    i32, i32, i32, f32, vp, vp, vp, vp, vp, vp]
        L.gdn_qsa_workspace_bytes.restype = ctypes.c_size_t
        L.gdn_qsa_workspace_bytes.argtypes = [vp, i32, i32, i32, i32, i32]
        L.gdn_qsa_indexer.restype = i32
        L.gdn_qsa_indexer.argtypes = [vp, vp, i32, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, f32, vp, vp,
                                      vp, ctypes.c_size_t, vp]
        L.gdn_qsa_token_sets.restype = i32
        L.gdn_qsa_token_sets.argtypes = [vp, vp, vp, i32, i32, i32, vp, vp, vp]
        L.gdn_status_string.restype = ctypes.c_char_p
        L.gdn_status_string.argtypes = [i32]
        L.gdn_device_error.restype = i32
        L.gdn_device_error.argtypes = [vp]
        L.gdn_version.restype = i32
        L.gdn_version.argtypes = []
        _lib = L
    return _lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return GDN_F32
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _cuda(t: torch.Tensor, name: str):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(fn: str, code: int):
    if code != 0:
        raise GdnError(fn, code)


_workspaces = {}


def _workspace(device, nbytes):
    """Device scratch for gdn_chunk_fwd, kept per device and grown on demand. One buffer
    serves every call on a device: the library indexes it by SM id, so calls on
    different streams do not collide."""
    if nbytes == 0:
        return None
    idx = device.index if device.index is not None else torch.cuda.current_device()
    ws = _workspaces.get(idx)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        _workspaces[idx] = ws
    return ws


def _chunk_setup(q, k, v, log_alpha, beta, cu_seqlens, S0, cu_seqlens_host, out, final_state,
                 state_out, y_dtype):
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (log_alpha, "log_alpha"), (beta, "beta"),
                 (cu_seqlens, "cu_seqlens")):
        _cuda(t, n)
    _cuda(S0, "S0")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    if log_alpha.dtype != torch.float32 or beta.dtype != torch.float32:
        raise TypeError("log_alpha and beta must be float32")
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    N, H, dk = q.shape
    dv = v.shape[2]
    n_seq = cu_seqlens.numel() - 1
    if cu_seqlens_host is None:
        cu_seqlens_host = cu_seqlens.to("cpu")
    cu_h = cu_seqlens_host.to(torch.int32).contiguous()
    y = out if out is not None else torch.empty((N, H, dv), dtype=y_dtype, device=q.device)
    _cuda(y, "out")
    S_T = None
    if final_state:
        S_T = (state_out if state_out is not None
               else torch.empty((n_seq, H, dv, dk), dtype=torch.float32, device=q.device))
        _cuda(S_T, "state_out")
    args = (_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(log_alpha), _ptr(beta), _ptr(S0),
            _ptr(cu_seqlens), ctypes.c_void_p(cu_h.data_ptr()), n_seq, H, dk, dv)
    return args, y, S_T, cu_h


def chunk_fwd(q, k, v, log_alpha, beta, cu_seqlens, S0=None, chunk=64, scale=1.0,
              cu_seqlens_host=None, out=None, final_state=True, y_dtype=torch.float32,
              state_out=None):
    """Chunked prefill over packed sequences. Returns (y, S_T or None).

    q, k [N, H, d_k] and v [N, H, d_v] (fp32 or bf16, same dtype); log_alpha, beta [N, H]
    fp32; cu_seqlens [n_seq + 1] int32 (device); S0 [n_seq, H, d_v, d_k] fp32 or None.
    y is returned in y_dtype (float32 by default; bfloat16 gives the round-to-nearest-even
    of the same fp32 result). out / state_out may supply the output tensors.
    """
    args, y, S_T, cu_h = _chunk_setup(q, k, v, log_alpha, beta, cu_seqlens, S0, cu_seqlens_host,
                                      out, final_state, state_out, y_dtype)
    L = lib()
    n_seq, H, dk, dv = args[9], args[10], args[11], args[12]
    ws_bytes = L.gdn_chunk_fwd_workspace_bytes(n_seq, q.shape[0], H, dk, dv, chunk)
    ws = _workspace(q.device, ws_bytes)
    rc = L.gdn_chunk_fwd(*args, int(chunk), float(scale), _ptr(y), _dtype_code(y), _ptr(S_T),
                         _ptr(ws), ws_bytes, _stream(q.device))
    _check("gdn_chunk_fwd", rc)
    return y, S_T


def chunk_fwd_gated(q, k, v, log_alpha, beta, cu_seqlens, z, w, eps=1e-6, S0=None, chunk=64,
                    scale=1.0, cu_seqlens_host=None, out=None, final_state=True,
                    o_dtype=torch.bfloat16, state_out=None):
    """chunk_fwd and the output epilogue in one library call: returns (o, S_T or None), where
    o = sigmoid(z) * y / sqrt(mean(y^2) + eps) * (1 + w) per (token, head) and y is the
    chunk_fwd output in o_dtype (written into o, then normalised in place). Tensor-core path
    only: bf16 q, k, v and z, d = 128, chunk 64 (other shapes raise GdnError
    GDN_ERR_UNSUPPORTED). w [d_v] fp32."""
    _cuda(z, "z")
    _cuda(w, "w")
    if z.dtype != torch.bfloat16 or z.shape != v.shape:
        raise TypeError("z must be bfloat16 with v's shape")
    if w.dtype != torch.float32 or w.numel() != v.shape[-1]:
        raise TypeError("w must be float32 [d_v]")
    args, o, S_T, cu_h = _chunk_setup(q, k, v, log_alpha, beta, cu_seqlens, S0, cu_seqlens_host,
                                      out, final_state, state_out, o_dtype)
    L = lib()
    n_seq, H, dk, dv = args[9], args[10], args[11], args[12]
    ws_bytes = L.gdn_chunk_fwd_workspace_bytes(n_seq, q.shape[0], H, dk, dv, chunk)
    ws = _workspace(q.device, ws_bytes)
    rc = L.gdn_chunk_fwd_gated(*args, int(chunk), float(scale), _ptr(z), _ptr(w), float(eps), _ptr(o),
                               _dtype_code(o), _ptr(S_T), _ptr(ws), ws_bytes, _stream(q.device))
    _check("gdn_chunk_fwd_gated", rc)
    return o, S_T


def backward(q, k, v, log_alpha, beta, cu_seqlens, dy, S0=None, dS_T=None, scale=1.0,
             cu_seqlens_host=None):
    """Gradients of L = sum <dy, y> + <dS_T, S_T> through the prefill.

    Inputs as chunk_fwd; dy [N, H, d_v] in q's dtype; dS_T [n_seq, H, d_v, d_k] fp32 or None.
    Returns (dq, dk, dv, dlog_alpha, dbeta, dS0), all fp32 (dS0 in the state layout)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (log_alpha, "log_alpha"), (beta, "beta"),
                 (cu_seqlens, "cu_seqlens"), (dy, "dy")):
        _cuda(t, n)
    _cuda(S0, "S0")
    _cuda(dS_T, "dS_T")
    if k.dtype != q.dtype or v.dtype != q.dtype or dy.dtype != q.dtype:
        raise TypeError("q, k, v, dy must share one dtype")
    N, H, dk = q.shape
    dv = v.shape[2]
    n_seq = cu_seqlens.numel() - 1
    if cu_seqlens_host is None:
        cu_seqlens_host = cu_seqlens.to("cpu")
    cu_h = cu_seqlens_host.to(torch.int32).contiguous()
    L = lib()
    ws_bytes = L.gdn_backward_workspace_bytes(ctypes.c_void_p(cu_h.data_ptr()), n_seq, H, dk, dv)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    f = dict(dtype=torch.float32, device=q.device)
    dq, dkk, dvv = torch.empty((N, H, dk), **f), torch.empty((N, H, dk), **f), torch.empty((N, H, dv), **f)
    dla, db = torch.empty((N, H), **f), torch.empty((N, H), **f)
    dS0 = torch.empty((n_seq, H, dv, dk), **f)
    rc = L.gdn_backward(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), _ptr(log_alpha), _ptr(beta), _ptr(S0),
                        _ptr(cu_seqlens), ctypes.c_void_p(cu_h.data_ptr()), n_seq, H, dk, dv, float(scale),
                        _ptr(dy), _ptr(dS_T), _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dla), _ptr(db), _ptr(dS0),
                        _ptr(ws), ws_bytes, _stream(q.device))
    _check("gdn_backward", rc)
    return dq, dkk, dvv, dla, db, dS0


def chunk_fwd_noalloc(q, k, v, log_alpha, beta, cu_seqlens, S0=None, chunk=64, scale=1.0,
                      cu_seqlens_host=None, out=None, final_state=True, y_dtype=torch.float32,
                      state_out=None):
    """chunk_fwd through gdn_chunk_fwd_noalloc: the library call allocates nothing (its
    scratch is a fixed device array of the library). Pass out / state_out (and a host
    cu_seqlens) for a call that allocates nothing on this side either."""
    args, y, S_T, cu_h = _chunk_setup(q, k, v, log_alpha, beta, cu_seqlens, S0, cu_seqlens_host,
                                      out, final_state, state_out, y_dtype)
    rc = lib().gdn_chunk_fwd_noalloc(*args, int(chunk), float(scale), _ptr(y), _dtype_code(y),
                                     _ptr(S_T), _stream(q.device))
    _check("gdn_chunk_fwd_noalloc", rc)
    return y, S_T


def decode_step(q, k, v, alpha, beta, S, scale=1.0, out=None, y_dtype=torch.float32):
    """One token per chain; S [n_seq, H, d_v, d_k] fp32 is updated in place. Returns y in
    y_dtype (float32 by default; bfloat16 gives the round-to-nearest-even of the same fp32
    result), or in out's dtype when out is given."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (alpha, "alpha"), (beta, "beta"), (S, "S")):
        _cuda(t, n)
    code = _dtype_code(q)
    n_seq, H, dk = q.shape
    dv = v.shape[2]
    y = out if out is not None else torch.empty((n_seq, H, dv), dtype=y_dtype, device=q.device)
    _cuda(y, "out")
    rc = lib().gdn_decode_step(_ptr(q), _ptr(k), _ptr(v), code, _ptr(alpha), _ptr(beta), _ptr(S),
                               n_seq, H, dk, dv, float(scale), _ptr(y), _dtype_code(y),
                               _stream(q.device))
    _check("gdn_decode_step", rc)
    return y


def decode_tokens(q, k, v, alpha, beta, S, scale=1.0, out=None, y_dtype=torch.float32):
    """n consecutive tokens per chain in one pass over the state (S updated in place).

    q, k [n_seq, n, H, d_k], v [n_seq, n, H, d_v] (fp32 or bf16, one dtype); alpha, beta
    [n_seq, n, H] fp32; S [n_seq, H, d_v, d_k] fp32. Returns y [n_seq, n, H, d_v] in
    y_dtype (float32 by default; bfloat16 gives the round-to-nearest-even of the same fp32
    result), or in out's dtype when out is given."""
    for t, nm in ((q, "q"), (k, "k"), (v, "v"), (alpha, "alpha"), (beta, "beta"), (S, "S")):
        _cuda(t, nm)
    code = _dtype_code(q)
    n_seq, n, H, dk = q.shape
    dv = v.shape[3]
    y = out if out is not None else torch.empty((n_seq, n, H, dv), dtype=y_dtype, device=q.device)
    _cuda(y, "out")
    rc = lib().gdn_decode_tokens(_ptr(q), _ptr(k), _ptr(v), code, _ptr(alpha), _ptr(beta), _ptr(S),
                                 n_seq, n, H, dk, dv, float(scale), _ptr(y), _dtype_code(y),
                                 _stream(q.device))
    _check("gdn_decode_tokens", rc)
    return y


def gate_norm(y, z, w, eps=1e-6, out=None, out_dtype=None):
    """o = sigmoid(z) * y / sqrt(mean(y^2) + eps) * (1 + w) over the last axis.

    y and z may each be float32 or bfloat16; o is out_dtype (default: y's dtype)."""
    for t, n in ((y, "y"), (z, "z"), (w, "w")):
        _cuda(t, n)
    if z.shape != y.shape:
        raise ValueError("z must have y's shape")
    if w.dtype != torch.float32 or w.numel() != y.shape[-1]:
        raise TypeError("w must be float32 [d_v]")
    dv = y.shape[-1]
    n_rows = y.numel() // dv
    if out is None:
        out = torch.empty(y.shape, dtype=out_dtype or y.dtype, device=y.device)
    _cuda(out, "out")
    o = out
    rc = lib().gdn_gate_norm(_ptr(y), _dtype_code(y), _ptr(z), _dtype_code(z), _ptr(w), n_rows,
                             dv, float(eps), _ptr(o), _dtype_code(o), _stream(y.device))
    _check("gdn_gate_norm", rc)
    return o


def featurize(xq, xk, xv, conv_q, conv_k, conv_v, beta_logit, alpha_logit, A, b_alpha, cu_seqlens,
              eps=1e-6, cu_seqlens_host=None, out=None):
    """Short causal convolution -> SiLU -> L2 norm (q, k), and the gates, for packed sequences.

    xq, xk [N, H, d_k] and xv [N, H, d_v] (one dtype, fp32 or bf16): the projected streams;
    conv_q, conv_k [H*d_k, W] and conv_v [H*d_v, W] fp32 (W <= 4; tap j multiplies the token
    W-1-j places back); beta_logit, alpha_logit [N, H] fp32; A, b_alpha [H] fp32;
    cu_seqlens [n_seq + 1] int32 (device). Returns (q, k, v, beta, log_alpha): q, k, v in
    the input dtype and beta, log_alpha fp32, ready for chunk_fwd. `out` may supply those
    five tensors."""
    for t, n in ((xq, "xq"), (xk, "xk"), (xv, "xv"), (conv_q, "conv_q"), (conv_k, "conv_k"),
                 (conv_v, "conv_v"), (beta_logit, "beta_logit"), (alpha_logit, "alpha_logit"),
                 (A, "A"), (b_alpha, "b_alpha"), (cu_seqlens, "cu_seqlens")):
        _cuda(t, n)
    if xk.dtype != xq.dtype or xv.dtype != xq.dtype:
        raise TypeError("xq, xk, xv must share one dtype")
    for t, n in ((conv_q, "conv_q"), (conv_k, "conv_k"), (conv_v, "conv_v"), (beta_logit, "beta_logit"),
                 (alpha_logit, "alpha_logit"), (A, "A"), (b_alpha, "b_alpha")):
        if t.dtype != torch.float32:
            raise TypeError(f"{n} must be float32")
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    N, H, dk = xq.shape
    dv = xv.shape[2]
    W = conv_q.shape[1]
    if tuple(conv_q.shape) != (H * dk, W) or tuple(conv_k.shape) != (H * dk, W) or \
            tuple(conv_v.shape) != (H * dv, W):
        raise ValueError("conv weights must be [H*d, W] with one W")
    n_seq = cu_seqlens.numel() - 1
    if cu_seqlens_host is None:
        cu_seqlens_host = cu_seqlens.to("cpu")
    cu_h = cu_seqlens_host.to(torch.int32).contiguous()
    if out is None:
        out = (torch.empty_like(xq), torch.empty_like(xk), torch.empty_like(xv),
               torch.empty((N, H), dtype=torch.float32, device=xq.device),
               torch.empty((N, H), dtype=torch.float32, device=xq.device))
    for t, n in zip(out, ("q", "k", "v", "beta", "log_alpha")):
        _cuda(t, n)
    q, k, v, beta, log_alpha = out
    rc = lib().gdn_featurize(_ptr(xq), _ptr(xk), _ptr(xv), _dtype_code(xq), _ptr(conv_q), _ptr(conv_k),
                             _ptr(conv_v), int(W), _ptr(beta_logit), _ptr(alpha_logit), _ptr(A),
                             _ptr(b_alpha), _ptr(cu_seqlens), ctypes.c_void_p(cu_h.data_ptr()), n_seq,
                             N, H, dk, dv, float(eps), _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                             _ptr(log_alpha), _stream(xq.device))
    _check("gdn_featurize", rc)
    return q, k, v, beta, log_alpha


def qsa_indexer(qx, kx, wq, wk, cu_seqlens, r=4, K=2048, rot=64, base=10000.0, eps=1e-6,
                cu_seqlens_host=None, out=None):
    """The QSA compressed indexer over packed sequences (see gdn_qsa_indexer in gdn.h).

    qx [N, Hq, 128] and kx [N, 128] (one dtype: bfloat16 runs the tensor-core scores,
    float32 the fp32 CUDA-core ones); wq, wk [128] fp32 (zero-centred RMSNorm weights);
    cu_seqlens [n_seq + 1] int32 (device). Returns (scores [N, nb_max] fp32, valid only for
    each token's visible blocks, blocks [N, ceil(K / r)] int32, -1 padded). `out` may
    supply (scores, blocks)."""
    for t, n in ((qx, "qx"), (kx, "kx"), (wq, "wq"), (wk, "wk"), (cu_seqlens, "cu_seqlens")):
        _cuda(t, n)
    if kx.dtype != qx.dtype:
        raise TypeError("qx and kx must share one dtype")
    if wq.dtype != torch.float32 or wk.dtype != torch.float32:
        raise TypeError("wq and wk must be float32")
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    N, Hq, d = qx.shape
    n_seq = cu_seqlens.numel() - 1
    if cu_seqlens_host is None:
        cu_seqlens_host = cu_seqlens.to("cpu")
    cu_h = cu_seqlens_host.to(torch.int32).contiguous()
    lens = (cu_h[1:] - cu_h[:-1]).tolist()
    nb_max = max([ln // r for ln in lens] + [0])
    kb = -(-K // r)
    if out is None:
        out = (torch.empty((N, max(nb_max, 1)), dtype=torch.float32, device=qx.device),
               torch.empty((N, kb), dtype=torch.int32, device=qx.device))
    scores, blocks = out
    _cuda(scores, "scores")
    _cuda(blocks, "blocks")
    L = lib()
    code = _dtype_code(qx)
    ws_bytes = L.gdn_qsa_workspace_bytes(ctypes.c_void_p(cu_h.data_ptr()), n_seq, Hq, d, r, code)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=qx.device)
    rc = L.gdn_qsa_indexer(_ptr(qx), _ptr(kx), code, _ptr(wq), _ptr(wk), _ptr(cu_seqlens),
                           ctypes.c_void_p(cu_h.data_ptr()), n_seq, Hq, d, int(r), int(K), int(rot),
                           float(base), float(eps), _ptr(scores), _ptr(blocks), _ptr(ws), ws_bytes,
                           _stream(qx.device))
    _check("gdn_qsa_indexer", rc)
    return scores[:, :nb_max], blocks


def qsa_token_sets(blocks, cu_seqlens, r=4, cu_seqlens_host=None):
    """Token sets of the QSA indexer's selection: (tokens [N, K_B * r + r - 1] int32 in
    ascending order, -1 padded, positions within each sequence; count [N] int32)."""
    _cuda(blocks, "blocks")
    _cuda(cu_seqlens, "cu_seqlens")
    if blocks.dtype != torch.int32:
        raise TypeError("blocks must be int32")
    N, kb = blocks.shape
    n_seq = cu_seqlens.numel() - 1
    if cu_seqlens_host is None:
        cu_seqlens_host = cu_seqlens.to("cpu")
    cu_h = cu_seqlens_host.to(torch.int32).contiguous()
    tokens = torch.empty((N, kb * r + r - 1), dtype=torch.int32, device=blocks.device)
    count = torch.empty((N,), dtype=torch.int32, device=blocks.device)
    rc = lib().gdn_qsa_token_sets(_ptr(blocks), _ptr(cu_seqlens), ctypes.c_void_p(cu_h.data_ptr()), n_seq, kb,
                                  int(r), _ptr(tokens), _ptr(count), _stream(blocks.device))
    _check("gdn_qsa_token_sets", rc)
    return tokens, count


def selftest_bounded_wait(limit_cycles=2_000_000, mode=0, device=None):
    """Runs the kernels' bounded wait on the device (see gdn_selftest_bounded_wait) and
    returns the device error status it leaves: "GDN_ERR_TIMEOUT" for mode 0 (the wait ran
    out), "GDN_OK" for modes 1 (aborted by another thread) and 2 (completed)."""
    dev = device if device is not None else torch.cuda.current_device()
    _check("gdn_selftest_bounded_wait", lib().gdn_selftest_bounded_wait(int(limit_cycles), int(mode), _stream(dev)))
    return device_error(dev)


def device_error(device=None) -> str:
    """Synchronises the current stream and returns (and clears) the device error status."""
    dev = device if device is not None else torch.cuda.current_device()
    return STATUS.get(lib().gdn_device_error(_stream(dev)), "?")
