"""Thin ctypes binding over libgdn.so (include/gdn.h): argument marshalling only.

Every function takes torch CUDA tensors, passes their device pointers and the current CUDA stream
to the C entry point of the same name, and raises ``GdnError`` on a non-OK status.  All arithmetic
happens in the library's kernels; there is no fallback of any kind -- if ``libgdn.so`` is missing
the first call raises.  torch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_TIMEOUT, \
    GDN_ERR_DEVICE_ARG = range(6)
GDN_BF16, GDN_F32 = 0, 1

# name -> (restype, argtypes); mirrors include/gdn.h
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t
SIGNATURES = {
    "gdn_status_string": (ctypes.c_char_p, [_I]),
    "gdn_gates": (_I, [_P, _P, _I, _P, _P, _I64, _I, _P, _P, _P]),
    "gdn_causal_conv1d_silu": (_I, [_P, _I, _P, _P, _I, _I64, _I, _I, _P, _I, _I, _I, _F, _P, _P,
                                    _P, _P]),
    "gdn_chunk_fwd": (_I, [_P, _P, _P, _P, _P, _I, _F, _P, _P, _I, _I, _I64, _I, _I, _I, _I, _I,
                           _P, _P, _P, _SZ, _P]),
    "gdn_chunk_fwd_strided": (_I, [_P, _I64, _P, _I64, _P, _I64, _P, _P, _I, _F, _P, _P, _I, _I,
                                   _I64, _I, _I, _I, _I, _I, _P, _P, _P, _SZ, _P]),
    "gdn_chunk_fwd_gated_norm": (_I, [_P, _I64, _P, _I64, _P, _I64, _P, _P, _P, _P, _P, _P, _F,
                                      _I, _F, _P, _P, _I, _I, _I64, _I, _I, _I, _I, _I, _P, _P,
                                      _P, _SZ, _P]),
    "gdn_chunk_fwd_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _F, _P, _P, _I, _I, _I64, _I, _I, _I,
                                   _I, _I, _P, _P, _P]),
    "gdn_chunk_fwd_workspace_size": (_SZ, [_I, _I, _I64, _I, _I, _I, _I, _I]),
    "gdn_workspace_status": (_I, [_P, _P, ctypes.POINTER(_I)]),
    "gdn_recurrent_step": (_I, [_P, _P, _P, _P, _P, _I, _F, _P, _I, _I, _I, _I, _I, _P, _P]),
    "gdn_gated_rmsnorm": (_I, [_P, _P, _I, _P, _F, _I64, _I, _P, _P]),
    "gdn_decode_layer_step": (_I, [_P, _P, _P, _P, _I, _P, _P, _I, _P, _P, _P, _P, _P, _F, _F, _F,
                                   _P, _I, _I, _I, _I, _I, _P, _P]),
}

_lib = None


class GdnError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)}")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libgdn.so (built by ``python -m gated_deltanet_fwd_b200.build``); raises if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"libgdn.so not found at {path}; build it with "
                               "`python -m gated_deltanet_fwd_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().gdn_status_string(int(status)).decode()


def _check(fn, status):
    if status != GDN_OK:
        raise GdnError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _dt(t):
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"unsupported activation dtype {t.dtype}")


def _cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _tok_stride(t):
    """Token stride of a [B, T, H, d] view whose heads are packed inside each token, else None."""
    B, T, H, d = t.shape
    if not t.is_cuda or t.stride(3) != 1 or t.stride(2) != d:
        return None
    if B > 1 and t.stride(0) != T * t.stride(1):
        return None
    return t.stride(1)


# ------------------------------------------------------------------------------ calls ------

def gdn_gates(a, b, A_log, dt_bias, g=None, beta=None):
    """beta = sigmoid(b), g = -exp(A_log) * softplus(a + dt_bias).  a, b: [..., Hv]."""
    _cuda(a, b, A_log, dt_bias, g, beta)
    Hv = A_log.numel()
    g = torch.empty(a.shape, dtype=torch.float32, device=a.device) if g is None else g
    beta = torch.empty(a.shape, dtype=torch.float32, device=a.device) if beta is None else beta
    _check("gdn_gates", load().gdn_gates(_ptr(a), _ptr(b), _dt(a), _ptr(A_log), _ptr(dt_bias),
                                         a.numel() // Hv, Hv, _ptr(g), _ptr(beta), _stream(a)))
    return g, beta


def gdn_causal_conv1d_silu(x, w, bias=None, cu_seqlens=None, n_l2norm_ch=0, l2norm_group=0,
                           l2_eps=1e-6, conv_state_in=None, conv_state_out=None, y=None):
    """Depthwise causal conv + SiLU (+ per-group L2 norm of the first n_l2norm_ch channels).

    x: [B, T, C]; w: [C, K] fp32; returns y [B, T, C] (x's dtype).
    """
    _cuda(x, w, bias, cu_seqlens, conv_state_in, conv_state_out, y)
    B, T, C = x.shape
    K = w.shape[1]
    N = cu_seqlens.numel() - 1 if cu_seqlens is not None else B
    y = torch.empty_like(x) if y is None else y
    _check("gdn_causal_conv1d_silu", load().gdn_causal_conv1d_silu(
        _ptr(x), _dt(x), _ptr(w), _ptr(bias), B, T, C, K, _ptr(cu_seqlens), N, n_l2norm_ch,
        l2norm_group, float(l2_eps), _ptr(conv_state_in), _ptr(conv_state_out), _ptr(y),
        _stream(x)))
    return y


def workspace_size(N, B, T, Hk, Hv, dk, dv, chunk):
    return int(load().gdn_chunk_fwd_workspace_size(N, B, T, Hk, Hv, dk, dv, chunk))


def workspace_status(workspace) -> int:
    """Blocks on the current stream, then returns the device status word of `workspace`."""
    out = ctypes.c_int(-1)
    _check("gdn_workspace_status", load().gdn_workspace_status(
        _ptr(workspace), _stream(workspace), ctypes.byref(out)))
    return out.value


def gdn_chunk_fwd(q, k, v, g, beta, scale=None, initial_state=None, cu_seqlens=None, chunk=64,
                  out=None, final_state=None, output_final_state=True, workspace=None):
    """Chunked prefill: (q, k, v, g, beta, initial_state, cu_seqlens) -> (out, final_state).

    q, k: [B, T, Hk, dk]; v: [B, T, Hv, dv]; g, beta: [B, T, Hv] fp32; states [N, Hv, dv, dk].
    q, k, v may be views whose tokens are not packed back to back (e.g. slices of the conv's
    [q | k | v] output); those go through gdn_chunk_fwd_strided.
    """
    _cuda(g, beta, initial_state, cu_seqlens, out, final_state, workspace)
    qs, ks, vs = _tok_stride(q), _tok_stride(k), _tok_stride(v)
    if qs is None or ks is None or vs is None:
        raise ValueError("q, k, v must be CUDA [B, T, H, d] tensors with each token's heads packed")
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    N = cu_seqlens.numel() - 1 if cu_seqlens is not None else B
    scale = dk ** -0.5 if scale is None else scale
    out = torch.empty(v.shape, dtype=v.dtype, device=v.device) if out is None else out
    if final_state is None and output_final_state:
        final_state = torch.empty((N, Hv, dv, dk), dtype=torch.float32, device=q.device)
    ws_bytes = workspace_size(N, B, T, Hk, Hv, dk, dv, chunk)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    ws_b = workspace.numel() * workspace.element_size()
    if (qs, ks, vs) == (Hk * dk, Hk * dk, Hv * dv):
        _check("gdn_chunk_fwd", load().gdn_chunk_fwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _dt(q), float(scale),
            _ptr(initial_state), _ptr(cu_seqlens), N, B, T, Hk, Hv, dk, dv, chunk, _ptr(out),
            _ptr(final_state), _ptr(workspace), ws_b, _stream(q)))
    else:
        _check("gdn_chunk_fwd_strided", load().gdn_chunk_fwd_strided(
            _ptr(q), qs, _ptr(k), ks, _ptr(v), vs, _ptr(g), _ptr(beta), _dt(q), float(scale),
            _ptr(initial_state), _ptr(cu_seqlens), N, B, T, Hk, Hv, dk, dv, chunk, _ptr(out),
            _ptr(final_state), _ptr(workspace), ws_b, _stream(q)))
    return out, final_state


def gdn_chunk_fwd_gated_norm(q, k, v, a, b, A_log, dt_bias, z, norm_w, norm_eps=1e-6, scale=None,
                             initial_state=None, cu_seqlens=None, y=None, final_state=None,
                             output_final_state=True, workspace=None):
    """Layer core after the conv in one call: gates(a, b) -> chunked delta rule -> gated RMSNorm
    with z.  q, k: [B, T, Hk, 128]; v: [B, T, Hv, 128] (may be strided views of the conv output);
    a, b: [B, T, Hv] bf16; z: [B, T, Hv, 128] bf16.  Returns (y, final_state)."""
    _cuda(a, b, A_log, dt_bias, z, norm_w, initial_state, cu_seqlens, y, final_state, workspace)
    if len({t.dtype for t in (q, k, v, a, b, z)}) != 1:
        raise TypeError("q, k, v, a, b and z must share one activation dtype")
    qs, ks, vs = _tok_stride(q), _tok_stride(k), _tok_stride(v)
    if qs is None or ks is None or vs is None:
        raise ValueError("q, k, v must be CUDA [B, T, H, d] tensors with each token's heads packed")
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    N = cu_seqlens.numel() - 1 if cu_seqlens is not None else B
    scale = dk ** -0.5 if scale is None else scale
    y = torch.empty(v.shape, dtype=v.dtype, device=v.device) if y is None else y
    if final_state is None and output_final_state:
        final_state = torch.empty((N, Hv, dv, dk), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(workspace_size(N, B, T, Hk, Hv, dk, dv, 64), dtype=torch.uint8,
                                device=q.device)
    _check("gdn_chunk_fwd_gated_norm", load().gdn_chunk_fwd_gated_norm(
        _ptr(q), qs, _ptr(k), ks, _ptr(v), vs, _ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias),
        _ptr(z), _ptr(norm_w), float(norm_eps), _dt(q), float(scale), _ptr(initial_state),
        _ptr(cu_seqlens), N, B, T, Hk, Hv, dk, dv, 64, _ptr(y), _ptr(final_state),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(q)))
    return y, final_state


def gdn_recurrent_step(q, k, v, g, beta, state, scale=None, out=None):
    """One decode token per sequence; `state` [N, Hv, dv, dk] fp32 is updated in place.

    q, k: [N, Hk, dk]; v: [N, Hv, dv]; g, beta: [N, Hv] fp32.  Returns out [N, Hv, dv].
    """
    _cuda(q, k, v, g, beta, state, out)
    N, Hk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    scale = dk ** -0.5 if scale is None else scale
    out = torch.empty_like(v) if out is None else out
    _check("gdn_recurrent_step", load().gdn_recurrent_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _dt(q), float(scale), _ptr(state), N, Hk,
        Hv, dk, dv, _ptr(out), _stream(q)))
    return out


def gdn_decode_layer_step(mix, a, b, z, conv_w, conv_state_in, conv_state_out, A_log, dt_bias,
                          norm_w, state, Hk, conv_bias=None, l2_eps=1e-6, norm_eps=1e-6,
                          scale=None, y=None):
    """One decode token of the layer core: conv (history in conv_state_in, advanced into
    conv_state_out) + SiLU + q/k L2 norm, gates, recurrent step on `state` (in place), gated
    RMSNorm with z.  mix: [N, C]; a, b: [N, Hv]; z: [N, Hv, dv]; returns y [N, Hv, dv]."""
    _cuda(mix, a, b, z, conv_w, conv_bias, conv_state_in, conv_state_out, A_log, dt_bias, norm_w,
          state, y)
    N, Hv, dv = z.shape
    dk = state.shape[3]
    K = conv_w.shape[1]
    scale = dk ** -0.5 if scale is None else scale
    y = torch.empty_like(z) if y is None else y
    _check("gdn_decode_layer_step", load().gdn_decode_layer_step(
        _ptr(mix), _ptr(a), _ptr(b), _ptr(z), _dt(mix), _ptr(conv_w), _ptr(conv_bias), K,
        _ptr(conv_state_in), _ptr(conv_state_out), _ptr(A_log), _ptr(dt_bias), _ptr(norm_w),
        float(l2_eps), float(norm_eps), float(scale), _ptr(state), N, Hk, Hv, dk, dv, _ptr(y),
        _stream(mix)))
    return y


def gdn_gated_rmsnorm(x, z, w, eps=1e-6, y=None):
    """y = x * rsqrt(mean(x^2) + eps) * (1 + w) * silu(z) over the last dim."""
    _cuda(x, z, w, y)
    dim = x.shape[-1]
    y = torch.empty_like(x) if y is None else y
    _check("gdn_gated_rmsnorm", load().gdn_gated_rmsnorm(
        _ptr(x), _ptr(z), _dt(x), _ptr(w), float(eps), x.numel() // dim, dim, _ptr(y),
        _stream(x)))
    return y
