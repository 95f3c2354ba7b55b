"""fp64 CPU oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  The CUDA library never imports it, and it never imports the CUDA library: the two
share no code.  The arithmetic lives in ``gdn_oracle.c`` (plain C, fp64, one token at a time);
this module compiles it with gcc on first use and marshals numpy / torch-CPU arrays into it.

Sources, by page title:
  [P2] "解密Qwen3-Next的Gated DeltaNet：如何用75%混合层实现长文本高效推理" (jsqmd.com)
  [P3] "Qwen3.5 Gated DeltaNet 核心机制解析" (wanger-sjtu.github.io)
  [P5] "Qwen3-Next大模型架构解析：混合注意力与MoE优化实践" (intelliparadigm.com)

Pins: every function here is checked in ``tests/test_oracle.py`` against closed forms, special
cases that reduce to library routines, and an exact brute force on tiny inputs -- never against
its own formula retyped.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "liboracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into _build/liboracle.so (plain gcc, IEEE fp64, no fast-math)."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
                           "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_gates.argtypes = [_D, _D, _D, _D, ctypes.c_int64, ctypes.c_int, _D, _D]
        lib.oracle_gates.restype = None
        lib.oracle_causal_conv1d_silu.argtypes = [
            _D, _D, _D, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int, _I32,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, _D, _D, _D]
        lib.oracle_causal_conv1d_silu.restype = None
        lib.oracle_gated_delta_rule.argtypes = [
            _D, _D, _D, _D, _D, ctypes.c_double, _D, _I32, ctypes.c_int, ctypes.c_int,
            ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _D, _D,
            ctypes.c_int]
        lib.oracle_gated_delta_rule.restype = ctypes.c_int
        lib.oracle_gated_rmsnorm.argtypes = [_D, _D, _D, ctypes.c_double, ctypes.c_int64,
                                             ctypes.c_int, _D]
        lib.oracle_gated_rmsnorm.restype = None
        _lib = lib
    return _lib


def _f64(x):
    """Any array-like (numpy, torch CPU tensor of any float dtype) -> contiguous float64."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: upcast exactly (bf16/fp32 -> fp64 is exact)
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_D)


def _i32(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.ascontiguousarray(x, dtype=np.int32)


def gates(a, b, A_log, dt_bias):
    """beta = sigmoid(b), g = -exp(A_log) * softplus(a + dt_bias)  ([P5] §2.2, [P3] flowchart).

    a, b: [..., Hv]; A_log, dt_bias: [Hv].  Returns (g, beta) as float64 arrays of a's shape.
    """
    a, b, A_log, dt_bias = _f64(a), _f64(b), _f64(A_log), _f64(dt_bias)
    Hv = A_log.shape[0]
    assert a.shape == b.shape and a.shape[-1] == Hv and dt_bias.shape == (Hv,)
    n_tok = a.size // Hv
    g = np.empty_like(a)
    beta = np.empty_like(a)
    _load().oracle_gates(_ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias), n_tok, Hv, _ptr(g),
                         _ptr(beta))
    return g, beta


def causal_conv1d_silu(x, w, bias=None, cu_seqlens=None, n_l2norm_ch=0, l2norm_group=128,
                       l2_eps=1e-6, conv_state_in=None, return_state=False):
    """Depthwise causal conv + SiLU + per-group L2 norm of the leading channels ([P3] conv layer).

    x: [B, T, C]; w: [C, K]; bias: [C] or None; cu_seqlens: [N+1] int32 (then B == 1);
    conv_state_in: [N, C, K-1] or None.  Returns y [B, T, C] (and conv_state_out if asked).
    """
    x, w, bias, cs_in = _f64(x), _f64(w), _f64(bias), _f64(conv_state_in)
    cu = _i32(cu_seqlens)
    B, T, C = x.shape
    K = w.shape[1]
    assert w.shape == (C, K)
    N = (cu.shape[0] - 1) if cu is not None else B
    if cu is not None:
        assert B == 1
    y = np.zeros_like(x)
    cs_out = np.zeros((N, C, K - 1)) if return_state else None
    _load().oracle_causal_conv1d_silu(
        _ptr(x), _ptr(w), _ptr(bias), B, T, C, K,
        None if cu is None else cu.ctypes.data_as(_I32), N, n_l2norm_ch, l2norm_group, l2_eps,
        _ptr(cs_in), _ptr(cs_out), _ptr(y))
    return (y, cs_out) if return_state else y


def gated_delta_rule(q, k, v, g, beta, scale, initial_state=None, cu_seqlens=None, nthreads=1):
    """Token-sequential gated delta rule ([P2] §2.2 call convention; state update of [P3]).

    q, k: [B, T, Hk, dk]; v: [B, T, Hv, dv]; g, beta: [B, T, Hv]; initial_state:
    [N, Hv, dv, dk] or None; cu_seqlens: [N+1] int32 or None (then N == B).
    Returns (out [B, T, Hv, dv], final_state [N, Hv, dv, dk]) in float64.
    """
    q, k, v, g, beta = _f64(q), _f64(k), _f64(v), _f64(g), _f64(beta)
    S0 = _f64(initial_state)
    cu = _i32(cu_seqlens)
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    assert k.shape == q.shape and v.shape[:2] == (B, T) and g.shape == (B, T, Hv)
    assert beta.shape == g.shape
    N = (cu.shape[0] - 1) if cu is not None else B
    out = np.zeros((B, T, Hv, dv))
    S_T = np.zeros((N, Hv, dv, dk))
    rc = _load().oracle_gated_delta_rule(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(S0),
        None if cu is None else cu.ctypes.data_as(_I32), N, B, T, Hk, Hv, dk, dv, _ptr(out),
        _ptr(S_T), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_gated_delta_rule: bad arguments")
    return out, S_T


def gated_rmsnorm(x, z, w, eps=1e-6):
    """y = x / sqrt(mean(x^2) + eps) * (1 + w) * silu(z) over the last dim ([P2] §3.2, [P3])."""
    x, z, w = _f64(x), _f64(z), _f64(w)
    dim = x.shape[-1]
    assert z.shape == x.shape and w.shape == (dim,)
    y = np.empty_like(x)
    _load().oracle_gated_rmsnorm(_ptr(x), _ptr(z), _ptr(w), float(eps), x.size // dim, dim,
                                 _ptr(y))
    return y
