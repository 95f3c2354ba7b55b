"""Seeded synthetic inputs for the gated delta rule.

This module draws random tensors only: it holds none of the method's arithmetic (no gates, no conv,
no recurrence), so both the CUDA path and the CPU oracle can be fed from it.  Everything is drawn
on the CPU with ``torch.Generator`` in fp32 and then cast to the stated dtype, so that both sides
see the same rounded values.

Distributions follow the workloads of the Qwen3-Next / Qwen3.5 Gated DeltaNet layer:
  * q, k ~ N(0, 1), then scaled to unit L2 norm per head (the layer normalises q and k per head
    before the delta rule); v ~ N(0, 1)
  * a, b ~ N(0, 1) (gate pre-activations; ``a_mean`` shifts a, e.g. -6 for slow decay)
  * A_log = log U[1, 16] per v-head; dt_bias ~ N(0, 0.1) per v-head
  * initial state ~ N(0, s0_std) fp32, independent per sequence, or zero
  * layer-core inputs: q|k|v mix, z ~ N(0, 1) bf16; conv weight ~ U(-1/sqrt(K), 1/sqrt(K));
    RMSNorm weight ~ N(0, 0.02)
"""
from __future__ import annotations

import math

import torch

# Workload shapes.  Seeds are 1000 + index of the workload in this list.
WORKLOADS = {
    "tiny_f32": dict(index=0, B=1, T=64, Hk=2, Hv=2, dk=16, dv=16, dtype="f32", chunk=16),
    "prefill_4k": dict(index=1, B=1, T=4096, Hk=16, Hv=32, dk=128, dv=128, dtype="bf16",
                       chunk=64),
    "prefill_varlen_32k": dict(index=2, B=1, T=32768, Hk=16, Hv=32, dk=128, dv=128,
                               dtype="bf16", chunk=64, seqlens=[16384, 8192, 6144, 2048],
                               s0_std=0.02),
    "decode_256": dict(index=3, N=256, Hk=16, Hv=32, dk=128, dv=128, dtype="bf16", steps=64,
                       s0_std=0.02),
    "layer_core_2x16k": dict(index=4, B=2, T=16384, Hk=16, Hv=32, dk=128, dv=128,
                             dtype="bf16", chunk=64, K=4, eps=1e-6),
    # the decode workload's shapes, one token of the whole layer core per step
    "decode_layer_256": dict(index=3, N=256, Hk=16, Hv=32, dk=128, dv=128, dtype="bf16",
                             steps=64, K=4, s0_std=0.02, eps=1e-6),
}


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _randn(gen, shape, std=1.0, mean=0.0):
    return torch.randn(*shape, generator=gen, dtype=torch.float32) * std + mean


def _unit_heads(x: torch.Tensor) -> torch.Tensor:
    """Scale each head vector (last dim) to unit length -- input preparation only."""
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def cu_from_lengths(lengths) -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


def rule_inputs(*, B, T, Hk, Hv, dk, dv, dtype="bf16", seed=0, seqlens=None, s0_std=None,
                a_mean=0.0, a_std=1.0, N=None, **_unused):
    """Inputs of the delta rule (prefill or, with T == 1, one decode step).

    Returns a dict of CPU tensors: q, k [B,T,Hk,dk] and v [B,T,Hv,dv] in ``dtype``; a, b
    [B,T,Hv] fp32 (gate pre-activations); A_log, dt_bias [Hv] fp32; initial_state
    [N,Hv,dv,dk] fp32 or None; cu_seqlens int32 [N+1] or None.
    """
    gen = _gen(seed)
    dt = torch_dtype(dtype)
    q = _unit_heads(_randn(gen, (B, T, Hk, dk))).to(dt)
    k = _unit_heads(_randn(gen, (B, T, Hk, dk))).to(dt)
    v = _randn(gen, (B, T, Hv, dv)).to(dt)
    a = _randn(gen, (B, T, Hv), std=a_std, mean=a_mean)
    b = _randn(gen, (B, T, Hv))
    A_log = torch.log(torch.rand(Hv, generator=gen, dtype=torch.float32) * 15.0 + 1.0)
    dt_bias = _randn(gen, (Hv,), std=0.1)
    cu = None
    if seqlens is not None:
        assert B == 1 and sum(seqlens) == T
        cu = cu_from_lengths(seqlens)
        N = len(seqlens)
    elif N is None:
        N = B
    S0 = None
    if s0_std:
        S0 = _randn(gen, (N, Hv, dv, dk), std=s0_std)
    return dict(q=q, k=k, v=v, a=a, b=b, A_log=A_log, dt_bias=dt_bias, initial_state=S0,
                cu_seqlens=cu, N=N)


def decode_inputs(*, N, Hk, Hv, dk, dv, dtype="bf16", seed=0, steps=1, s0_std=0.02,
                  **_unused):
    """Inputs of `steps` consecutive one-token decode steps for N sequences.

    Returns state [N,Hv,dv,dk] fp32 and per-step lists of q, k [N,Hk,dk], v [N,Hv,dv] (dtype),
    a, b [N,Hv] fp32, plus A_log, dt_bias [Hv].
    """
    gen = _gen(seed)
    dt = torch_dtype(dtype)
    state = _randn(gen, (N, Hv, dv, dk), std=s0_std)
    A_log = torch.log(torch.rand(Hv, generator=gen, dtype=torch.float32) * 15.0 + 1.0)
    dt_bias = _randn(gen, (Hv,), std=0.1)
    qs, ks, vs, as_, bs = [], [], [], [], []
    for _ in range(steps):
        qs.append(_unit_heads(_randn(gen, (N, Hk, dk))).to(dt))
        ks.append(_unit_heads(_randn(gen, (N, Hk, dk))).to(dt))
        vs.append(_randn(gen, (N, Hv, dv)).to(dt))
        as_.append(_randn(gen, (N, Hv)))
        bs.append(_randn(gen, (N, Hv)))
    return dict(state=state, q=qs, k=ks, v=vs, a=as_, b=bs, A_log=A_log, dt_bias=dt_bias)


def decode_layer_inputs(*, N, Hk, Hv, dk, dv, K=4, dtype="bf16", seed=0, steps=1, s0_std=0.02,
                        **_unused):
    """Inputs of `steps` decode tokens of the whole layer core for N sequences.

    Per step: mix [N, C] (the token's [q | k | v] projections before the conv), a, b [N, Hv] and
    z [N, Hv, dv], all in ``dtype`` and ~ N(0, 1).  Once: conv_w [C, K] ~ U(+-1/sqrt(K)); the conv
    history conv_state [N, C, K-1] (fp32 holding bf16-rounded N(0, 1) values, like past inputs);
    A_log, dt_bias [Hv]; norm_w [dv] ~ N(0, 0.02); state [N, Hv, dv, dk] ~ N(0, s0_std).
    """
    gen = _gen(seed)
    dt = torch_dtype(dtype)
    C = 2 * Hk * dk + Hv * dv
    bound = 1.0 / math.sqrt(K)
    conv_w = (torch.rand(C, K, generator=gen, dtype=torch.float32) * 2.0 - 1.0) * bound
    conv_state = _randn(gen, (N, C, K - 1)).to(dt).float()
    A_log = torch.log(torch.rand(Hv, generator=gen, dtype=torch.float32) * 15.0 + 1.0)
    dt_bias = _randn(gen, (Hv,), std=0.1)
    norm_w = _randn(gen, (dv,), std=0.02)
    state = _randn(gen, (N, Hv, dv, dk), std=s0_std)
    mix, a, b, z = [], [], [], []
    for _ in range(steps):
        mix.append(_randn(gen, (N, C)).to(dt))
        a.append(_randn(gen, (N, Hv)).to(dt))
        b.append(_randn(gen, (N, Hv)).to(dt))
        z.append(_randn(gen, (N, Hv, dv)).to(dt))
    return dict(mix=mix, a=a, b=b, z=z, conv_w=conv_w, conv_state=conv_state, A_log=A_log,
                dt_bias=dt_bias, norm_w=norm_w, state=state, C=C)


def layer_core_inputs(*, B, T, Hk, Hv, dk, dv, K=4, dtype="bf16", seed=0, seqlens=None,
                      **_unused):
    """Inputs of the layer core (projection outputs given as random tensors).

    mix [B,T,2*Hk*dk + Hv*dv] ordered [q | k | v] with each head's channels contiguous;
    z [B,T,Hv,dv]; a, b [B,T,Hv] (dtype); A_log, dt_bias [Hv]; conv_w [C,K];
    norm_w [dv] fp32.
    """
    gen = _gen(seed)
    dt = torch_dtype(dtype)
    C = 2 * Hk * dk + Hv * dv
    mix = _randn(gen, (B, T, C)).to(dt)
    z = _randn(gen, (B, T, Hv, dv)).to(dt)
    a = _randn(gen, (B, T, Hv)).to(dt)
    b = _randn(gen, (B, T, Hv)).to(dt)
    A_log = torch.log(torch.rand(Hv, generator=gen, dtype=torch.float32) * 15.0 + 1.0)
    dt_bias = _randn(gen, (Hv,), std=0.1)
    bound = 1.0 / math.sqrt(K)
    conv_w = (torch.rand(C, K, generator=gen, dtype=torch.float32) * 2.0 - 1.0) * bound
    norm_w = _randn(gen, (dv,), std=0.02)
    cu = cu_from_lengths(seqlens) if seqlens is not None else None
    return dict(mix=mix, z=z, a=a, b=b, A_log=A_log, dt_bias=dt_bias, conv_w=conv_w,
                norm_w=norm_w, cu_seqlens=cu, C=C)


def fused_core_inputs(*, B, T, Hk, Hv, dk, dv, seed=0, seqlens=None, s0_std=None, a_mean=0.0,
                      **_unused):
    """Inputs of the layer core after the conv (q, k, v already L2-normalised as the conv leaves
    them): rule_inputs' q, k, v, initial state and cu_seqlens in bf16, with a, b rounded to bf16
    (they come out of a bf16 projection), z [B,T,Hv,dv] bf16 ~ N(0, 1) and norm_w [dv] fp32
    ~ N(0, 0.02)."""
    x = rule_inputs(B=B, T=T, Hk=Hk, Hv=Hv, dk=dk, dv=dv, dtype="bf16", seed=seed,
                    seqlens=seqlens, s0_std=s0_std, a_mean=a_mean)
    gen = _gen(seed + 7919)
    x["a"] = x["a"].to(torch.bfloat16)
    x["b"] = x["b"].to(torch.bfloat16)
    x["z"] = _randn(gen, (B, T, Hv, dv)).to(torch.bfloat16)
    x["norm_w"] = _randn(gen, (dv,), std=0.02)
    return x
