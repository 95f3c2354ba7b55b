"""GPU parity of gdn_chunk_fwd (chunked prefill) against the fp64 oracle.

Every case, the full-size workloads included, is compared element by element on every output
and every final state; the full-size workloads run in the launch configuration the bench times.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_fwd_b200 import gdn, inputs
from gdn_testutil import assert_bf16_close, assert_f32_close, oracle_gates_f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gpu_chunk(x, g, beta, chunk, scale, workspace_bytes=None):
    cu = x["cu_seqlens"]
    S0 = x["initial_state"]
    ws = None
    if workspace_bytes is not None:
        ws = torch.empty(workspace_bytes, dtype=torch.uint8, device=DEV)
    out, S = gdn.gdn_chunk_fwd(x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV), g.to(DEV),
                               beta.to(DEV), scale=scale,
                               initial_state=None if S0 is None else S0.to(DEV),
                               cu_seqlens=None if cu is None else cu.to(DEV), chunk=chunk,
                               workspace=ws)
    torch.cuda.synchronize()
    if ws is not None:
        assert gdn.workspace_status(ws) == gdn.GDN_OK
    return out.cpu(), S.cpu()


NTHREADS = max(1, os.cpu_count() or 1)


def _full_oracle(x, g, beta, scale):
    return oracle.gated_delta_rule(x["q"], x["k"], x["v"], g, beta, scale,
                                   initial_state=x["initial_state"],
                                   cu_seqlens=x["cu_seqlens"], nthreads=NTHREADS)


def _check(dtype, out, S, o_ref, S_ref, what):
    if dtype == "bf16":
        assert_bf16_close(out, o_ref, what + " out")
        assert_bf16_close(S, S_ref, what + " state")
    else:
        assert_f32_close(out, o_ref, what + " out")
        assert_f32_close(S, S_ref, what + " state")


def test_tiny_f32_workload():
    """The tiny all-fp32 check: B=1, T=64, 2 heads, d=16, chunk 16, zero initial state."""
    w = inputs.WORKLOADS["tiny_f32"]
    x = inputs.rule_inputs(**w, seed=1000 + w["index"])
    g, beta = oracle_gates_f32(x)
    out, S = _gpu_chunk(x, g, beta, w["chunk"], w["dk"] ** -0.5)
    o_ref, S_ref = _full_oracle(x, g, beta, w["dk"] ** -0.5)
    _check("f32", out, S, o_ref, S_ref, "tiny")


CASES = [
    # B, T, Hk, Hv, dk, dv, chunk, dtype, seqlens, s0, a_mean
    (1, 200, 1, 2, 128, 128, 64, "bf16", None, 0.02, 0.0),   # tensor-core shape, ragged tail
    (2, 130, 2, 4, 128, 128, 64, "bf16", None, None, -6.0),  # slow decay, batch rows
    (1, 333, 2, 4, 128, 128, 64, "bf16", [1, 64, 0, 65, 127, 76], 0.02, -6.0),  # varlen
    (1, 96, 2, 2, 128, 128, 64, "bf16", None, 0.05, -6.0),   # Hk == Hv
    (1, 150, 1, 2, 128, 128, 32, "bf16", None, 0.02, -6.0),  # CUDA-core path, bf16
    (1, 150, 1, 2, 128, 128, 16, "f32", None, 0.02, -6.0),   # all fp32
    (1, 100, 2, 4, 64, 32, 64, "f32", [37, 0, 63], 0.1, -6.0),
    (1, 81, 1, 1, 16, 48, 16, "f32", None, 0.1, -3.0),
    (1, 70, 1, 2, 128, 64, 64, "bf16", None, 0.02, -6.0),    # dk != dv
]


@pytest.mark.parametrize("case", CASES)
def test_chunk_small_cases(case):
    B, T, Hk, Hv, dk, dv, chunk, dtype, seqlens, s0, a_mean = case
    x = inputs.rule_inputs(B=B, T=T, Hk=Hk, Hv=Hv, dk=dk, dv=dv, dtype=dtype, seed=T + dk,
                           seqlens=seqlens, s0_std=s0, a_mean=a_mean)
    g, beta = oracle_gates_f32(x)
    out, S = _gpu_chunk(x, g, beta, chunk, dk ** -0.5)
    o_ref, S_ref = _full_oracle(x, g, beta, dk ** -0.5)
    _check(dtype, out, S, o_ref, S_ref, str(case))


@pytest.mark.parametrize("case", [c for c in CASES if c[4] == c[5] == 128 and c[6] == 64
                                  and c[7] == "bf16"])
def test_chunk_small_workspace_path(case):
    """The tensor-core shape with only the 256-byte status workspace: the path that keeps no
    per-chunk operands in the workspace (one CTA pair per sequence and head)."""
    B, T, Hk, Hv, dk, dv, chunk, dtype, seqlens, s0, a_mean = case
    x = inputs.rule_inputs(B=B, T=T, Hk=Hk, Hv=Hv, dk=dk, dv=dv, dtype=dtype, seed=T + dk + 1,
                           seqlens=seqlens, s0_std=s0, a_mean=a_mean)
    g, beta = oracle_gates_f32(x)
    out, S = _gpu_chunk(x, g, beta, chunk, dk ** -0.5, workspace_bytes=256)
    o_ref, S_ref = _full_oracle(x, g, beta, dk ** -0.5)
    _check(dtype, out, S, o_ref, S_ref, "small workspace " + str(case))


def test_prefill_varlen_32k_small_workspace_path():
    """The 32K varlen workload on the path without per-chunk workspace, every element."""
    w = inputs.WORKLOADS["prefill_varlen_32k"]
    x = inputs.rule_inputs(**w, seed=1000 + w["index"])
    g, beta = oracle_gates_f32(x)
    out, S = _gpu_chunk(x, g, beta, 64, 128 ** -0.5, workspace_bytes=256)
    o_ref, S_ref = _full_oracle(x, g, beta, 128 ** -0.5)
    assert_bf16_close(out, o_ref, "32k small-workspace path out")
    assert_bf16_close(S, S_ref, "32k small-workspace path final states")


def _no_scan_workspace_bytes(N, n_tok, Hv):
    """Workspace with room for the per-chunk operands but not for the scan's state arrays: the
    tensor-core path then runs one chain per (sequence, v-head).  Layout as in the library:
    1024 header bytes + (ceil(n_tok / 64) + N) chunk slots x Hv x (16384 + 512) bytes."""
    return 1024 + (-(-n_tok // 64) + N) * Hv * (16384 + 512)


SCAN_CASES = [
    # T, seqlens, Hk, Hv, s0, a_mean, zero_g
    (3000, None, 1, 2, 0.02, -6.0, False),          # one sequence, six segments
    (3000, None, 1, 2, 0.02, 0.0, True),            # g = 0: the state carries through every segment
    (4300, [1500, 100, 0, 2600, 100], 2, 4, 0.05, -3.0, False),  # varlen: split and unsplit
    (2049, None, 1, 1, None, -6.0, False),          # Hk = Hv, zero initial state, ragged tail
]


@pytest.mark.parametrize("case", SCAN_CASES)
def test_chunk_intra_sequence_scan(case):
    """Sequences longer than two segments run as the intra-sequence scan (segment 0 and the middle
    segments' affine maps in parallel, a prefix over the maps, then the later segments from their
    entry states); against the oracle, and against the same call without the scan."""
    T, seqlens, Hk, Hv, s0, a_mean, zero_g = case
    x = inputs.rule_inputs(B=1, T=T, Hk=Hk, Hv=Hv, dk=128, dv=128, dtype="bf16", seed=T + Hv,
                           seqlens=seqlens, s0_std=s0, a_mean=a_mean)
    g, beta = oracle_gates_f32(x)
    if zero_g:
        g = torch.zeros_like(g)
    N = x["N"]
    out, S = _gpu_chunk(x, g, beta, 64, 128 ** -0.5)
    o_ref, S_ref = _full_oracle(x, g, beta, 128 ** -0.5)
    _check("bf16", out, S, o_ref, S_ref, "scan " + str(case))
    out1, S1 = _gpu_chunk(x, g, beta, 64, 128 ** -0.5,
                          workspace_bytes=_no_scan_workspace_bytes(N, T, Hv))
    _check("bf16", out1, S1, o_ref, S_ref, "one chain " + str(case))


def test_chunk_zero_decay():
    """g = 0 (no forgetting): nothing damps an error carried between chunks."""
    x = inputs.rule_inputs(B=1, T=256, Hk=1, Hv=2, dk=128, dv=128, seed=4, s0_std=0.02)
    g, beta = oracle_gates_f32(x)
    g = torch.zeros_like(g)
    out, S = _gpu_chunk(x, g, beta, 64, 128 ** -0.5)
    o_ref, S_ref = _full_oracle(x, g, beta, 128 ** -0.5)
    _check("bf16", out, S, o_ref, S_ref, "g=0")


def test_chunk_empty_and_no_state():
    """A zero-length sequence returns its initial state; a NULL initial state means zeros."""
    x = inputs.rule_inputs(B=1, T=64, Hk=1, Hv=2, dk=128, dv=128, seed=9, seqlens=[0, 64],
                           s0_std=0.02)
    g, beta = oracle_gates_f32(x)
    out, S = _gpu_chunk(x, g, beta, 64, 0.1)
    assert torch.equal(S[0], x["initial_state"][0])
    x["initial_state"] = None
    out, S = _gpu_chunk(x, g, beta, 64, 0.1)
    o_ref, S_ref = _full_oracle(x, g, beta, 0.1)
    _check("bf16", out, S, o_ref, S_ref, "no S0")


def _full_size(wname, a_mean=0.0):
    """A full-size workload on the GPU against the oracle over every element of `out` and every
    final state."""
    w = inputs.WORKLOADS[wname]
    x = inputs.rule_inputs(**w, seed=1000 + w["index"], a_mean=a_mean)
    g, beta = oracle_gates_f32(x)
    scale = w["dk"] ** -0.5
    out, S = _gpu_chunk(x, g, beta, w["chunk"], scale)
    o_ref, S_ref = _full_oracle(x, g, beta, scale)
    tag = f"{wname} a_mean={a_mean}"
    assert_bf16_close(out, o_ref, tag + " out (all elements)")
    assert_bf16_close(S, S_ref, tag + " final states (all)")


def test_prefill_4k_full():
    """B=1, T=4096, 16 q/k heads, 32 v heads, d=128, bf16, chunk 64, zero initial state."""
    _full_size("prefill_4k")


def test_prefill_4k_slow_decay_full():
    _full_size("prefill_4k", a_mean=-6.0)


def test_prefill_varlen_32k_full():
    """32768 tokens as 4 sequences (16384/8192/6144/2048) with per-sequence initial states."""
    _full_size("prefill_varlen_32k")


def test_prefill_varlen_32k_slow_decay_full():
    _full_size("prefill_varlen_32k", a_mean=-6.0)


def test_prefill_16k_zero_decay_long_chain():
    """One 16384-token sequence with g = 0: nothing forgets, so any rounding the chunk path
    carries from chunk to chunk (its state operand is rounded to bf16 every chunk) accumulates
    over all 256 chunks instead of being damped away."""
    x = inputs.rule_inputs(B=1, T=16384, Hk=1, Hv=2, dk=128, dv=128, seed=16384, s0_std=0.02)
    g, beta = oracle_gates_f32(x)
    g = torch.zeros_like(g)
    out, S = _gpu_chunk(x, g, beta, 64, 128 ** -0.5)
    o_ref, S_ref = _full_oracle(x, g, beta, 128 ** -0.5)
    assert_bf16_close(out, o_ref, "16k g=0 out")
    assert_bf16_close(S, S_ref, "16k g=0 final state")


@pytest.mark.parametrize("chunk,dtype", [(64, "bf16"), (32, "bf16"), (16, "f32")])
def test_chunk_on_conv_output_views(chunk, dtype):
    """q, k, v as strided views into one [B, T, Hk*dk | Hk*dk | Hv*dv] buffer (the conv's output
    layout), read in place through gdn_chunk_fwd_strided; must equal the dense call exactly."""
    B, T, Hk, Hv, d = 2, 150, 2, 4, 128
    x = inputs.rule_inputs(B=B, T=T, Hk=Hk, Hv=Hv, dk=d, dv=d, dtype=dtype, seed=31,
                           s0_std=0.02, a_mean=-6.0)
    g, beta = oracle_gates_f32(x)
    mix = torch.cat([x["q"].reshape(B, T, -1), x["k"].reshape(B, T, -1),
                     x["v"].reshape(B, T, -1)], dim=-1).to(DEV)
    qv = mix[:, :, :Hk * d].view(B, T, Hk, d)
    kv = mix[:, :, Hk * d:2 * Hk * d].view(B, T, Hk, d)
    vv = mix[:, :, 2 * Hk * d:].view(B, T, Hv, d)
    S0 = x["initial_state"].to(DEV)
    o1, S1 = gdn.gdn_chunk_fwd(qv, kv, vv, g.to(DEV), beta.to(DEV), initial_state=S0,
                               chunk=chunk)
    o2, S2 = gdn.gdn_chunk_fwd(x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV), g.to(DEV),
                               beta.to(DEV), initial_state=S0, chunk=chunk)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
