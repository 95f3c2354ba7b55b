"""Device-detected faults on the GPU, in the forms that fault, trap or hang nothing.

A malformed cu_seqlens (decreasing, or past T, or negative) is only visible on the device.  The
chunk kernels check each sequence's range before any access that uses it and record
GDN_ERR_DEVICE_ARG in the workspace status word; the conv bounds every access by the token count
and the sequence count whatever cu_seqlens holds.  After each such call the same context must
still run a correct call: a fault that lost the context would show there.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_fwd_b200 import gdn, inputs
from gdn_testutil import (assert_bf16_close, assert_bf16_rounding_close, assert_f32_close,
                          oracle_gates_f32)

pytestmark = pytest.mark.gpu
DEV = "cuda"

BAD_CU = {
    "decreasing": [0, 100, 50, 200],
    "past_T": [0, 100, 150, 205],
    "negative": [-3, 100, 150, 200],
}


def _good_call(chunk, dtype):
    x = inputs.rule_inputs(B=1, T=200, Hk=1, Hv=2, dk=128, dv=128, dtype=dtype, seed=5,
                           seqlens=[100, 50, 50], s0_std=0.02, a_mean=-6.0)
    g, beta = oracle_gates_f32(x)
    ws = torch.empty(gdn.workspace_size(3, 1, 200, 1, 2, 128, 128, chunk), dtype=torch.uint8,
                     device=DEV)
    out, S = gdn.gdn_chunk_fwd(x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV), g.to(DEV),
                               beta.to(DEV), initial_state=x["initial_state"].to(DEV),
                               cu_seqlens=x["cu_seqlens"].to(DEV), chunk=chunk, workspace=ws)
    assert gdn.workspace_status(ws) == gdn.GDN_OK
    o_ref, S_ref = oracle.gated_delta_rule(x["q"], x["k"], x["v"], g, beta, 128 ** -0.5,
                                           initial_state=x["initial_state"],
                                           cu_seqlens=x["cu_seqlens"])
    if dtype == "bf16":
        assert_bf16_close(out, o_ref, "after bad cu_seqlens: out")
        assert_bf16_close(S, S_ref, "after bad cu_seqlens: state")
    else:
        assert_f32_close(out, o_ref, "after bad cu_seqlens: out")
        assert_f32_close(S, S_ref, "after bad cu_seqlens: state")
    return x, g, beta


@pytest.mark.parametrize("kind", sorted(BAD_CU))
@pytest.mark.parametrize("chunk,dtype", [(64, "bf16"), (32, "bf16"), (16, "f32")])
def test_chunk_bad_cu_seqlens_reports_device_arg(kind, chunk, dtype):
    """Tensor-core path (chunk 64, bf16) and CUDA-core path (chunk 32 / fp32)."""
    x, g, beta = _good_call(chunk, dtype)
    cu_bad = torch.tensor(BAD_CU[kind], dtype=torch.int32, device=DEV)
    ws = torch.empty(gdn.workspace_size(3, 1, 200, 1, 2, 128, 128, chunk), dtype=torch.uint8,
                     device=DEV)
    out = torch.zeros(1, 200, 2, 128, dtype=x["v"].dtype, device=DEV)
    S = torch.zeros(3, 2, 128, 128, device=DEV)
    gdn.gdn_chunk_fwd(x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV), g.to(DEV), beta.to(DEV),
                      initial_state=x["initial_state"].to(DEV), cu_seqlens=cu_bad, chunk=chunk,
                      out=out, final_state=S, workspace=ws)
    assert gdn.workspace_status(ws) == gdn.GDN_ERR_DEVICE_ARG
    _good_call(chunk, dtype)  # the context is still usable


@pytest.mark.parametrize("kind", sorted(BAD_CU))
def test_conv_bad_cu_seqlens_stays_in_bounds(kind):
    """The conv has no status word: a malformed cu_seqlens gives unspecified values for the
    tokens it misdescribes, but no access leaves x, y or the conv states, and the next call on
    the same context is exact."""
    gen = torch.Generator().manual_seed(8)
    C, K, T = 512, 4, 200
    xin = torch.randn(1, T, C, generator=gen).to(torch.bfloat16)
    w = (torch.rand(C, K, generator=gen) * 2 - 1) / K ** 0.5
    s_in = torch.randn(3, C, K - 1, generator=gen)
    s_out = torch.empty(3, C, K - 1, device=DEV)
    gdn.gdn_causal_conv1d_silu(xin.to(DEV), w.to(DEV), None,
                               cu_seqlens=torch.tensor(BAD_CU[kind], dtype=torch.int32,
                                                       device=DEV),
                               n_l2norm_ch=256, l2norm_group=128, conv_state_in=s_in.to(DEV),
                               conv_state_out=s_out)
    torch.cuda.synchronize()
    cu = torch.tensor([0, 100, 150, 200], dtype=torch.int32)
    y = gdn.gdn_causal_conv1d_silu(xin.to(DEV), w.to(DEV), None, cu_seqlens=cu.to(DEV),
                                   n_l2norm_ch=256, l2norm_group=128,
                                   conv_state_in=s_in.to(DEV), conv_state_out=s_out)
    ref, s_ref = oracle.causal_conv1d_silu(xin, w, None, cu_seqlens=cu, n_l2norm_ch=256,
                                           l2norm_group=128, conv_state_in=s_in,
                                           return_state=True)
    assert_bf16_rounding_close(y, ref, "conv after bad cu_seqlens")
    assert np.array_equal(s_out.cpu().double().numpy(), s_ref)


DEBUG_LIB = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                         "gated_deltanet_fwd_b200", "libgdn_debug.so")


@pytest.mark.parametrize("T,skip", [(600, 3), (2000, 2)])
def test_chunk_wait_timeout_reports_and_recovers(T, skip):
    """The failure-test build of the library (every bounded device wait gives up after about a
    millisecond) withholds one chunk's tiles from the tensor-core prefill, so nothing lands for the
    waits on that stage: they run out, the kernels record GDN_ERR_TIMEOUT and every CTA leaves with
    no copy or MMA in flight.  T = 2000 also runs the intra-sequence scan (three phases).  A normal
    call on the same context afterwards must be correct: nothing was left allocated or hung."""
    import ctypes
    assert os.path.exists(DEBUG_LIB), "build the failure-test library: __graft_entry__.build()"
    prev = gdn._lib
    gdn._lib = None
    try:
        lib = gdn.load(DEBUG_LIB)
        lib.gdn_debug_set_skip_chunk.argtypes = [ctypes.c_int]
        lib.gdn_debug_set_skip_chunk.restype = None
        x = inputs.rule_inputs(B=1, T=T, Hk=1, Hv=2, dk=128, dv=128, seed=T, s0_std=0.02,
                               a_mean=-6.0)
        g, beta = oracle_gates_f32(x)
        args = (x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV), g.to(DEV), beta.to(DEV))
        S0 = x["initial_state"].to(DEV)
        ws = torch.empty(gdn.workspace_size(1, 1, T, 1, 2, 128, 128, 64), dtype=torch.uint8,
                         device=DEV)
        lib.gdn_debug_set_skip_chunk(skip)
        try:
            gdn.gdn_chunk_fwd(*args, initial_state=S0, workspace=ws)
            assert gdn.workspace_status(ws) == gdn.GDN_ERR_TIMEOUT
        finally:
            lib.gdn_debug_set_skip_chunk(-1)
        out, S = gdn.gdn_chunk_fwd(*args, initial_state=S0, workspace=ws)
        assert gdn.workspace_status(ws) == gdn.GDN_OK
        o_ref, S_ref = oracle.gated_delta_rule(x["q"], x["k"], x["v"], g, beta, 128 ** -0.5,
                                               initial_state=x["initial_state"])
        assert_bf16_close(out, o_ref, "after a timed-out call: out")
        assert_bf16_close(S, S_ref, "after a timed-out call: state")
    finally:
        gdn._lib = prev
