"""gdn_chunk_fwd_noalloc: the chunked prefill for callers that cannot allocate device memory.

Such callers (a plugin inside an engine that owns and pre-plans all device memory, a host with a
fixed device-memory budget) hand over inputs and outputs only, so this entry point uses a fixed
scratch array inside the library instead of a caller workspace.  The test calls it through the C
ABI twice in a row and checks both results against gdn_chunk_fwd with a caller workspace.  The file
name makes pytest collect it last.
"""
import ctypes

import pytest
import torch

from gated_deltanet_fwd_b200 import gdn, inputs
from gdn_testutil import assert_bf16_close, oracle_gates_f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(q, k, v, g, beta, S0, cu, chunk, out, S_T):
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    N = cu.numel() - 1 if cu is not None else B
    st = gdn.load().gdn_chunk_fwd_noalloc(
        _p(q), _p(k), _p(v), _p(g), _p(beta), gdn.GDN_BF16, float(dk ** -0.5), _p(S0), _p(cu), N,
        B, T, Hk, Hv, dk, dv, chunk, _p(out), _p(S_T),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == gdn.GDN_OK, gdn.status_string(st)


@pytest.mark.parametrize("chunk", [64, 32])
def test_noalloc_matches_workspace_call_twice(chunk):
    x = inputs.rule_inputs(B=1, T=333, Hk=2, Hv=4, dk=128, dv=128, seed=77,
                           seqlens=[100, 0, 64, 169], s0_std=0.02, a_mean=-6.0)
    g, beta = oracle_gates_f32(x)
    q, k, v = x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV)
    g, beta = g.to(DEV), beta.to(DEV)
    S0, cu = x["initial_state"].to(DEV), x["cu_seqlens"].to(DEV)
    # the reference call gets a caller workspace of gdn_chunk_fwd_workspace_size() bytes: both calls
    # then take the same kernel path and must agree bit for bit
    ws = torch.empty(gdn.workspace_size(4, 1, 333, 2, 4, 128, 128, chunk), dtype=torch.uint8,
                     device=DEV)
    ref_out, ref_S = gdn.gdn_chunk_fwd(q, k, v, g, beta, initial_state=S0, cu_seqlens=cu,
                                       chunk=chunk, workspace=ws)
    assert gdn.workspace_status(ws) == gdn.GDN_OK
    for _ in range(2):  # two calls in a row share the library's scratch
        out = torch.full_like(ref_out, float("nan"))
        S_T = torch.full_like(ref_S, float("nan"))
        _noalloc(q, k, v, g, beta, S0, cu, chunk, out, S_T)
        torch.cuda.synchronize()
        assert_bf16_close(out, ref_out, "noalloc out")
        assert_bf16_close(S_T, ref_S, "noalloc final state")
        assert torch.equal(out, ref_out) and torch.equal(S_T, ref_S)
