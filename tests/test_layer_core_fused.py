"""GPU parity of gdn_chunk_fwd_gated_norm (gates -> chunked delta rule -> gated RMSNorm in one
call) against the fp64 oracle's composition of the same three steps, and against the library's
own unfused calls.

The layer's dataflow after the conv ("Qwen3.5 Gated DeltaNet 核心机制解析", flowchart: split ->
gates -> delta rule -> RMSNormGated(core_attn_out, z); "解密Qwen3-Next的Gated DeltaNet" §3.2 for the
zero-centred norm).  Cases span several chunks, ragged tails, an empty sequence, initial states,
sequences long enough for the intra-sequence scan, and the workspace that runs without it.
"""
import os

import pytest
import torch

import oracle
from gated_deltanet_fwd_b200 import gdn, inputs
from gdn_testutil import BF16_REL_L2, assert_bf16_close, max_abs, record_margin, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"
NTHREADS = max(1, os.cpu_count() or 1)
EPS = 1e-6


def _no_scan_workspace_bytes(N, n_tok, Hv):
    """Room for the per-chunk operands only (1024 header bytes + (ceil(n_tok / 64) + N) chunk
    slots x Hv x (16384 + 512) bytes): the call then runs one chain per (sequence, v-head)."""
    return 1024 + (-(-n_tok // 64) + N) * Hv * (16384 + 512)


def _oracle(x, scale):
    g, beta = oracle.gates(x["a"].float(), x["b"].float(), x["A_log"], x["dt_bias"])
    o, S = oracle.gated_delta_rule(x["q"], x["k"], x["v"], g, beta, scale,
                                   initial_state=x["initial_state"], cu_seqlens=x["cu_seqlens"],
                                   nthreads=NTHREADS)
    return oracle.gated_rmsnorm(o, x["z"], x["norm_w"], eps=EPS), S


def _to(t):
    return None if t is None else t.to(DEV)


def _fused(x, scale, workspace_bytes=None):
    ws = None
    if workspace_bytes is not None:
        ws = torch.empty(workspace_bytes, dtype=torch.uint8, device=DEV)
    y, S = gdn.gdn_chunk_fwd_gated_norm(
        _to(x["q"]), _to(x["k"]), _to(x["v"]), _to(x["a"]), _to(x["b"]), _to(x["A_log"]),
        _to(x["dt_bias"]), _to(x["z"]), _to(x["norm_w"]), norm_eps=EPS, scale=scale,
        initial_state=_to(x["initial_state"]), cu_seqlens=_to(x["cu_seqlens"]), workspace=ws)
    torch.cuda.synchronize()
    if ws is not None:
        assert gdn.workspace_status(ws) == gdn.GDN_OK
    return y.cpu(), S.cpu()


def _unfused(x, scale):
    g, beta = gdn.gdn_gates(_to(x["a"]), _to(x["b"]), _to(x["A_log"]), _to(x["dt_bias"]))
    o, S = gdn.gdn_chunk_fwd(_to(x["q"]), _to(x["k"]), _to(x["v"]), g, beta, scale=scale,
                             initial_state=_to(x["initial_state"]),
                             cu_seqlens=_to(x["cu_seqlens"]), chunk=64)
    y = gdn.gdn_gated_rmsnorm(o, _to(x["z"]), _to(x["norm_w"]), eps=EPS)
    torch.cuda.synchronize()
    return y.cpu(), S.cpu()


CASES = [
    # T, seqlens, Hk, Hv, s0_std, a_mean, workspace
    (1000, [0, 1, 63, 64, 65, 300, 507], 2, 4, 0.02, 0.0, "full"),   # ragged, one empty sequence
    (3000, None, 1, 2, 0.02, -6.0, "full"),                          # long enough to be split
    (3000, None, 1, 2, 0.02, -6.0, "noscan"),                        # the same, one chain
    (2049, [1500, 549], 2, 4, None, -3.0, "full"),                   # zero initial state
]


@pytest.mark.parametrize("case", CASES, ids=[f"T{c[0]}-{c[6]}" for c in CASES])
def test_fused_layer_core_parity(case):
    T, seqlens, Hk, Hv, s0, a_mean, ws_mode = case
    x = inputs.fused_core_inputs(B=1, T=T, Hk=Hk, Hv=Hv, dk=128, dv=128, seed=T + Hv,
                                 seqlens=seqlens, s0_std=s0, a_mean=a_mean)
    scale = 128 ** -0.5
    N = x["N"]
    wsb = _no_scan_workspace_bytes(N, T, Hv) if ws_mode == "noscan" else None
    y, S = _fused(x, scale, wsb)
    y_ref, S_ref = _oracle(x, scale)
    r = rel_l2(y, y_ref)
    record_margin(f"fused layer core y {case}", rel_l2=r, rel_l2_tol=BF16_REL_L2,
                  max_abs=max_abs(y, y_ref))
    assert r <= BF16_REL_L2
    assert_bf16_close(S, S_ref, f"fused layer core state {case}")
    # the same three steps as separate calls: they differ only in where the gates are evaluated
    y_u, S_u = _unfused(x, scale)
    assert rel_l2(y, y_u) <= BF16_REL_L2
    assert rel_l2(S, S_u) <= 1e-5


def test_fused_layer_core_rejects_fp32():
    x = inputs.fused_core_inputs(B=1, T=64, Hk=1, Hv=1, dk=128, dv=128, seed=3)
    f = {n: x[n].float().to(DEV) for n in ("q", "k", "v", "a", "b", "z")}
    with pytest.raises(gdn.GdnError) as e:
        gdn.gdn_chunk_fwd_gated_norm(f["q"], f["k"], f["v"], f["a"], f["b"], _to(x["A_log"]),
                                     _to(x["dt_bias"]), f["z"], _to(x["norm_w"]))
    assert e.value.status == gdn.GDN_ERR_UNSUPPORTED
