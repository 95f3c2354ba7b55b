"""The layer core end to end on the GPU against the oracle's composition, at full size.

The layer-core workload (B = 2 batch rows of 16384 tokens, a [q | k | v] mix of 8192 channels,
16 q/k heads, 32 v heads, d = 128, conv kernel 4, gated RMSNorm eps 1e-6) runs through the library
the way the bench times it:

    gdn_causal_conv1d_silu (conv + SiLU + q/k L2 norm)  ->  gdn_gates (a, b)  ->
    gdn_chunk_fwd on q, k, v read in place from the conv output  ->  gdn_gated_rmsnorm(core, z)

and every element of every stage is compared with the fp64 oracle's composition of the same four
steps (oracle conv -> oracle gates -> oracle delta rule -> oracle gated RMSNorm), which never sees
a bf16 intermediate.  This follows the layer's dataflow in "Qwen3.5 Gated DeltaNet 核心机制解析"
(flowchart: conv before the q/k/v split, then the gates, the delta rule, and the norm of the core
output gated by z).
"""
import os

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_fwd_b200 import gdn, inputs
from gdn_testutil import (BF16_REL_L2, assert_bf16_close, assert_bf16_rounding_close, max_abs,
                          record_margin, rel_l2)

pytestmark = pytest.mark.gpu
DEV = "cuda"
NTHREADS = max(1, os.cpu_count() or 1)


def test_layer_core_end_to_end_full_size():
    w = inputs.WORKLOADS["layer_core_2x16k"]
    x = inputs.layer_core_inputs(**w, seed=1000 + w["index"])
    B, T, Hk, Hv, d, K = w["B"], w["T"], w["Hk"], w["Hv"], w["dk"], w["K"]
    C = x["C"]
    scale = d ** -0.5

    # ---- GPU, as the bench runs it
    mix = x["mix"].to(DEV)
    y = torch.empty_like(mix)
    cs_out = torch.empty(B, C, K - 1, device=DEV)
    gdn.gdn_causal_conv1d_silu(mix, x["conv_w"].to(DEV), None, n_l2norm_ch=2 * Hk * d,
                               l2norm_group=d, conv_state_out=cs_out, y=y)
    g, beta = gdn.gdn_gates(x["a"].to(DEV), x["b"].to(DEV), x["A_log"].to(DEV),
                            x["dt_bias"].to(DEV))
    qv = y[:, :, :Hk * d].view(B, T, Hk, d)
    kv = y[:, :, Hk * d:2 * Hk * d].view(B, T, Hk, d)
    vv = y[:, :, 2 * Hk * d:].view(B, T, Hv, d)
    core, S_T = gdn.gdn_chunk_fwd(qv, kv, vv, g, beta, scale=scale, chunk=64)
    yn = gdn.gdn_gated_rmsnorm(core, x["z"].to(DEV), x["norm_w"].to(DEV), eps=w["eps"])
    # the same after the conv as one call (gates and norm fused into the chunk kernels)
    yf, Sf = gdn.gdn_chunk_fwd_gated_norm(qv, kv, vv, x["a"].to(DEV), x["b"].to(DEV),
                                          x["A_log"].to(DEV), x["dt_bias"].to(DEV),
                                          x["z"].to(DEV), x["norm_w"].to(DEV), norm_eps=w["eps"],
                                          scale=scale)
    torch.cuda.synchronize()
    y_gpu, cs_gpu = y.cpu(), cs_out.cpu()
    core_gpu, S_gpu, yn_gpu = core.cpu(), S_T.cpu(), yn.cpu()
    yf_gpu, Sf_gpu = yf.cpu(), Sf.cpu()
    del mix, y, qv, kv, vv, core, S_T, yn, yf, Sf

    # ---- oracle composition in fp64 (one batch row at a time keeps host memory bounded)
    g_ref, b_ref = oracle.gates(x["a"], x["b"], x["A_log"], x["dt_bias"])
    worst_conv = 0.0
    for bi in range(B):
        y_ref, cs_ref = oracle.causal_conv1d_silu(x["mix"][bi:bi + 1], x["conv_w"], None,
                                                  n_l2norm_ch=2 * Hk * d, l2norm_group=d,
                                                  return_state=True)
        # conv stage: one bf16 rounding per element; the carried state is data movement: exact
        worst_conv = max(worst_conv, assert_bf16_rounding_close(
            y_gpu[bi:bi + 1], y_ref, f"layer core conv output, row {bi}"))
        assert max_abs(cs_gpu[bi:bi + 1], cs_ref) == 0.0
        q_ref = y_ref[:, :, :Hk * d].reshape(1, T, Hk, d)
        k_ref = y_ref[:, :, Hk * d:2 * Hk * d].reshape(1, T, Hk, d)
        v_ref = y_ref[:, :, 2 * Hk * d:].reshape(1, T, Hv, d)
        del y_ref
        o_ref, S_ref = oracle.gated_delta_rule(q_ref, k_ref, v_ref, g_ref[bi:bi + 1],
                                               b_ref[bi:bi + 1], scale, nthreads=NTHREADS)
        del q_ref, k_ref, v_ref
        # delta-rule stage, the method's bf16 tolerance on outputs and final state
        assert_bf16_close(core_gpu[bi:bi + 1], o_ref, f"layer core chunk output, row {bi}")
        assert_bf16_close(S_gpu[bi:bi + 1], S_ref, f"layer core final state, row {bi}")
        # normed output: RMSNorm rescales each row, so its error is the core output's relative
        # error plus one bf16 rounding; held to the same relative L2 bound
        yn_ref = oracle.gated_rmsnorm(o_ref, x["z"][bi:bi + 1], x["norm_w"], eps=w["eps"])
        r = rel_l2(yn_gpu[bi:bi + 1], yn_ref)
        record_margin(f"layer core normed output, row {bi}", rel_l2=r, rel_l2_tol=BF16_REL_L2,
                      max_abs=max_abs(yn_gpu[bi:bi + 1], yn_ref))
        assert r <= BF16_REL_L2
        # the fused call: same bound on its normed output and final state
        rf = rel_l2(yf_gpu[bi:bi + 1], yn_ref)
        record_margin(f"layer core fused normed output, row {bi}", rel_l2=rf,
                      rel_l2_tol=BF16_REL_L2, max_abs=max_abs(yf_gpu[bi:bi + 1], yn_ref))
        assert rf <= BF16_REL_L2
        assert_bf16_close(Sf_gpu[bi:bi + 1], S_ref, f"layer core fused final state, row {bi}")
