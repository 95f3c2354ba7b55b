"""GPU parity of gdn_decode_layer_step (one decode token of the whole layer core in one launch)
against the fp64 oracle's composition of the same steps:

    oracle conv (one token, the cached history as conv_state_in) + SiLU + q/k L2 norm ->
    oracle gates -> oracle delta rule (one token, cached state) -> oracle gated RMSNorm(., z)

with the conv history and the delta-rule state carried from step to step, as the decode path of
"Qwen3.5 Gated DeltaNet 核心机制解析" (cache and state switching) advances its conv_states and
recurrent_states caches.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_fwd_b200 import gdn, inputs
from gdn_testutil import (BF16_REL_L2, F32_REL, assert_bf16_close, assert_f32_close, max_abs,
                          record_margin, rel_l2)

pytestmark = pytest.mark.gpu
DEV = "cuda"
NTHREADS = max(1, os.cpu_count() or 1)


def _oracle_step(d, s, cs, S, Hk, dk, scale, eps):
    """One token of the layer core in fp64; returns y [N, Hv, dv], new history, new state."""
    mix = d["mix"][s]
    N, C = mix.shape
    y_conv, cs_new = oracle.causal_conv1d_silu(mix[:, None, :], d["conv_w"], None,
                                               n_l2norm_ch=2 * Hk * dk, l2norm_group=dk,
                                               conv_state_in=cs, return_state=True)
    Hv = d["z"][s].shape[1]
    q = y_conv[:, :, :Hk * dk].reshape(N, 1, Hk, dk)
    k = y_conv[:, :, Hk * dk:2 * Hk * dk].reshape(N, 1, Hk, dk)
    v = y_conv[:, :, 2 * Hk * dk:].reshape(N, 1, Hv, -1)
    g, beta = oracle.gates(d["a"][s], d["b"][s], d["A_log"], d["dt_bias"])
    o, S_new = oracle.gated_delta_rule(q, k, v, g[:, None], beta[:, None], scale,
                                       initial_state=S, nthreads=NTHREADS)
    y = oracle.gated_rmsnorm(o[:, 0], d["z"][s], d["norm_w"], eps)
    return y, cs_new, S_new


def _run(d, Hk, dk, steps, dtype, K):
    """GPU and oracle over `steps` tokens; checks every output, the histories and the states."""
    scale, eps = dk ** -0.5, 1e-6
    conv_w = d["conv_w"].to(DEV)
    A_log, dt_bias, norm_w = d["A_log"].to(DEV), d["dt_bias"].to(DEV), d["norm_w"].to(DEV)
    state = d["state"].to(DEV)
    cs = [d["conv_state"].to(DEV), torch.empty_like(d["conv_state"]).to(DEV)]
    cs_ref, S_ref = d["conv_state"].double().numpy(), d["state"].double().numpy()
    for s in range(steps):
        y = gdn.gdn_decode_layer_step(d["mix"][s].to(DEV), d["a"][s].to(DEV), d["b"][s].to(DEV),
                                      d["z"][s].to(DEV), conv_w, cs[s & 1] if K > 1 else None,
                                      cs[(s + 1) & 1] if K > 1 else None, A_log, dt_bias,
                                      norm_w, state, Hk)
        y_ref, cs_ref, S_ref = _oracle_step(d, s, cs_ref, S_ref, Hk, dk, scale, eps)
        what = f"decode layer ({dtype}, K={K}) step {s}"
        r = rel_l2(y, y_ref)
        tol = BF16_REL_L2 if dtype == "bf16" else F32_REL
        record_margin(what + " y", rel_l2=r, rel_l2_tol=tol, max_abs=max_abs(y, y_ref))
        assert r <= tol
        if K > 1:  # the history is data movement: exact
            assert max_abs(cs[(s + 1) & 1], cs_ref) == 0.0
    if dtype == "bf16":
        assert_bf16_close(state, S_ref, f"decode layer states after {steps} steps")
    else:
        assert_f32_close(state, S_ref, f"decode layer states after {steps} steps")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("K", [4, 1, 8])
def test_decode_layer_small(dtype, K):
    d = inputs.decode_layer_inputs(N=3, Hk=2, Hv=4, dk=128, dv=128, K=K, dtype=dtype, seed=21 + K,
                                   steps=3)
    _run(d, 2, 128, 3, dtype, K)


@pytest.mark.parametrize("Hk,Hv", [(2, 2), (1, 4), (3, 6)])
def test_decode_layer_head_sharing(Hk, Hv):
    """Other head-sharing ratios than the workload's Hv = 2 Hk (which takes the paired-head
    kernel): one v-head per k-head, four per k-head, and three pairs."""
    d = inputs.decode_layer_inputs(N=3, Hk=Hk, Hv=Hv, dk=128, dv=128, K=4, dtype="bf16",
                                   seed=40 + Hk + Hv, steps=2)
    _run(d, Hk, 128, 2, "bf16", 4)


def test_decode_layer_full_size():
    """256 sequences, 16 q/k heads, 32 v heads, conv kernel 4, 64 consecutive tokens: every
    output of every step, every history and every final state."""
    w = inputs.WORKLOADS["decode_layer_256"]
    d = inputs.decode_layer_inputs(**w, seed=1000 + w["index"])
    _run(d, w["Hk"], w["dk"], w["steps"], "bf16", w["K"])


def test_decode_layer_matches_unfused_calls():
    """The fused step against the unfused sequence of library calls on the same token (conv with
    history -> gates -> recurrent step -> gated RMSNorm); they differ only by the bf16 rounding of
    q, k, v that the unfused conv writes."""
    Hk, Hv, d_, K = 2, 4, 128, 4
    d = inputs.decode_layer_inputs(N=5, Hk=Hk, Hv=Hv, dk=d_, dv=d_, K=K, seed=33, steps=1)
    N, C = d["mix"][0].shape
    conv_w = d["conv_w"].to(DEV)
    A_log, dt_bias, norm_w = d["A_log"].to(DEV), d["dt_bias"].to(DEV), d["norm_w"].to(DEV)
    cs_in = d["conv_state"].to(DEV)
    st1, st2 = d["state"].to(DEV), d["state"].to(DEV)
    cs1, cs2 = torch.empty_like(cs_in), torch.empty_like(cs_in)
    y1 = gdn.gdn_decode_layer_step(d["mix"][0].to(DEV), d["a"][0].to(DEV), d["b"][0].to(DEV),
                                   d["z"][0].to(DEV), conv_w, cs_in, cs1, A_log, dt_bias, norm_w,
                                   st1, Hk)
    yc = gdn.gdn_causal_conv1d_silu(d["mix"][0].to(DEV)[:, None, :], conv_w, None,
                                    n_l2norm_ch=2 * Hk * d_, l2norm_group=d_, conv_state_in=cs_in,
                                    conv_state_out=cs2)
    g, beta = gdn.gdn_gates(d["a"][0].to(DEV), d["b"][0].to(DEV), A_log, dt_bias)
    q = yc[:, 0, :Hk * d_].reshape(N, Hk, d_).contiguous()
    k = yc[:, 0, Hk * d_:2 * Hk * d_].reshape(N, Hk, d_).contiguous()
    v = yc[:, 0, 2 * Hk * d_:].reshape(N, Hv, d_).contiguous()
    o = gdn.gdn_recurrent_step(q, k, v, g, beta, st2)
    y2 = gdn.gdn_gated_rmsnorm(o, d["z"][0].to(DEV), norm_w)
    torch.cuda.synchronize()
    assert torch.equal(cs1, cs2)
    assert rel_l2(y1, y2) <= BF16_REL_L2
    assert_bf16_close(st1, st2, "fused vs unfused state")
