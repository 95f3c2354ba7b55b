"""GPU parity of gdn_recurrent_step (one-token decode, state in place) against the oracle."""
import os

import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_fwd_b200 import gdn, inputs
from gdn_testutil import assert_bf16_close, assert_f32_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run_steps(d, steps, dtype, sample=None):
    """Runs `steps` decode steps on the GPU and the same steps in the oracle on sampled
    sequences; returns per-step outputs and final states of both."""
    gates = [oracle.gates(d["a"][s], d["b"][s], d["A_log"], d["dt_bias"]) for s in range(steps)]
    gates = [(torch.from_numpy(g).float(), torch.from_numpy(b).float()) for g, b in gates]
    state = d["state"].to(DEV)
    Hk = d["q"][0].shape[1]
    scale = d["q"][0].shape[2] ** -0.5
    outs = []
    for s in range(steps):
        o = gdn.gdn_recurrent_step(d["q"][s].to(DEV), d["k"][s].to(DEV), d["v"][s].to(DEV),
                                   gates[s][0].to(DEV), gates[s][1].to(DEV), state, scale=scale)
        outs.append(o.cpu())
    sample = list(range(d["state"].shape[0])) if sample is None else sample
    S = d["state"][sample].double().numpy()
    ref_outs = []
    for s in range(steps):
        # one decode step of N sequences == the rule over B = N batch rows of length 1
        q = d["q"][s][sample].unsqueeze(1)
        k = d["k"][s][sample].unsqueeze(1)
        v = d["v"][s][sample].unsqueeze(1)
        g = gates[s][0][sample].unsqueeze(1)
        b = gates[s][1][sample].unsqueeze(1)
        o, S = oracle.gated_delta_rule(q, k, v, g, b, scale, initial_state=S,
                                       nthreads=max(1, os.cpu_count() or 1))
        ref_outs.append(o[:, 0])
    return [o[sample] for o in outs], state.cpu()[sample], ref_outs, S


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dv", [128, 64, 8])
def test_recurrent_small(dtype, dv):
    d = inputs.decode_inputs(N=5, Hk=2, Hv=4, dk=128, dv=dv, dtype=dtype, seed=7, steps=3)
    outs, S, ref_outs, S_ref = _run_steps(d, 3, dtype)
    for s in range(3):
        if dtype == "bf16":
            assert_bf16_close(outs[s], ref_outs[s], f"out step {s}")
        else:
            assert_f32_close(outs[s], ref_outs[s], f"out step {s}")
    if dtype == "bf16":
        assert_bf16_close(S, S_ref, "state")
    else:
        assert_f32_close(S, S_ref, "state")


def test_recurrent_hk_equals_hv():
    d = inputs.decode_inputs(N=3, Hk=4, Hv=4, dk=128, dv=128, dtype="f32", seed=8, steps=2)
    outs, S, ref_outs, S_ref = _run_steps(d, 2, "f32")
    assert_f32_close(outs[1], ref_outs[1], "out")
    assert_f32_close(S, S_ref, "state")


def test_recurrent_decode_full_size():
    """The decode workload at full size (256 sequences, 32 v-heads, 128 x 128 fp32 states,
    64 consecutive steps, state carried in place) in the launch configuration the bench times;
    the oracle follows every sequence through all 64 steps and every output is compared."""
    w = inputs.WORKLOADS["decode_256"]
    d = inputs.decode_inputs(**w, seed=1000 + w["index"])
    outs, S, ref_outs, S_ref = _run_steps(d, w["steps"], "bf16")
    for s in range(w["steps"]):
        assert_bf16_close(outs[s], ref_outs[s], f"decode out step {s}")
    assert_bf16_close(S, S_ref, "decode states after 64 steps")
