"""Cross-mode consistency on the GPU: the chunked prefill agrees with the decode step run token by
token, with itself split and chained through the state, and across chunk sizes."""
import pytest
import torch

from gated_deltanet_fwd_b200 import gdn, inputs
from gdn_testutil import assert_bf16_close, assert_f32_close, oracle_gates_f32, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_chunk_equals_recurrent_stepped(dtype):
    B, T, Hk, Hv, d = 2, 150, 2, 4, 128
    x = inputs.rule_inputs(B=B, T=T, Hk=Hk, Hv=Hv, dk=d, dv=d, dtype=dtype, seed=21,
                           s0_std=0.02, a_mean=-6.0)
    g, beta = oracle_gates_f32(x)
    q, k, v = x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV)
    g, beta = g.to(DEV), beta.to(DEV)
    S0 = x["initial_state"].to(DEV)
    out, S = gdn.gdn_chunk_fwd(q, k, v, g, beta, initial_state=S0, chunk=64)
    state = S0.clone()
    outs = []
    for t in range(T):
        outs.append(gdn.gdn_recurrent_step(q[:, t].contiguous(), k[:, t].contiguous(),
                                           v[:, t].contiguous(), g[:, t].contiguous(),
                                           beta[:, t].contiguous(), state))
    rec = torch.stack(outs, dim=1)
    check = assert_bf16_close if dtype == "bf16" else assert_f32_close
    check(out, rec, "chunk vs stepped out")
    check(S, state, "chunk vs stepped state")


def test_split_and_chain():
    """prefill(T) == prefill(t1) then prefill(T - t1) from its final state."""
    x = inputs.rule_inputs(B=1, T=300, Hk=2, Hv=4, dk=128, dv=128, seed=22, s0_std=0.02,
                           a_mean=-6.0)
    g, beta = oracle_gates_f32(x)
    q, k, v = x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV)
    g, beta = g.to(DEV), beta.to(DEV)
    S0 = x["initial_state"].to(DEV)
    out, S = gdn.gdn_chunk_fwd(q, k, v, g, beta, initial_state=S0)
    t1 = 100  # not a multiple of the chunk
    sl = lambda t, a, b: t[:, a:b].contiguous()
    o1, S1 = gdn.gdn_chunk_fwd(sl(q, 0, t1), sl(k, 0, t1), sl(v, 0, t1), sl(g, 0, t1),
                               sl(beta, 0, t1), initial_state=S0)
    o2, S2 = gdn.gdn_chunk_fwd(sl(q, t1, 300), sl(k, t1, 300), sl(v, t1, 300), sl(g, t1, 300),
                               sl(beta, t1, 300), initial_state=S1)
    assert_bf16_close(torch.cat([o1, o2], dim=1), out, "split out")
    assert_bf16_close(S2, S, "split state")


def test_chunk_sizes_agree():
    x = inputs.rule_inputs(B=1, T=200, Hk=1, Hv=2, dk=128, dv=128, seed=23, s0_std=0.02,
                           a_mean=-6.0)
    g, beta = oracle_gates_f32(x)
    args = [x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV), g.to(DEV), beta.to(DEV)]
    S0 = x["initial_state"].to(DEV)
    res = [gdn.gdn_chunk_fwd(*args, initial_state=S0, chunk=c) for c in (16, 32, 64)]
    for o, S in res[:2]:
        assert_bf16_close(o, res[2][0], "chunk-size out")
        assert_bf16_close(S, res[2][1], "chunk-size state")


def test_varlen_equals_separate_calls():
    lens = [70, 1, 129, 64]
    x = inputs.rule_inputs(B=1, T=sum(lens), Hk=2, Hv=4, dk=128, dv=128, seed=24,
                           seqlens=lens, s0_std=0.02, a_mean=-6.0)
    g, beta = oracle_gates_f32(x)
    cu = x["cu_seqlens"]
    out, S = gdn.gdn_chunk_fwd(x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV), g.to(DEV),
                               beta.to(DEV), initial_state=x["initial_state"].to(DEV),
                               cu_seqlens=cu.to(DEV))
    for n in range(len(lens)):
        a, b = int(cu[n]), int(cu[n + 1])
        sl = lambda t: t[:, a:b].contiguous().to(DEV)
        o_n, S_n = gdn.gdn_chunk_fwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(g), sl(beta),
                                     initial_state=x["initial_state"][n:n + 1].to(DEV))
        # identical per-sequence work: bit-identical results
        assert torch.equal(out[:, a:b], o_n)
        assert torch.equal(S[n:n + 1], S_n)
