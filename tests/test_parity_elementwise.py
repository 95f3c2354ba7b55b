"""GPU parity of the elementwise calls (gates, causal conv + SiLU + L2 norm, gated RMSNorm)
against the fp64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_fwd_b200 import gdn, inputs
from gdn_testutil import assert_bf16_rounding_close, assert_f32_close, max_abs, rel_l2

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(1, 1, 1), (2, 333, 32), (1, 4097, 7)])
def test_gates(dtype, shape):
    gen = torch.Generator().manual_seed(11)
    Hv = shape[-1]
    a = (torch.randn(*shape, generator=gen) * 4).to(inputs.torch_dtype(dtype))
    b = (torch.randn(*shape, generator=gen) * 4).to(inputs.torch_dtype(dtype))
    A_log = torch.log(torch.rand(Hv, generator=gen) * 15 + 1)
    dt_bias = torch.randn(Hv, generator=gen) * 0.1
    g, beta = gdn.gdn_gates(a.to(DEV), b.to(DEV), A_log.to(DEV), dt_bias.to(DEV))
    g_ref, b_ref = oracle.gates(a, b, A_log, dt_bias)
    assert_f32_close(g, g_ref, "g", tol=2e-6)
    assert_f32_close(beta, b_ref, "beta", tol=2e-6)
    assert np.max(np.abs(g.cpu().double().numpy() - g_ref) / np.maximum(np.abs(g_ref), 1e-30)) < 1e-5


def _conv_case(B, T, Hk, Hv, d, K, dtype, seed, cu=None, with_state=False):
    gen = torch.Generator().manual_seed(seed)
    C = 2 * Hk * d + Hv * d
    x = torch.randn(B, T, C, generator=gen).to(inputs.torch_dtype(dtype))
    w = (torch.rand(C, K, generator=gen) * 2 - 1) / K ** 0.5
    bias = torch.randn(C, generator=gen) * 0.1
    N = (len(cu) - 1) if cu is not None else B
    s_in = torch.randn(N, C, K - 1, generator=gen) if with_state else None
    cu_t = torch.tensor(cu, dtype=torch.int32) if cu is not None else None
    return x, w, bias, s_in, cu_t, C, N


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("K", [1, 3, 4, 8])
def test_conv_batch(dtype, K):
    Hk, Hv, d = 2, 4, 64
    x, w, bias, _, _, C, _ = _conv_case(2, 77, Hk, Hv, d, K, dtype, seed=K)
    y = gdn.gdn_causal_conv1d_silu(x.to(DEV), w.to(DEV), bias.to(DEV), n_l2norm_ch=2 * Hk * d,
                                   l2norm_group=d)
    ref = oracle.causal_conv1d_silu(x, w, bias, n_l2norm_ch=2 * Hk * d, l2norm_group=d)
    if dtype == "bf16":
        assert_bf16_rounding_close(y, ref, "conv y")
    else:
        assert_f32_close(y, ref, "conv y", tol=1e-5)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_conv_varlen_with_state(dtype):
    """Ragged sequences (empty, shorter than K-1, crossing tile edges) with a carried state."""
    Hk, Hv, d, K = 1, 2, 128, 4
    cu = [0, 5, 5, 7, 70, 71, 140]
    x, w, bias, s_in, cu_t, C, N = _conv_case(1, cu[-1], Hk, Hv, d, K, dtype, seed=3, cu=cu,
                                              with_state=True)
    s_out = torch.empty(N, C, K - 1, device=DEV)
    y = gdn.gdn_causal_conv1d_silu(x.to(DEV), w.to(DEV), None, cu_seqlens=cu_t.to(DEV),
                                   n_l2norm_ch=2 * Hk * d, l2norm_group=d,
                                   conv_state_in=s_in.to(DEV), conv_state_out=s_out)
    ref, s_ref = oracle.causal_conv1d_silu(x, w, None, cu_seqlens=cu_t, n_l2norm_ch=2 * Hk * d,
                                           l2norm_group=d, conv_state_in=s_in, return_state=True)
    if dtype == "bf16":
        assert_bf16_rounding_close(y, ref, "conv y")
    else:
        assert_f32_close(y, ref, "conv y", tol=1e-5)
    # the carried state is pure data movement: exact
    assert max_abs(s_out, s_ref) == 0.0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("K", [2, 5, 6, 7])
def test_conv_ragged_slabs_and_groups(dtype, K):
    """Channel count that leaves a partial warp in a second channel slab (2056 = 2048 + 8),
    32-channel norm groups whose normalised range ends inside a warp (1184 channels), window
    lengths on every unrolling path, and ragged varlen sequences (empty, shorter than K-1, long
    enough to split across blocks) with a carried state."""
    gen = torch.Generator().manual_seed(40 + K)
    C, n_l2, group = 2056, 1184, 32
    cu = [0, 3, 3, 200, 201, 777, 1000]
    N, T = len(cu) - 1, cu[-1]
    x = torch.randn(1, T, C, generator=gen).to(inputs.torch_dtype(dtype))
    w = (torch.rand(C, K, generator=gen) * 2 - 1) / K ** 0.5
    bias = torch.randn(C, generator=gen) * 0.1
    s_in = torch.randn(N, C, K - 1, generator=gen)
    cu_t = torch.tensor(cu, dtype=torch.int32)
    s_out = torch.empty(N, C, K - 1, device=DEV)
    y = gdn.gdn_causal_conv1d_silu(x.to(DEV), w.to(DEV), bias.to(DEV), cu_seqlens=cu_t.to(DEV),
                                   n_l2norm_ch=n_l2, l2norm_group=group,
                                   conv_state_in=s_in.to(DEV), conv_state_out=s_out)
    ref, s_ref = oracle.causal_conv1d_silu(x, w, bias, cu_seqlens=cu_t, n_l2norm_ch=n_l2,
                                           l2norm_group=group, conv_state_in=s_in,
                                           return_state=True)
    if dtype == "bf16":
        assert_bf16_rounding_close(y, ref, "conv y")
    else:
        assert_f32_close(y, ref, "conv y", tol=1e-5)
    assert max_abs(s_out, s_ref) == 0.0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dim", [64, 128, 256])
def test_gated_rmsnorm(dtype, dim):
    gen = torch.Generator().manual_seed(dim)
    rows = 1031
    x = (torch.randn(rows, dim, generator=gen) * 2).to(inputs.torch_dtype(dtype))
    z = torch.randn(rows, dim, generator=gen).to(inputs.torch_dtype(dtype))
    w = torch.randn(dim, generator=gen) * 0.02
    y = gdn.gdn_gated_rmsnorm(x.to(DEV), z.to(DEV), w.to(DEV), eps=1e-6)
    ref = oracle.gated_rmsnorm(x, z, w, eps=1e-6)
    if dtype == "bf16":
        assert_bf16_rounding_close(y, ref, "rmsnorm y")
    else:
        assert_f32_close(y, ref, "rmsnorm y", tol=1e-5)


def test_gated_rmsnorm_in_place_layer_core_size():
    w_ = inputs.WORKLOADS["layer_core_2x16k"]
    gen = torch.Generator().manual_seed(5)
    rows = w_["B"] * w_["T"] * w_["Hv"]
    x = torch.randn(rows, 128, generator=gen).to(torch.bfloat16)
    z = torch.randn(rows, 128, generator=gen).to(torch.bfloat16)
    w = torch.randn(128, generator=gen) * 0.02
    xd = x.to(DEV)
    y = gdn.gdn_gated_rmsnorm(xd, z.to(DEV), w.to(DEV), eps=1e-6, y=xd)  # in place
    ref = oracle.gated_rmsnorm(x, z, w, eps=1e-6)
    assert_bf16_rounding_close(y.cpu(), ref, "rmsnorm in place, all rows")
