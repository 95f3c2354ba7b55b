"""Pins of the fp64 oracle against what the pages and the mathematics fix (CPU only).

Nothing here retypes the oracle's own formula: every expected value is a closed form, a hand-worked
example, an invariant, a library routine (numpy / scipy / torch) or an independent brute force
(dense transfer-matrix products in numpy).

Sources, by page title:
  [P2] "解密Qwen3-Next的Gated DeltaNet：如何用75%混合层实现长文本高效推理" (jsqmd.com)
  [P3] "Qwen3.5 Gated DeltaNet 核心机制解析" (wanger-sjtu.github.io)
  [P5] "Qwen3-Next大模型架构解析：混合注意力与MoE优化实践" (intelliparadigm.com)
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle

RNG = np.random.default_rng(20261202)


def _rand_rule(B=1, T=6, Hk=1, Hv=1, dk=5, dv=3, unit_keys=False, s0=True, seed=None):
    rng = np.random.default_rng(seed) if seed is not None else RNG
    q = rng.standard_normal((B, T, Hk, dk))
    k = rng.standard_normal((B, T, Hk, dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, Hv, dv))
    g = -rng.uniform(0.0, 1.5, (B, T, Hv))
    beta = rng.uniform(0.0, 1.0, (B, T, Hv))
    S0 = rng.standard_normal((B, Hv, dv, dk)) if s0 else None
    return q, k, v, g, beta, S0


# ------------------------------------------------------------------ the recurrence --------

def test_single_token_from_zero_state():
    """One token from S0 = 0: S = beta v k^T and o = scale * beta (k.q) v, whatever g is."""
    q, k, v, g, beta, _ = _rand_rule(T=1, dk=5, dv=3, s0=False)
    scale = 0.37
    out, S = oracle.gated_delta_rule(q, k, v, g, beta, scale)
    b = beta[0, 0, 0]
    np.testing.assert_allclose(S[0, 0], b * np.outer(v[0, 0, 0], k[0, 0, 0]), rtol=1e-14,
                               atol=1e-15)
    np.testing.assert_allclose(out[0, 0, 0], scale * b * (k[0, 0, 0] @ q[0, 0, 0]) * v[0, 0, 0],
                               rtol=1e-13, atol=1e-15)


def test_beta0_g0_is_identity():
    """beta = 0 and g = 0: the state never changes and o_t = scale * S0 q_t."""
    q, k, v, g, beta, S0 = _rand_rule(T=7)
    g[:] = 0.0
    beta[:] = 0.0
    out, S = oracle.gated_delta_rule(q, k, v, g, beta, 0.5, initial_state=S0)
    np.testing.assert_array_equal(S, S0)
    for t in range(7):
        np.testing.assert_allclose(out[0, t, 0], 0.5 * S0[0, 0] @ q[0, t, 0], rtol=1e-13)


def test_beta0_pure_decay():
    """beta = 0, any g: S_T = exp(sum_t g_t) S0 -- the decay multiplies the whole state."""
    q, k, v, g, beta, S0 = _rand_rule(T=9)
    beta[:] = 0.0
    _, S = oracle.gated_delta_rule(q, k, v, g, beta, 1.0, initial_state=S0)
    np.testing.assert_allclose(S, math.exp(g.sum()) * S0, rtol=1e-12)


def test_orthonormal_keys_retrieve_exactly():
    """g = 0, beta = 1, orthonormal keys, S0 = 0: S k_i = v_i for every written pair."""
    dk, dv, n = 8, 4, 6
    Qm, _ = np.linalg.qr(RNG.standard_normal((dk, dk)))
    k = Qm[:, :n].T.reshape(1, n, 1, dk)
    v = RNG.standard_normal((1, n, 1, dv))
    q = RNG.standard_normal((1, n, 1, dk))
    g = np.zeros((1, n, 1))
    beta = np.ones((1, n, 1))
    _, S = oracle.gated_delta_rule(q, k, v, g, beta, 1.0)
    for i in range(n):
        np.testing.assert_allclose(S[0, 0] @ k[0, i, 0], v[0, i, 0], atol=1e-12)


def test_same_key_is_overwritten():
    """Writing the same unit key twice with beta = 1, g = 0 leaves S k = v_second: the delta rule
    deletes the old association ([P2] §2.1 table: DeltaNet's precise deletion / selective update).
    Directions orthogonal to k keep what S0 held."""
    dk, dv = 6, 4
    k1 = RNG.standard_normal(dk)
    k1 /= np.linalg.norm(k1)
    k = np.stack([k1, k1]).reshape(1, 2, 1, dk)
    v = RNG.standard_normal((1, 2, 1, dv))
    q = RNG.standard_normal((1, 2, 1, dk))
    S0 = RNG.standard_normal((1, 1, dv, dk))
    _, S = oracle.gated_delta_rule(q, k, v, np.zeros((1, 2, 1)), np.ones((1, 2, 1)), 1.0,
                                   initial_state=S0)
    np.testing.assert_allclose(S[0, 0] @ k1, v[0, 1, 0], atol=1e-12)
    w = RNG.standard_normal(dk)
    w -= (w @ k1) * k1
    np.testing.assert_allclose(S[0, 0] @ w, S0[0, 0] @ w, atol=1e-12)


def test_hand_worked_two_tokens():
    """A two-token example worked by hand in exact arithmetic (dk = dv = 2, scale = 1).

    token 1: S0 = 0, k = (1, 0), v = (1, 2), beta = 1/2, g = 0, q = (1, 1)
             S1 = 1/2 v k^T = [[0.5, 0], [1, 0]];            o1 = S1 q = (0.5, 1)
    token 2: k = (0.6, 0.8), v = (0, 1), beta = 1, g = ln(1/2), q = (0, 1)
             S1 k = (0.3, 0.6);  S1 - (S1 k) k^T = [[0.32, -0.24], [0.64, -0.48]]
             S2 = 1/2 * that + v k^T = [[0.16, -0.12], [0.92, 0.56]];   o2 = (-0.12, 0.56)
             (and S2 k = (0, 1) = v: the decayed state is corrected onto v exactly)
    """
    q = np.array([[1.0, 1.0], [0.0, 1.0]]).reshape(1, 2, 1, 2)
    k = np.array([[1.0, 0.0], [0.6, 0.8]]).reshape(1, 2, 1, 2)
    v = np.array([[1.0, 2.0], [0.0, 1.0]]).reshape(1, 2, 1, 2)
    g = np.array([0.0, math.log(0.5)]).reshape(1, 2, 1)
    beta = np.array([0.5, 1.0]).reshape(1, 2, 1)
    out, S = oracle.gated_delta_rule(q, k, v, g, beta, 1.0)
    np.testing.assert_allclose(out[0, 0, 0], [0.5, 1.0], atol=1e-15)
    np.testing.assert_allclose(out[0, 1, 0], [-0.12, 0.56], atol=1e-15)
    np.testing.assert_allclose(S[0, 0], [[0.16, -0.12], [0.92, 0.56]], atol=1e-15)


def _brute_force(q, k, v, g, beta, scale, S0):
    """Dense transfer form for one head, numpy fp64, a code path independent of the oracle:
    with A_t = e^{g_t} (I - beta_t k_t k_t^T),
        S_t = S0 A_1 ... A_t + sum_{s<=t} beta_s v_s k_s^T A_{s+1} ... A_t,   o_t = scale S_t q_t.
    """
    T, dk = k.shape
    dv = v.shape[1]
    A = [math.exp(g[t]) * (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) for t in range(T)]
    outs, S_t = [], None
    for t in range(T):
        prod = np.eye(dk)
        for s in range(t + 1):
            prod = prod @ A[s]
        S_t = (S0 if S0 is not None else np.zeros((dv, dk))) @ prod
        for s in range(t + 1):
            tail = np.eye(dk)
            for r in range(s + 1, t + 1):
                tail = tail @ A[r]
            S_t = S_t + beta[s] * np.outer(v[s], k[s]) @ tail
        outs.append(scale * S_t @ q[t])
    return np.array(outs), S_t


@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_brute_force_transfer_product(T):
    """Brute force on T <= 8 with decay, non-unit keys, dk != dv, GQA (Hv = 2 Hk) and S0 != 0."""
    Hk, Hv, dk, dv = 2, 4, 5, 3
    q, k, v, g, beta, S0 = _rand_rule(T=T, Hk=Hk, Hv=Hv, dk=dk, dv=dv)
    out, S = oracle.gated_delta_rule(q, k, v, g, beta, 0.3, initial_state=S0)
    for h in range(Hv):
        hk = h // (Hv // Hk)
        o_ref, S_ref = _brute_force(q[0, :, hk], k[0, :, hk], v[0, :, h], g[0, :, h],
                                    beta[0, :, h], 0.3, S0[0, h])
        np.testing.assert_allclose(out[0, :, h], o_ref, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(S[0, h], S_ref, rtol=1e-11, atol=1e-12)


def test_linear_in_state_and_values():
    """out and S_T are jointly linear in (S0, V) for fixed q, k, g, beta."""
    q, k, v1, g, beta, S1 = _rand_rule(T=6, Hk=1, Hv=2)
    _, _, v2, _, _, S2 = _rand_rule(T=6, Hk=1, Hv=2)
    al, be = 0.7, -1.3
    o1, T1 = oracle.gated_delta_rule(q, k, v1, g, beta, 0.4, initial_state=S1)
    o2, T2 = oracle.gated_delta_rule(q, k, v2, g, beta, 0.4, initial_state=S2)
    o3, T3 = oracle.gated_delta_rule(q, k, al * v1 + be * v2, g, beta, 0.4,
                                     initial_state=al * S1 + be * S2)
    np.testing.assert_allclose(o3, al * o1 + be * o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(T3, al * T1 + be * T2, rtol=1e-11, atol=1e-12)


def test_split_and_chain():
    """Running [0, T) at once equals [0, t1) then [t1, T) from the first part's final state --
    the chunk loop of [P2] §2.2 that feeds initial_state from the previous call's state."""
    q, k, v, g, beta, S0 = _rand_rule(T=11, Hk=1, Hv=2, dk=4, dv=4)
    o, S = oracle.gated_delta_rule(q, k, v, g, beta, 0.5, initial_state=S0)
    t1 = 4
    oa, Sa = oracle.gated_delta_rule(q[:, :t1], k[:, :t1], v[:, :t1], g[:, :t1], beta[:, :t1],
                                     0.5, initial_state=S0)
    ob, Sb = oracle.gated_delta_rule(q[:, t1:], k[:, t1:], v[:, t1:], g[:, t1:], beta[:, t1:],
                                     0.5, initial_state=Sa)
    np.testing.assert_allclose(np.concatenate([oa, ob], axis=1), o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(Sb, S, rtol=1e-13, atol=1e-14)


def test_varlen_equals_separate_sequences_and_batch():
    """cu_seqlens packing gives the same per-sequence results as separate calls, and a batch of
    equal-length rows equals the packed form."""
    lens = [3, 1, 5, 4]
    parts = [_rand_rule(T=n, Hk=1, Hv=2, dk=4, dv=3) for n in lens]
    cat = lambda i: np.concatenate([p[i] for p in parts], axis=1)
    S0 = np.concatenate([p[5] for p in parts], axis=0)
    cu = np.cumsum([0] + lens).astype(np.int32)
    o, S = oracle.gated_delta_rule(cat(0), cat(1), cat(2), cat(3), cat(4), 0.5,
                                   initial_state=S0, cu_seqlens=cu)
    for n, p in enumerate(parts):
        on, Sn = oracle.gated_delta_rule(*p[:5], 0.5, initial_state=p[5])
        np.testing.assert_allclose(o[:, cu[n]:cu[n + 1]], on, rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(S[n], Sn[0], rtol=1e-14, atol=1e-15)
    # batch form: two rows of 4 tokens == packed [4, 4]
    q, k, v, g, beta, S0 = _rand_rule(B=2, T=4, Hk=1, Hv=1, dk=3, dv=3)
    ob, Sb = oracle.gated_delta_rule(q, k, v, g, beta, 1.0, initial_state=S0)
    pk = lambda x: x.reshape(1, 8, *x.shape[2:])
    op, Sp = oracle.gated_delta_rule(pk(q), pk(k), pk(v), pk(g), pk(beta), 1.0,
                                     initial_state=S0, cu_seqlens=np.array([0, 4, 8], np.int32))
    np.testing.assert_allclose(op.reshape(ob.shape), ob, rtol=1e-14)
    np.testing.assert_allclose(Sp, Sb, rtol=1e-14)


def test_threads_do_not_change_results():
    q, k, v, g, beta, S0 = _rand_rule(B=3, T=5, Hk=2, Hv=4, dk=4, dv=4)
    o1, S1 = oracle.gated_delta_rule(q, k, v, g, beta, 0.5, initial_state=S0, nthreads=1)
    o4, S4 = oracle.gated_delta_rule(q, k, v, g, beta, 0.5, initial_state=S0, nthreads=4)
    np.testing.assert_array_equal(o1, o4)
    np.testing.assert_array_equal(S1, S4)


def test_empty_sequence_keeps_state():
    """A zero-length sequence in cu_seqlens returns its initial state unchanged."""
    q, k, v, g, beta, S0 = _rand_rule(T=3, Hk=1, Hv=1, dk=3, dv=3)
    S0 = np.concatenate([S0, S0 * 2], axis=0)
    _, S = oracle.gated_delta_rule(q, k, v, g, beta, 1.0, initial_state=S0,
                                   cu_seqlens=np.array([0, 0, 3], np.int32))
    np.testing.assert_array_equal(S[0], S0[0])


# ------------------------------------------------------------------ gates ------------------

def test_gates_spot_values():
    """b = 0 -> beta = 1/2; a + dt_bias = 0 with A_log = 0 -> g = -ln 2 ([P5] §2.2 formulas)."""
    a = np.array([[0.0, 1.5]])
    b = np.array([[0.0, 0.0]])
    g, beta = oracle.gates(a, b, np.array([0.0, 0.0]), np.array([0.0, -1.5]))
    np.testing.assert_allclose(beta, 0.5, rtol=0, atol=0)
    np.testing.assert_allclose(g, -math.log(2.0), rtol=1e-15)


def test_gates_against_library_routines():
    """beta vs scipy.special.expit, g vs -exp(A_log) * numpy.logaddexp(0, a + dt_bias)."""
    Hv = 6
    a = RNG.standard_normal((50, Hv)) * 8
    b = RNG.standard_normal((50, Hv)) * 8
    A_log = np.log(RNG.uniform(1, 16, Hv))
    dt_bias = RNG.standard_normal(Hv) * 0.1
    g, beta = oracle.gates(a, b, A_log, dt_bias)
    np.testing.assert_allclose(beta, scipy.special.expit(b), rtol=1e-14)
    np.testing.assert_allclose(g, -np.exp(A_log) * np.logaddexp(0.0, a + dt_bias), rtol=1e-14)
    assert np.all(g < 0) and np.all((beta > 0) & (beta < 1))
    # extreme pre-activations stay finite: softplus -> 0 / identity, sigmoid -> 0 / 1
    g2, b2 = oracle.gates(np.array([[-800.0, 800.0]]), np.array([[-800.0, 800.0]]),
                          np.zeros(2), np.zeros(2))
    assert g2[0, 0] == 0.0 or abs(g2[0, 0]) < 1e-300
    assert g2[0, 1] == -800.0 and b2[0, 0] == 0.0 and b2[0, 1] == 1.0


# ------------------------------------------------------------------ conv --------------------

def _silu(x):
    return x * scipy.special.expit(x)


def test_conv_delta_input_reproduces_taps():
    """A unit impulse at t0 gives silu(w[c, K-1-(t-t0)]) for t0 <= t < t0+K: cross-correlation
    with the current token on tap K-1."""
    T, C, K, t0 = 12, 8, 4, 5
    x = np.zeros((1, T, C))
    x[0, t0, :] = 1.0
    w = RNG.standard_normal((C, K))
    y = oracle.causal_conv1d_silu(x, w)
    for t in range(T):
        lag = t - t0
        pre = w[:, K - 1 - lag] if 0 <= lag < K else np.zeros(C)
        np.testing.assert_allclose(y[0, t], _silu(pre), rtol=1e-15, atol=1e-300)


def test_conv_against_numpy_convolve():
    """Per channel, pre = numpy.convolve(x, flipped w)[:T] + bias; K = 1 is a pure scale."""
    for K in (1, 3, 4):
        T, C = 20, 16
        x = RNG.standard_normal((1, T, C))
        w = RNG.standard_normal((C, K))
        bias = RNG.standard_normal(C)
        y = oracle.causal_conv1d_silu(x, w, bias)
        for c in range(C):
            pre = np.convolve(x[0, :, c], w[c, ::-1])[:T] + bias[c]
            np.testing.assert_allclose(y[0, :, c], _silu(pre), rtol=1e-13, atol=1e-14)


def test_conv_l2norm_groups():
    """Normalised groups have unit norm (up to eps); channels past n_l2norm_ch are untouched."""
    T, C, K, G = 9, 48, 4, 8
    x = RNG.standard_normal((1, T, C))
    w = RNG.standard_normal((C, K))
    y0 = oracle.causal_conv1d_silu(x, w)
    y = oracle.causal_conv1d_silu(x, w, n_l2norm_ch=32, l2norm_group=G, l2_eps=0.0)
    for c0 in range(0, 32, G):
        np.testing.assert_allclose(np.linalg.norm(y[0, :, c0:c0 + G], axis=-1), 1.0, rtol=1e-14)
        ratio = y[0, :, c0:c0 + G] / y0[0, :, c0:c0 + G]
        np.testing.assert_allclose(ratio, ratio[:, :1].repeat(G, 1), rtol=1e-12)
    np.testing.assert_array_equal(y[0, :, 32:], y0[0, :, 32:])


def test_conv_varlen_and_state_chaining():
    """No mixing across cu_seqlens boundaries; splitting a sequence and passing conv_state_out
    as the next conv_state_in reproduces the single call; the state is the last K-1 inputs."""
    C, K = 8, 4
    lens = [7, 2, 5]
    x = RNG.standard_normal((1, sum(lens), C))
    w = RNG.standard_normal((C, K))
    cu = np.cumsum([0] + lens).astype(np.int32)
    y, st = oracle.causal_conv1d_silu(x, w, cu_seqlens=cu, return_state=True)
    for n in range(3):
        yn, stn = oracle.causal_conv1d_silu(x[:, cu[n]:cu[n + 1]], w, return_state=True)
        np.testing.assert_array_equal(y[:, cu[n]:cu[n + 1]], yn)
        np.testing.assert_array_equal(st[n], stn[0])
    np.testing.assert_array_equal(st[0], x[0, 4:7].T)          # len 7 >= K-1
    np.testing.assert_array_equal(st[1][:, 1:], x[0, 7:9].T)   # len 2 < K-1: zero-padded
    np.testing.assert_array_equal(st[1][:, 0], 0.0)
    # chaining, including a middle piece shorter than K-1
    full, st_full = oracle.causal_conv1d_silu(x[:, :7], w, return_state=True)
    y1, s1 = oracle.causal_conv1d_silu(x[:, :3], w, return_state=True)
    y2, s2 = oracle.causal_conv1d_silu(x[:, 3:5], w, conv_state_in=s1, return_state=True)
    y3, s3 = oracle.causal_conv1d_silu(x[:, 5:7], w, conv_state_in=s2, return_state=True)
    np.testing.assert_allclose(np.concatenate([y1, y2, y3], axis=1), full, rtol=1e-15)
    np.testing.assert_array_equal(s3, st_full)


# ------------------------------------------------------------------ gated RMSNorm ----------

def test_rmsnorm_against_torch_rms_norm():
    """y = torch rms_norm(x, weight = 1 + w, eps) * silu(z), all in float64 ([P2] §3.2)."""
    x = RNG.standard_normal((37, 128)) * 3
    z = RNG.standard_normal((37, 128))
    w = RNG.standard_normal(128) * 0.02
    y = oracle.gated_rmsnorm(x, z, w, eps=1e-6)
    xt = torch.from_numpy(x)
    ref = torch.nn.functional.rms_norm(xt, (128,), weight=torch.from_numpy(1.0 + w), eps=1e-6)
    ref = ref * torch.nn.functional.silu(torch.from_numpy(z))
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-13, atol=1e-15)


def test_rmsnorm_special_rows():
    """w = 0 and a unit-RMS row give x * silu(z); a constant row c gives
    sign(c) |c| / sqrt(c^2 + eps) (1 + w) silu(z); the result is invariant to scaling x."""
    dim = 64
    x = RNG.standard_normal(dim)
    x /= np.sqrt(np.mean(x * x))
    z = RNG.standard_normal(dim)
    y = oracle.gated_rmsnorm(x[None], z[None], np.zeros(dim), eps=0.0)
    np.testing.assert_allclose(y[0], x * _silu(z), rtol=1e-14)
    w = RNG.standard_normal(dim) * 0.02
    c = -2.5
    y = oracle.gated_rmsnorm(np.full((1, dim), c), z[None], w, eps=1e-6)
    np.testing.assert_allclose(y[0], c / math.sqrt(c * c + 1e-6) * (1 + w) * _silu(z),
                               rtol=1e-14)
    xr = RNG.standard_normal((3, dim))
    np.testing.assert_allclose(oracle.gated_rmsnorm(7.0 * xr, np.ones((3, dim)), w, eps=0.0),
                               oracle.gated_rmsnorm(xr, np.ones((3, dim)), w, eps=0.0),
                               rtol=1e-14)


# ------------------------------------------------------------------ stored regression -------

def _load_golden():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_f32_oracle.txt")
    rows = [l for l in open(path) if not l.startswith("#")]
    return np.array(rows[0].split(), float), np.array(rows[1].split(), float)


def test_golden_tiny_regression():
    """The oracle still reproduces the stored tiny-workload values it wrote earlier."""
    import importlib.util, os
    spec = importlib.util.spec_from_file_location(
        "make_golden", os.path.join(os.path.dirname(__file__), "golden", "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    out, S = mg.compute()
    S_ref, o_ref = _load_golden()
    np.testing.assert_allclose(S.ravel(), S_ref, rtol=1e-15, atol=1e-16)
    np.testing.assert_allclose(out[0, mg.TOKENS].ravel(), o_ref, rtol=1e-15, atol=1e-16)
