"""Shared helpers of the GPU parity tests: error metrics, tolerances, and per-(sequence, head)
oracle sampling for full-size workloads.  No arithmetic of the method lives here."""
import json
import os

import numpy as np
import torch

import oracle

# Tolerances stated for the method: bf16 activations with fp32 state vs the fp64 oracle, and the
# all-fp32 mode.
BF16_REL_L2 = 5e-3
BF16_MAX_ABS = 2e-2
F32_REL = 1e-4


def to64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def rel_l2(x, ref):
    x, ref = to64(x), to64(ref)
    den = np.linalg.norm(ref.ravel())
    return float(np.linalg.norm((x - ref).ravel()) / (den if den > 0 else 1.0))


def max_abs(x, ref):
    x, ref = to64(x), to64(ref)
    return float(np.max(np.abs(x - ref))) if x.size else 0.0


def record_margin(what, **metrics):
    """Prints the measured error next to its tolerance (shown with `pytest -s` or `-rA`) and,
    when GDN_MARGINS names a file, appends it there as one JSON line."""
    print("MARGIN " + what + " " + " ".join(f"{k}={v:.3e}" if isinstance(v, float) else f"{k}={v}"
                                            for k, v in metrics.items()), flush=True)
    path = os.environ.get("GDN_MARGINS")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(dict(what=what, **metrics)) + "\n")


def assert_bf16_close(x, ref, what=""):
    r, m = rel_l2(x, ref), max_abs(x, ref)
    record_margin(what, rel_l2=r, rel_l2_tol=BF16_REL_L2, max_abs=m, max_abs_tol=BF16_MAX_ABS)
    assert r <= BF16_REL_L2 and m <= BF16_MAX_ABS, f"{what}: rel_L2={r:.3e} max_abs={m:.3e}"
    return r, m


def assert_f32_close(x, ref, what="", tol=F32_REL):
    r = rel_l2(x, ref)
    record_margin(what, rel_l2=r, rel_l2_tol=tol)
    assert r <= tol, f"{what}: rel_L2={r:.3e} > {tol:.1e}"
    return r


# Elementwise kernels with bf16 outputs (conv, RMSNorm): the result is one round-to-nearest of
# an fp32 value, so each element may differ from the exact value by the bf16 unit roundoff 2^-8
# relative, plus fp32 evaluation error (a few 1e-7 relative), plus an absolute floor for values
# near zero.
BF16_UNIT_ROUNDOFF = 2.0 ** -8


def assert_bf16_rounding_close(x, ref, what="", abs_floor=1e-6):
    x, ref = to64(x), to64(ref)
    err = np.abs(x - ref)
    bound = (BF16_UNIT_ROUNDOFF + 1e-5) * np.abs(ref) + abs_floor
    bad = err > bound
    record_margin(what, worst_err_over_bound=float(np.max(err / bound)) if err.size else 0.0,
                  rel_l2=rel_l2(x, ref))
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements beyond bf16 rounding, worst "
                           f"err {err[bad].max():.3e} at |ref| {np.abs(ref[bad]).max():.3e}")
    return rel_l2(x, ref)


def oracle_gates_f32(inp):
    """g, beta for the delta rule from the oracle's gates, rounded to fp32 (what both sides see)."""
    g, beta = oracle.gates(inp["a"], inp["b"], inp["A_log"], inp["dt_bias"])
    return torch.from_numpy(g).float(), torch.from_numpy(beta).float()


def oracle_units(q, k, v, g, beta, scale, S0, cu, units, B=None, T=None, nthreads=8):
    """Oracle outputs for selected (sequence n, v-head h) units only.

    Each unit is independent, so it is run alone on its slice of the inputs (Hk = Hv = 1).
    Returns {(n, h): (out [L, dv], S_T [dv, dk])}.
    """
    Hk, Hv = q.shape[2], v.shape[2]
    res = {}
    for (n, h) in units:
        hk = h // (Hv // Hk)
        if cu is not None:
            s0, s1 = int(cu[n]), int(cu[n + 1])
            sl = lambda x, hh: x[0:1, s0:s1, hh:hh + 1]
        else:
            sl = lambda x, hh, n=n: x[n:n + 1, :, hh:hh + 1]
        qq, kk, vv = sl(q, hk), sl(k, hk), sl(v, h)
        if cu is not None:
            gg, bb = g[0:1, s0:s1, h:h + 1], beta[0:1, s0:s1, h:h + 1]
        else:
            gg, bb = g[n:n + 1, :, h:h + 1], beta[n:n + 1, :, h:h + 1]
        st = None if S0 is None else S0[n:n + 1, h:h + 1]
        o, S = oracle.gated_delta_rule(qq, kk, vv, gg, bb, scale, initial_state=st,
                                       nthreads=1)
        res[(n, h)] = (o[0, :, 0], S[0, 0])
    return res
