"""Writes tests/golden/tiny_f32_oracle.txt from the oracle alone (no CUDA path involved).

Workload: tiny fp32 check (B=1, T=64, Hk=Hv=2, dk=dv=16, zero initial state, scale 16^-0.5),
seed 1000, inputs from gated_deltanet_fwd_b200.inputs; g and beta from the oracle's gates.
Stored: the final state (2 x 16 x 16) and the outputs of every 7th token, as %.17g text.
Run:  python tests/golden/make_golden.py
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from gated_deltanet_fwd_b200 import inputs  # noqa: E402

TOKENS = list(range(0, 64, 7))


def compute():
    w = inputs.WORKLOADS["tiny_f32"]
    x = inputs.rule_inputs(**w, seed=1000 + w["index"])
    g, beta = oracle.gates(x["a"], x["b"], x["A_log"], x["dt_bias"])
    out, S = oracle.gated_delta_rule(x["q"], x["k"], x["v"], g, beta, 16 ** -0.5)
    return out, S


def main():
    out, S = compute()
    path = os.path.join(HERE, "tiny_f32_oracle.txt")
    with open(path, "w") as f:
        f.write("# written by tests/golden/make_golden.py from the fp64 oracle only\n")
        f.write("# final_state[h, j, i] for h<2, j<16, i<16, row-major\n")
        f.write(" ".join("%.17g" % x for x in S.ravel()) + "\n")
        f.write("# out[0, t, h, j] for t in %s\n" % TOKENS)
        f.write(" ".join("%.17g" % x for x in out[0, TOKENS].ravel()) + "\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
