"""Runs one workload a few times for profiler captures (ncu): few launches, ~1 GB on the device.

    python -m gated_deltanet_fwd_b200.profile_driver prefill|prefill4k|decode|conv [repeats]

prefill    gdn_gates + gdn_chunk_fwd on the 32768-token varlen workload (4 sequences)
prefill4k  gdn_gates + gdn_chunk_fwd on B=1, T=4096
decode     consecutive gdn_recurrent_step calls on 256 sequences x 32 heads of 128 x 128 state
conv       gdn_causal_conv1d_silu on the [2, 16384, 8192] mix, then gdn_gated_rmsnorm on the
           v channels viewed as 128-wide rows
"""
import sys

import torch

from . import gdn, inputs


def main(argv):
    mode = argv[1] if len(argv) > 1 else "prefill"
    reps = int(argv[2]) if len(argv) > 2 else 2
    dev = torch.device("cuda", 0)
    if mode in ("prefill", "prefill4k"):
        name = "prefill_varlen_32k" if mode == "prefill" else "prefill_4k"
        w = inputs.WORKLOADS[name]
        x = inputs.rule_inputs(**w, seed=1000 + w["index"])
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
        for _ in range(reps):
            g, beta = gdn.gdn_gates(d["a"], d["b"], d["A_log"], d["dt_bias"])
            gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], g, beta, initial_state=d["initial_state"],
                              cu_seqlens=d["cu_seqlens"], chunk=w["chunk"])
    elif mode == "decode":
        w = dict(inputs.WORKLOADS["decode_256"], steps=max(reps, 1))
        x = inputs.decode_inputs(**w, seed=1000 + w["index"])
        st = x["state"].to(dev)
        A_log, dt_bias = x["A_log"].to(dev), x["dt_bias"].to(dev)
        for s in range(w["steps"]):
            g, beta = gdn.gdn_gates(x["a"][s].to(dev), x["b"][s].to(dev), A_log, dt_bias)
            gdn.gdn_recurrent_step(x["q"][s].to(dev), x["k"][s].to(dev), x["v"][s].to(dev), g,
                                   beta, st)
    elif mode == "conv":
        w = inputs.WORKLOADS["layer_core_2x16k"]
        x = inputs.layer_core_inputs(**w, seed=1000 + w["index"])
        mix, cw = x["mix"].to(dev), x["conv_w"].to(dev)
        z, nw = x["z"].to(dev).view(-1, w["dv"]), x["norm_w"].to(dev)
        nqk = 2 * w["Hk"] * w["dk"]
        for _ in range(reps):
            y = gdn.gdn_causal_conv1d_silu(mix, cw, None, n_l2norm_ch=nqk, l2norm_group=w["dk"])
            gdn.gdn_gated_rmsnorm(y[:, :, nqk:].contiguous().view(-1, w["dv"]), z, nw)
    else:
        raise SystemExit(__doc__)
    torch.cuda.synchronize()
    print("done", mode)


if __name__ == "__main__":
    main(sys.argv)
