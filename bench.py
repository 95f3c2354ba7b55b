#!/usr/bin/env python
"""Benchmark of the gated delta rule on B200: prefill tokens/s at T = 32K and decode seqs/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on stdout (rank 0).  The headline `value` is prefill tokens/s of the packed
32768-token varlen workload (4 sequences of 16384/8192/6144/2048 tokens, 16 q/k heads, 32 v heads,
d = 128, bf16, chunk 64, per-sequence fp32 initial states, final states returned); one step is
gdn_gates + gdn_chunk_fwd over that batch.  The same line carries `decode` (256 sequences x 32
heads of 128 x 128 fp32 state, one step = 64 consecutive gdn_recurrent_step calls, seqs/s) and
`layer_core` (B = 2 x 16384 tokens: conv, then gates + chunk + gated RMSNorm in one fused call, tokens/s;
 the four unfused calls timed beside it), each with the
roofline of its dominant kernel.  Every input is larger than L2, so no flush is needed between
iterations.

Multi-GPU: one process per GPU (torchrun); every rank runs its own independent copy of each
workload (sequences and heads are independent units, so nothing is exchanged): weak scaling,
whole-job value = units of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_deltanet_fwd_b200 import inputs  # noqa: E402

METRIC = "gated-delta-rule prefill tokens/s (T=32K) & decode seqs/s; % of roofline"
# Algorithmic work of the chunk form per token per v-head (d = 128, chunk C = 64): 2 FLOP per
# multiply-add x (4*C*d for K K^T, Q K^T, the triangular apply and the intra-chunk output, + 3*d^2
# for K S^T, Q S^T and the state update) = 163,840 FLOP.
CHUNK_FLOP_PER_TOKEN_HEAD = 2 * (4 * 64 * 128 + 3 * 128 * 128)

# Kernels one bf16 d = 128 chunk call launches with a workspace of gdn_chunk_fwd_workspace_size():
# the scan planner, the per-chunk prep, chain phase 1, the state prefix, chain phase 3.
CHUNK_LAUNCHES = 5


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant kernels, from one ncu
# capture each (summaries under profiles/), tied to the kernel source they were taken from: once
# the source changes the bench reports traffic as null until it is captured again.
MEASURED_TRAFFIC = {
    # one gdn_chunk_fwd call on the 32K varlen workload (scan plan, prep, chain phase 1, state
    # prefix, chain phase 3), ncu dram__bytes_read.sum + dram__bytes_write.sum summed over the
    # five kernels: 1,391.3 MB read + 461.7 MB written
    "gdn_chunk_fwd": dict(sources=["csrc/chunk_prep.cu", "csrc/chunk_chain.cu",
                                   "csrc/chunk_scan.cu", "csrc/chunk_tm.cuh", "csrc/ptx.cuh"],
                          sha256_16="fe6069ea6d4d9046", bytes_per_launch=1.85296e9),
    # recurrent_step_kernel on 256 sequences x 32 heads: 541.2 MB read + 479.2 MB written
    "gdn_recurrent_step": dict(sources=["csrc/recurrent.cu"], sha256_16="a413ca6c4c9f6c5e",
                               bytes_per_launch=1.02039e9),
    # decode_fused_pair_kernel on 256 sequences x 32 heads: 574.8 MB read + 505.3 MB written
    "gdn_decode_layer_step": dict(sources=["csrc/decode_fused.cu"], sha256_16="9cc12723f08fc19a",
                                  bytes_per_launch=1.08017e9),
}


def _sources_sha(sources):
    h = hashlib.sha256()
    for src in sources:
        with open(os.path.join(ROOT, "gated_deltanet_fwd_b200", src), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(kernel, units):
    """ncu DRAM bytes per launch of `kernel` scaled to `units`, or None once a source it was
    measured on has changed."""
    m = MEASURED_TRAFFIC[kernel]
    try:
        sha = _sources_sha(m["sources"])
    except OSError:
        return None
    if sha != m["sha256_16"]:
        return None
    return m.get("bytes_per_launch", m.get("bytes_per_token", 0.0) * units)


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p["bf16_tflops_sustained"]), source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ------------------------------------------------------------------ distributed ------------

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False

    def init(self, backend):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            if torch.cuda.is_available():
                dist.barrier(device_ids=[self.local])
            else:
                dist.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.float64,
                         device=f"cuda:{self.local}" if torch.cuda.is_available() else "cpu")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


# ------------------------------------------------------------------ clocks -----------------

class ClockSampler:
    """nvidia-smi sampling (200 ms) of SM clock and throttle reasons around a timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        self.sel = None
        try:
            p = torch.cuda.get_device_properties(device_index)
            self.sel = "%08x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
        except Exception:
            self.sel = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu=timestamp,{self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "200"]
        if self.sel:
            cmd[1:1] = ["-i", self.sel]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        self.t0 = time.time()

    def stop(self):
        if self.proc is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=[], samples=0,
                        note="nvidia-smi unavailable")
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i] == "Active"})
        loaded = [s for s in sm if mx and s > 0.3 * max(mx)]
        return dict(sm_mhz=statistics.median(loaded or sm) if sm else None,
                    sm_max_mhz=max(mx) if mx else None, reasons=reasons, samples=len(rows))


# ------------------------------------------------------------------ timing helpers ---------

def timed_region(dist, step, K, W):
    """W untimed warm-up steps, then exactly K steps between CUDA events on the current stream,
    bracketed by a barrier and a device synchronize on both sides.  Returns max-over-ranks ms."""
    for _ in range(W):
        step(False)
    torch.cuda.synchronize()
    dist.barrier()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(K):
        step(True)
    e1.record(s)
    e1.synchronize()
    torch.cuda.synchronize()
    dist.barrier()
    return dist.max(e0.elapsed_time(e1))


class KernelTimer:
    """CUDA events around one call inside the timed region (same stream as its launch)."""

    def __init__(self):
        self.pairs = []

    def __call__(self, fn):
        s = torch.cuda.current_stream()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        r = fn()
        b.record(s)
        self.pairs.append((a, b))
        return r

    def mean_ms(self):
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in self.pairs) / max(1, len(self.pairs))


# ------------------------------------------------------------------ workloads --------------

def _prefill_inputs():
    w = inputs.WORKLOADS["prefill_varlen_32k"]
    x = inputs.rule_inputs(**w, seed=1000 + w["index"])
    return w, x


def bench_prefill(dist, gdn, K, W, peaks):
    w, x = _prefill_inputs()
    dev = torch.device("cuda", torch.cuda.current_device())
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    T, Hv, dk = w["T"], w["Hv"], w["dk"]
    scale = dk ** -0.5
    g = torch.empty(1, T, Hv, device=dev)
    beta = torch.empty(1, T, Hv, device=dev)
    out = torch.empty_like(d["v"])
    S_T = torch.empty_like(d["initial_state"])
    ws = torch.empty(gdn.workspace_size(4, 1, T, 16, Hv, dk, dk, 64), dtype=torch.uint8,
                     device=dev)
    kt = KernelTimer()

    def step(timed):
        gdn.gdn_gates(d["a"], d["b"], d["A_log"], d["dt_bias"], g=g, beta=beta)
        call = lambda: gdn.gdn_chunk_fwd(d["q"], d["k"], d["v"], g, beta, scale=scale,
                                         initial_state=d["initial_state"],
                                         cu_seqlens=d["cu_seqlens"], chunk=64, out=out,
                                         final_state=S_T, workspace=ws)
        kt(call) if timed else call()

    ms = timed_region(dist, step, K, W)
    status = gdn.workspace_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after prefill")
    chunk_ms = kt.mean_ms()
    tokens = T * dist.world
    flop = T * Hv * CHUNK_FLOP_PER_TOKEN_HEAD
    achieved = flop / (chunk_ms * 1e-3) / 1e12
    res = dict(value=tokens * K / (ms * 1e-3), ms_per_step=ms / K, chunk_ms=chunk_ms,
               roofline=dict(bound="tensor", kernel="gdn_chunk_fwd", achieved=achieved,
                             peak=peaks["bf16"], unit="TFLOP/s", frac=achieved / peaks["bf16"],
                             traffic=_traffic("gdn_chunk_fwd", T),
                             traffic_unit="bytes per launch", flop_per_launch=flop,
                             peak_source=peaks["source"] + " bf16 burst"),
               gpu_launches=(1 + CHUNK_LAUNCHES) * K)

    # end to end through the public API from pinned host buffers, H2D and D2H inside the region
    host = {k: x[k].pin_memory() for k in ("q", "k", "v", "a", "b", "initial_state")}
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h_S = torch.empty(S_T.shape, dtype=S_T.dtype).pin_memory()
    bi = sum(t.numel() * t.element_size() for t in host.values())
    bo = h_out.numel() * h_out.element_size() + h_S.numel() * h_S.element_size()

    # Sequences are pipelined over three streams: copy-in of sequence i+1 overlaps the compute of
    # sequence i and the copy-out of sequence i-1 (both PCIe directions busy at once).  Longest
    # first, so the tail after the last copy-in is the shortest sequence's compute and copy-out.
    cu_h = [int(c) for c in x["cu_seqlens"]]
    n_seq = len(cu_h) - 1
    s_in, s_cmp, s_out = (torch.cuda.Stream() for _ in range(3))

    def e2e_step(timed):
        cur = torch.cuda.current_stream()
        s_in.wait_stream(cur)
        for i in range(n_seq):
            a0, a1 = cu_h[i], cu_h[i + 1]
            with torch.cuda.stream(s_in):
                for k_ in ("q", "k", "v", "a", "b"):
                    d[k_][:, a0:a1].copy_(host[k_][:, a0:a1], non_blocking=True)
                d["initial_state"][i].copy_(host["initial_state"][i], non_blocking=True)
                e_in = torch.cuda.Event()
                e_in.record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(e_in)
                gdn.gdn_gates(d["a"][:, a0:a1], d["b"][:, a0:a1], d["A_log"], d["dt_bias"],
                              g=g[:, a0:a1], beta=beta[:, a0:a1])
                gdn.gdn_chunk_fwd(d["q"][:, a0:a1], d["k"][:, a0:a1], d["v"][:, a0:a1],
                                  g[:, a0:a1], beta[:, a0:a1], scale=scale,
                                  initial_state=d["initial_state"][i:i + 1], chunk=64,
                                  out=out[:, a0:a1], final_state=S_T[i:i + 1], workspace=ws)
                e_c = torch.cuda.Event()
                e_c.record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_c)
                h_out[:, a0:a1].copy_(out[:, a0:a1], non_blocking=True)
                h_S[i].copy_(S_T[i], non_blocking=True)
        cur.wait_stream(s_out)

    ke = max(2, min(K, 5))
    ms_e2e = timed_region(dist, e2e_step, ke, 1)
    res["e2e"] = dict(value=tokens * ke / (ms_e2e * 1e-3), unit="tokens/s",
                      h2d_bytes_per_step=bi, d2h_bytes_per_step=bo)
    return res


def bench_decode(dist, gdn, K, W, peaks):
    w = inputs.WORKLOADS["decode_256"]
    steps = w["steps"]
    x = inputs.decode_inputs(**w, seed=1000 + w["index"])
    dev = torch.device("cuda", torch.cuda.current_device())
    N, Hv, dv, dk, Hk = w["N"], w["Hv"], w["dv"], w["dk"], w["Hk"]
    state = x["state"].to(dev)
    A_log, dt_bias = x["A_log"].to(dev), x["dt_bias"].to(dev)
    q = [t.to(dev) for t in x["q"]]
    k = [t.to(dev) for t in x["k"]]
    v = [t.to(dev) for t in x["v"]]
    a = [t.to(dev) for t in x["a"]]
    b = [t.to(dev) for t in x["b"]]
    g = torch.empty(N, Hv, device=dev)
    beta = torch.empty(N, Hv, device=dev)
    out = torch.empty(N, Hv, dv, dtype=torch.bfloat16, device=dev)
    kt = KernelTimer()
    scale = dk ** -0.5

    def step(timed):
        for s in range(steps):
            gdn.gdn_gates(a[s], b[s], A_log, dt_bias, g=g, beta=beta)
            call = lambda: gdn.gdn_recurrent_step(q[s], k[s], v[s], g, beta, state, scale=scale,
                                                  out=out)
            kt(call) if timed else call()

    ms = timed_region(dist, step, K, W)
    rec_ms = kt.mean_ms()
    state_bytes = N * Hv * dv * dk * 4
    io_bytes = (2 * N * Hk * dk + 2 * N * Hv * dv) * 2 + 2 * N * Hv * 4
    bytes_per_launch = 2 * state_bytes + io_bytes
    achieved = bytes_per_launch / (rec_ms * 1e-3) / 1e9
    return dict(value=N * steps * K * dist.world / (ms * 1e-3), unit="seqs/s",
                ms_per_step=ms / K, decode_token_us=rec_ms * 1e3,
                roofline=dict(bound="hbm", kernel="gdn_recurrent_step", achieved=achieved,
                              peak=peaks["hbm"], unit="GB/s", frac=achieved / peaks["hbm"],
                              frac_of_nominal_8tbs=achieved / 8000.0,
                              traffic=_traffic("gdn_recurrent_step", 0),
                              traffic_unit="bytes per launch",
                              bytes_per_launch=bytes_per_launch,
                              peak_source=peaks["source"] + " HBM copy"),
                gpu_launches=2 * steps * K)


def bench_decode_layer(dist, gdn, K, W, peaks):
    """The decode workload's shapes with one token of the whole layer core per launch
    (gdn_decode_layer_step: conv with the cached history, gates, recurrent step, gated RMSNorm);
    one step = 64 consecutive tokens."""
    w = inputs.WORKLOADS["decode_layer_256"]
    steps = w["steps"]
    x = inputs.decode_layer_inputs(**w, seed=1000 + w["index"])
    dev = torch.device("cuda", torch.cuda.current_device())
    N, Hk, Hv, dk, dv, Kc = w["N"], w["Hk"], w["Hv"], w["dk"], w["dv"], w["K"]
    C = x["C"]
    state = x["state"].to(dev)
    cs = [x["conv_state"].to(dev), torch.empty_like(x["conv_state"]).to(dev)]
    conv_w, A_log, dt_bias = x["conv_w"].to(dev), x["A_log"].to(dev), x["dt_bias"].to(dev)
    norm_w = x["norm_w"].to(dev)
    mix = [t.to(dev) for t in x["mix"]]
    a = [t.to(dev) for t in x["a"]]
    b = [t.to(dev) for t in x["b"]]
    z = [t.to(dev) for t in x["z"]]
    y = torch.empty(N, Hv, dv, dtype=torch.bfloat16, device=dev)
    kt = KernelTimer()

    def step(timed):
        for s_ in range(steps):
            call = lambda: gdn.gdn_decode_layer_step(mix[s_], a[s_], b[s_], z[s_], conv_w,
                                                     cs[s_ & 1], cs[(s_ + 1) & 1], A_log,
                                                     dt_bias, norm_w, state, Hk, y=y)
            kt(call) if timed else call()

    ms = timed_region(dist, step, K, W)
    k_ms = kt.mean_ms()
    state_bytes = N * Hv * dv * dk * 4
    hist_bytes = N * C * (Kc - 1) * 4
    io_bytes = (N * C + 2 * N * Hv + 2 * N * Hv * dv) * 2  # mix, a, b, z in; y out (bf16)
    bytes_per_launch = 2 * state_bytes + 2 * hist_bytes + io_bytes
    achieved = bytes_per_launch / (k_ms * 1e-3) / 1e9
    return dict(value=N * steps * K * dist.world / (ms * 1e-3), unit="seqs/s",
                ms_per_step=ms / K, token_us=k_ms * 1e3,
                roofline=dict(bound="hbm", kernel="gdn_decode_layer_step", achieved=achieved,
                              peak=peaks["hbm"], unit="GB/s", frac=achieved / peaks["hbm"],
                              frac_of_nominal_8tbs=achieved / 8000.0,
                              traffic=_traffic("gdn_decode_layer_step", 1),
                              traffic_unit="bytes per launch",
                              bytes_per_launch=bytes_per_launch,
                              peak_source=peaks["source"] + " HBM copy"),
                gpu_launches=steps * K)


def bench_layer_core(dist, gdn, K, W, peaks):
    w = inputs.WORKLOADS["layer_core_2x16k"]
    x = inputs.layer_core_inputs(**w, seed=1000 + w["index"])
    dev = torch.device("cuda", torch.cuda.current_device())
    B, T, Hk, Hv, d = w["B"], w["T"], w["Hk"], w["Hv"], w["dk"]
    mix = x["mix"].to(dev)
    z = x["z"].to(dev)
    a, b = x["a"].to(dev), x["b"].to(dev)
    A_log, dt_bias = x["A_log"].to(dev), x["dt_bias"].to(dev)
    conv_w, norm_w = x["conv_w"].to(dev), x["norm_w"].to(dev)
    C = x["C"]
    y = torch.empty_like(mix)
    g = torch.empty(B, T, Hv, device=dev)
    beta = torch.empty(B, T, Hv, device=dev)
    core = torch.empty(B, T, Hv, d, dtype=torch.bfloat16, device=dev)
    S_T = torch.empty(B, Hv, d, d, device=dev)
    cs_out = torch.empty(B, C, w["K"] - 1, device=dev)
    ws = torch.empty(gdn.workspace_size(B, B, T, Hk, Hv, d, d, 64), dtype=torch.uint8, device=dev)
    # q, k, v are views into the conv output [q | k | v] (token stride C): no copies
    kt = {"conv": KernelTimer(), "core": KernelTimer()}
    qv = y[:, :, :Hk * d].view(B, T, Hk, d)
    kv = y[:, :, Hk * d:2 * Hk * d].view(B, T, Hk, d)
    vv = y[:, :, 2 * Hk * d:].view(B, T, Hv, d)
    yout = torch.empty_like(core)

    def conv():
        gdn.gdn_causal_conv1d_silu(mix, conv_w, None, n_l2norm_ch=2 * Hk * d, l2norm_group=d,
                                   conv_state_out=cs_out, y=y)

    # the layer core as two calls: conv (+ SiLU + q/k L2 norm), then gates + chunked delta rule +
    # gated RMSNorm fused into the chunk kernels
    def step(timed):
        run = (lambda name, f: kt[name](f)) if timed else (lambda name, f: f())
        run("conv", conv)
        run("core", lambda: gdn.gdn_chunk_fwd_gated_norm(
            qv, kv, vv, a, b, A_log, dt_bias, z, norm_w, norm_eps=w["eps"], scale=d ** -0.5,
            y=yout, final_state=S_T, workspace=ws))

    ms = timed_region(dist, step, K, W)
    status = gdn.workspace_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status} after the fused layer core")
    per = {k_: t.mean_ms() for k_, t in kt.items()}

    # the same four steps as separate calls, for comparison
    ku = {"conv": KernelTimer(), "gates": KernelTimer(), "chunk": KernelTimer(),
          "norm": KernelTimer()}

    def step_unfused(timed):
        run = (lambda name, f: ku[name](f)) if timed else (lambda name, f: f())
        run("conv", conv)
        run("gates", lambda: gdn.gdn_gates(a, b, A_log, dt_bias, g=g, beta=beta))
        run("chunk", lambda: gdn.gdn_chunk_fwd(qv, kv, vv, g, beta, scale=d ** -0.5, chunk=64,
                                               out=core, final_state=S_T, workspace=ws))
        run("norm", lambda: gdn.gdn_gated_rmsnorm(core, z, norm_w, eps=w["eps"], y=yout))

    ms_u = timed_region(dist, step_unfused, K, W)
    per_u = {k_: t.mean_ms() for k_, t in ku.items()}
    n_tok = B * T
    conv_bytes = 2 * n_tok * C * 2
    flop = n_tok * Hv * CHUNK_FLOP_PER_TOKEN_HEAD
    return dict(value=n_tok * K * dist.world / (ms * 1e-3), unit="tokens/s", ms_per_step=ms / K,
                kernels_ms=per,
                conv_hbm_frac=conv_bytes / (per["conv"] * 1e-3) / 1e9 / peaks["hbm"],
                core_tensor_frac=flop / (per["core"] * 1e-3) / 1e12 / peaks["bf16"],
                unfused=dict(ms_per_step=ms_u / K, kernels_ms=per_u),
                gpu_launches=(1 + CHUNK_LAUNCHES + 1) * K)


# ------------------------------------------------------------------ CPU oracle --------------

def oracle_prefill_sample(seqs=(0, 1, 2, 3)):
    """The fp64 oracle on a bounded sample of the prefill workload: the given sequences, all
    32 v-heads, on every host core.  Returns (tokens/s, cores, description)."""
    import oracle
    w, x = _prefill_inputs()
    cu = x["cu_seqlens"]
    g, beta = oracle.gates(x["a"], x["b"], x["A_log"], x["dt_bias"])
    cores = os.cpu_count() or 1
    t0 = time.time()
    tokens = 0
    for n in seqs:
        s0, s1 = int(cu[n]), int(cu[n + 1])
        oracle.gated_delta_rule(x["q"][:, s0:s1], x["k"][:, s0:s1], x["v"][:, s0:s1],
                                g[:, s0:s1], beta[:, s0:s1], w["dk"] ** -0.5,
                                initial_state=x["initial_state"][n:n + 1], nthreads=cores)
        tokens += s1 - s0
    dt = time.time() - t0
    desc = (f"sequences {list(seqs)} of the 32K varlen workload ({tokens} tokens x 32 v-heads), "
            f"fp64, {cores} threads, {dt:.1f} s")
    return tokens / dt, cores, desc


def run_reference(args, dist):
    if dist.rank != 0:
        return 0
    rates = []
    desc = ""
    cores = os.cpu_count() or 1
    for i in range(args.warmup + args.steps):
        r, cores, desc = oracle_prefill_sample(seqs=(3,))
        if i >= args.warmup:
            rates.append(r)
    value = statistics.mean(rates)
    line = dict(metric=METRIC, value=value, unit="tokens/s", n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=2048 / value * 1e3, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                impl="reference",
                config=dict(workload="prefill_varlen_32k", tokens=32768,
                            seqlens=[16384, 8192, 6144, 2048], Hk=16, Hv=32, dk=128, dv=128,
                            chunk=64, l2="inputs larger than L2"),
                cpu_baseline=dict(value=value, unit="tokens/s", cores=cores, kind="oracle",
                                  sample="each step: " + desc),
                e2e=dict(value=value, unit="tokens/s", h2d_bytes_per_step=0,
                         d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ profiling -------------

def run_profile(mode, reps):
    """Runs one workload a few times and nothing else, for ncu captures (few launches, at most a
    few GB on the device):

    prefill    gdn_gates + gdn_chunk_fwd on the 32768-token varlen workload (4 sequences)
    prefill4k  gdn_gates + gdn_chunk_fwd on B=1, T=4096
    decode     consecutive gdn_gates + gdn_recurrent_step calls on 256 sequences x 32 heads
    conv       gdn_causal_conv1d_silu on the [2, 16384, 8192] mix, then gdn_gated_rmsnorm on the
               v channels viewed as 128-wide rows
    layercore  the layer core on B = 2 x 16384 tokens: gdn_causal_conv1d_silu, then
               gdn_chunk_fwd_gated_norm on q, k, v read in place from the conv output
    decodelayer  consecutive gdn_decode_layer_step calls on 256 sequences x 32 heads
    """
    from gated_deltanet_fwd_b200 import gdn
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
    elif mode == "decodelayer":
        w = dict(inputs.WORKLOADS["decode_layer_256"], steps=max(reps, 1))
        x = inputs.decode_layer_inputs(**w, seed=1000 + w["index"])
        st = x["state"].to(dev)
        cs = [x["conv_state"].to(dev), torch.empty_like(x["conv_state"]).to(dev)]
        cw, A_log, dt_bias = x["conv_w"].to(dev), x["A_log"].to(dev), x["dt_bias"].to(dev)
        nw = x["norm_w"].to(dev)
        for s_ in range(w["steps"]):
            gdn.gdn_decode_layer_step(x["mix"][s_].to(dev), x["a"][s_].to(dev),
                                      x["b"][s_].to(dev), x["z"][s_].to(dev), cw, cs[s_ & 1],
                                      cs[(s_ + 1) & 1], A_log, dt_bias, nw, st, w["Hk"])
    elif mode == "layercore":
        w = inputs.WORKLOADS["layer_core_2x16k"]
        x = inputs.layer_core_inputs(**w, seed=1000 + w["index"])
        B, T, Hk, Hv, d = w["B"], w["T"], w["Hk"], w["Hv"], w["dk"]
        mix, cw = x["mix"].to(dev), x["conv_w"].to(dev)
        a, b, z = x["a"].to(dev), x["b"].to(dev), x["z"].to(dev)
        A_log, dt_bias, nw = x["A_log"].to(dev), x["dt_bias"].to(dev), x["norm_w"].to(dev)
        for _ in range(reps):
            y = gdn.gdn_causal_conv1d_silu(mix, cw, None, n_l2norm_ch=2 * Hk * d, l2norm_group=d)
            gdn.gdn_chunk_fwd_gated_norm(y[:, :, :Hk * d].view(B, T, Hk, d),
                                         y[:, :, Hk * d:2 * Hk * d].view(B, T, Hk, d),
                                         y[:, :, 2 * Hk * d:].view(B, T, Hv, d), a, b, A_log,
                                         dt_bias, z, nw, norm_eps=w["eps"])
    else:
        raise SystemExit(run_profile.__doc__)
    torch.cuda.synchronize()
    print("done", mode, flush=True)
    return 0


# ------------------------------------------------------------------ main -------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", default=None,
                    help="run one workload for a profiler capture: "
                         "prefill|prefill4k|decode|conv|layercore|decodelayer")
    ap.add_argument("--repeats", type=int, default=2, help="launches per --profile run")
    args = ap.parse_args()
    if args.profile:
        return run_profile(args.profile, args.repeats)
    args.warmup = max(args.warmup, 3)
    dist = Dist()
    if args.impl == "reference":
        return run_reference(args, dist)

    from gated_deltanet_fwd_b200 import gdn
    gdn.load()
    torch.cuda.set_device(dist.local)
    dist.init("nccl")
    peaks = _peaks()
    clocks = ClockSampler(dist.local)
    clocks.start()
    pre = bench_prefill(dist, gdn, args.steps, args.warmup, peaks)
    clk = clocks.stop()
    clocks.start()
    dec = bench_decode(dist, gdn, max(2, args.steps // 4), args.warmup, peaks)
    dec["clocks"] = clocks.stop()
    clocks.start()
    dec_layer = bench_decode_layer(dist, gdn, max(2, args.steps // 4), args.warmup, peaks)
    dec_layer["clocks"] = clocks.stop()
    clocks.start()
    core = bench_layer_core(dist, gdn, max(2, args.steps // 4), args.warmup, peaks)
    core["clocks"] = clocks.stop()
    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        r, cores, desc = oracle_prefill_sample()
        cpu = dict(value=r, unit="tokens/s", cores=cores, kind="oracle", sample=desc)
    if dist.rank == 0:
        line = dict(metric=METRIC, value=pre["value"], unit="tokens/s", n_gpus=dist.world,
                    steps=args.steps, warmup=args.warmup, ms_per_step=pre["ms_per_step"],
                    higher_is_better=True, scaling="weak", vs_baseline=None, dtype="bf16",
                    data="synthetic",
                    config=dict(workload="prefill_varlen_32k", tokens=32768,
                                seqlens=[16384, 8192, 6144, 2048], Hk=16, Hv=32, dk=128, dv=128,
                                chunk=64, state="fp32", step="gdn_gates + gdn_chunk_fwd",
                                l2="inputs larger than L2 (no flush)",
                                parallelism=f"replica x{dist.world}"),
                    roofline=pre["roofline"], e2e=pre["e2e"], gpu_launches=pre["gpu_launches"],
                    clocks=clk, cpu_baseline=cpu, decode=dec, decode_layer=dec_layer,
                    layer_core=core)
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
