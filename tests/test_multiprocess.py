"""The N > 1 launch path of bench.py, on CPU with the gloo backend: each rank is an independent
replica, so the only collectives are the timing barrier and the max-over-ranks reduction of the
elapsed time; and under torchrun the reference (oracle) arm prints from rank 0 alone while the
other ranks exit 0 without work."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_SCRIPT = r"""
import sys
sys.path.insert(0, sys.argv[1])
import bench
d = bench.Dist()
d.init("gloo")
d.barrier()
m = d.max(float(d.rank) + 0.5)
d.barrier()
d.close()
print("RESULT", d.rank, d.world, m, flush=True)
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(**kw):
    env = dict(os.environ)
    env.update({k: str(v) for k, v in kw.items()})
    env["CUDA_VISIBLE_DEVICES"] = ""
    return env


def test_dist_barrier_and_max_two_gloo_ranks():
    port = _free_port()
    procs = [subprocess.Popen([sys.executable, "-c", RANK_SCRIPT, ROOT],
                              env=_env(RANK=r, LOCAL_RANK=r, WORLD_SIZE=2,
                                       MASTER_ADDR="127.0.0.1", MASTER_PORT=port),
                              stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
             for r in range(2)]
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err[-2000:]
        outs.append(out)
    results = sorted(l.split() for o in outs for l in o.splitlines() if l.startswith("RESULT"))
    # both ranks agree on the maximum over ranks (rank 1's 1.5)
    assert [r[1:] for r in results] == [["0", "2", "1.5"], ["1", "2", "1.5"]]


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    p = subprocess.run(cmd, cwd=ROOT, env=_env(), capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout[-2000:]
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["warmup"] >= 3
    assert rec["value"] > 0 and rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["value"] == rec["value"]
