"""The multi-rank host logic of bench.py, on CPU with two gloo ranks launched by
torch.distributed.run (the same launcher the multi-GPU bench uses)."""
import json
import os
import socket
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _torchrun(args, timeout=300):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port())] + args
    env = dict(os.environ, OMP_NUM_THREADS="1")
    return subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=timeout, env=env)


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks([3, 1.5], 1) == [3.0, 1.5]


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(2, 2048, 0.5) == 2 * 2048 / 0.5e-3
    assert bench.job_throughput(1, 2048, 0.5) == 2048 / 0.5e-3


def test_max_over_ranks_two_gloo_ranks():
    out = os.path.join(ROOT, "_build", "multirank")  # build scratch inside the repository
    os.makedirs(out, exist_ok=True)
    for k in range(2):
        if os.path.exists(os.path.join(out, f"rank{k}.json")):
            os.remove(os.path.join(out, f"rank{k}.json"))
    r = _torchrun([os.path.join("tests", "_rank_helper.py"), out])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.load(open(os.path.join(out, f"rank{k}.json"))) for k in range(2)]
    assert sorted(d["rank"] for d in lines) == [0, 1]
    for d in lines:
        assert d["world"] == 2
        assert d["max"] == [2.0, 10.0, 5.0]  # element-wise max of the two ranks' timings
        assert d["value"] == 2 * 100 / (2.0 * 1e-3)  # both ranks' rows over the slowest rank's time


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    r = _torchrun(["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
                   "--workload", "tiny_m64_k256_n1024_p98"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
