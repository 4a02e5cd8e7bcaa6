"""bench.py with two ranks on CPU (gloo): the process group plumbing the GPU
runs use over NCCL (barrier, max of the timings over ranks), weak scaling (each
rank its own seeded batch of the same shapes), the whole-job throughput, and
the reference arm run by rank 0 alone."""
import json
import os
import socket
import subprocess
import sys

import bench

HERE = os.path.dirname(os.path.abspath(__file__))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_over_gloo():
    port = free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), OMP_NUM_THREADS="2")
        procs.append(subprocess.Popen([sys.executable, os.path.join(HERE, "rank_child.py")], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True))
    outs = []
    for p in procs:
        try:
            out, _ = p.communicate(timeout=240)
        finally:
            if p.poll() is None:
                p.kill()
        assert p.returncode == 0, out
        outs.append(out)
    res = {}
    for out in outs:
        line = [l for l in out.splitlines() if l.startswith("RESULT ")][-1]
        r = json.loads(line[len("RESULT "):])
        res[r["rank"]] = r
    assert sorted(res) == [0, 1] and all(r["world"] == 2 for r in res.values())
    # max over ranks reaches every rank
    assert res[0]["max"] == res[1]["max"] == 11.0
    # head split: contiguous ranges of the 5 heads; their kept work sums to the layer's
    assert res[0]["heads"] == [0, 3] and res[1]["heads"] == [3, 2]
    assert res[0]["flops_sum"] == res[1]["flops_sum"] == res[0]["flops_layer"]
    # weak scaling: same shapes, own seed, different data
    assert res[0]["q_shape"] == res[1]["q_shape"]
    assert res[0]["seed"] != res[1]["seed"] and res[0]["q_sum"] != res[1]["q_sum"]
    # the reference arm: one JSON line from rank 0, nothing from rank 1
    assert res[1]["reference_out"] == ""
    line = json.loads(res[0]["reference_out"].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_whole_job_throughput_is_all_ranks_work_over_the_slowest_time():
    # 2 ranks x 10 steps x 1 TFLOP in 1 s (the max over ranks) = 20 TFLOP/s
    assert bench.whole_job_tflops(2, 10, 1e12, 1000.0) == 20.0
    assert bench.whole_job_tflops(1, 5, 2e12, 500.0) == 20.0
    # a head split: one layer of 3 TFLOP per step shared by the ranks, 10 steps in 1 s
    assert bench.job_tflops(10, 3e12, 1000.0) == 30.0
