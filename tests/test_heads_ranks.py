"""Head-parallel layout of the layer (sparse_linear_hybrid_b200/heads.py): the
ranges of heads cover every head exactly once, and two ranks over gloo on CPU,
each running the oracle layer on its own heads, gather the output of the layer
run on all heads at once (the (b, h) units are independent; SALAD summary
section 2.1)."""
import json
import os
import socket
import subprocess
import sys

import pytest

from sparse_linear_hybrid_b200.heads import head_ranges

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("heads,world", [(40, 8), (12, 5), (12, 1), (7, 7), (5, 2), (1, 1)])
def test_head_ranges_cover_every_head_once(heads, world):
    rs = head_ranges(heads, world)
    assert len(rs) == world
    covered = [h for b, c in rs for h in range(b, b + c)]
    assert covered == list(range(heads))                      # contiguous, in rank order, each once
    counts = [c for _, c in rs]
    assert max(counts) - min(counts) <= 1 and min(counts) >= 1


def test_head_ranges_reject_more_ranks_than_heads():
    with pytest.raises(ValueError):
        head_ranges(4, 5)


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_gather_the_whole_layer():
    port = free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), OMP_NUM_THREADS="2")
        procs.append(subprocess.Popen([sys.executable, os.path.join(HERE, "heads_child.py")], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True))
    res = {}
    for p in procs:
        try:
            out, _ = p.communicate(timeout=240)
        finally:
            if p.poll() is None:
                p.kill()
        assert p.returncode == 0, out
        line = [l for l in out.splitlines() if l.startswith("RESULT ")][-1]
        r = json.loads(line[len("RESULT "):])
        res[r["rank"]] = r
    assert res[0]["range"] == [0, 3] and res[1]["range"] == [3, 2]
    for r in res.values():
        assert r["slice_max_diff"] == 0.0          # a head's output does not depend on the other heads
        assert r["gathered_max_diff"] == 0.0       # the gather puts every range in its place
        assert r["untouched_zero"]
