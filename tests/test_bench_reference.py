"""Host check of the reference arm's JSON line (bench.py --impl reference, the
CPU oracle on a bounded sample): the time it claims as measured fits inside the
wall clock of the run, and the extrapolated whole-step time is labelled apart."""
import argparse
import contextlib
import io
import json
import time

import bench
import salad_inputs as si


def test_reference_line_claims_no_more_time_than_the_run_had():
    args = argparse.Namespace(steps=5, warmup=3)
    buf = io.StringIO()
    t0 = time.perf_counter()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, si.TINY)
    wall = time.perf_counter() - t0
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 5
    assert line["steps"] * line["ms_per_step"] / 1e3 <= wall
    assert line["timed_s"] <= line["wall_s_of_timed_loop"] + 1e-3 <= wall
    assert line["query_blocks_per_step"] >= 1
    assert line["ms_per_full_step_extrapolated"] > 0 and line["extrapolated_from_s"] >= line["timed_s"]
    assert line["cpu_baseline"]["value"] == line["value"] == line["e2e"]["value"]
