"""The benchmark's reference arm (the oracle on the host cores) prints one JSON line with
the fields the driver reads. It needs no GPU, so it is checked here on the tiny
workload.
"""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    res = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                          "--steps", "2", "--warmup", "1"],
                         cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 2 and line["value"] > 0
    assert line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["config"]["workload"].startswith("tiny")
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_l2_rule_of_the_timed_steps():
    """Steps that read at least twice the 126 MB L2 run back to back (inputs larger than
    L2); the others are timed after a 256 MB L2 write. Of the benchmark's workloads only
    tiny (and the FP8 decode, at 656 bytes per token) fall below the bar."""
    sys.path.insert(0, ROOT)
    import bench
    from mla_paged_kv_06_b200 import workloads as wl

    assert bench.L2_FLUSH_BYTES > bench.L2_BYTES
    assert bench.flush_free(2 * bench.L2_BYTES) and not bench.flush_free(2 * bench.L2_BYTES - 1)
    for name, expect in (("v3", True), ("uniform", True), ("skewed", True), ("spec", True),
                         ("tiny", False)):
        w = wl.WORKLOADS[name]
        lens = wl.draw_seqlens(w.seqlen, w.batch, 0)
        nbytes = wl.algorithmic_work(lens, w.s_q, w.h_q, w.causal)[0]
        assert bench.flush_free(nbytes) == expect, (name, nbytes)
        assert ("no flush" in bench.l2_note(nbytes, expect)) == expect
    tokens = int(wl.draw_seqlens(wl.WORKLOADS["uniform"].seqlen, wl.WORKLOADS["uniform"].batch, 0).sum())
    assert not bench.flush_free(tokens * 656)
