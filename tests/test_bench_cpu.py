"""The benchmark's JSON contract on the CPU: the reference arm (the fp64 oracle timed on the host
cores) prints one line with the keys the GPU arm's line also carries."""

import io
import json
import os
import sys
from contextlib import redirect_stdout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line():
    sys.path.insert(0, ROOT)
    import bench

    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--config", "1", "--steps", "2", "--warmup", "3"])
    assert rc == 0
    lines = [ln for ln in buf.getvalue().splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3 and d["value"] > 0
    assert d["config"]["workload"].startswith("cfg1")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_bench_rejects_too_few_warmup_steps():
    sys.path.insert(0, ROOT)
    import bench
    import pytest

    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--config", "1", "--warmup", "2"])


def test_reference_arm_prints_on_rank_zero_only(monkeypatch):
    """Under torchrun every rank runs the reference arm's command; only rank 0 works and prints."""
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--gpus", "2", "--config", "1", "--steps", "1", "--warmup", "3"])
    assert rc == 0 and buf.getvalue().strip() == ""


def test_recorded_traffic_only_for_the_captured_launch():
    """The roofline's DRAM traffic comes from a capture of the same kernel sources on the same
    launch: a layout or length override, or the other walk order over striped shards, must not
    pick up the default launch's figure (and the tile walk must find its own)."""
    sys.path.insert(0, ROOT)
    import dataclasses

    import bench
    from ring_blockwise_softmax_b200 import inputs as I

    w3 = I.WORKLOADS[3]  # striped, d = 128
    keys = {
        bench.traffic_key(w3),
        bench.traffic_key(w3, walk="tile"),
        bench.traffic_key(dataclasses.replace(w3, layout="contiguous")),
        bench.traffic_key(dataclasses.replace(w3, N=w3.N // 4)),
        bench.traffic_key(w3, backward=True),
    }
    assert len(keys) == 5
    assert bench.traffic_key(w3) == "cfg3"
    # the walk order only matters for striped shards at d > 64
    w2 = I.WORKLOADS[2]
    assert bench.traffic_key(w2, walk="tile") == bench.traffic_key(w2)
    rec = json.load(open(os.path.join(ROOT, "profiles", "fmha_traffic.json")))
    if rec["kernel_sources_sha256"] == bench.kernel_sources_hash():
        assert bench.recorded_traffic(bench.traffic_key(w3), "fused") is not None
        assert bench.recorded_traffic(bench.traffic_key(w3, walk="tile"), "fused") is not None
        assert bench.recorded_traffic(bench.traffic_key(dataclasses.replace(w3, layout="contiguous")), "fused") is None
        assert bench.recorded_traffic(bench.traffic_key(w3), "stepwise") is None
