"""The benchmark's host-side logic, on CPU: the reference arm -- the fp64
oracle timed on the host cores -- keeps the one-JSON-line contract, alone and
under torchrun (rank 0 alone runs and prints; the other ranks exit 0 without
work); the rule that sends a timed run round again on a bad clock record; and
the roofline's byte accounting against the keys the oracle reads."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
ARGS = ["bench.py", "--impl", "reference", "--steps", "2", "--warmup", "3", "--workload", "tiny"]


def _json_lines(text):
    return [json.loads(line) for line in text.splitlines() if line.startswith("{")]


def _check_line(d, n_gpus):
    assert d["impl"] == "reference"
    for key in ("metric", "unit", "dtype", "data", "scaling"):
        assert isinstance(d[key], str) and d[key]
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["n_gpus"] == n_gpus and d["steps"] == 2 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["config"]["workload"] == "tiny"
    # the same config dict the GPU arm prints (the driver compares them key by key)
    import synth
    import bench
    assert d["config"] == bench.bench_config(synth.WORKLOADS["tiny"], False, n_gpus)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable] + ARGS, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_line(lines[0], 1)


def test_reference_arm_under_torchrun_prints_on_rank_zero_only():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port)] + ARGS + ["--gpus", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_line(lines[0], 2)


def test_clock_records_that_disqualify_a_timed_region():
    """Hardware or thermal slowdown, or SM clocks stuck well below their
    maximum with no reason reported, send the main timed run round once more;
    a power cap alone does not."""
    import sys
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench
    ok = {"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": []}
    assert not bench.clocks_rejected(ok)
    assert not bench.clocks_rejected({"sm_mhz": 1320.0, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]})
    for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clocks_rejected({"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": [r]})
    assert bench.clocks_rejected({"sm_mhz": 1100.0, "sm_max_mhz": 1965, "reasons": []})  # a leftover clock lock
    assert not bench.clocks_rejected({"sm_mhz": None, "sm_max_mhz": None, "reasons": []})  # no NVML: nothing to judge



@pytest.mark.parametrize("per_head", [0, 1])
def test_roofline_key_bytes_agree_with_the_oracles_key_count(per_head):
    """The K/V bytes the roofline counts per step (2 x D x 2 bytes per key of
    the union of each unit's fresh ranges, from the step's decisions) equal
    the keys the oracle actually reads, on a stream with hits and misses."""
    import sys
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench
    import oracle
    import synth
    wl = synth.WORKLOADS["tiny"].with_(steps=40, head_labels=bool(per_head))
    stream, cache = synth.queries(wl), synth.kv_cache(wl)
    orc = oracle.Oracle.for_workload(wl, cache, per_head=per_head)
    hits = 0
    for t in range(wl.steps):
        r = orc.step(stream.q[t], stream.rope_pos[t], cache.K, cache.V, cache.block_table, stream.seq_lens[t])
        _, _, kv = bench.step_bytes(wl, r.hit, r.match_pos, stream.seq_lens[t], min(t, wl.W))
        assert kv == r.keys_read * 2 * wl.D * 2, t
        hits += int(r.hit.sum())
    assert 0 < hits < wl.steps * r.hit.size


def test_compact_line_keeps_five_significant_digits():
    """The one JSON line rounds floats to five significant digits (the full
    record goes to stderr) and leaves every other value as it is."""
    import bench
    rec = {"value": 14396.609269749571, "frac": 0.6022880969335624, "n": 20, "ok": True, "none": None,
           "nested": {"us": [20.285333041101694, 143.22400093078613], "name": "x"}, "inf": float("inf")}
    out = bench._compact(rec)
    assert out["value"] == 14397.0 and out["frac"] == 0.60229 and out["n"] == 20 and out["ok"] is True
    assert out["none"] is None and out["nested"]["name"] == "x" and out["inf"] == float("inf")
    assert out["nested"]["us"] == [20.285, 143.22]
