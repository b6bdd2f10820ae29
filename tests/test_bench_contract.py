"""The benchmark's one-line JSON report: the keys and invariants its readers rely on.

The reference arm (the fp64 oracle on the host cores) runs here on the CPU; the
device arm runs a short default step on the GPU.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
COMMON = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
          "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def _run(args, timeout):
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=timeout)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]       # exactly one JSON line
    return json.loads(lines[0])


def _check_common(d):
    missing = COMMON - set(d)
    assert not missing, missing
    assert d["n_gpus"] == 1 and d["scaling"] == "weak" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["warmup"] >= 3
    assert isinstance(d["config"], dict) and d["config"]["workload"].startswith("gqa70b")
    e = d["e2e"]
    assert {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"} <= set(e) and e["unit"] == d["unit"]


def test_reference_arm_line():
    d = _run(["--impl", "reference", "--steps", "1", "--warmup", "3"], timeout=600)
    _check_common(d)
    assert d["impl"] == "reference" and d["dtype"] == "f64"
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["cores"] >= 1 and c["sample"] and c["value"] == d["value"]
    assert d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


@pytest.mark.gpu
def test_device_arm_line():
    d = _run(["--steps", "5", "--warmup", "3", "--no-cpu-baseline"], timeout=900)
    _check_common(d)
    assert "impl" not in d or d["impl"] != "reference"
    r = d["roofline"]
    assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(r)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    assert 0.3 < r["frac"] < 1.3                       # above 1 a little is possible; far above is a bug
    assert d["gpu_launches"] > 0 and d["device_errors"] == 0
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["d2h_bytes_per_step"] > 0
    c = d["clocks"]
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(c)
    s = d["us_decode_spread"]
    assert s["p10"] <= s["median"] <= s["p90"]
    # the other configurations of the benchmark, each with its own roofline and errors
    cf = d["configs"]
    assert set(cf) == {"mha13b", "shared_prefix", "fp8_long", "beam", "prefill70b"}
    for name, e in cf.items():
        assert e["value"] > 0 and e["device_errors"] == 0, name
        assert {"bound", "achieved", "peak", "unit", "frac", "traffic"} <= set(e["roofline"]), name
        # the beam step (68 MB of unique KV, few long work units) is latency-bound well below
        # the copy bandwidth; far above 1 would mean the timed kernel skipped work
        assert 0.05 < e["roofline"]["frac"] < 1.3, (name, e["roofline"])
    assert cf["shared_prefix"]["unique_kv_bytes_per_step"] < cf["shared_prefix"]["logical_kv_bytes_per_step"]
    assert cf["beam"]["unique_kv_bytes_per_step"] < cf["beam"]["logical_kv_bytes_per_step"]


def test_unique_kv_bytes_counts_a_shared_block_once():
    """Two sequences sharing their first two blocks: 16 + 16 shared tokens, then
    8 and 3 tokens in their own last blocks; a block's count is the most tokens
    any sequence reads from it."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    tables = np.array([[5, 6, 7], [5, 6, 9]], np.int32)
    assert bench.unique_kv_bytes(tables, np.array([40, 35]), 10) == (16 + 16 + 8 + 3) * 10
    assert bench.unique_kv_bytes(tables, np.array([20, 40]), 1) == 16 + 16 + 8      # block 6: 4 vs 16 tokens
    assert bench.unique_kv_bytes(tables, np.array([0, 0]), 1) == 0


def test_source_hash_ignores_comments_only():
    """The committed ncu traffic is keyed to the kernels' code: comments and blank
    lines may change, code (inline PTX strings included) may not."""
    import bench
    base = 'int f(int a) {  // twice\n    return 2 * a;\n}\nasm("add.u32 %0; // in the string");\n'
    same = '/* doubles */\nint f(int a) {\n\n    return 2 * a;   // comment\n}\nasm("add.u32 %0; // in the string");\n'
    other = 'int f(int a) {\n    return 3 * a;\n}\nasm("add.u32 %0; // in the string");\n'
    ptx = 'int f(int a) {\n    return 2 * a;\n}\nasm("add.u32 %0; // changed");\n'
    h = lambda text: bench.kernel_source_hash(("x.cu",), read=lambda f: text)
    assert h(base) == h(same)
    assert h(base) != h(other) and h(base) != h(ptx)


def test_every_traffic_entry_matches_the_current_kernels():
    """Each workload's committed DRAM traffic was captured from the code that is in
    the tree now (otherwise the bench line reports null traffic for it)."""
    import bench
    data = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
    for w in ("gqa70b", "mha13b", "fp8_long", "shared_prefix", "beam", "prefill70b", "prefill70b_fp8"):
        assert w in data, w
        assert bench.ncu_traffic(w) == data[w]["dram_bytes_per_launch"], "stale traffic entry: %s" % w
