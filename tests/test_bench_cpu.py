"""bench.py's reference arm (the CPU oracle) runs without a GPU: its JSON line
keeps the contract's keys, with zero host<->device bytes."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
         "--warmup", "0", "--cpu-seconds", "2"],
        cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"] == "lumina_mgpt_768"  # the default headline workload
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"]


def test_reference_arm_takes_the_variant_flags():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
         "--warmup", "0", "--cpu-seconds", "1", "--workload", "llamagen_xl",
         "--cls-queries", "8", "--cfg-pairing", "halves",
         "--mode", "uniform", "--unstratified"],
        cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    d = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][0])
    c = d["config"]
    assert c["grouping_queries"] == 8 and c["cfg_pairing"] == "halves"
    assert c["budgets"] == "uniform" and c["strata"] == "pooled"
    assert d["value"] > 0


def test_planted_recovery():
    """Labels equal to the planted kinds recover everything; all-Global
    labels recover nothing; the shares count (layer, sequence, head)."""
    import numpy as np

    sys.path.insert(0, ROOT)
    import bench
    from kv_cache_compression_hkv_b200.inputs import WORKLOADS, planted_local_heads
    w = WORKLOADS["llamagen_xl"].scaled(num_layers=3, num_seqs=2)
    planted = np.stack([planted_local_heads(w, l, 5).numpy() for l in range(3)])
    perfect = np.repeat(planted[:, None, :], 2, axis=1).astype(np.uint8)
    assert bench.planted_recovery(w, perfect, 5) == {"local_as_local": 1.0,
                                                     "global_as_local": 0.0}
    none = np.zeros_like(perfect)
    assert bench.planted_recovery(w, none, 5) == {"local_as_local": 0.0, "global_as_local": 0.0}
    flipped = 1 - perfect
    assert bench.planted_recovery(w, flipped, 5) == {"local_as_local": 0.0,
                                                     "global_as_local": 1.0}
    # one planted Local head of one sequence missed: 1 of 3 * 2 * 12
    part = perfect.copy()
    part[0, 0, int(np.flatnonzero(planted[0])[0])] = 0
    r = bench.planted_recovery(w, part, 5)
    assert abs(r["local_as_local"] - (1 - 1 / 72)) < 1e-12 and r["global_as_local"] == 0.0
