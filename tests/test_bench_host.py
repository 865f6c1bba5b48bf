"""Host logic of the benchmark that needs no GPU: the flop count of the
block-sparse step (pairs the tile mask selects, ragged last tiles included)
and the clock sampler's parsing of nvidia-smi samples around a timed region
shorter than the sampling period (a fake nvidia-smi on PATH)."""
import os
import stat
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from quantization_aware_attention_nvfp4_b200 import workloads as W  # noqa: E402


def test_selected_pairs_counts_ragged_tiles():
    w = W.custom(2, 3, 300, 200, 64, seed_index=5)
    mask = W.random_tile_mask(w, 0.5)
    T = W.SPARSE_TILE
    brute = 0
    for b in range(w.B):
        for h in range(w.H):
            for i in range(w.Lq):
                for j in range(w.Lk):
                    brute += int(mask[b, h, i // T, j // T])
    assert bench.selected_pairs(w, mask) == brute
    assert bench.selected_pairs(w, np.ones_like(mask)) == w.B * w.H * w.Lq * w.Lk


def test_topk_tiles_follows_the_selection_formula():
    # max(1, min(ceil((1 - sparsity) * n), n))
    assert W.topk_tiles(244, 0.9) == 25
    assert W.topk_tiles(10, 0.9) == 1
    assert W.topk_tiles(5, 0.0) == 5
    assert W.topk_tiles(7, 1.0) == 1
    m = W.tile_mask(W.get("wan_6h_31200"), 0.9)
    assert m.shape == (1, 6, 244, 244) and np.all(m.sum(-1) == 25)


def _fake_smi(tmp_path, reason):
    script = tmp_path / "nvidia-smi"
    script.write_text("#!/bin/sh\nsleep 0.2\nfor i in $(seq 1 200); do echo '0, 1800, 1965, 700.0, 0x4, Not Active, "
                      "Not Active, Not Active, %s'; sleep 0.05; done\n" % reason)
    script.chmod(script.stat().st_mode | stat.S_IEXEC)
    return str(tmp_path)


def test_clock_sampler_brackets_a_short_region(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, "Active") + os.pathsep + os.environ["PATH"])
    with bench.ClockSampler(0) as c:
        time.sleep(0.01)  # far shorter than the 50 ms sampling period
    s = c.summary()
    assert s["samples"] >= 2
    assert s["sm_mhz"] == 1800.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))  # nothing to run
    with bench.ClockSampler(0) as c:
        pass
    assert c.summary()["reasons"] == ["nvidia-smi unavailable"]


def test_default_metric_and_workload_names():
    import argparse
    a = argparse.Namespace(sparsity=None, causal=False, flags=15, workload="wan_6h_31200", tile=128)
    w = W.get("wan_6h_31200")
    assert bench.metric_name(a, w) == bench.METRIC
    assert bench.workload_name(a, w) == "wan_6h_31200"
    a.flags = 7
    assert bench.workload_name(a, w) == "wan_6h_31200_flags7"
    assert bench.flag_names(7) == "q,k,v" and bench.flag_names(0) == "none"
    a.causal = True
    assert bench.metric_name(a, w).startswith("Causal") and bench.workload_name(a, w) == "causal_wan_6h_31200_flags7"


def test_dtype_weighted_peak():
    # four units, one on a pipe four times faster: floor 3 + 1/4 unit-times
    assert abs(bench.dtype_weighted_peak(1000.0, 4, 1) - 1000.0 * 4 / 3.25) < 1e-9
    assert bench.dtype_weighted_peak(1000.0, 2, 0) == 1000.0


def test_oracle_sample_rows_scale_with_key_length():
    assert bench.sample_rows(W.get("wan_6h_31200"), 6144) == 6144
    assert bench.sample_rows(W.get("large_40h_75600"), 6144) == int(6144 * 31200 / 75600)
    assert bench.sample_rows(W.get("tiny"), 6144) == 256  # capped at Lq


def test_metric_names_of_every_leg_and_workload():
    import argparse
    for w in W.WORKLOADS:
        for flags in (15, 7, 0):
            for sparsity, causal in ((None, False), (0.9, False), (None, True)):
                a = argparse.Namespace(sparsity=sparsity, causal=causal, flags=flags, workload=w.name, tile=128)
                name = bench.metric_name(a, w)
                assert "B%d H%d L%d" % (w.B, w.H, w.Lq) in name or name == bench.METRIC
                assert bench.workload_name(a, w).endswith(w.name if flags == 15 else "%s_flags%d" % (w.name, flags))
    a = argparse.Namespace(sparsity=None, causal=False, flags=15, workload="tiny", tile=128)
    assert bench.metric_name(a, W.get("tiny")) == "Attn-QAT fwd+bwd ms & TFLOP/s at B1 H2 L256 D64; % of B200 BF16 peak"


def test_selected_pairs_of_64_token_blocks():
    w = W.custom(1, 2, 300, 200, 64, seed_index=6)
    rng = np.random.default_rng(1)
    mask = (rng.random((1, 2, 5, 4)) < 0.5).astype(np.uint8)
    brute = sum(int(mask[0, h, i // 64, j // 64]) for h in range(2) for i in range(300) for j in range(200))
    assert bench.selected_pairs(w, mask, 64) == brute


def test_attention_digest_ignores_comments_not_code():
    """The digest that ties profiles/traffic.json to the kernels is the same
    after a comment edit and different after a code edit."""
    from quantization_aware_attention_nvfp4_b200 import build
    base = {n: open(os.path.join(build.CSRC, n)).read() for n in build.ATTENTION_SOURCES}
    d0 = build.attention_sources_digest(lambda n: base[n])
    assert d0 == build.attention_sources_digest()
    commented = dict(base)
    commented["fwd.cu"] = "// a new line comment\n/* and a\n block one */\n" + base["fwd.cu"].replace(";", ";  // note", 1)
    assert build.attention_sources_digest(lambda n: commented[n]) == d0
    edited = dict(base)
    edited["bwd.cu"] = base["bwd.cu"].replace("kBN", "kBM", 1)
    assert build.attention_sources_digest(lambda n: edited[n]) != d0
    assert build.code_only("a = 1; // x\n/* y */ b  =\n 2;") == "a = 1; b = 2;"


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the float64 oracle on the host cores) prints
    one JSON line with the keys the benchmark contract names."""
    import json
    import subprocess
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    p = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "1", "--workload", "tiny"], capture_output=True, text=True, timeout=600,
                       cwd=root)
    assert p.returncode == 0, p.stderr
    lines = [ln for ln in p.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1 and d["value"] > 0
    assert d["config"]["workload"] == "tiny"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
