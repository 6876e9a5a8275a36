"""bench.py's reference arm (the CPU oracle on the host cores) and its JSON
line, on CPU: the keys the benchmark contract asks for, the oracle sample
description, and the algorithmic byte and operation counts it reports
(checked against the layer shapes). No GPU."""
import json
import subprocess
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))

import bench  # noqa: E402
from quantized_lora_merge_b200 import workloads as wl  # noqa: E402


def test_reference_arm_json_line():
    res = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1", "--config", "linear320"],
                         capture_output=True, text=True, timeout=600, cwd=str(ROOT))
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    one = line["cpu_baseline"]["single_core"]
    assert one["cores"] == 1 and one["value"] > 0 and one["unit"] == line["unit"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_reference_arm_bounds_its_steps_with_a_row_block():
    """Many steps on a large config: each step's sample shrinks to a block of
    the first layer's rows, so the run stays near --reference-seconds."""
    res = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--impl", "reference", "--steps", "4",
                          "--warmup", "1", "--config", "llama3_8b", "--reference-seconds", "2"],
                         capture_output=True, text=True, timeout=600, cwd=str(ROOT))
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    assert line["steps"] == 4 and line["value"] > 0
    assert "rows of layer0.q (4096x4096) taken as one layer" in line["cpu_baseline"]["sample"]
    assert line["ms_per_step"] < 2000.0


@pytest.mark.parametrize("cfg", ["sd_unet", "llama3_8b", "dit_3072"])
def test_algorithmic_counts(cfg):
    layers = wl.CONFIGS[cfg]()
    for l in layers[:4]:
        code = 0.5 if l.w_bits == 4 else 1.0
        assert bench.prepare_bytes(l) == l.numel * (8 + code) + l.d * 8
        assert bench.ste_bytes(l) == 2 * l.numel + 6 * l.r * (l.d + l.n)
        assert bench.merge_bytes(l) > l.numel * code
        assert bench.merge_ops(l) == l.numel * (22 + l.r + (5.5 if l.variant == "mul" else 8.0))
        # the tensor cores form A B in the fused kernel: no rank term on the lanes
        assert bench.merge_ops(l, True) == l.numel * (22 + (5.5 if l.variant == "mul" else 8.0))


def test_host_room_for_pinned_arenas(tmp_path):
    """The end-to-end leg's pinned arenas are checked against the node's
    available host memory for every rank on the node (10 % margin)."""
    mi = tmp_path / "meminfo"
    mi.write_text("MemTotal:       209715200 kB\nMemAvailable:   104857600 kB\n")   # 100 GiB free
    need = 40 << 30
    assert bench.host_room(need, 1, str(mi)) == (True, "")
    assert bench.host_room(need, 2, str(mi)) == (True, "")        # 80 GiB x 1.1 < 100 GiB
    ok, why = bench.host_room(need, 3, str(mi))
    assert not ok and "3 rank(s)" in why
    # no MemAvailable line: nothing to compare against, the leg runs
    mi.write_text("MemTotal:       209715200 kB\n")
    assert bench.host_room(need, 8, str(mi)) == (True, "")
