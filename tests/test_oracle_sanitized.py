"""The CPU oracle built with AddressSanitizer and UndefinedBehaviorSanitizer
runs every entry point on small and ragged inputs without a report: no
out-of-bounds access, use after free, signed overflow or invalid shift in the
code that every parity claim rests on. CPU only."""
import os
import shutil
import subprocess
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]


def _asan_runtime():
    if shutil.which("gcc") is None:
        return None
    p = subprocess.run(["gcc", "-print-file-name=libasan.so"], capture_output=True, text=True).stdout.strip()
    return p if os.path.isabs(p) and os.path.exists(p) else None


def test_oracle_under_address_and_undefined_behaviour_sanitizers(tmp_path):
    asan = _asan_runtime()
    if asan is None:
        pytest.skip("gcc's sanitizer runtime is not installed")
    lib = tmp_path / "liboracle_sanitized.so"
    subprocess.run(["gcc", "-std=c11", "-O1", "-g", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
                    "-fPIC", "-shared", "-fsanitize=address,undefined", "-fno-sanitize-recover=all",
                    "-fno-omit-frame-pointer", str(ROOT / "oracle" / "intlora_oracle.c"), "-o", str(lib),
                    "-lm"], check=True, timeout=300)
    env = dict(os.environ, LD_PRELOAD=asan, ASAN_OPTIONS="detect_leaks=0",
               UBSAN_OPTIONS="print_stacktrace=1")
    run = [sys.executable, str(ROOT / "tests" / "oracle_sanitize_run.py"), str(lib)]
    res = subprocess.run(run, env=env, capture_output=True, text=True, timeout=600, cwd=str(ROOT))
    assert res.returncode == 0, res.stderr[-3000:]
    assert res.stdout.strip().endswith("done")
    assert "runtime error" not in res.stderr and "AddressSanitizer" not in res.stderr
    # the pin suite's own calls (large draws, brute force, worked examples)
    res = subprocess.run(run + ["--pins"], env=env, capture_output=True, text=True, timeout=900,
                         cwd=str(ROOT))
    assert res.returncode == 0, (res.stdout[-2000:], res.stderr[-3000:])
    assert " passed" in res.stdout
    assert "runtime error" not in res.stderr and "AddressSanitizer" not in res.stderr
