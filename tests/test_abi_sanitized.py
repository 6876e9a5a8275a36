"""The C ABI's host code (argument validation, batching, workspace sizing)
built with AddressSanitizer and UndefinedBehaviorSanitizer passes the whole
host-validation suite (tests/test_abi.py) without a report. CPU only: no call
reaches a launch. The sanitized build is cached under _build/ by the hash of
the sources."""
import hashlib
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor
from pathlib import Path

import pytest

import quantized_lora_merge_b200.build as qbuild

ROOT = Path(__file__).resolve().parents[1]
SAN = ["-Xcompiler", "-fsanitize=address", "-Xcompiler", "-fsanitize=undefined",
       "-Xcompiler", "-fno-omit-frame-pointer"]


def _asan_runtime():
    if shutil.which("gcc") is None:
        return None
    p = subprocess.run(["gcc", "-print-file-name=libasan.so"], capture_output=True, text=True).stdout.strip()
    return p if os.path.isabs(p) and os.path.exists(p) else None


def _sanitized_library() -> Path:
    srcs = qbuild.sources()
    deps = sorted(srcs) + sorted(qbuild.CSRC.glob("*.cuh")) + sorted(qbuild.CSRC.glob("*.h")) + \
        sorted(qbuild.INCLUDE.glob("*.h"))
    digest = hashlib.sha256(b"".join(p.read_bytes() for p in deps) + " ".join(SAN).encode()).hexdigest()
    out = ROOT / "_build" / "sanitized"
    lib, stamp = out / "libintlora.so", out / "libintlora.so.sha256"
    if lib.exists() and stamp.exists() and stamp.read_text().strip() == digest:
        return lib
    out.mkdir(parents=True, exist_ok=True)
    objs = [str(out / (s.stem + ".o")) for s in srcs]
    cmds = [[qbuild.NVCC, *qbuild.ARCH, "-O1", "-std=c++17", "-Xcompiler", "-fPIC", *SAN,
             "--expt-relaxed-constexpr", "-I", str(qbuild.INCLUDE), "-I", str(qbuild.CSRC), "-c", str(s),
             "-o", o] for s, o in zip(srcs, objs)]
    with ThreadPoolExecutor(max_workers=max(1, min(len(cmds), os.cpu_count() or 1))) as pool:
        for f in [pool.submit(subprocess.run, c, check=True, capture_output=True) for c in cmds]:
            f.result()
    subprocess.run([qbuild.NVCC, *qbuild.ARCH, "-shared", "-Xcompiler", "-fPIC", *SAN, *objs, "-o",
                    str(lib)], check=True, capture_output=True)
    stamp.write_text(digest + "\n")
    return lib


def test_c_abi_host_code_under_address_and_undefined_behaviour_sanitizers():
    asan = _asan_runtime()
    if asan is None or not Path(qbuild.NVCC).exists():
        pytest.skip("nvcc or gcc's sanitizer runtime is not installed")
    lib = _sanitized_library()
    env = dict(os.environ, LD_PRELOAD=asan,
               ASAN_OPTIONS="detect_leaks=0:detect_odr_violation=0:alloc_dealloc_mismatch=0",
               UBSAN_OPTIONS="print_stacktrace=1:halt_on_error=1")
    res = subprocess.run([sys.executable, str(ROOT / "tests" / "abi_sanitize_run.py"), str(lib)], env=env,
                         capture_output=True, text=True, timeout=900, cwd=str(ROOT))
    assert res.returncode == 0, (res.stdout[-2000:], res.stderr[-3000:])
    assert "passed" in res.stdout
    assert "runtime error" not in res.stderr and "AddressSanitizer" not in res.stderr
