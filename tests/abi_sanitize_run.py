"""Runs tests/test_abi.py (host-side validation of every C-ABI entry point,
no GPU) against the library given on the command line: a build with
AddressSanitizer and UndefinedBehaviorSanitizer on its host code, loaded with
the sanitizer runtime preloaded (see tests/test_abi_sanitized.py). Exits with
pytest's status; the sanitizers abort the process on a report."""
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))

import pytest  # noqa: E402

import quantized_lora_merge_b200.build as qbuild  # noqa: E402
from quantized_lora_merge_b200 import binding as B  # noqa: E402

B.LIB_PATH = Path(sys.argv[1])
qbuild.build = lambda force=False, verbose_ptxas=False: B.LIB_PATH    # never rebuild here

if __name__ == "__main__":
    # -s: a sanitizer report goes straight to stderr instead of a capture file
    sys.exit(pytest.main(["-q", "-x", "-s", "-p", "no:cacheprovider", str(ROOT / "tests" / "test_abi.py")]))
