"""The product path stays independent of the oracle and has no fallback,
checked on the sources and on CPU:

- nothing under quantized_lora_merge_b200/ imports, loads or runs oracle/;
- bench.py reaches oracle/ only from its CPU baseline and reference-arm code
  (functions named for them, or a block guarded by the cpu-baseline switch);
- oracle/ imports nothing from the package's CUDA path;
- the binding raises when libintlora.so is absent instead of computing
  anything another way."""
import ast
import subprocess
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parents[1]
PKG = ROOT / "quantized_lora_merge_b200"


def _imports(tree):
    """(module name, node) of every import statement in a module."""
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name, node
        elif isinstance(node, ast.ImportFrom):
            yield (node.module or ""), node


def test_package_never_imports_the_oracle():
    for path in sorted(PKG.rglob("*.py")):
        tree = ast.parse(path.read_text())
        for name, _ in _imports(tree):
            assert name.split(".")[0] != "oracle", f"{path.name} imports {name}"
        # no dynamic route either (importlib, ctypes load of the oracle's C library)
        assert "liboracle" not in path.read_text() and "importlib" not in path.read_text(), path.name


def test_bench_uses_the_oracle_only_for_its_cpu_legs():
    src = (ROOT / "bench.py").read_text()
    tree = ast.parse(src)
    allowed_functions = {"oracle_sample", "single_core", "cpu_baseline", "run_reference"}
    parents = {}
    for node in ast.walk(tree):
        for child in ast.iter_child_nodes(node):
            parents[child] = node
    found = 0
    for name, node in _imports(tree):
        if name.split(".")[0] != "oracle":
            continue
        found += 1
        ok = False
        p = parents.get(node)
        while p is not None and not ok:
            if isinstance(p, ast.FunctionDef) and p.name in allowed_functions:
                ok = True
            if isinstance(p, ast.If) and "cpu_baseline" in ast.unparse(p.test):
                ok = True
            p = parents.get(p)
        assert ok, f"bench.py line {node.lineno} imports the oracle outside its CPU legs"
    assert found >= 1
    # never at module level: importing bench.py does not load the oracle
    assert all(not isinstance(n, (ast.Import, ast.ImportFrom)) or
               all(a.name.split(".")[0] != "oracle" for a in getattr(n, "names", []))
               for n in tree.body)


def test_oracle_does_not_reach_the_cuda_path():
    for path in sorted((ROOT / "oracle").rglob("*")):
        if path.suffix not in (".py", ".c", ".h"):
            continue
        text = path.read_text()
        assert "libintlora" not in text, path.name
        assert "quantized_lora_merge_b200.binding" not in text, path.name
        assert "csrc" not in text, path.name
        if path.suffix == ".py":
            for name, _ in _imports(ast.parse(text)):
                assert not name.startswith("quantized_lora_merge_b200") or name.endswith("workloads"), \
                    f"{path.name} imports {name}"


def test_binding_fails_loudly_without_the_library(tmp_path):
    code = (
        "import sys; from pathlib import Path; sys.path.insert(0, sys.argv[1])\n"
        "from quantized_lora_merge_b200 import binding as B\n"
        "B.LIB_PATH = Path(sys.argv[2]) / 'libintlora.so'\n"
        "try:\n"
        "    B.lib()\n"
        "except OSError as e:\n"
        "    print('raised', 'missing' in str(e))\n"
        "else:\n"
        "    print('loaded')\n")
    res = subprocess.run([sys.executable, "-c", code, str(ROOT), str(tmp_path)],
                         capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stderr[-2000:]
    assert res.stdout.strip() == "raised True"
