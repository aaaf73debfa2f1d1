"""Structural rules of the product, checked without a GPU:
  * the product package never imports the oracle (the oracle is test infrastructure);
  * bench.py touches the oracle only in its CPU-baseline and reference legs;
  * without the native library the binding fails loudly instead of falling back;
  * the reference arm prints one JSON line with the contract's keys.
"""
import ast
import glob
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _oracle_imports(path):
    tree = ast.parse(open(path).read())
    found = []
    for fn in [n for n in ast.walk(tree) if isinstance(n, (ast.FunctionDef, ast.Module))]:
        for sub in ast.walk(fn):
            if isinstance(sub, ast.ImportFrom) and sub.module and sub.module.split(".")[0] == "oracle":
                found.append(getattr(fn, "name", "<module>"))
            if isinstance(sub, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in sub.names):
                found.append(getattr(fn, "name", "<module>"))
    return found


def test_product_package_does_not_import_the_oracle():
    for path in glob.glob(os.path.join(ROOT, "kv_cache_vector_encode_b200", "**", "*.py"), recursive=True):
        assert not _oracle_imports(path), path
    for path in glob.glob(os.path.join(ROOT, "kv_cache_vector_encode_b200", "csrc", "*")):
        assert "oracle" not in open(path, errors="ignore").read().lower() or path.endswith(".md"), path


def test_bench_uses_the_oracle_only_in_its_baseline_legs():
    users = set(_oracle_imports(os.path.join(ROOT, "bench.py"))) - {"<module>"}
    assert users <= {"oracle_step", "oracle_per_workload", "run_reference", "cpu_baseline_measure"}, users
    # and the oracle helpers themselves are only reached from those legs
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    for helper in ("oracle_step", "oracle_per_workload"):
        callers = {fn.name for fn in ast.walk(tree) if isinstance(fn, ast.FunctionDef)
                   for c in ast.walk(fn) if isinstance(c, ast.Call) and getattr(c.func, "id", "") == helper}
        assert callers <= {"run_reference", "cpu_baseline_measure"}, (helper, callers)


def test_missing_native_library_fails_loudly():
    code = ("import kv_cache_vector_encode_b200 as tq\n"
            "tq.LIB_PATH = '/nonexistent/libtq.so'\n"
            "try:\n    tq.lib()\nexcept RuntimeError as e:\n    print('raised', e)\nelse:\n    print('loaded')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert "raised" in r.stdout and "loaded" not in r.stdout, r.stdout + r.stderr


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "3", "--warmup", "3"], cwd=ROOT,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 3
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
