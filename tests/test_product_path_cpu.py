"""The product path has no CPU fallback and never touches the oracle."""
import os
import re
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "decode_kv_cache_paged_b200")


def test_package_without_library_fails_loudly(tmp_path):
    """A copy of the package without libkvc.so must refuse to import."""
    dst = tmp_path / "decode_kv_cache_paged_b200"
    dst.mkdir()
    for name in ("__init__.py", "workloads.py"):
        shutil.copy(os.path.join(PKG, name), dst / name)
    r = subprocess.run([sys.executable, "-c", "import decode_kv_cache_paged_b200"], cwd=tmp_path,
                       capture_output=True, text=True, env={**os.environ, "PYTHONPATH": str(tmp_path)})
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "no CPU fallback" in r.stderr


def test_product_code_never_references_the_oracle():
    """Neither the binding nor the CUDA sources import, load or call oracle/."""
    pattern = re.compile(r"^\s*(import|from)\s+oracle\b|import_module\(.oracle|liboracle|\borc_[a-z]")
    offenders = []
    for dirpath, _, files in os.walk(PKG):
        if "_build" in dirpath:
            continue
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                with open(os.path.join(dirpath, f), encoding="utf-8") as fh:
                    for i, line in enumerate(fh, 1):
                        if pattern.search(line):
                            offenders.append(f"{f}:{i}: {line.strip()}")
    assert not offenders, offenders
