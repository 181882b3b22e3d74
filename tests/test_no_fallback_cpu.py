"""The product path has no CPU fallback: without libq4gemv.so the package
refuses to import, and nothing in the package or its native sources refers
to the oracle (test infrastructure) or to a host re-implementation."""
import os
import re
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "q4_quantized_decode_b200")


def test_import_fails_loudly_without_the_library(tmp_path):
    dst = tmp_path / "q4_quantized_decode_b200"
    dst.mkdir()
    for f in os.listdir(PKG):
        if f.endswith(".py"):
            shutil.copy(os.path.join(PKG, f), dst / f)          # sources only, no .so
    r = subprocess.run([sys.executable, "-c", "import q4_quantized_decode_b200"],
                       cwd=tmp_path, capture_output=True, text=True,
                       env={**os.environ, "PYTHONPATH": str(tmp_path)})
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libq4gemv.so is missing" in r.stderr


def test_package_never_refers_to_the_oracle():
    pat = re.compile(r"\boracle\b|q4_oracle|import\s+numpy")
    hits = []
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                p = os.path.join(dirpath, f)
                for n, line in enumerate(open(p, encoding="utf-8"), 1):
                    if pat.search(line):
                        hits.append(f"{os.path.relpath(p, ROOT)}:{n}: {line.strip()}")
    assert not hits, "\n".join(hits)
