"""The library and the oracles share no code and neither imports the other.

Only the seeded input generators (``synthetic.py``, no method arithmetic) serve both sides, and the
oracles take plain arrays, so they import neither the package nor its generators."""

import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_sparse_long_dual_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _sources(top, exts):
    for d, _, files in os.walk(top):
        for f in files:
            if f.endswith(exts):
                yield os.path.join(d, f)


def test_library_sources_never_reach_the_oracle():
    pat = re.compile(r"^\s*(from\s+oracle\b|import\s+oracle\b|#\s*include\s*[<\"].*oracle)", re.M)
    hits = [p for p in _sources(PKG, (".py", ".cu", ".cuh", ".h", ".cpp", ".c"))
            if pat.search(open(p, encoding="utf-8").read())]
    assert not hits, hits


def test_oracles_import_only_the_standard_library_and_numpy():
    allowed = {"__future__", "math", "dataclasses", "numpy"}
    for p in _sources(ORACLE, (".py",)):
        mods = re.findall(r"^\s*(?:from\s+(\S+)\s+import|import\s+(\S+))", open(p, encoding="utf-8").read(), re.M)
        used = {(a or b).split(".")[0] for a, b in mods}
        assert used <= allowed, (p, used - allowed)


def test_importing_the_binding_loads_no_oracle_module():
    code = ("import sys; import block_sparse_long_dual_b200.sfa, block_sparse_long_dual_b200.synthetic; "
            "print(sorted(m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')))")
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "[]"
