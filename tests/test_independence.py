"""The oracle and the CUDA path share nothing, and the product never reaches
the oracle: a source scan on the CPU.

* No file of the library (the package, its CUDA sources, the C header) names
  the oracle.  The input generators import neither side and hold none of the
  method's arithmetic (no quantiser, plan or score: they draw numbers and
  round them to bf16).
* The oracle includes no header of the library and no file of it includes
  the oracle's.
* Importing the library's binding imports no oracle module."""
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PRODUCT_DIRS = ("decode_fathom_plan_b200", "include")
SOURCE_EXT = (".py", ".cu", ".cuh", ".h", ".c", ".cpp")


def _sources(top):
    for base, dirs, files in os.walk(os.path.join(ROOT, top)):
        dirs[:] = [d for d in dirs if not d.startswith(("_build", "__pycache__"))]
        for f in files:
            if f.endswith(SOURCE_EXT):
                yield os.path.join(base, f)


def test_product_sources_never_name_the_oracle():
    pat = re.compile(r"\boracle\b|fathom_oracle|\bfo_[a-z]")
    hits = []
    for top in PRODUCT_DIRS:
        for path in _sources(top):
            for i, line in enumerate(open(path, encoding="utf-8"), 1):
                if pat.search(line):
                    hits.append(f"{os.path.relpath(path, ROOT)}:{i}: {line.strip()}")
    assert not hits, "\n".join(hits)


def test_input_generators_import_no_oracle():
    """The generators serve both sides (their docstring may say so), but import
    neither of them."""
    for path in _sources("synth"):
        for line in open(path, encoding="utf-8"):
            if re.match(r"\s*(import|from)\s", line):
                assert "oracle" not in line and "decode_fathom_plan_b200" not in line, line


def test_oracle_includes_nothing_of_the_library():
    src = open(os.path.join(ROOT, "oracle", "fathom_oracle.c"), encoding="utf-8").read()
    includes = re.findall(r'#include\s*[<"]([^>"]+)[>"]', src)
    assert includes and all(h in ("math.h", "stdint.h", "stdlib.h", "string.h") for h in includes), includes
    py = open(os.path.join(ROOT, "oracle", "__init__.py"), encoding="utf-8").read()
    assert "decode_fathom_plan_b200" not in py and "libfathom" not in py


def test_input_generators_hold_no_method_arithmetic():
    src = open(os.path.join(ROOT, "synth", "__init__.py"), encoding="utf-8").read()
    for word in ("quantiz", "water", "plan_", "bit plane", "topk", "argsort", "scale_c"):
        assert word not in src.lower(), word


def test_importing_the_binding_loads_no_oracle_module():
    code = ("import sys; import decode_fathom_plan_b200, synth; "
            "bad = [m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')]; "
            "print(bad); sys.exit(1 if bad else 0)")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
