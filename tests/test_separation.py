"""The oracle and the CUDA path stay apart, and the product path has no fallback.

Checked on the host from the sources:
- No file of the package (its Python or its CUDA/C++ sources, or the public header) imports,
  includes, loads or names the oracle.
- The oracle's C file includes only standard C headers and OpenMP. Its Python wrapper imports
  nothing of the package.
- The input generators that feed both sides import neither.
- Outside the tests, only the bench's CPU-baseline function and the smoke check import the
  oracle, each inside its own function.
- Without libsq.so the binding raises instead of computing anything.
"""
import ast
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "bit_quantized_frozen_b200")


def read(rel):
    with open(os.path.join(ROOT, rel)) as f:
        return f.read()


def imported_modules(rel):
    """(module name, enclosing function or None) for every import in a Python file."""
    tree = ast.parse(read(rel))
    out = []

    def visit(node, fn):
        for child in ast.iter_child_nodes(node):
            f = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else fn
            if isinstance(child, ast.Import):
                out.extend((a.name.split(".")[0], fn) for a in child.names)
            elif isinstance(child, ast.ImportFrom) and child.module:
                out.append((child.module.split(".")[0], fn))
            visit(child, f)
    visit(tree, None)
    return out


def package_files():
    for dirpath, _, names in os.walk(PKG):
        for n in names:
            if n.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                yield os.path.relpath(os.path.join(dirpath, n), ROOT)


def test_package_never_touches_the_oracle():
    for rel in list(package_files()) + ["include/sq.h"]:
        text = read(rel)
        if rel.endswith(".py"):
            assert "oracle" not in {m for m, _ in imported_modules(rel)}, rel
        assert not re.search(r"liboracle|sq_oracle|oracle/", text), rel
        assert not re.search(r"\bor_[a-z0-9_]+\s*\(", text), rel      # no call of an oracle routine


def test_oracle_includes_and_imports_nothing_of_the_package():
    includes = re.findall(r"#include\s*[<\"]([^>\"]+)[>\"]", read("oracle/sq_oracle.c"))
    assert set(includes) <= {"math.h", "stdint.h", "string.h", "stdlib.h", "omp.h"}, includes
    mods = {m for m, _ in imported_modules("oracle/__init__.py")}
    assert "bit_quantized_frozen_b200" not in mods and "bench" not in mods, mods


def test_input_generators_import_neither_side():
    mods = {m for m, _ in imported_modules("synth_inputs.py")}
    assert not mods & {"oracle", "bit_quantized_frozen_b200"}, mods


def test_oracle_users_outside_the_tests():
    bench = [fn for m, fn in imported_modules("bench.py") if m == "oracle"]
    assert bench == ["cpu_sample"], bench
    entry = [fn for m, fn in imported_modules("__graft_entry__.py") if m == "oracle"]
    assert entry and set(entry) <= {"build", "smoke"}, entry


def test_missing_library_raises():
    code = ("import bit_quantized_frozen_b200 as sq\n"
            "try:\n"
            "    sq.lib()\n"
            "except RuntimeError as e:\n"
            "    print('raised:', e)\n"
            "else:\n"
            "    print('loaded')\n")
    env = dict(os.environ, SQ_LIBSQ_PATH=os.path.join(ROOT, "no_such_dir", "libsq.so"))
    p = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert p.returncode == 0, p.stderr
    assert p.stdout.startswith("raised:") and "libsq.so not found" in p.stdout, p.stdout
