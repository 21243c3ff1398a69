"""The oracle and the CUDA path share no code, and the product has no fallback.

- Nothing under cross_loop_sparse_b200/ (the binding, the build script, the
  CUDA sources) imports or includes anything from oracle/ or workload/.
- oracle/ imports nothing from cross_loop_sparse_b200/; its only project
  import is workload/ for the bf16 conversions of the seeded inputs.
- workload/ (the seeded input generators both sides use) imports neither.
- The binding refuses to import when the built library is missing: no CPU
  path stands in for it.
"""
import ast
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _py_imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            if node.level == 0 and node.module:
                names.add(node.module.split(".")[0])
    return names


def _files(sub, exts):
    for dirpath, _dirs, files in os.walk(os.path.join(ROOT, sub)):
        if "__pycache__" in dirpath:
            continue
        for f in files:
            if f.endswith(exts):
                yield os.path.join(dirpath, f)


def test_product_imports_neither_oracle_nor_workload():
    for path in _files("cross_loop_sparse_b200", (".py",)):
        bad = _py_imports(path) & {"oracle", "workload"}
        assert not bad, (path, bad)
    for path in _files("cross_loop_sparse_b200", (".cu", ".cuh", ".h")):
        src = open(path).read()
        assert not re.search(r'#\s*include\s*[<"][^>"]*(oracle|workload)', src), path
    for path in _files("include", (".h",)):
        assert "oracle" not in open(path).read().lower(), path


def test_oracle_and_inputs_do_not_import_the_product():
    for path in _files("oracle", (".py",)):
        imports = _py_imports(path)
        assert "cross_loop_sparse_b200" not in imports, path
        assert imports <= {"__future__", "math", "numpy", "workload", "dataclasses", "typing", "itertools",
                           "functools", "collections"}, (path, imports)
    for path in _files("workload", (".py",)):
        assert not (_py_imports(path) & {"oracle", "cross_loop_sparse_b200"}), path


def test_binding_refuses_to_load_without_the_library(tmp_path):
    """A copy of the package without libflashloop.so must fail at import."""
    pkg = tmp_path / "cross_loop_sparse_b200"
    pkg.mkdir()
    for f in ("__init__.py", "flashloop.py"):
        (pkg / f).write_text(open(os.path.join(ROOT, "cross_loop_sparse_b200", f)).read())
    code = "import cross_loop_sparse_b200.flashloop"
    out = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True, text=True, timeout=300)
    assert out.returncode != 0
    assert "ImportError" in out.stderr and "libflashloop.so is missing" in out.stderr
