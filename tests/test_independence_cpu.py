"""The oracle and the CUDA path stay apart, and the product path has no CPU fallback.

- nothing in the package (Python, CUDA, headers) imports, loads or includes the oracle;
- the oracle includes nothing of the package or the C ABI;
- bench.py and __graft_entry__.py import the oracle only inside the functions allowed to
  use it: the CPU-baseline and reference legs, build() (which compiles it) and smoke();
- the binding raises when the CUDA library is missing instead of computing anything.
"""
import ast
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "protein_pair_representation_b200")


def _files(top, exts):
    for d, _, names in os.walk(top):
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def test_package_never_touches_the_oracle():
    offenders = []
    for path in _files(PKG, (".py", ".cu", ".cuh", ".h", ".cpp")):
        with open(path) as f:
            text = f.read()
        if "oracle" in text:
            offenders.append(os.path.relpath(path, ROOT))
    assert not offenders, f"the product package mentions the oracle: {offenders}"


def test_oracle_includes_nothing_of_the_package():
    for path in _files(os.path.join(ROOT, "oracle"), (".py", ".c", ".h")):
        with open(path) as f:
            text = f.read()
        for name in ("protein_pair_representation_b200", "trimul.h", "kernels.h", "sm100.cuh", "libtrimul"):
            assert name not in text, f"{os.path.relpath(path, ROOT)} refers to {name}"


# bench.py: the cpu_baseline leg (cpu_oracle_layer_ms, and cpu_oracle_probe run in a child process
# per thread count) and the reference arm
ALLOWED = {"bench.py": {"cpu_oracle_layer_ms", "cpu_oracle_probe", "run_reference"}, "__graft_entry__.py": {"build", "smoke"}}


@pytest.mark.parametrize("name", sorted(ALLOWED))
def test_oracle_imported_only_where_allowed(name):
    with open(os.path.join(ROOT, name)) as f:
        tree = ast.parse(f.read())
    found = set()

    def visit(node, func):
        for child in ast.iter_child_nodes(node):
            here = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else func
            if isinstance(child, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in child.names):
                found.add(func)
            if isinstance(child, ast.ImportFrom) and (child.module or "").split(".")[0] == "oracle":
                found.add(func)
            visit(child, here)

    visit(tree, None)
    assert found, f"{name} is expected to use the oracle somewhere"
    assert found <= ALLOWED[name], f"{name} imports the oracle in {sorted(found - ALLOWED[name])}"


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    from protein_pair_representation_b200 import build, trimul as tm
    monkeypatch.setattr(build, "LIB_PATH", str(tmp_path / "missing" / "libtrimul.so"))
    monkeypatch.setattr(tm, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        tm.load_library()
