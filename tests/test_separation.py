"""The oracle and the CUDA path stay apart, and the product path has no fallback.

* No module of the CUDA package imports the oracle, and the oracle imports
  nothing from the package; ``gen`` (seeded inputs and storage formats) imports
  neither.
* ``bench.py`` and the entry points import the oracle only inside the functions
  allowed to run it: the CPU baseline / reference arm and ``smoke()``.
* Without ``libmoe.so`` the package raises instead of computing anything.
"""
import ast
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = "int4_expert_ffn_top_b200"


def _imports(path: str):
    """(top-level module name, qualified enclosing class/function or None) for every import in a file."""
    tree = ast.parse(open(path).read(), path)
    out = []

    def visit(node, fn):
        for child in ast.iter_child_nodes(node):
            f = fn
            if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef, ast.ClassDef)):
                f = f"{fn}.{child.name}" if fn else child.name
            if isinstance(child, ast.Import):
                out.extend((a.name.split(".")[0], fn) for a in child.names)
            elif isinstance(child, ast.ImportFrom):
                if child.level:  # relative: stays inside its own package
                    out.append((".", fn))
                else:
                    out.append((child.module.split(".")[0], fn))
            visit(child, f)

    visit(tree, None)
    return out


def _py_files(d: str):
    for dirpath, _, files in os.walk(os.path.join(ROOT, d)):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(dirpath, f)


def test_package_and_oracle_never_import_each_other():
    for f in _py_files(PKG):
        assert "oracle" not in {m for m, _ in _imports(f)}, f
    for f in _py_files("oracle"):
        assert not {m for m, _ in _imports(f)} & {PKG, "gen", "torch"}, f
    for f in _py_files("gen"):
        assert not {m for m, _ in _imports(f)} & {PKG, "oracle", "torch"}, f


def test_cuda_sources_name_no_oracle_file():
    csrc = os.path.join(ROOT, PKG, "csrc")
    for f in os.listdir(csrc):
        src = open(os.path.join(csrc, f)).read()
        assert "oracle" not in src.lower(), f


def test_oracle_is_imported_only_where_it_may_run():
    allowed = {"bench.py": {"OracleTokenPass.__init__"}, "__graft_entry__.py": {"smoke"}}
    for name, fns in allowed.items():
        uses = [fn for m, fn in _imports(os.path.join(ROOT, name)) if m == "oracle"]
        assert uses, name
        assert all(fn in fns for fn in uses), (name, uses)


def test_missing_library_raises_instead_of_falling_back():
    missing = os.path.join(ROOT, "_build", "no_such_dir", "libmoe.so")
    code = f"import {PKG}._lib as L\ntry:\n    L.load({missing!r})\nexcept RuntimeError as e:\n    print('raised', e)\n"
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.startswith("raised") and "not built" in r.stdout, r.stdout + r.stderr
