"""The oracle and the product stay independent (CPU only, static checks).

  * Nothing in the package fp8_moe_expert_top_b200/ imports the oracle, and
    the oracle imports nothing but numpy and the standard library (in
    particular neither the package nor torch).
  * bench.py reaches the oracle only from its CPU-baseline / reference
    functions, and __graft_entry__.py only from smoke(); neither imports it at
    module level.
  * The seeded input generators (inputs.py), the one module both sides use,
    import neither side.
  * No committed source refers to the scratch folder or to the source pages'
    directory.
"""

import ast
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "fp8_moe_expert_top_b200")


def _imports(path):
    """(module name, enclosing function name or None) of every import in a file."""
    tree = ast.parse(open(path).read(), filename=path)
    out = []

    def visit(node, func):
        for child in ast.iter_child_nodes(node):
            f = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else func
            if isinstance(child, ast.Import):
                out.extend((a.name, func) for a in child.names)
            elif isinstance(child, ast.ImportFrom):
                mod = ("." * child.level) + (child.module or "")
                out.append((mod, func))
            visit(child, f)

    visit(tree, None)
    return out


def _py_files(folder):
    for dirpath, _, files in os.walk(folder):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(dirpath, f)


def test_package_never_imports_the_oracle():
    for path in _py_files(PKG):
        for mod, _ in _imports(path):
            assert not mod.split(".")[0] == "oracle", (path, mod)


def test_oracle_imports_only_numpy_and_the_standard_library():
    allowed = {"numpy", "math", "fractions"}
    for path in _py_files(os.path.join(ROOT, "oracle")):
        for mod, _ in _imports(path):
            if mod.startswith("."):
                continue                       # its own modules
            assert mod.split(".")[0] in allowed, (path, mod)


def test_inputs_module_imports_neither_side():
    for mod, _ in _imports(os.path.join(PKG, "inputs.py")):
        assert not mod.startswith("."), mod                # no sibling module of the package
        assert mod.split(".")[0] not in ("oracle", "fp8_moe_expert_top_b200"), mod


@pytest.mark.parametrize("fname,allowed", [
    ("bench.py", {"_oracle_quantize", "oracle_sample", "time_oracle"}),
    ("__graft_entry__.py", {"smoke"}),
])
def test_entry_points_reach_the_oracle_only_where_allowed(fname, allowed):
    uses = [(mod, func) for mod, func in _imports(os.path.join(ROOT, fname)) if mod.split(".")[0] == "oracle"]
    assert uses, f"{fname} is expected to use the oracle in {sorted(allowed)}"
    for mod, func in uses:
        assert func in allowed, (fname, mod, func)


def test_no_committed_source_refers_to_scratch_or_the_pages():
    files = subprocess.run(["git", "ls-files"], cwd=ROOT, capture_output=True, text=True).stdout.split()
    if not files:
        pytest.skip("not a git checkout")
    src = [f for f in files if f.endswith((".py", ".cu", ".cuh", ".h", ".c", ".ini"))]
    assert src
    scratch = "_" + "work/"                      # spelled in two parts so this file does not match itself
    pages = "/root/" + "reference"
    for f in src:
        text = open(os.path.join(ROOT, f)).read()
        assert scratch not in text, f
        assert pages not in text, f


def test_importing_the_package_does_not_load_the_oracle():
    code = ("import sys; import fp8_moe_expert_top_b200.layer, fp8_moe_expert_top_b200.binding, "
            "fp8_moe_expert_top_b200.inputs; print(any(m == 'oracle' or m.startswith('oracle.') for m in sys.modules))")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == "False"
