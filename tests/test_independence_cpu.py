"""The oracle and the CUDA path share no code: the product package never
imports, includes or loads anything of the oracle, the oracle never refers
to the product's sources, and the seeded input module imports neither.
bench.py may use the oracle only inside its CPU-baseline and reference-arm
functions (never at module level), and __graft_entry__ only in build() and
smoke()."""
import ast
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_discrete_diffusion_dd_b200")


def _imports(path):
    """(module names imported at top level, {function: imported names})."""
    tree = ast.parse(open(path).read())
    top, inner = set(), {}

    def names(node):
        if isinstance(node, ast.Import):
            return {a.name.split(".")[0] for a in node.names}
        if isinstance(node, ast.ImportFrom) and node.module:
            return {node.module.split(".")[0]}
        return set()

    for node in tree.body:
        top |= names(node)
    for node in ast.walk(tree):
        if isinstance(node, ast.FunctionDef):
            got = set()
            for sub in ast.walk(node):
                got |= names(sub)
            inner[node.name] = got
    return top, inner


def test_package_never_reaches_the_oracle():
    for path in glob.glob(os.path.join(PKG, "**", "*.py"), recursive=True):
        top, inner = _imports(path)
        assert "oracle" not in top, path
        assert all("oracle" not in v for v in inner.values()), path
    for path in glob.glob(os.path.join(PKG, "csrc", "*")):
        text = open(path, errors="replace").read()
        assert not re.search(r'#include\s*[<"][^>"]*oracle', text), path
        assert "liboracle" not in text, path


def test_oracle_never_reaches_the_package():
    for path in glob.glob(os.path.join(ROOT, "oracle", "*.c")):
        text = open(path).read()
        includes = re.findall(r'#include\s*[<"]([^>"]+)[>"]', text)
        assert all(not i.startswith("dd") for i in includes), (path, includes)
    top, inner = _imports(os.path.join(ROOT, "oracle", "__init__.py"))
    allowed = {"__future__", "ctypes", "os", "subprocess", "numpy", "torch"}
    used = top.union(*inner.values())
    assert used <= allowed, used - allowed


def test_input_module_imports_neither():
    top, inner = _imports(os.path.join(ROOT, "workloads", "__init__.py"))
    used = top.union(*inner.values())
    assert "oracle" not in used and "block_discrete_diffusion_dd_b200" not in used


def test_bench_and_entry_use_the_oracle_only_where_allowed():
    top, inner = _imports(os.path.join(ROOT, "bench.py"))
    assert "oracle" not in top
    users = {f for f, v in inner.items() if "oracle" in v}
    # the two CPU legs and the timed sample they share
    assert users <= {"cpu_baseline", "run_reference", "_oracle_sample"}, users
    top, inner = _imports(os.path.join(ROOT, "__graft_entry__.py"))
    assert "oracle" not in top
    users = {f for f, v in inner.items() if "oracle" in v}
    assert users <= {"build", "smoke"}, users
