"""CPU checks of two structural rules of this repository.

1. The product (the package grouped_gemm_route_b200: its Python modules and
   its CUDA sources) never imports, includes, links or loads anything under
   oracle/, and the oracle never imports the package: the two share only the
   seeded input generator, which holds none of the layer's arithmetic.
2. The oracle is reached only from tests/, __graft_entry__ and bench.py's
   CPU-baseline / reference-arm functions.
"""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "grouped_gemm_route_b200")


def _py_imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    names = []
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names += [a.name for a in node.names]
        elif isinstance(node, ast.ImportFrom):
            mod = node.module or ""
            names += [mod] + [f"{mod}.{a.name}" for a in node.names]
    return names


def _files(top, exts):
    for d, _, fs in os.walk(top):
        for f in fs:
            if f.endswith(exts):
                yield os.path.join(d, f)


def test_package_python_never_imports_the_oracle():
    for path in _files(PKG, (".py",)):
        for name in _py_imports(path):
            assert not name.startswith("oracle") and "moe_oracle" not in name, (path, name)


def test_cuda_sources_never_include_or_load_the_oracle():
    for path in _files(PKG, (".cu", ".cuh", ".h", ".cpp")):
        src = open(path).read()
        assert not re.search(r'#\s*include\s*[<"][^>"]*oracle', src), path
        assert "libmoe_oracle" not in src and "moe_oracle" not in src, path


def test_oracle_never_imports_the_package():
    for path in _files(os.path.join(ROOT, "oracle"), (".py",)):
        for name in _py_imports(path):
            assert not name.startswith("grouped_gemm_route_b200"), (path, name)
    for path in _files(os.path.join(ROOT, "oracle"), (".cpp", ".h", ".hpp", ".cu", ".cuh")):
        src = open(path).read()
        assert "grouped_gemm_route_b200" not in src and "moe.h" not in src, path


def test_bench_reaches_the_oracle_only_from_its_baseline_functions():
    path = os.path.join(ROOT, "bench.py")
    tree = ast.parse(open(path).read(), filename=path)
    allowed = {"time_oracle_step", "oracle_threads"}  # called by cpu_baseline and run_reference only
    for fn in [n for n in ast.walk(tree) if isinstance(n, ast.FunctionDef)]:
        for node in ast.walk(fn):
            if isinstance(node, ast.ImportFrom) and (node.module or "").startswith("oracle"):
                assert fn.name in allowed, (fn.name, node.module)
    callers = {fn.name for fn in ast.walk(tree) if isinstance(fn, ast.FunctionDef)
               for node in ast.walk(fn) if isinstance(node, ast.Call) and isinstance(node.func, ast.Name)
               and node.func.id in allowed}
    assert callers <= allowed | {"cpu_baseline", "run_reference"}, callers
    top = [n for n in tree.body if isinstance(n, (ast.Import, ast.ImportFrom))]
    for node in top:  # nothing at module level
        mods = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module or ""]
        assert not any(m.startswith("oracle") for m in mods)
