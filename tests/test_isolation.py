"""The oracle and the CUDA path share no code, and only test code reaches the oracle.

Checked on the sources, nothing imported:

- the package never imports the oracle;
- the oracle imports neither the package nor its input generator;
- the CUDA sources include only their own headers and the public one;
- in bench.py the oracle is imported only by the CPU sampler that serves the CPU-baseline
  and reference legs, and in __graft_entry__.py only by smoke().
"""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "scale_calibration_lh_b200")
CSRC = os.path.join(PKG, "csrc")


def _py_files(d):
    for base, _, files in os.walk(d):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(base, f)


def _imports(path):
    """(imported module, enclosing function name or None) for every import in a file."""
    tree = ast.parse(open(path).read(), filename=path)
    out = []

    def visit(node, fn):
        for child in ast.iter_child_nodes(node):
            if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)):
                visit(child, child.name if fn is None else fn)
                continue
            if isinstance(child, ast.Import):
                out.extend((a.name, fn) for a in child.names)
            elif isinstance(child, ast.ImportFrom):
                out.append(("." * child.level + (child.module or ""), fn))
            visit(child, fn)

    visit(tree, None)
    return out


def _is_oracle(mod):
    return mod == "oracle" or mod.startswith("oracle.") or "lhcal_oracle" in mod


def test_package_never_imports_the_oracle():
    for path in _py_files(PKG):
        assert not [m for m, _ in _imports(path) if _is_oracle(m)], path
        assert "lhcal_oracle" not in open(path).read(), path


def test_oracle_imports_nothing_of_the_cuda_path():
    oracle_dir = os.path.join(ROOT, "oracle")
    for path in _py_files(oracle_dir):
        for mod, _ in _imports(path):
            assert not mod.startswith("scale_calibration_lh_b200"), (path, mod)
            assert "synth" not in mod and not mod.startswith(".."), (path, mod)
    assert not [f for f in os.listdir(oracle_dir) if f.endswith((".cu", ".cuh", ".h", ".so"))]


def test_cuda_sources_include_only_their_own_headers():
    own = set(os.listdir(CSRC)) | set(os.listdir(os.path.join(ROOT, "include")))
    for f in os.listdir(CSRC):
        if not f.endswith((".cu", ".cuh", ".h")):
            continue
        for inc in re.findall(r'#include\s+"([^"]+)"', open(os.path.join(CSRC, f)).read()):
            assert inc in own and "oracle" not in inc, (f, inc)


def test_oracle_reached_only_from_the_cpu_sampler_and_smoke():
    bench = [fn for m, fn in _imports(os.path.join(ROOT, "bench.py")) if _is_oracle(m)]
    assert bench and set(bench) == {"oracle_sample_step"}
    entry = [fn for m, fn in _imports(os.path.join(ROOT, "__graft_entry__.py")) if _is_oracle(m)]
    assert entry and set(entry) == {"smoke"}
