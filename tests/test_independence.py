"""The oracle and the CUDA path share no code: nothing under oracle/ imports the
package or loads its library, and the package never imports the oracle (only
tests, __graft_entry__.smoke() and bench.py's CPU legs may).  Checked on the
import statements of every source file, so it needs no GPU."""
import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.level == 0 and node.module:
            names.add(node.module.split(".")[0])
    return names


def _py_files(d):
    for base, _, files in os.walk(os.path.join(ROOT, d)):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(base, f)


def test_oracle_does_not_use_the_cuda_path():
    files = list(_py_files("oracle"))
    assert files
    for f in files:
        assert "sparse_linear_layers_b200" not in _imports(f), f
        text = open(f).read()
        assert "libsbl" not in text and "ctypes" not in text, f


def test_package_does_not_use_the_oracle():
    files = list(_py_files("sparse_linear_layers_b200"))
    assert files
    for f in files:
        assert "oracle" not in _imports(f), f


def test_kernel_sources_do_not_include_the_oracle():
    csrc = os.path.join(ROOT, "sparse_linear_layers_b200", "csrc")
    for f in os.listdir(csrc):
        if f.endswith((".cu", ".cuh", ".h")):
            for line in open(os.path.join(csrc, f)):
                assert not (line.lstrip().startswith("#include") and "oracle" in line), (f, line)
