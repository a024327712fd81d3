"""The oracle and the CUDA path stay apart (static checks on the sources).

- Nothing in the product package (the binding, the build script, the input
  generators) imports the oracle, and no kernel source or public header
  includes anything of it.
- The oracle imports nothing of the product package and includes no kernel
  header: the two share no code.
- bench.py imports the oracle only in its CPU-baseline leg and in the
  reference arm (`cpu_baseline`, `reference`, and the cpu_baseline entry of
  `ours`)."""
import ast
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
PKG = os.path.join(ROOT, "fp8_block_scaled_10_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _imported_modules(tree):
    """(top-level module name, enclosing function name or None) per import."""
    out = []

    def visit(node, func):
        for child in ast.iter_child_nodes(node):
            f = func
            if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)):
                f = child.name if func is None else func
            if isinstance(child, ast.Import):
                out.extend((a.name.split(".")[0], f) for a in child.names)
            elif isinstance(child, ast.ImportFrom):
                if child.level == 0 and child.module:
                    out.append((child.module.split(".")[0], f))
            visit(child, f)

    visit(tree, None)
    return out


def _py_files(folder):
    return [os.path.join(folder, f) for f in sorted(os.listdir(folder)) if f.endswith(".py")]


def _c_includes(path):
    return re.findall(r'^\s*#\s*include\s*[<"]([^>"]+)[>"]', open(path).read(), re.M)


def test_product_package_never_imports_the_oracle():
    for path in _py_files(PKG):
        mods = {m for m, _ in _imported_modules(ast.parse(open(path).read()))}
        assert "oracle" not in mods, path


def test_kernel_sources_include_nothing_of_the_oracle():
    csrc = os.path.join(PKG, "csrc")
    srcs = [os.path.join(csrc, f) for f in os.listdir(csrc)] + \
        [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))]
    for path in srcs:
        for inc in _c_includes(path):
            assert "oracle" not in inc, (path, inc)


def test_oracle_shares_no_code_with_the_product():
    for path in _py_files(ORACLE):
        mods = {m for m, _ in _imported_modules(ast.parse(open(path).read()))}
        assert "fp8_block_scaled_10_b200" not in mods, path
    for name in os.listdir(ORACLE):
        if name.endswith((".c", ".h")):
            for inc in _c_includes(os.path.join(ORACLE, name)):
                assert not inc.endswith((".cuh", "fp8bs.h")) and "csrc" not in inc, (name, inc)


def test_bench_imports_the_oracle_only_in_its_cpu_legs():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    where = {f for m, f in _imported_modules(tree) if m == "oracle"}
    assert where and where <= {"cpu_baseline", "reference", "ours"}, where
    # inside `ours` the oracle itself runs only through cpu_baseline(); the
    # function reads nothing from the module but its thread count
    ours = next(n for n in tree.body if isinstance(n, ast.FunctionDef) and n.name == "ours")
    used = {n.attr for n in ast.walk(ours)
            if isinstance(n, ast.Attribute) and isinstance(n.value, ast.Name)
            and n.value.id == "oracle"}
    assert used <= {"num_threads"}, used
