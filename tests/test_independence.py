"""The CUDA path and the oracle share no code.

The product package never imports the oracle (and importing it loads no oracle module); the
CUDA / C sources of the product never include the oracle's, nor the oracle the product's; the
oracle imports nothing from the product; the one module both sides use, the seeded input
generator, holds none of the method's arithmetic.
"""
import ast
import glob
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "global_attention_sink_softmax_b200")


def imported_modules(path):
    tree = ast.parse(open(path).read())
    mods = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            mods.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            if node.level:  # relative import inside the package
                mods.add("." + (node.module or ""))
            elif node.module:
                mods.add(node.module.split(".")[0])
    return mods


def test_product_python_never_imports_the_oracle():
    for path in glob.glob(os.path.join(PKG, "*.py")):
        assert "oracle" not in imported_modules(path), path


def test_oracle_imports_nothing_from_the_product():
    for path in glob.glob(os.path.join(ROOT, "oracle", "*.py")):
        mods = imported_modules(path)
        assert "global_attention_sink_softmax_b200" not in mods, path


def includes(path):
    return re.findall(r'^\s*#\s*include\s*[<"]([^>"]+)[>"]', open(path).read(), flags=re.M)


def test_sources_include_nothing_across_the_line():
    product = glob.glob(os.path.join(PKG, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*"))
    oracle_files = {os.path.basename(p) for p in glob.glob(os.path.join(ROOT, "oracle", "*"))}
    product_files = {os.path.basename(p) for p in product}
    for path in product:
        for inc in includes(path):
            assert os.path.basename(inc) not in oracle_files and "oracle" not in inc, (path, inc)
    for path in glob.glob(os.path.join(ROOT, "oracle", "*.c")):
        for inc in includes(path):
            assert os.path.basename(inc) not in product_files, (path, inc)
            assert inc in {"math.h", "stdint.h", "stdlib.h", "string.h"}, (path, inc)


def test_importing_the_package_loads_no_oracle():
    code = ("import sys, global_attention_sink_softmax_b200 as sa; "
            "assert 'oracle' not in sys.modules, sorted(m for m in sys.modules if 'oracle' in m)")
    subprocess.run([sys.executable, "-c", code], cwd=ROOT, check=True)


def test_input_generator_holds_no_attention_arithmetic():
    path = os.path.join(PKG, "workloads.py")
    mods = imported_modules(path)
    assert mods <= {"math", "dataclasses", "typing", "torch", "__future__"}, mods
    # no call of the method's operations and no matrix product in its code (prose may name them)
    forbidden = {"softmax", "log_softmax", "logsumexp", "exp", "exp2", "log", "matmul", "mm", "bmm",
                 "einsum", "sin", "cos", "scaled_dot_product_attention"}
    tree = ast.parse(open(path).read())
    for node in ast.walk(tree):
        if isinstance(node, ast.Call):
            f = node.func
            name = f.attr if isinstance(f, ast.Attribute) else getattr(f, "id", None)
            assert name not in forbidden, (name, node.lineno)
        assert not (isinstance(node, ast.BinOp) and isinstance(node.op, ast.MatMult)), node.lineno
