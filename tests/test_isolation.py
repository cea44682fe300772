"""The oracle and the CUDA path stay independent: the package and the input generators never
import the oracle, the oracle imports neither of them, and bench.py reaches the oracle only
from its CPU-baseline and reference legs."""
import ast
import glob
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(path):
    """(top-level module name, enclosing function name or None) for every import in a file."""
    tree = ast.parse(open(path).read())
    out = []

    def visit(node, func):
        for child in ast.iter_child_nodes(node):
            f = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else func
            if isinstance(child, ast.Import):
                out.extend((a.name.split(".")[0], func) for a in child.names)
            elif isinstance(child, ast.ImportFrom) and child.level == 0 and child.module:
                out.append((child.module.split(".")[0], func))
            visit(child, f)
    visit(tree, None)
    return out


def _files(*dirs):
    return [p for d in dirs for p in glob.glob(os.path.join(ROOT, d, "**", "*.py"), recursive=True)]


def test_product_and_generators_never_import_the_oracle():
    for p in _files("block_quant_gemv_b200", "synth"):
        assert "oracle" not in [m for m, _ in _imports(p)], p


def test_oracle_imports_neither_the_product_nor_the_generators():
    for p in _files("oracle"):
        mods = [m for m, _ in _imports(p)]
        assert "block_quant_gemv_b200" not in mods and "synth" not in mods, p


def test_bench_reaches_the_oracle_only_from_its_cpu_legs():
    legs = {"oracle_sample", "oracle_moe_sample", "oracle_prefill_sample", "run_reference"}
    for mod, func in _imports(os.path.join(ROOT, "bench.py")):
        if mod == "oracle":
            assert func in legs, f"bench.py imports the oracle in {func}"


def test_kernel_sources_do_not_reference_the_oracle():
    for p in glob.glob(os.path.join(ROOT, "block_quant_gemv_b200", "csrc", "*")) + [os.path.join(ROOT, "include", "bqg.h")]:
        assert "oracle" not in open(p).read().lower(), p
