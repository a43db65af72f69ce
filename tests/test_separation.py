"""The oracle and the CUDA path share no code: no product module imports the oracle, the
oracle imports nothing of the product, and bench.py reaches the oracle only from its CPU
baseline and reference-arm functions."""
import ast
import glob
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(tree):
    """(top-level module name, enclosing function name or None) of every import."""
    out = []

    def walk(node, fn):
        for child in ast.iter_child_nodes(node):
            f = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else fn
            if isinstance(child, ast.Import):
                out.extend((a.name.split(".")[0], fn) for a in child.names)
            elif isinstance(child, ast.ImportFrom):
                if child.level:                       # relative import inside a package
                    out.append((".", fn))
                else:
                    out.append((child.module.split(".")[0], fn))
            walk(child, f)
    walk(tree, None)
    return out


def _parse(path):
    return ast.parse(open(path).read(), path)


def test_product_never_imports_the_oracle():
    for path in glob.glob(os.path.join(ROOT, "quantized_vit_encoder_b200", "**", "*.py"), recursive=True):
        mods = {m for m, _ in _imports(_parse(path))}
        assert "oracle" not in mods, path
    for path in glob.glob(os.path.join(ROOT, "quantized_vit_encoder_b200", "csrc", "*")):
        assert "oracle" not in open(path).read(), path


def test_oracle_imports_nothing_of_the_product():
    for path in glob.glob(os.path.join(ROOT, "oracle", "*.py")):
        mods = {m for m, _ in _imports(_parse(path))}
        assert "quantized_vit_encoder_b200" not in mods and "bench" not in mods, path


def test_bench_reaches_the_oracle_only_from_its_cpu_legs():
    uses = [fn for m, fn in _imports(_parse(os.path.join(ROOT, "bench.py"))) if m == "oracle"]
    assert uses and set(uses) <= {"cpu_baseline", "run_reference"}, uses
