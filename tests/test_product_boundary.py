"""Static checks of the product boundary (CPU only).

The float64 oracle is test infrastructure: the package (Python binding, ring
driver, build script) and the seeded input generators must never import it, and
bench.py may reach it only from its CPU-baseline and reference-arm functions.
Nothing committed may read the scratch folder `_work/`.
"""
import ast
import glob
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "tiled_exact_attention_forward_b200")


def _imports(tree):
    """(module name, enclosing top-level function or None) of every import."""
    out = []

    def visit(node, fn):
        for child in ast.iter_child_nodes(node):
            f = fn
            if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) and fn is None:
                f = child.name
            if isinstance(child, ast.Import):
                out.extend((a.name, f) for a in child.names)
            elif isinstance(child, ast.ImportFrom):
                out.append((child.module or "", f))
            visit(child, f)

    visit(tree, None)
    return out


def _parse(path):
    with open(path) as fh:
        return ast.parse(fh.read(), filename=path)


def test_package_and_input_generators_never_import_the_oracle():
    files = glob.glob(os.path.join(PKG, "*.py")) + [os.path.join(ROOT, "workloads.py")]
    assert len(files) >= 4
    for path in files:
        for mod, _ in _imports(_parse(path)):
            assert not mod.split(".")[0] == "oracle", f"{os.path.relpath(path, ROOT)} imports {mod}"


def test_cuda_sources_do_not_reach_the_oracle():
    for path in glob.glob(os.path.join(PKG, "csrc", "*")):
        with open(path, errors="replace") as fh:
            text = fh.read()
        assert "oracle" not in text.lower(), os.path.relpath(path, ROOT)


def test_bench_uses_the_oracle_only_for_the_cpu_baseline_and_reference_arm():
    uses = [(m, f) for m, f in _imports(_parse(os.path.join(ROOT, "bench.py"))) if m.split(".")[0] == "oracle"]
    assert uses, "the CPU-baseline leg is expected to time the oracle"
    assert {f for _, f in uses} <= {"oracle_sample", "run_reference"}, uses


def test_nothing_committed_reads_the_scratch_folder():
    files = subprocess.run(["git", "ls-files"], cwd=ROOT, capture_output=True, text=True).stdout.split()
    if not files:  # not a git checkout: check the tree instead
        files = [os.path.relpath(p, ROOT) for p in glob.glob(os.path.join(ROOT, "**", "*.py"), recursive=True)]
    for rel in files:
        if rel.startswith("_work/") or not rel.endswith((".py", ".cu", ".cuh", ".h", ".sh", ".toml", ".cfg")):
            continue
        if rel == "tests/test_product_boundary.py":
            continue
        with open(os.path.join(ROOT, rel), errors="replace") as fh:
            assert "_work/" not in fh.read(), rel
