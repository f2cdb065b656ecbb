"""The oracle and the CUDA library share no code and neither imports the other;
the product package never reaches the oracle."""
import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(path):
    with open(path) as f:
        tree = ast.parse(f.read())
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module:
            names.add(node.module.split(".")[0])
    return names


def _py_files(d):
    for dp, _, fs in os.walk(os.path.join(ROOT, d)):
        for f in fs:
            if f.endswith(".py"):
                yield os.path.join(dp, f)


def test_oracle_does_not_import_the_package():
    for p in _py_files("oracle"):
        assert "paged_kv_cache_438_b200" not in _imports(p), p


def test_package_does_not_import_the_oracle():
    for p in _py_files("paged_kv_cache_438_b200"):
        assert "oracle" not in _imports(p), p
        with open(p) as f:
            src = f.read()
        assert "import oracle" not in src and "from oracle" not in src, p


def test_native_sources_do_not_reference_the_oracle():
    csrc = os.path.join(ROOT, "paged_kv_cache_438_b200", "csrc")
    for dp, _, fs in os.walk(csrc):
        for f in fs:
            with open(os.path.join(dp, f), errors="ignore") as fh:
                assert "oracle" not in fh.read().lower(), f
