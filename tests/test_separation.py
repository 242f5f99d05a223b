"""The CUDA product path and the fp64 oracle stay independent: the package
never imports the oracle (or any CPU fallback), the oracle never imports the
package, and the binding fails loudly when the compiled library is missing."""
import ast
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            names.add(node.module.split(".")[0])
    return names


def _py_files(sub):
    for dirpath, _, files in os.walk(os.path.join(ROOT, sub)):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(dirpath, f)


def test_package_does_not_import_the_oracle():
    for path in _py_files("draft_model_b200"):
        assert "oracle" not in _imports(path), path


def test_oracle_does_not_import_the_package():
    for path in _py_files("oracle"):
        assert not ({"draft_model_b200", "synth"} & _imports(path)), path


def test_cuda_sources_do_not_reach_into_the_oracle():
    for dirpath, _, files in os.walk(os.path.join(ROOT, "draft_model_b200", "csrc")):
        for f in files:
            text = open(os.path.join(dirpath, f), encoding="utf-8").read()
            assert "oracle" not in text.lower(), f


def test_bench_reaches_the_oracle_only_in_its_cpu_legs():
    """bench.py imports the oracle only inside the CPU-baseline and reference
    helpers, and nothing from tests/ (whose harness imports the oracle)."""
    path = os.path.join(ROOT, "bench.py")
    tree = ast.parse(open(path).read(), filename=path)
    allowed = {"oracle_block_rate", "OracleFraction"}
    for node in tree.body:
        name = getattr(node, "name", None)
        sub = ast.Module(body=[node], type_ignores=[])
        found = set()
        for n in ast.walk(sub):
            if isinstance(n, ast.Import):
                found.update(a.name.split(".")[0] for a in n.names)
            elif isinstance(n, ast.ImportFrom) and n.module:
                found.add(n.module.split(".")[0])
        assert "_harness" not in found, name
        if "oracle" in found:
            assert name in allowed, f"bench.py imports the oracle in {name!r}"
    assert "\"tests\"" not in open(path).read()


def test_missing_library_raises(monkeypatch):
    from draft_model_b200 import _binding
    monkeypatch.setattr(_binding, "_lib", None)
    monkeypatch.setattr(_binding, "_LIB_PATH", os.path.join(ROOT, "no_such_libdomino.so"))
    with pytest.raises(RuntimeError):
        _binding.load_library()
