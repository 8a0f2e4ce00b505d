"""The product path never touches the oracle, and the oracle never touches the product path.

The package (library binding, inputs, device plumbing, parallel exchanges) must not import or read
anything under oracle/, and the oracle must not import the package's compute (it may share only the
seeded input generators, which hold none of the method's arithmetic)."""

import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            names.add(("." * node.level) + (node.module or ""))
            names.update(("." * node.level) + (node.module or "") + "." + a.name for a in node.names)
    return names


def _py_files(d):
    for root, _, files in os.walk(os.path.join(ROOT, d)):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(root, f)


def test_package_does_not_import_the_oracle():
    for path in _py_files("grouped_nf4_expert_b200"):
        bad = [n for n in _imports(path) if n.split(".")[0] == "oracle" or ".oracle" in n]
        assert not bad, (path, bad)
        assert "oracle/" not in open(path).read(), path


def test_oracle_uses_no_package_compute():
    allowed = {"inputs"}  # seeded draws only
    for path in _py_files("oracle"):
        for n in _imports(path):
            if n.startswith("grouped_nf4_expert_b200"):
                assert n.split(".")[-1] in allowed, (path, n)


def test_native_sources_do_not_reference_the_oracle():
    csrc = os.path.join(ROOT, "grouped_nf4_expert_b200", "csrc")
    for f in os.listdir(csrc):
        if f.endswith((".cu", ".cuh", ".h", ".cpp")):
            assert "oracle" not in open(os.path.join(csrc, f)).read().lower(), f
