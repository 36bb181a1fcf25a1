"""The oracle and the CUDA path share no code: no source of one includes or imports the other,
and the package never touches the oracle.  Only the seeded generators (synth/) serve both."""
import ast
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "attention_frame_decode_b200")


def _includes(path):
    return re.findall(r'^\s*#\s*include\s*[<"]([^>"]+)[>"]', open(path).read(), flags=re.M)


def _imports(path):
    tree = ast.parse(open(path).read())
    mods = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            mods.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module:
            mods.add(node.module.split(".")[0])
    return mods


def test_oracle_sources_include_nothing_of_the_cuda_path():
    for path in glob.glob(os.path.join(ROOT, "oracle", "*.[ch]")):
        for inc in _includes(path):
            assert not re.search(r"vc\.h|csrc|attention_frame_decode_b200|\.cuh", inc), (path, inc)
    assert _imports(os.path.join(ROOT, "oracle", "__init__.py")).isdisjoint({"attention_frame_decode_b200"})


def test_cuda_sources_include_nothing_of_the_oracle():
    paths = glob.glob(os.path.join(PKG, "csrc", "*.cu")) + glob.glob(os.path.join(PKG, "csrc", "*.cuh"))
    paths.append(os.path.join(ROOT, "include", "vc.h"))
    assert len(paths) > 10
    for path in paths:
        for inc in _includes(path):
            assert "oracle" not in inc and "synth" not in inc, (path, inc)


def test_package_never_imports_the_oracle():
    for path in glob.glob(os.path.join(PKG, "*.py")):
        assert "oracle" not in _imports(path), path
