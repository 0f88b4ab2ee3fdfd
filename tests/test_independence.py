"""The oracle and the CUDA path share no code (checked on the sources, CPU only).

- Nothing under oracle/ imports the library package or the device-side input
  helper.
- Nothing in the package (binding, build script, CUDA sources) refers to the
  oracle.
- The seeded input generators (csa_synth, apart from its device upload
  helper) import neither side.
- In bench.py the oracle is imported only by the CPU legs: the oracle
  baseline and the reference arm.
"""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = "indexer_selected_sparse_csa2_b200"


def _imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    out = []
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            out += [(a.name, node) for a in node.names]
        elif isinstance(node, ast.ImportFrom):
            mod = node.module or ""
            if node.level:                                  # relative import inside a package
                mod = "." + mod
            out.append((mod, node))
    return out, tree


def _py_files(d):
    for dp, _, fs in os.walk(os.path.join(ROOT, d)):
        for f in fs:
            if f.endswith(".py"):
                yield os.path.join(dp, f)


def test_oracle_imports_neither_the_library_nor_the_device_helper():
    for path in _py_files("oracle"):
        for mod, _ in _imports(path)[0]:
            assert not mod.startswith(PKG), (path, mod)
            assert mod != "csa_synth.device", (path, mod)


def test_library_never_refers_to_the_oracle():
    pkg = os.path.join(ROOT, PKG)
    for dp, _, fs in os.walk(pkg):
        for f in fs:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dp, f)).read()
                assert not re.search(r"\boracle\b", txt), os.path.join(dp, f)
    for path in _py_files(PKG):
        for mod, _ in _imports(path)[0]:
            assert not mod.startswith("oracle"), (path, mod)


def test_input_generators_import_neither_side():
    for path in _py_files("csa_synth"):
        if path.endswith(os.path.join("csa_synth", "device.py")):
            continue                                        # uploads through the library by design
        for mod, _ in _imports(path)[0]:
            assert not mod.startswith("oracle") and not mod.startswith(PKG), (path, mod)


def test_bench_imports_the_oracle_only_in_its_cpu_legs():
    path = os.path.join(ROOT, "bench.py")
    _, tree = _imports(path)
    allowed = {"_oracle_case", "_time_oracle", "run_reference", "cpu_baseline"}
    for fn in ast.walk(tree):
        if not isinstance(fn, ast.FunctionDef):
            continue
        for node in ast.walk(fn):
            mods = []
            if isinstance(node, ast.Import):
                mods = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                mods = [node.module or ""]
            if any(m.startswith("oracle") for m in mods):
                assert fn.name in allowed, (fn.name, mods)
    for node in tree.body:                                  # and not at module level
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            mods = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module or ""]
            assert not any(m.startswith("oracle") for m in mods)
