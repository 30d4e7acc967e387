"""The oracle stays test infrastructure: nothing in the library package imports it or shares
code with it, the library has no CPU path for the kernels' work, and bench.py reaches it only
from its CPU-baseline / reference function.  Static checks over the sources."""
import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "mixed_format_paged_mkv_b200")


def imported_modules(path):
    tree = ast.parse(open(path).read())
    out = []
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            out += [(a.name, node) for a in node.names]
        elif isinstance(node, ast.ImportFrom) and node.module:
            out.append((node.module, node))
    return tree, out


def test_library_package_never_imports_the_oracle():
    for name in os.listdir(PKG):
        if name.endswith(".py"):
            _, mods = imported_modules(os.path.join(PKG, name))
            assert not any(m.split(".")[0] == "oracle" for m, _ in mods), name


def test_native_sources_do_not_reference_the_oracle():
    for d in (os.path.join(PKG, "csrc"), os.path.join(ROOT, "include")):
        for name in os.listdir(d):
            text = open(os.path.join(d, name), errors="replace").read()
            assert "oracle" not in text.lower(), name


def test_oracle_does_not_import_the_library():
    odir = os.path.join(ROOT, "oracle")
    for name in os.listdir(odir):
        if name.endswith(".py"):
            _, mods = imported_modules(os.path.join(odir, name))
            assert not any(m.startswith("mixed_format_paged_mkv_b200") for m, _ in mods), name
            head = open(os.path.join(odir, name)).read(2000)
            if name != "__init__.py":
                assert "test infrastructure" in head, name


def test_bench_reaches_the_oracle_only_from_its_baseline_function():
    tree, mods = imported_modules(os.path.join(ROOT, "bench.py"))
    funcs = [n for n in ast.walk(tree) if isinstance(n, ast.FunctionDef)]
    for m, node in mods:
        if m.split(".")[0] != "oracle":
            continue
        owner = [f.name for f in funcs if f.lineno <= node.lineno <= f.end_lineno]
        assert owner == ["oracle_sample"], owner
    calls = [f.name for f in funcs
             for n in ast.walk(f) if isinstance(n, ast.Call)
             and getattr(n.func, "id", None) == "oracle_sample"]
    assert sorted(set(calls)) == ["run_gpu", "run_reference"]


def test_binding_fails_loudly_without_the_library(tmp_path, monkeypatch):
    from mixed_format_paged_mkv_b200 import api
    monkeypatch.setattr(api, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(api, "_lib", None)
    try:
        api.lib()
    except RuntimeError as e:
        assert "not built" in str(e)
    else:
        raise AssertionError("the binding loaded without its library")
