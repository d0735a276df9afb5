"""The oracle and the CUDA path stay independent (static checks, no device).

* No module of the product package or of the shared generators imports the
  oracle; the oracle imports numpy, the standard library and, from the
  generators' module, only the two configuration records.
* bench.py imports the oracle only inside its CPU-baseline functions, and
  __graft_entry__ only inside smoke(); a module-level import would put the
  oracle on the product path.
* The native sources and the public header never mention or include the
  oracle, and the binding raises on a missing library instead of falling back.
"""
import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "token_skipping_sparse_step_b200")


def _py_files(top):
    for dirpath, _, files in os.walk(top):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(dirpath, f)


def _imports(tree):
    """(module name, enclosing function name or None) for every import."""
    out = []

    def visit(node, fn):
        for child in ast.iter_child_nodes(node):
            name = fn
            if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)):
                name = child.name
            if isinstance(child, ast.Import):
                out.extend((a.name.split(".")[0], fn) for a in child.names)
            elif isinstance(child, ast.ImportFrom) and child.module and not child.level:
                out.append((child.module.split(".")[0], fn))
            visit(child, name)

    visit(tree, None)
    return out


def _parse(path):
    with open(path) as f:
        return ast.parse(f.read(), filename=path)


def test_product_and_generators_never_import_the_oracle():
    for top in (PKG, os.path.join(ROOT, "synth")):
        for path in _py_files(top):
            mods = {m for m, _ in _imports(_parse(path))}
            assert "oracle" not in mods, path


def test_oracle_imports_only_numpy_the_standard_library_and_config_types():
    allowed = {"math", "numpy", "dataclasses", "typing", "__future__", "functools", "itertools", "synth"}
    for path in _py_files(os.path.join(ROOT, "oracle")):
        tree = _parse(path)
        mods = {m for m, _ in _imports(tree)}
        assert mods <= allowed, (path, mods - allowed)
        for node in ast.walk(tree):   # from the generators, only the configuration records
            if isinstance(node, ast.ImportFrom) and node.module == "synth":
                assert {a.name for a in node.names} <= {"ModelDims", "RunConfig"}, path


def test_entry_points_import_the_oracle_only_in_their_cpu_legs():
    legs = {"bench.py": {"oracle_sample", "run_reference"}, "__graft_entry__.py": {"smoke"}}
    for name, fns in legs.items():
        for mod, fn in _imports(_parse(os.path.join(ROOT, name))):
            if mod == "oracle":
                assert fn in fns, (name, fn)


def test_native_sources_do_not_reference_the_oracle():
    tops = [os.path.join(PKG, "csrc"), os.path.join(ROOT, "include")]
    for top in tops:
        for dirpath, _, files in os.walk(top):
            for f in files:
                with open(os.path.join(dirpath, f), errors="replace") as fh:
                    assert "oracle" not in fh.read().lower(), f


def test_binding_has_no_fallback():
    with open(os.path.join(PKG, "__init__.py")) as f:
        src = f.read()
    assert "raise ImportError" in src
    for word in ("numpy.linalg", "torch.matmul", "torch.nn.functional", "F.scaled_dot_product_attention"):
        assert word not in src, word
