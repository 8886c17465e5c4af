"""The oracle and the CUDA path share no code, and the product path never reaches the oracle.

Checked on the source text, without a GPU:
* nothing in the package (Python binding, build script, CUDA sources and headers) imports,
  includes or names a file of ``oracle/``;
* the oracle imports only the standard library and numpy (not the package, not its inputs);
* in ``bench.py`` only the CPU-oracle arms (functions named ``oracle_*``) import the oracle,
  and the GPU timing functions call none of them;
* the package's input generator, the one module both sides start from, holds no step of the
  method (no softmax, top-k or attention arithmetic).
"""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "long_context_sparse_hs2_b200")


def _files(top, exts):
    for d, _, names in os.walk(top):
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def test_package_never_names_the_oracle():
    hits = []
    for p in _files(PKG, (".py", ".cu", ".cuh", ".h", ".c", ".cpp")):
        text = open(p, encoding="utf-8").read()
        for pat in (r"^\s*(from|import)\s+oracle\b", r"#\s*include\s*[<\"][^>\"]*oracle", r"hs2_oracle"):
            if re.search(pat, text, re.M):
                hits.append((os.path.relpath(p, ROOT), pat))
    assert not hits, hits


def _imported_modules(tree):
    mods = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            mods |= {a.name.split(".")[0] for a in node.names}
        elif isinstance(node, ast.ImportFrom) and node.level == 0:
            mods.add(node.module.split(".")[0])
    return mods


def test_oracle_imports_only_numpy_and_the_standard_library():
    allowed = {"numpy", "math", "dataclasses", "typing", "__future__"}
    for p in _files(os.path.join(ROOT, "oracle"), (".py",)):
        mods = _imported_modules(ast.parse(open(p).read()))
        assert mods <= allowed, (p, mods - allowed)


def _functions(tree):
    return {n.name: n for n in ast.walk(tree) if isinstance(n, ast.FunctionDef)}


def test_bench_reaches_the_oracle_only_in_its_cpu_arms():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    funcs = _functions(tree)
    # module-level imports of the oracle would load it for every run
    top = [n for n in tree.body if isinstance(n, (ast.Import, ast.ImportFrom))]
    assert "oracle" not in _imported_modules(ast.Module(body=top, type_ignores=[]))
    importers = {name for name, f in funcs.items() if "oracle" in _imported_modules(f)}
    assert importers and all(name.startswith("oracle_") for name in importers), importers

    # the GPU measurement (run_gpu: warm-up, timed steps, end-to-end copies) and every bench
    # function it calls reach no oracle arm
    def calls(f):
        return {c.func.id for c in ast.walk(f) if isinstance(c, ast.Call) and isinstance(c.func, ast.Name)}

    seen, todo = set(), ["run_gpu"]
    while todo:
        name = todo.pop()
        if name in seen or name not in funcs:
            continue
        seen.add(name)
        todo += list(calls(funcs[name]))
    assert "run_gpu" in seen and not (seen & {n for n in funcs if n.startswith("oracle_")}), seen


def _code_only(path):
    """The module's syntax tree with every docstring and other bare string expression dropped."""
    tree = ast.parse(open(path).read())
    for node in ast.walk(tree):
        body = getattr(node, "body", None)
        if isinstance(body, list):
            node.body = [b for b in body if not (isinstance(b, ast.Expr) and isinstance(b.value, ast.Constant)
                                                 and isinstance(b.value.value, str))] or [ast.Pass()]
    return tree


def test_input_generator_holds_no_step_of_the_method():
    tree = _code_only(os.path.join(PKG, "inputs.py"))
    names = {n.id for n in ast.walk(tree) if isinstance(n, ast.Name)}
    names |= {n.attr for n in ast.walk(tree) if isinstance(n, ast.Attribute)}
    names |= {n.name for n in ast.walk(tree) if isinstance(n, ast.FunctionDef)}
    banned = ("softmax", "logsumexp", "argpartition", "topk", "lse", "attend", "sdpa", "scaled_dot")
    assert not [n for n in names if any(b in n.lower() for b in banned)]
    # no matrix products: the generator draws numbers, it does not contract them
    assert not [n for n in ast.walk(tree) if isinstance(n, ast.BinOp) and isinstance(n.op, ast.MatMult)]
    assert not ({"matmul", "einsum", "dot", "tensordot", "bmm", "mm"} & names)
