"""The oracle is test infrastructure and the product path never reaches it: the package and its CUDA
sources neither import, include nor load anything under oracle/, the oracle does not use the package,
and bench.py touches the oracle only in its CPU legs (the cpu_baseline sample and the reference arm)."""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_flashattention_b200")


def _files(top, exts):
    for dirpath, _, names in os.walk(top):
        for n in names:
            if n.endswith(exts):
                yield os.path.join(dirpath, n)


def test_package_never_reaches_the_oracle():
    pat = re.compile(r"\boracle\b|sfa_oracle")
    for f in _files(PKG, (".py", ".cu", ".cuh", ".h", ".cpp")):
        for i, line in enumerate(open(f, encoding="utf-8"), 1):
            code = line.split("//")[0] if f.endswith((".cu", ".cuh", ".h", ".cpp")) else line.split("#")[0]
            assert not pat.search(code), f"{os.path.relpath(f, ROOT)}:{i} names the oracle: {line.strip()}"


def test_oracle_does_not_use_the_package():
    """No import of the package, no #include of its sources, no load of its library."""
    bad = re.compile(r"^\s*(import|from)\s+sparse_flashattention_b200|^\s*#\s*include\s*[<\"].*(sfa\.h|sfa_|csrc)"
                     r"|libsfa\.so|dlopen|CDLL\([^)]*libsfa[^_]", re.M)
    for f in _files(os.path.join(ROOT, "oracle"), (".py", ".c", ".h")):
        m = bad.search(open(f, encoding="utf-8").read())
        assert m is None, f"{os.path.relpath(f, ROOT)} uses the package: {m.group(0)}"


def test_bench_uses_the_oracle_only_in_its_cpu_legs():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py"), encoding="utf-8").read())
    allowed = {"cpu_oracle_rate", "main_reference"}
    top_imports = [n for n in tree.body if isinstance(n, (ast.Import, ast.ImportFrom))]
    for n in top_imports:
        names = [a.name for a in n.names] + ([n.module] if isinstance(n, ast.ImportFrom) and n.module else [])
        assert "oracle" not in names, "bench.py imports the oracle at module level"
    for fn in ast.walk(tree):
        if not isinstance(fn, ast.FunctionDef):
            continue
        for n in ast.walk(fn):
            if isinstance(n, ast.Import) and any(a.name == "oracle" for a in n.names):
                assert fn.name in allowed, f"bench.py imports the oracle inside {fn.name}"


def test_binding_fails_loudly_without_the_library():
    src = open(os.path.join(PKG, "__init__.py"), encoding="utf-8").read()
    assert "raise ImportError" in src and "no fallback" in src
