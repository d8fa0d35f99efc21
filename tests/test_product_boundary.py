"""The product path and the oracle stay apart.

No module of the package imports the oracle or names its compiled library, and the oracle imports
nothing of the package and includes none of its headers.  bench.py may use the oracle only in its
CPU-baseline and reference legs (functions whose names say so)."""
import ast
from pathlib import Path

ROOT = Path(__file__).resolve().parents[1]
PKG = ROOT / "entmax_tcgen05_tma_b200"


def _imports(path: Path):
    tree = ast.parse(path.read_text())
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield node, a.name
        elif isinstance(node, ast.ImportFrom):
            yield node, node.module or ""


def test_package_never_imports_the_oracle():
    for f in sorted(PKG.rglob("*.py")):
        for _, name in _imports(f):
            assert not name.split(".")[0] == "oracle", (f, name)
        assert "entmax_oracle" not in f.read_text(), f


def test_package_sources_do_not_name_the_oracle_library():
    for f in sorted((PKG / "csrc").glob("*")):
        assert "entmax_oracle" not in f.read_text(), f


def test_bench_uses_the_oracle_only_in_its_baseline_legs():
    tree = ast.parse((ROOT / "bench.py").read_text())
    users = set()
    for fn in ast.walk(tree):
        if isinstance(fn, (ast.FunctionDef, ast.AsyncFunctionDef)):
            for node in ast.walk(fn):
                if isinstance(node, (ast.Import, ast.ImportFrom)):
                    mods = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module or ""]
                    if any(m.split(".")[0] == "oracle" for m in mods):
                        users.add(fn.name)
    top = [n for n in tree.body if isinstance(n, (ast.Import, ast.ImportFrom))]
    for node in top:
        mods = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module or ""]
        assert not any(m.split(".")[0] == "oracle" for m in mods), "module-level oracle import in bench.py"
    assert users and users <= {"oracle_baseline", "run_reference"}, users


def test_oracle_never_imports_the_package():
    for f in sorted((ROOT / "oracle").glob("*.py")):
        for _, name in _imports(f):
            assert name.split(".")[0] != "entmax_tcgen05_tma_b200", (f, name)
    for f in sorted((ROOT / "oracle").glob("*.c")):
        text = f.read_text()
        for line in text.splitlines():
            if line.startswith("#include"):
                assert "<" in line and "entmax_attn" not in line, (f, line)
