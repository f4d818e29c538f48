"""Host-side guarantees of the product path (no GPU): it never reaches the
oracle, it fails loudly without its library, and bench.py reports the ncu
traffic of a kernel only while the kernel is the one that was profiled."""
import ast
import os

import pytest

from conftest import ROOT
from speculative_decoding_draft_sample_b200 import binding as bn

PKG = os.path.join(ROOT, "speculative_decoding_draft_sample_b200")


def imported_modules(path):
    tree = ast.parse(open(path).read(), filename=path)
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name, node
        elif isinstance(node, ast.ImportFrom):
            yield (node.module or ""), node


def test_the_package_never_imports_the_oracle():
    for name in sorted(os.listdir(PKG)):
        if name.endswith(".py"):
            for mod, _ in imported_modules(os.path.join(PKG, name)):
                assert not mod.split(".")[0] == "oracle", f"{name} imports {mod}"


def test_bench_imports_the_oracle_only_in_its_cpu_legs():
    """bench.py may run the oracle only for the CPU baseline and the reference arm."""
    path = os.path.join(ROOT, "bench.py")
    tree = ast.parse(open(path).read())
    allowed = {"cpu_baseline", "reference_arm"}
    for fn in ast.walk(tree):
        if isinstance(fn, ast.FunctionDef):
            for node in ast.walk(fn):
                mod = None
                if isinstance(node, ast.ImportFrom):
                    mod = node.module or ""
                elif isinstance(node, ast.Import):
                    mod = node.names[0].name
                if mod is not None and mod.split(".")[0] == "oracle":
                    assert fn.name in allowed, f"bench.py:{fn.name} imports {mod}"
    for node in tree.body:  # nothing at module level
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            mod = node.module if isinstance(node, ast.ImportFrom) else node.names[0].name
            assert (mod or "").split(".")[0] != "oracle"


def test_missing_library_raises(monkeypatch, tmp_path):
    monkeypatch.setattr(bn, "LIB_PATH", str(tmp_path / "libdspark.so"))
    monkeypatch.setattr(bn, "_lib", None)
    with pytest.raises(bn.DSparkError, match="missing"):
        bn.lib()
    with pytest.raises(bn.DSparkError, match="missing"):
        bn.version()


def test_profiled_traffic_follows_the_kernel_sources(monkeypatch, tmp_path):
    import bench
    files = bench.DRAFT_KERNEL_SOURCES
    sha = bench.sources_sha256(files)
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "k.txt").write_text(f"source_sha256: {sha}\ndram_bytes_per_launch: 123.0\n")
    (prof / "stale.txt").write_text("source_sha256: 00\ndram_bytes_per_launch: 123.0\n")
    real_join = os.path.join

    def join(*parts):  # profiles/ of the temporary tree, sources of the real one
        if parts[:2] == (bench.ROOT, "profiles"):
            return real_join(str(tmp_path), *parts[1:])
        return real_join(*parts)

    monkeypatch.setattr(bench.os.path, "join", join)
    assert bench.profiled_traffic(files, "k.txt")[0] == 123.0
    assert bench.profiled_traffic(files, "stale.txt")[0] is None
    assert bench.profiled_traffic(files, "absent.txt")[0] is None
