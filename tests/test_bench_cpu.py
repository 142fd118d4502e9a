"""bench.py loads on a machine without a GPU: the module compiles and imports,
its tables are well formed, and the profile subcommand parses its arguments."""
import importlib.util
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_bench_imports_and_tables_are_well_formed():
    b = _bench()
    for name, rec in b.NCU_TRAFFIC.items():
        assert set(rec) == {"bytes_per_launch", "source_sha"}, name
        assert isinstance(rec["bytes_per_launch"], int) and rec["bytes_per_launch"] > 0
        assert len(rec["source_sha"]) == 16
    assert {d[0] for d in b.DECODES} <= set(b.NCU_TRAFFIC) | {"decode"}
    assert len(b.kernel_sha("attn_fwd_sm100.cuh")) == 16


def test_profile_subcommand_parses():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "profile", "fwd", "--help"],
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert "--causal" in out.stdout
