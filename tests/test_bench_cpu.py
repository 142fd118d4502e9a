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


def test_launch_count_follows_the_split_rule():
    """The step's launch count: a non-causal call whose last round holds at most
    half as many 256-row query blocks as SMs makes a second launch."""
    b = _bench()
    assert b.fwd_launch_count(2, 32, 2048, True, 148) == 1
    assert b.fwd_launch_count(2, 32, 2048, False, 148) == 2   # 512 blocks: last round 68 <= 74
    assert b.fwd_launch_count(8, 16, 2048, False, 148) == 1   # 1024 blocks: last round 136 > 74
    assert b.fwd_launch_count(1, 37, 1024, False, 148) == 1   # 148 blocks: no last round
    assert b.fwd_launch_count(1, 1, 128, False, 148) == 1     # one key tile: nothing to split
    assert b.fwd_launch_count(1, 1, 256, False, 148) == 2     # one block, two key tiles
    assert len(b.CAUSAL_SWEEP) >= 3
