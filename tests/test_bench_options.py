"""bench.py's workload selection: --swa W runs the sliding window (block 1, window W),
--block/--window override the block rule and --rope adds the rotary embedding, all on the
config's own shapes and seeds."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class Args:
    config, examples, swa, block, window = 3, 0, 0, 0, 0


def test_default_is_the_configured_workload():
    b = _bench()
    w = b.config_workload(Args())
    assert (w.block, w.window) == (256, 2) and "block 256, window 2" in w.name


def test_sliding_window_option():
    b = _bench()
    a = Args()
    a.swa = 512
    w = b.config_workload(a)
    assert (w.block, w.window) == (1, 512)
    assert "sliding window 512 tokens" in w.name and "block 256" not in w.name
    base = b.config_workload(Args())
    assert (w.batch, w.heads, w.head_dim, w.seed) == (base.batch, base.heads, base.head_dim, base.seed)


def test_block_window_overrides():
    b = _bench()
    a = Args()
    a.block, a.window = 64, 1
    w = b.config_workload(a)
    assert (w.block, w.window) == (64, 1) and "block 64, window 1" in w.name


def test_job_totals_single_rank_is_identity():
    b = _bench()
    assert b.job_totals(5.0, 7.0, 3.0) == (5.0, 7.0, 3.0)


def test_rope_option_keeps_the_workload_and_covers_the_longest_example():
    b = _bench()
    a = Args()
    a.rope = True
    w = b.config_workload(a)
    base = b.config_workload(Args())
    assert w.name == base.name + ", rotary q/k"
    assert (w.block, w.window, w.batch, w.heads, w.head_dim, w.seed) == \
        (base.block, base.window, base.batch, base.heads, base.head_dim, base.seed)
    cos, sin = b.tables_for([64, 4096, 17], 128)
    assert cos.shape == sin.shape == (4096, 64)


def test_reference_arm_prints_one_contract_line():
    """bench.py --impl reference (the oracle on the host cores) prints one JSON
    line with the contract's keys; config 2 (one 1024-token example per step)
    keeps it to seconds."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "2",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert "workload" in d["config"]


def test_gdpa_option_names_the_activation_and_refuses_skip_flags():
    import pytest
    b = _bench()
    a = Args()
    a.gdpa = "silu"
    w = b.config_workload(a)
    assert w.name.endswith(", GDPA silu") and (w.block, w.window) == (256, 2)
    a.config = 5
    with pytest.raises(SystemExit):
        b.config_workload(a)


def test_mx_option_names_the_operands_and_refuses_rope_and_gdpa():
    import pytest
    b = _bench()
    a = Args()
    a.mx = True
    w = b.config_workload(a)
    assert w.name.endswith(", MXFP8 Q/K") and w.head_dim == 128
    a.rope = True
    with pytest.raises(SystemExit):
        b.config_workload(a)
    assert b.parse(["--mx"]).mx and not b.parse([]).mx
