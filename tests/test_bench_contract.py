"""bench.py's command line and JSON contract, on CPU.

The reference arm (the float64 oracle on the host's cores) runs here on the small
decode workload and must print one JSON line with the contract's keys; fewer
than three warm-up steps are refused; and the product arm, which has no CPU
fallback, must fail without printing a result when no GPU is present.
"""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args, timeout=240):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          cwd=ROOT, timeout=timeout)


def test_reference_arm_prints_one_contract_line():
    r = run_bench("--impl", "reference", "--config", "tiny", "--steps", "2", "--warmup", "3")
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["vs_baseline"] is None and d["config"]["name"] == "tiny" and "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_fewer_than_three_warmup_steps_are_refused():
    r = run_bench("--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "2")
    assert r.returncode != 0 and not r.stdout.strip()
    assert "warmup" in r.stderr


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_product_arm_fails_loudly_without_a_gpu():
    r = run_bench("--steps", "1", "--warmup", "3")
    assert r.returncode != 0
    assert not r.stdout.strip()                      # no result line from any fallback


@pytest.mark.parametrize("config", ["tiny", "prefill", "prefill_fp8"])
def test_product_arm_adds_the_cpu_baseline(config, monkeypatch, capsys):
    """main()'s product arm after the GPU timing, with the timing replaced by a stub returning a
    fixed line on the small workload: the cpu_baseline the oracle adds is complete."""
    import bench
    from paged_kv_cache_324_b200 import workload as wl
    stub = {"metric": "m", "value": 1.0, "unit": "u"}
    if config == "tiny":
        monkeypatch.setattr(bench, "run_ours", lambda *a: (dict(stub), wl.make("tiny")))
    else:
        monkeypatch.setattr(bench, "run_prefill", lambda *a: (dict(stub), wl.make_prefill(small=True)))
    monkeypatch.setattr(sys, "argv", ["bench.py", "--config", config, "--steps", "1", "--warmup", "3",
                                      "--cpu-budget", "0.05"])
    for var in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(var, raising=False)
    bench.main()
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    cb = json.loads(lines[0])["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1 and cb["sample"]
    if config == "tiny":
        assert cb["one_core"]["cores"] == 1 and cb["one_core"]["value"] > 0


def test_reference_arm_runs_on_rank_zero_only():
    """Under two ranks the reference arm prints one line from rank 0; rank 1 exits at once."""
    outs = []
    for rank in (0, 1):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                            "--gpus", "2", "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                           cwd=ROOT, env=env, timeout=240)
        assert r.returncode == 0, r.stderr
        outs.append([ln for ln in r.stdout.splitlines() if ln.strip()])
    assert len(outs[0]) == 1 and json.loads(outs[0][0])["n_gpus"] == 2
    assert outs[1] == []


def test_config_rows_name_decode_workloads():
    """Every workload the default run times under "configs" is a decode workload the generator knows,
    and the shared-prefix rows are the ones with shared prompts."""
    import bench
    from paged_kv_cache_324_b200 import workload as wl
    names = set(wl.NAMES) | set(wl.EXTRA_NAMES)
    assert bench.CONFIG_ROWS
    for name, shared in bench.CONFIG_ROWS:
        assert name in names, name
        if shared:
            assert name.startswith("prefix")
    # the large-batch rows the 75%-of-HBM target names are among them
    assert {"gqa", "fp8", "fp8_b32"} <= {n for n, _ in bench.CONFIG_ROWS}


def test_l2_note_names_the_regime():
    import bench
    assert "more than the 126 MB L2" in bench.l2_note(2 * 10 ** 9)
    assert "fit in the 126 MB L2" in bench.l2_note(50 * 10 ** 6)
