"""bench.py's JSON-line contract, checked on the CPU through its reference
arm (the oracle timed on host cores): required keys, the workload names of
the options, and that only rank 0 prints under a multi-rank launch."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                         capture_output=True, text=True, cwd=ROOT, env=env, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    return [json.loads(l) for l in res.stdout.splitlines() if l.startswith("{")]


@pytest.mark.parametrize("extra,suffix", [([], ""), (["--shared-expert"], "_shared1"),
                                          (["--fp8-intermediate"], "_a8")])
def test_reference_line_moe(extra, suffix):
    (line,) = _run(["--steps", "1", "--warmup", "1", "--ref-layers", "1", *extra])
    assert KEYS <= set(line)
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["higher_is_better"] is True and line["n_gpus"] == 1
    assert line["config"]["workload"] == "ling_layer_M1_gap" + suffix
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_line_lm_head():
    (line,) = _run(["--op", "lm_head", "--steps", "1", "--warmup", "1", "--ref-rows", "2048"])
    assert KEYS <= set(line)
    assert line["config"]["workload"] == "lm_head_fp8_V157184_H2560_M1" and line["value"] > 0


def test_reference_other_ranks_print_nothing():
    assert _run(["--steps", "1", "--warmup", "1", "--ref-layers", "1"],
                {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []
    assert _run(["--op", "lm_head", "--steps", "1", "--warmup", "1", "--ref-rows", "256"],
                {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []


def test_split_needs_one_part_per_rank():
    """--parts under a multi-rank launch must match the number of ranks (checked
    before any device work)."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--parts", "3"], capture_output=True,
                         text=True, cwd=ROOT, env=env, timeout=600)
    assert res.returncode != 0 and "--parts must equal the number of ranks" in res.stderr
