"""The JSON line bench.py prints for the reference arm (the oracle on the host
cores) carries the keys the benchmark contract asks for.  CPU only: the tiny
workload, one timed step."""
import contextlib
import io
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_arm_json_line(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--workload", "tiny_w4a8", "--steps", "1",
                         "--warmup", "3", "--cpu-budget-s", "0.5"])
    assert rc == 0
    lines = [l for l in buf.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "impl", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TOPS"
    assert d["steps"] == 1 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny_w4a8"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_kernel_hash_ignores_comments_only():
    """The DRAM-traffic figure is reported only for the kernel it was measured
    on; the hash that decides this sees code, not comments or layout."""
    src = ('// header "quoted" /* not a block */\n'
           'const char* s = "a // b /* c */";  /* block\n comment */ int x = \'"\';\n'
           'int   y  =  1; // trailing\n')
    code = bench._c_code_only(src)
    assert code == 'const char* s = "a // b /* c */"; int x = \'"\'; int y = 1;'
    assert bench._c_code_only(src.replace("trailing", "other words")) == code
    assert bench._c_code_only(src.replace("y  =  1", "y = 2")) != code



def test_reference_step_sample_is_bounded():
    """With the default 2000 timed steps the reference arm has about 75 ms of
    host time per step: its sample must shrink to that (rows of every M,
    against 64 channels) instead of quantizing every row of X each step."""
    import oracle
    import synthetic_inputs as si
    layer = si.LAYERS["llama3_8b_qkv"]
    ref = oracle.quantize_weights(si.weights(layer, 0), layer.group)
    budget = bench.REFERENCE_RUN_S / 2020
    rows, n_cols = bench.oracle_sample_plan(layer, budget, oracle, ref["dq"])
    assert n_cols == 64 and sum(rows) < sum(layer.ms) // 4
    assert all(1 <= r <= M for r, M in zip(rows, layer.ms))
    Xs = [si.activations(layer, M, seed=0)[:r] for M, r in zip(layer.ms, rows)]
    ops, dt = bench.run_oracle_pass(layer, oracle, ref["dq"], ref["s1"], Xs, n_cols)
    assert ops == sum(2 * r * n_cols * layer.K for r in rows)
    assert dt < 5 * budget + 0.2
