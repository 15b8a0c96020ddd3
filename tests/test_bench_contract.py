"""The benchmark's JSON line on CPU: every workload's line carries the keys
and units the measurement contract needs (metric, whole-job value, roofline
with achieved / peak / frac / traffic, clocks, launches, e2e), computed from a
synthetic result record whose numbers are known, so the arithmetic of
`achieved` and `frac` is checked as well."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

PK = dict(hbm=6540.8, bf16=1645.8, bf16_sus=1369.4, src="measured")
CLOCKS = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 10}


def _prefill_res(T, steps, world=1):
    flops_idx = 1024.0 * T * (T + 1) / 2
    # indexer: 2 launches per step, each taking half of 0.5 s per step
    return dict(ms=800.0 * steps, tokens=T * steps * world, steps=steps, flops_idx=flops_idx,
                flops_attn=0.1 * flops_idx, kern={"indexer": (2 * steps, 500.0 * steps), "attention": (2, 1.0)},
                launches=4 * steps, clocks=CLOCKS,
                e2e=dict(value=1.0, unit="tokens/s", h2d_bytes_per_step=10, d2h_bytes_per_step=5))


def _decode_res(steps, world=1):
    return dict(ms=24.0 * steps, tokens=64 * 32 * steps * world, steps=steps, bytes_indexer=4.3e9,
                bytes_step=4.4e9 * 32, kern={"decode_indexer": (32 * steps, 0.65 * 32 * steps)},
                launches=100, clocks=CLOCKS, calls=32 * steps)


@pytest.mark.parametrize("name", list(bench.WORKLOADS))
def test_line_has_contract_keys(name):
    wl = bench.WORKLOADS[name]
    steps = 5
    res = _decode_res(steps) if wl["kind"] == "decode" else _prefill_res(wl["T"] - wl.get("L_old", 0), steps)
    line = bench.line_for(name, res, 1, steps, 3, PK)
    json.dumps(line)   # serialisable
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "clocks", "gpu_launches"):
        assert k in line, k
    assert line["config"]["workload"] == name
    assert line["scaling"] == "weak" and line["higher_is_better"] is True
    r = line["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in r, k
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    assert line["value"] == pytest.approx(res["tokens"] / (res["ms"] / 1e3))
    if wl["kind"] == "decode":
        assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == PK["hbm"]
        # 4.3 GB per launch in 0.65 ms
        assert r["achieved"] == pytest.approx(4.3e9 / 0.65e-3 / 1e9)
    else:
        assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] == PK["bf16_sus"]
        # FLOPs of one step over two launches of 250 ms each
        assert r["achieved"] == pytest.approx(res["flops_idx"] / 2 / 0.25 / 1e12)


def test_whole_job_value_counts_every_rank():
    res = _decode_res(5, world=4)
    line = bench.line_for("decode_64x256k", res, 4, 5, 3, PK)
    assert line["n_gpus"] == 4
    assert line["value"] == pytest.approx(4 * 64 * 32 * 5 / (24.0 * 5 / 1e3))


def test_reference_arm_line(tmp_path):
    """`--impl reference` on rank 0 prints one JSON line with the oracle as the
    arm (a tiny stand-in workload keeps the CPU time short)."""
    code = (
        "import sys, runpy; sys.argv = ['bench.py', '--impl', 'reference', '--steps', '1', '--warmup', '3',"
        " '--workload', 'prefill_32k'];"
        "import bench; bench.cpu_sample = lambda wl, target_s=12.0: (12.5, dict(sample='stub', elapsed=1.0));"
        "bench.main()")
    p = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300,
                       env=dict(os.environ, RANK="0", WORLD_SIZE="1"))
    assert p.returncode == 0, p.stderr
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] == 12.5
    assert line["ms_per_step"] == 1000.0 and line["warmup"] == 3   # one sampled step's wall time
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
