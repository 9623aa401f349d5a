"""The benchmark's command line on CPU.

The reference arm (the fp64 oracle on the host cores) prints exactly one JSON
line carrying the keys of the result contract, with its own value repeated in
`cpu_baseline` and `e2e`.  The product arm has no CPU path: without a GPU it
exits with an error and prints no result line.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CONTRACT = {
    "metric": str, "value": float, "unit": str, "n_gpus": int, "steps": int, "warmup": int,
    "ms_per_step": float, "higher_is_better": bool, "scaling": str,
    "vs_baseline": (type(None), float), "dtype": str, "data": str, "config": dict,
    "impl": str, "cpu_baseline": dict, "e2e": dict,
}


def run_bench(*args):
    return subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True,
                          text=True, timeout=300)


def test_reference_arm_prints_one_contract_line():
    out = run_bench("--impl", "reference", "--steps", "2", "--warmup", "0",
                    "--workload", "tiny_f32_t64")
    assert out.returncode == 0, out.stderr
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    r = json.loads(lines[0])
    for key, typ in CONTRACT.items():
        assert isinstance(r[key], typ), key
    assert r["impl"] == "reference" and r["n_gpus"] == 1
    assert r["steps"] == 2 and r["warmup"] == 0
    assert r["unit"] == "tokens/s" and r["higher_is_better"] is True
    assert r["dtype"] == "f64" and r["data"] == "synthetic" and r["vs_baseline"] is None
    assert r["config"]["workload"] == "tiny_f32_t64"
    # value = tokens of the bounded sample per step over the time of a step
    tok = r["config"]["sample_tokens_per_step"]
    assert r["value"] == pytest.approx(tok / (r["ms_per_step"] / 1e3), rel=1e-3)
    cb = r["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == r["value"] and cb["cores"] >= 1
    assert cb["sample"]
    assert r["e2e"] == {"value": r["value"], "unit": r["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_product_arm_has_no_cpu_path():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    out = run_bench("--steps", "1", "--warmup", "3")
    assert out.returncode != 0
    assert not any(ln.lstrip().startswith("{") for ln in out.stdout.splitlines())


def test_launches_per_step_match_the_profiled_launch_lists():
    """The kernel count per step that bench.py reports as gpu_launches, against the
    ncu launch lists in profiles/ (kernels per graph replay: 36 in 3 prefill steps,
    100 in 20 decode steps, 100 in 20 NVFP4 decode steps, 180 in 20 latent steps)."""
    import bench
    import synth
    want = {"prefill_bf16_t16384": 12, "decode_bf16_t8": 5, "decode_nvfp4_t8": 5,
            "decode_latent_bf16_t8": 9}
    for name, n in want.items():
        assert bench.launches_per_step(synth.CONFIGS[name]) == n, name
