"""bench.py's reference arm on the host (CPU only): it times the oracle on
bounded samples and prints one JSON line with the contract's keys."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "toy", "--steps", "2",
                        "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "dtype", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["steps"] == 2 and line["warmup"] == 3 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "toy"


def _bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_algorithmic_work_counts():
    """The roofline numerators, worked by hand for the Mixtral-shaped batch
    (29450 kept rows) and the 64-token decode batch (128 rows, all 8 experts)."""
    b = _bench_module()
    d, d_ff = 4096, 14336
    # two GEMMs of R x d x d_ff multiply-adds, two flops each
    assert b.ffn_flops(29450, d, d_ff) == 2 * 2 * 29450 * d * d_ff == 6917246156800
    # bf16: both weight matrices of each touched expert once, x_g read, H written and read, y written
    counts = [16] * 8
    weights = 8 * 2 * d * d_ff * 2
    rows = 128 * d * 2 + 2 * 128 * d_ff * 2 + 128 * d * 2
    assert b.ffn_bytes(counts, d, d_ff, 2) == weights + rows == 1888485376
    # an expert without rows costs no weight bytes
    assert b.ffn_bytes([32, 0] + [16] * 6, d, d_ff, 2) == 7 * 2 * d * d_ff * 2 + rows


def test_traffic_lookup_is_keyed_by_source():
    """A DRAM figure is reported only for the GEMM source it was measured on."""
    b = _bench_module()
    import hashlib
    src = os.path.join(ROOT, "sparse_mixture_experts_noisy_b200", "csrc", "gemm_tc.cu")
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    keyed = {}
    for line in open(os.path.join(ROOT, "profiles", "traffic.txt")):
        parts = line.split()
        if len(parts) >= 3 and not line.startswith("#"):
            keyed[(parts[0], parts[1])] = float(parts[2])
    for tag in ("prefill_mixtral", "prefill_fine", "decode"):
        assert b.ncu_traffic(tag) == keyed.get((tag, h))
    assert b.ncu_traffic("no_such_workload") is None
