"""bench.py's JSON line, checked on the host: the reference arm (the oracle on the host
cores) prints one line with every key of the contract, and a GPU-less run of the
product arm fails loudly instead of falling back to the CPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, timeout=300):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, capture_output=True,
                          text=True, timeout=timeout)


def test_reference_arm_prints_one_contract_line():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-rows", "4")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["data"] == "synthetic"
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_warmup_below_three_is_refused():
    r = _run("--impl", "reference", "--steps", "1", "--warmup", "1", "--ref-rows", "4")
    assert r.returncode != 0
    assert "warmup" in r.stderr


def test_product_arm_without_a_gpu_fails_loudly():
    import torch
    if torch.cuda.is_available():
        return  # the GPU suite runs the product arm for real
    r = _run("--steps", "1", "--warmup", "3")
    assert r.returncode != 0


def test_reference_arm_under_torchrun_prints_once_from_rank_zero():
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
                        "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-rows", "4"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2


def _bench_module():
    sys.path.insert(0, ROOT)
    import bench
    return bench


def test_attention_flops_count_the_visible_pairs():
    bench = _bench_module()
    for S in (1, 2, 7, 130):
        pairs = sum(1 for i in range(S) for j in range(S) if j <= i)
        assert bench.attention_flops(S, 3, 16) == 4 * 16 * 3 * pairs  # QK^T and PV, 2 flops per multiply-add
    assert bench.attention_flops(8704, 16, 128) == 310_347_038_720


def test_select_path_bytes_at_the_128k_workload():
    bench = _bench_module()
    # gate: residual read, W1, b1/W2 (+b2), scores written; top-K: scores + mask read, kept
    # indices (+count) written; gather: indices, rows read and written, scores gathered
    assert bench.select_path_bytes(131072, 2048, 256, 8704) == 610_543_110


def test_clock_sampler_reads_median_clock_and_reasons():
    bench = _bench_module()

    class _Proc:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    cs = bench.ClockSampler(0)
    cs.proc = _Proc()
    cs.lines = ["0, 1965, 1965, 900.1, 0x4, Not Active, Not Active, Not Active, Active",
                "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
                "0, 1900, 1965, 950.0, 0x0, Not Active, Not Active, Not Active, Not Active",
                "garbage line"]
    out = cs.stop()
    assert out["sm_mhz"] == 1900 and out["sm_max_mhz"] == 1965 and out["samples"] == 3
    assert out["reasons"] == ["sw_power_cap"]


def test_attention_algorithmic_bytes_at_the_128k_layer():
    bench = _bench_module()
    read, write = bench.attention_bytes(8704, 16, 8, 128)
    # Q (16 heads) + K + V (8 heads each) in bf16, the key scores and the gains read once; O written once
    assert read == (16 + 8 + 8) * 128 * 2 * 8704 + 4 * 8704 + 4 * 16 == 71_338_048
    assert write == 16 * 128 * 2 * 8704 == 35_651_584


def test_sweep_covers_every_workload_budget():
    bench = _bench_module()
    from learned_token_pruning_mlp_b200 import workloads as W
    for name, w in W.WORKLOADS.items():
        listed = sorted(k for nm, k in bench.SWEEP if nm == name)
        if w.varlen:
            assert listed == [None]          # one line for the packed batch (per-request budgets)
        elif name != "tiny_n512":            # the tiny case is a parity case, not a bench line
            assert listed == sorted(w.budgets), name
