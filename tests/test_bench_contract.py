"""The benchmark's JSON contract on the host: the reference arm (the oracle on a bounded sample)
prints one line with the required keys for an activation workload and for the K/V-only one, and
each workload's L2 statement follows its input sizes."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"}


@pytest.mark.parametrize("workload", ["tiny-768", "kv-4096"])
def test_reference_arm_line(workload):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", workload, "--steps", "2",
                          "--warmup", "1", "--ref-budget-s", "5"], cwd=ROOT, env=env, capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert KEYS <= set(d)
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["config"]["workload"] == workload


def test_l2_statement_follows_input_sizes():
    sys.path.insert(0, ROOT)
    import bench
    from post_activation_quantization_b200 import workloads as W
    assert "larger than L2" in bench.workload_config(W.WORKLOADS["opt175b-12288"])["l2"]
    assert "larger than L2" in bench.workload_config(W.WORKLOADS["kv-4096"])["l2"]
    assert "fit in the 126 MB L2" in bench.workload_config(W.WORKLOADS["tiny-768"])["l2"]
    assert "fit in the 126 MB L2" in bench.workload_config(W.WORKLOADS["opt6.7b-4096"])["l2"]


def test_stage_accounting_per_workload():
    """Stages, algorithmic bytes and launch counts of a step (the basis of `value` and of the
    `gpu_launches` claim): by hand for the bench workload and the K/V-only one."""
    sys.path.insert(0, ROOT)
    import bench
    from post_activation_quantization_b200 import workloads as W
    st = bench.stage_list(W.WORKLOADS["opt175b-12288"])
    assert [s[0] for s in st] == ["calib_ln", "kv_calib", "kmeans", "ln_quant_plan", "ln_reorder_quant",
                                  "ln_reorder_quant_unplanned", "explicit_reorder_baseline", "dynamic_ranges",
                                  "linear_prepare", "reordered_linear", "kv_quant", "kv_quant_cluster_ordered",
                                  "dequant_act", "dequant_kv", "kv_append", "kv_decode_attention"]
    b = dict((n, v) for n, v, _ in st)
    T, C, Tc, kv = 32768, 12288, 262144, 8 * 96 * 2048 * 128
    assert b["calib_ln"] == Tc * C * 2
    assert b["kv_calib"] == 2 * kv * 2
    assert b["ln_reorder_quant"] == b["ln_reorder_quant_unplanned"] == T * C * 2 + T * C * 3 // 8
    assert b["ln_quant_plan"] == 28 * C
    assert b["kv_quant"] == 2 * (kv * 2 + kv * 3 // 8)
    assert b["kv_quant_cluster_ordered"] == kv * 2 + kv * 3 // 8
    assert b["dequant_act"] == T * C * 3 // 8 + T * C * 2
    assert b["dequant_kv"] == 2 * (kv * 3 // 8 + kv * 2)
    assert b["kv_append"] == 2 * (8 * 96 * 128 * 2 + 8 * 96 * 128 * 3 // 8)
    assert b["kv_decode_attention"] == 2 * kv * 3 // 8 + 2 * 8 * 96 * 128 * 4
    assert b["explicit_reorder_baseline"] == T * C * 2 + 4 * T * C * 4 + T * C * 3 // 8
    assert b["dynamic_ranges"] == T * C * 2
    # the Q/K/V projection (N = 3C) on a 2048-token micro-batch: its operand preparation reads
    # the 4-bit codes and writes fp16 plus two floats per row; the GEMM is counted in FLOPs
    N = 3 * C
    assert b["linear_prepare"] == N * C // 2 + N * C * 2 + 8 * N and b["reordered_linear"] == 0
    assert bench.stage_flops(W.WORKLOADS["opt175b-12288"]) == {"reordered_linear": 2 * 2048 * C * N}
    assert sum(l for _, _, l in st) == 30  # 2 + 4 + 6 + 1 + 1 + 1 + 3 + 3 + 1 + 1 + 1 + 1 + 1 + 2 + 1 + 1
    st = bench.stage_list(W.WORKLOADS["kv-4096"])
    assert [s[0] for s in st] == ["kv_calib", "kmeans", "kv_quant", "kv_quant_cluster_ordered", "dequant_kv", "kv_append",
                                  "kv_decode_attention"]
    assert sum(l for _, _, l in st) == 4 + 4 + 1 + 1 + 2 + 1 + 1
    st = bench.stage_list(W.WORKLOADS["tiny-768"])
    assert [s[0] for s in st] == ["calib_ln", "kmeans", "ln_quant_plan", "ln_reorder_quant", "ln_reorder_quant_unplanned",
                                  "explicit_reorder_baseline", "dynamic_ranges", "linear_prepare", "reordered_linear",
                                  "dequant_act"]
    assert sum(l for _, _, l in st) == 2 + 2 + 1 + 1 + 1 + 3 + 3 + 1 + 1 + 1
    assert bench.stage_flops(W.WORKLOADS["tiny-768"]) == {"reordered_linear": 2 * 512 * 768 * 2304}


def test_gpus_n_starts_n_ranks():
    """`--gpus 2` outside a launcher starts two ranks under torchrun (checked without a GPU:
    --dry-run makes each rank report its place and exit)."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    env.pop("WORLD_SIZE", None)
    out = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--dry-run"], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    ranks = [json.loads(l) for l in out.stdout.splitlines() if l.startswith("{")]
    assert sorted(r["rank"] for r in ranks) == [0, 1]
    assert all(r["world_size"] == 2 for r in ranks)


def test_world_size_mismatch_is_refused():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, "bench.py", "--gpus", "4", "--dry-run"], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode != 0 and "--gpus 4" in out.stderr
