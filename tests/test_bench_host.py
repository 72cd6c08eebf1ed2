"""Host-side pieces of bench.py (no GPU): the roofline arithmetic, the
workload block of the JSON line and the oracle CPU baseline."""
import math

import bench
import synth

PEAKS = {"sm_max_mhz": 1965.0, "bf16_tflops": 1640.9, "bf16_tflops_sustained": 1416.7}


def test_subset_roofline_counts_elements_and_lanes():
    wl = synth.CONFIGS["large_subset_bf16"]
    r = bench._alu_roofline(wl, 176.7, PEAKS)
    elems = wl.T * wl.K * (wl.S + 1)
    assert r["elements"] == elems and r["ops_per_element"] == 14
    assert math.isclose(r["achieved"], elems * 14 / 0.1767 / 1e12, rel_tol=1e-12)
    assert math.isclose(r["peak"], 148 * 128 * 1965e6 / 1e12, rel_tol=1e-12)
    assert math.isclose(r["frac"], r["achieved"] / r["peak"], rel_tol=1e-12)
    assert r["bound"] == "alu" and 0.28 < r["frac"] < 0.30     # the verdict's 0.29 at 176.7 ms
    alt = r["with_accumulate"]
    assert alt["ops_per_element"] == 20 and math.isclose(alt["frac"], r["frac"] * 20 / 14)
    sfu = r["sfu"]
    assert math.isclose(sfu["peak"], 148 * 16 * 1965e6 / 1e12, rel_tol=1e-12)
    assert math.isclose(sfu["frac"], elems / 0.1767 / (148 * 16 * 1965e6), rel_tol=1e-12)
    assert 0.16 < sfu["frac"] < 0.18


def test_full_vocab_roofline_counts_one_generation():
    wl = synth.CONFIGS["full_bf16"]
    r = bench._alu_roofline(wl, 29.8, PEAKS)
    assert r["elements"] == wl.T * wl.K * wl.V and r["kernel"] == "full_draws"


def test_attention_roofline_splits_tensor_and_cuda_core_work():
    for name, rows_expected in (("attn_q_bf16", True), ("attn_k_bf16", True),
                                ("attn_v_bf16", False)):
        wl = synth.CONFIGS[name]
        r = bench._attn_roofline(wl, 10.0, PEAKS)
        L, H, dh = wl.seq_len, wl.n_heads, wl.head_dim
        rows = (wl.T // L) * L * (L + 1) // 2 if rows_expected else 0
        ops = wl.K * H * (rows * bench.ATTN_OPS_PER_ROW + wl.T * dh * bench.ATTN_OPS_PER_NOISE)
        assert r["ops"] == ops
        assert math.isclose(r["achieved"], ops / 0.01 / 1e12, rel_tol=1e-12)
        if rows_expected:
            assert r["tensor"]["flops"] == 6 * dh * wl.K * H * rows
        else:
            assert "tensor" not in r


def test_mlp_roofline_flops():
    for name in ("mlp_bf16", "mlp_down_bf16", "attn_out_bf16"):
        wl = synth.CONFIGS[name]
        r = bench._mlp_roofline(wl, 300.0, PEAKS)
        d, dff, V = wl.d, wl.d_ff, wl.V
        per_row = 2 * d * V                          # dz = dh W_head^T
        if name != "mlp_down_bf16":
            per_row += 2 * dff * d                   # dh = da W_down^T
        if name == "attn_out_bf16":
            per_row += 2 * d * dff                   # du = (sigma eps) W_up^T
        assert math.isclose(r["flops"], per_row * wl.T * wl.K, rel_tol=1e-12)
        # dz and dh on the hi planes only, plus a correction per row (2d, and
        # 2 d_ff where dh comes from da); du on both planes of sigma eps
        executed = per_row + 2 * d
        if name != "mlp_down_bf16":
            executed += 2 * dff
        if name == "attn_out_bf16":
            executed += 2 * d * dff
        assert math.isclose(r["executed"]["flops"], executed * wl.T * wl.K, rel_tol=1e-12)
        assert r["bound"] == "tensor" and r["peak"] == PEAKS["bf16_tflops_sustained"]
    # the up-projection's 82.0 MFLOP per token-draw
    alg, _ = bench._mlp_flops_per_row(synth.CONFIGS["mlp_bf16"])
    assert round(alg / 1e6, 1) == 82.0


def test_gemm_report():
    g = bench._gemm_report(2.0 * 16384 * 1024 * 50304, 2.0, PEAKS)
    assert math.isclose(g["tflops"], 2.0 * 16384 * 1024 * 50304 / 2e-3 / 1e12)
    assert math.isclose(g["frac_burst"], g["tflops"] / 1640.9)


def test_config_block():
    class Args:
        config = "attn_q_bf16"
    cfg = bench._config(Args, synth.CONFIGS["attn_q_bf16"], 1)
    assert cfg["workload"] == "attn_q_bf16" and cfg["parallelism"] == "dp1"
    assert (cfg["seq_len"], cfg["n_heads"], cfg["head_dim"]) == (1024, 12, 64)
    Args.config = "large_subset_bf16"
    cfg = bench._config(Args, synth.CONFIGS["large_subset_bf16"], 2)
    assert "seq_len" not in cfg and cfg["parallelism"].startswith("dp2")
    assert (cfg["T_per_gpu"], cfg["K"], cfg["S"]) == (16384, 16384, 512)


def test_cpu_baseline_on_a_small_sample():
    cb = bench.cpu_baseline("tiny_fp32", budget_tokens=2)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1
    assert cb["host_cores"] >= cb["cores"] and cb["seconds"] > 0
    assert "2 tokens x all 16 draws of tiny_fp32" in cb["sample"]


def _run_bench(*args, env=None, rc=0):
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    e = dict(os.environ, **(env or {}))
    res = subprocess.run([sys.executable, "bench.py", *args], cwd=root, env=e,
                         capture_output=True, text=True, timeout=600)
    assert res.returncode == rc, res.stderr[-2000:]
    lines = [json.loads(s) for s in res.stdout.splitlines() if s.startswith("{")]
    return lines


def test_reference_arm_prints_one_contract_line():
    # the reference arm times the oracle on the host: one JSON line with the
    # metric, unit and workload of the product arm, marked impl=reference
    lines = _run_bench("--impl", "reference", "--steps", "1", "--warmup", "0",
                       "--config", "tiny_fp32")
    assert len(lines) == 1
    ln = lines[0]
    assert ln["impl"] == "reference" and ln["metric"] == bench.METRIC and ln["unit"] == bench.UNIT
    assert ln["n_gpus"] == 1 and ln["steps"] == 1 and ln["higher_is_better"] is True
    assert ln["config"]["workload"] == "tiny_fp32" and ln["value"] > 0
    cb = ln["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == ln["value"]
    assert ln["e2e"] == {"value": ln["value"], "unit": ln["unit"], "h2d_bytes_per_step": 0,
                         "d2h_bytes_per_step": 0}
    assert ln["ms_per_step"] > 0 and ln["dtype"] == "f64"


def test_reference_arm_other_ranks_exit_quietly():
    lines = _run_bench("--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
                       "--config", "tiny_fp32", env={"RANK": "1", "WORLD_SIZE": "2"})
    assert lines == []


def test_gpus_flag_starts_that_many_ranks():
    """bench.py --gpus 2 without a launcher starts two ranks itself; rank 0's
    line reports n_gpus 2, rank 1 prints nothing (the reference arm needs no
    GPU, so the launch runs here)."""
    lines = _run_bench("--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
                       "--config", "tiny_fp32", "--ref-tokens", "2")
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2
    assert lines[0]["config"]["parallelism"].startswith("dp2")


def test_gpus_flag_must_match_the_launcher():
    lines = _run_bench("--impl", "reference", "--gpus", "4", "--steps", "1", "--warmup", "0",
                       "--config", "tiny_fp32", env={"RANK": "0", "WORLD_SIZE": "2"}, rc=2)
    assert lines == []
