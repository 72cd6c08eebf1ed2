"""Benchmark of the Dust per-token activation-space gradient estimator.

One step = one full estimator call over one batch of synthetic input: clean
logits GEMM, log-sum-exp, the K perturbed draws with rewards and the
reward-weighted noise average g, and the G_W GEMM. The default workload is
the LM head at d=1024, V=50304 with T=16384 tokens, K=16384 draws and
vocabulary-subset draws of S=512 (the large-subset workload); ``--config``
selects another one.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl dust|reference]

``--gpus N`` with N > 1 starts N ranks itself (torch.distributed.run, one
process per GPU) unless a launcher already did; under a launcher it must
equal WORLD_SIZE. Rank 0 prints one JSON line. With N > 1 each rank runs its own
token shard (token_offset = rank * T, so the noise is that of one N*T-token
run) and the step ends with the one exchange the path has, a sum all-reduce
of G_W over NCCL: weak scaling, value = all ranks' token-draws / the slowest
rank's time. ``--impl reference`` times the CPU oracle on a bounded sample
of the same workload. ``--tokens N`` cuts the workload to its first N tokens
(profiling slices).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "token-draws/sec of Dust gradient estimate (LM head d=1024,V=50304); % roofline"
UNIT = "token-draws/s"
SM_COUNT = 148
LANES_PER_SM = 128           # 4 schedulers x 32 lanes issue per clock
SFU_PER_SM = 16              # transcendental (MUFU) lanes per SM per clock
# Algorithmic minimum of issue slots per perturbed element (the roofline's
# `frac`): Philox4x32-10 10 (2.5 rounds per word, each two wide multiplies and
# two three-input XORs), the Gaussian 2 (half of a log, a square root and a
# sine/cosine pair, one slot each), the expm1 1 and one multiply-add 1.
ALU_OPS_PER_ELEM = 14
# A second count, reported beside it: the same generator with the sine and
# cosine as two slots and the expm1 as two (a degree-3 series), the p operand
# load that feeds the reward's multiply-add, and the g accumulation's
# multiply and shared-memory add, which the fused kernel must also issue.
ALU_OPS_PER_ELEM_WITH_ACCUMULATE = 20
# attention internals: per (draw, head, row visited) a d_h-long dot product
# on the tensor cores, taken as three fp16 products (6 d_h flops), and on the
# CUDA cores an expm1 (8 lane operations) and two multiply-adds; per noise
# entry the generator's 14 lane operations (Philox 10, Gaussian 4)
ATTN_OPS_PER_ROW = 10
ATTN_OPS_PER_NOISE = 14
ATTN_TC_FLOPS_PER_ROW_DH = 6
ATTN_SAMPLE_DRAWS = 4
# DRAM bytes (read + write) per token of the subset-draw kernel on the
# large-subset workload: ncu dram__bytes_read.sum + dram__bytes_write.sum of
# one launch over its first 2048 tokens (415.33 + 179.30 MB), per token; the
# kernel's traffic is per token (the logit row in, the fp16 g operand out).
SUBSET_DRAM_BYTES_PER_TOKEN = (415.334144e6 + 179.300096e6) / 2048
PROFILED_SUBSET_WORKLOAD = "large_subset_bf16"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "sm_max_mhz": 1965.0}, "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "pci.bus_id")

    def __init__(self, out_path=None):
        self.proc = None
        self.path = out_path or os.path.join(os.environ.get("DUST_CLOCKS_DIR", tempfile.gettempdir()),
                                             f"dust_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
        if not rows:
            return None
        mine = [r for r in rows if _same_bus(r[9])] or [r for r in rows if r[0] == rows[0][0]]
        sm = [float(r[1]) for r in mine if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in mine if r[2].replace(".", "").isdigit()]
        reasons = sorted({CLOCK_REASONS[k] for r in mine for k in range(4)
                          if r[5 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(mine)}


def _same_bus(bus_id: str) -> bool:
    """Whether nvidia-smi's PCI bus id ("00000000:18:00.0") is this rank's GPU."""
    try:
        import torch
        pr = torch.cuda.get_device_properties(torch.cuda.current_device())
        dom, bus, rest = bus_id.split(":")
        dev = rest.split(".")[0]
        return (int(dom, 16), int(bus, 16), int(dev, 16)) == (
            pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
    except (ValueError, AttributeError, RuntimeError):
        return False


CLOCK_REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


def _merge_clocks(clk, world: int, device: str = "cuda"):
    """The clock record of the whole job: the lowest median SM clock and the
    union of the throttle reasons over all ranks (every rank calls this; the
    tensors live on the process group's device)."""
    if world == 1:
        return clk
    import torch
    import torch.distributed as dist
    sm = clk["sm_mhz"] if clk and clk["sm_mhz"] is not None else float("inf")
    bits = sum(1 << k for k, n in enumerate(CLOCK_REASONS) if clk and n in clk["reasons"])
    hi = torch.tensor([clk["sm_max_mhz"] or 0.0 if clk else 0.0, float(bits),
                       float(clk["samples"] if clk else 0)], dtype=torch.float64, device=device)
    lo = torch.tensor([sm], dtype=torch.float64, device=device)
    dist.all_reduce(hi, op=dist.ReduceOp.MAX)
    dist.all_reduce(lo, op=dist.ReduceOp.MIN)
    if float(hi[2]) == 0.0:
        return None
    b = int(hi[1].item())
    return {"sm_mhz": None if lo.item() == float("inf") else float(lo.item()),
            "sm_max_mhz": float(hi[0]) or None,
            "reasons": [n for k, n in enumerate(CLOCK_REASONS) if b >> k & 1],
            "samples": int(hi[2]), "ranks": world}


# ----------------------------------------------------------------------------- oracle baseline
def _oracle_tokens(args):
    """Worker: the oracle on a few tokens of a workload (spawned process).

    Returns (token-draws done, seconds spent in the oracle); input generation is
    not timed."""
    import oracle
    import synth
    name, toks = args
    wl = synth.CONFIGS[name]
    if wl.variant == "head":
        inp = synth.make_head_inputs(wl)
        t0 = time.perf_counter()
        for t in toks:
            prm = oracle.Params(T=1, d=wl.d, V=wl.V, K=wl.K, S=wl.S, sigma=wl.sigma,
                                seed=wl.seed, token_offset=t)
            oracle.head_grad(inp["H"][t:t + 1], inp["W"], inp["targets"][t:t + 1], prm)
    elif wl.variant.startswith("attn_") and wl.variant != "attn_out":
        # the oracle recomputes the whole perturbed sequence per draw: the
        # sample is the first ATTN_SAMPLE_DRAWS draws of each token
        inp = synth.make_attn_inputs(wl)
        which = wl.variant[-1]
        L, H, D = wl.seq_len, wl.n_heads, wl.n_heads * wl.head_dim
        t0 = time.perf_counter()
        for t in toks:
            b, pos = divmod(t, L)
            rows = slice(b * L, (b + 1) * L)
            Ob, _ = oracle.attention_seq(inp["Q"][rows], inp["K"][rows], inp["V"][rows], H)
            for i in range(ATTN_SAMPLE_DRAWS):
                eps = oracle.gaussians(wl.seed, t, np.arange(i, i + 1), np.arange(D),
                                       oracle.attn.WHICH_TAG[which])
                oracle.attn_draws(inp["Q"][rows], inp["K"][rows], inp["V"][rows], Ob,
                                  inp["E"][rows], H, pos, which, eps, float(np.float32(wl.sigma)))
        return len(toks) * ATTN_SAMPLE_DRAWS, time.perf_counter() - t0
    else:
        inp = synth.make_mlp_inputs(wl)
        t0 = time.perf_counter()
        for t in toks:
            prm = oracle.Params(T=1, d=wl.d, V=wl.V, d_ff=wl.d_ff, K=wl.K, sigma=wl.sigma,
                                seed=wl.seed, token_offset=t)
            if wl.variant == "attn_out":
                oracle.attn_out_grad(inp["X"][t:t + 1], inp["O"][t:t + 1], inp["W_up"],
                                     inp["W_down"], inp["W_head"], inp["targets"][t:t + 1], prm)
            else:
                fn = oracle.mlp_down_grad if wl.variant == "mlp_down" else oracle.mlp_grad
                fn(inp["X"][t:t + 1], inp["W_up"], inp["W_down"], inp["W_head"],
                   inp["targets"][t:t + 1], prm)
    return len(toks) * wl.K, time.perf_counter() - t0


def cpu_baseline(name: str, budget_tokens: int = 0) -> dict:
    """Time the oracle as it stands on a bounded token sample.

    The sample is spread over spawned single-threaded worker processes (one
    per host core, at most 16); each worker times only its oracle calls and
    the sample's throughput is tokens x K / the slowest worker's time."""
    import multiprocessing as mp
    import synth
    wl = synth.CONFIGS[name]
    attn = wl.variant.startswith("attn_") and wl.variant != "attn_out"
    # attention oracle workers hold a few (heads x L x L) fp64 arrays each
    cores = max(1, min(os.cpu_count() or 1, 8 if attn else 16))
    ntok = min(budget_tokens or cores, wl.T)
    toks = [int(t) for t in np.linspace(0, wl.T - 1, ntok).round()] if ntok > 1 else [0]
    chunks = [(name, toks[i::cores]) for i in range(cores) if toks[i::cores]]
    saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS",
                                            "MKL_NUM_THREADS")}
    for k in saved:
        os.environ[k] = "1"
    try:
        with mp.get_context("spawn").Pool(len(chunks)) as pool:
            res = pool.map(_oracle_tokens, chunks, chunksize=1)
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    done = sum(r[0] for r in res)       # token-draws
    dt = max(r[1] for r in res)
    value = done / dt
    what = (f"{len(toks)} tokens x the first {ATTN_SAMPLE_DRAWS} draws" if attn
            else f"{len(toks)} tokens x all {wl.K} draws")
    return {"value": value, "unit": UNIT, "cores": len(chunks), "kind": "oracle",
            "host_cores": os.cpu_count(), "cpu_model": _cpu_model(), "seconds": dt,
            "sample": f"{what} of {name}, fp64 NumPy oracle, "
                      f"{len(chunks)} spawned single-threaded workers on a host of "
                      f"{os.cpu_count()} cores, slowest {dt:.1f} s"}


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ----------------------------------------------------------------------------- helpers
def _dist_init():
    """One rank per GPU: the rank's device is made current before the NCCL
    group is created, and the group is bound to it (its communicator is set
    up at once, so a failure shows here rather than in the first step)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def _max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The largest x over all ranks (every rank returns it); the device is the
    process group's (cuda under NCCL)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world):
    import torch
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def _alu_roofline(wl, draw_ms: float, peaks) -> dict:
    """ALU-issue roofline of the draw kernel: algorithmic elements x the minimum
    issue slots per element / time, against every lane issuing each clock; the
    SFU (exp) ceiling and the second instruction count are reported beside it.
    Full-vocabulary draws generate the noise once (one pass) or twice (a
    reward pass, then a g pass, where no one-pass plan fits); the algorithmic
    count is one generation."""
    if wl.S > 0:
        elems = wl.T * wl.K * (wl.S + 1)
    else:
        elems = wl.T * wl.K * wl.V
    t = draw_ms * 1e-3
    f = float(peaks.get("sm_max_mhz", 1965.0)) * 1e6
    peak = SM_COUNT * LANES_PER_SM * f / 1e12
    achieved = elems * ALU_OPS_PER_ELEM / t / 1e12                   # T lane-ops/s
    alt = elems * ALU_OPS_PER_ELEM_WITH_ACCUMULATE / t / 1e12
    sfu_peak = SM_COUNT * SFU_PER_SM * f / 1e12                        # T exp/s
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Tops/s",
            "frac": achieved / peak, "traffic": None,
            "kernel": "subset_draws" if wl.S > 0 else "full_draws",
            "elements": elems, "ops_per_element": ALU_OPS_PER_ELEM, "kernel_ms": draw_ms,
            "peak_basis": f"{SM_COUNT} SMs x {LANES_PER_SM} lanes x {f / 1e6:.0f} MHz (sm_max_mhz)",
            "with_accumulate": {"ops_per_element": ALU_OPS_PER_ELEM_WITH_ACCUMULATE,
                                "achieved": alt, "frac": alt / peak},
            "sfu": {"exp_per_element": 1, "achieved": elems / t / 1e12, "peak": sfu_peak,
                    "unit": "Texp/s", "frac": elems / t / 1e12 / sfu_peak,
                    "peak_basis": f"{SM_COUNT} SMs x {SFU_PER_SM} SFU lanes x {f / 1e6:.0f} MHz"}}


def _attn_roofline(wl, draws_ms: float, peaks) -> dict:
    """Roofline of the attention draw stage. Query and key noise: tensor-core
    products plus a CUDA-core epilogue, bound by the larger of the two times
    (the CUDA-core side here); value noise: CUDA cores only."""
    L, H, dh = wl.seq_len, wl.n_heads, wl.head_dim
    rows = (wl.T // L) * L * (L + 1) // 2 if wl.variant in ("attn_q", "attn_k") else 0
    ops = wl.K * H * (rows * ATTN_OPS_PER_ROW + wl.T * dh * ATTN_OPS_PER_NOISE)
    flops = ATTN_TC_FLOPS_PER_ROW_DH * dh * wl.K * H * rows
    t = draws_ms * 1e-3
    f = float(peaks.get("sm_max_mhz", 1965.0)) * 1e6
    peak = SM_COUNT * LANES_PER_SM * f / 1e12
    tc_peak = float(peaks.get("bf16_tflops", 1640.9))   # fp16 runs at the bf16 rate
    roof = {"bound": "alu", "achieved": ops / t / 1e12, "peak": peak, "unit": "Tops/s",
            "frac": ops / t / 1e12 / peak, "traffic": None, "kernel": "attn_draws", "ops": ops,
            "kernel_ms": draws_ms,
            "ops_basis": (f"K H (rows visited x {ATTN_OPS_PER_ROW} + T d_h x "
                          f"{ATTN_OPS_PER_NOISE}) on CUDA cores"),
            "peak_basis": f"{SM_COUNT} SMs x {LANES_PER_SM} lanes x {f / 1e6:.0f} MHz (sm_max_mhz)"}
    if flops:
        roof["tensor"] = {"flops": flops, "achieved_tflops": flops / t / 1e12,
                          "peak_tflops": tc_peak, "frac": flops / t / 1e12 / tc_peak,
                          "basis": f"{ATTN_TC_FLOPS_PER_ROW_DH} d_h flops per (draw, head, row): "
                                   "fp16 hi/lo split, three products; peak = measured bf16 burst"}
    return roof


def _mlp_flops_per_row(wl) -> tuple:
    """(algorithmic, executed) flops of the perturbed pass per (token, draw):
    the method's GEMMs dh = da W_down^T (up), du = (sigma eps) W_up^T and dh
    (attention output projection) and dz = dh W_head^T. dz and dh contract
    the hi planes of their bf16 operands only (the lo planes' first-order
    effects are added per row: 2d flops, and 2 d_ff where dh comes from da);
    du contracts both planes of sigma eps, twice its depth. Above sigma = 0.05
    every contraction takes both planes."""
    d, dff, V = wl.d, wl.d_ff, wl.V
    alg = exe = 2.0 * d * V + 2.0 * d
    if wl.variant in ("mlp", "attn_out"):
        alg += 2.0 * dff * d
        exe += 2.0 * dff * d + 2.0 * dff
    if wl.variant == "attn_out":
        alg += 2.0 * d * dff
        exe += 2.0 * 2.0 * d * dff
    alg -= 2.0 * d
    if wl.sigma > 0.05:  # both planes everywhere, no corrections
        exe = 2.0 * alg
    return alg, exe


def _mlp_roofline(wl, perturbed_ms: float, peaks) -> dict:
    """Tensor-core roofline of the MLP-block perturbed pass: the method's flops
    per (token, draw) over the stage time, against the sustained bf16 peak (a
    pass of hundreds of milliseconds runs under the power cap); the flops the
    GEMMs execute are reported beside it."""
    alg, exe = _mlp_flops_per_row(wl)
    rows = wl.T * wl.K
    t = perturbed_ms * 1e-3
    peak = float(peaks.get("bf16_tflops_sustained", 1416.7))
    return {"bound": "tensor", "achieved": alg * rows / t / 1e12, "peak": peak, "unit": "TFLOP/s",
            "frac": alg * rows / t / 1e12 / peak, "traffic": None, "kernel": "perturbed GEMMs",
            "flops": alg * rows, "kernel_ms": perturbed_ms,
            "flops_basis": "algorithmic flops of the perturbed pass's GEMMs per (token, draw)",
            "peak_basis": "measured bf16 sustained (power-capped) peak",
            "executed": {"flops": exe * rows, "achieved": exe * rows / t / 1e12,
                         "frac": exe * rows / t / 1e12 / peak,
                         "basis": ("dz and dh on the hi planes of their operands plus a "
                                   "correction per row; du on both planes of sigma eps")}}


def _gemm_report(flops: float, ms: float, peaks) -> dict:
    """Algorithmic TFLOP/s of one GEMM stage and its share of the measured bf16 peaks."""
    tf = flops / (ms * 1e-3) / 1e12
    return {"ms": ms, "tflops": tf,
            "frac_burst": tf / float(peaks.get("bf16_tflops", 1640.9)),
            "frac_sustained": tf / float(peaks.get("bf16_tflops_sustained", 1416.7))}


L2_NOTE = ("GPU arm: a 256 MiB write flushes L2 between timed steps; "
           "the oracle arm runs on the host cores")


def _config(args, wl, world: int) -> dict:
    """The workload of a JSON line (the same dict on both arms)."""
    cfg = {"workload": args.config, "T_per_gpu": wl.T, "d": wl.d, "V": wl.V, "K": wl.K,
           "S": wl.S, "sigma": wl.sigma, "dtype_inputs": wl.dtype, "d_ff": wl.d_ff, "l2": L2_NOTE,
           "parallelism": (f"dp{world}: token-sharded, G_W summed by NCCL all-reduce"
                           if world > 1 else "dp1")}
    if wl.seq_len:
        cfg.update(seq_len=wl.seq_len, n_heads=wl.n_heads, head_dim=wl.head_dim)
    return cfg


# ----------------------------------------------------------------------------- main arms
def run_reference(args):
    """The oracle on the host, each step a bounded token sample of the workload
    (all K draws of each sampled token): value = the sample's token-draws / its
    time, ms_per_step = the sample's measured time. Rank 0 alone runs."""
    world, rank = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synth
    wl = synth.CONFIGS[args.config]
    per_step, secs = [], []
    cb = None
    for _ in range(args.warmup):
        cpu_baseline(args.config, budget_tokens=args.ref_tokens)
    for _ in range(args.steps):
        cb = cpu_baseline(args.config, budget_tokens=args.ref_tokens)
        per_step.append(cb["value"])
        secs.append(cb["seconds"])
    value = statistics.median(per_step)
    cb["value"] = value
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * statistics.median(secs),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": _config(args, wl, world),
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_dust(args):
    import numpy as np
    import torch
    import synth
    import zeroth_order_transformer_dust_b200 as dust

    world, rank, local = _dist_init()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks, peak_kind = _peaks()
    wl = synth.CONFIGS[args.config]
    ctx = dust.Context(local)
    t_off = rank * wl.T

    if wl.variant == "head":
        inp = synth.make_head_inputs(wl)
        tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        H = torch.from_numpy(inp["H"]).to(tdt)
        W = torch.from_numpy(inp["W"]).to(tdt)
        y = torch.from_numpy(inp["targets"]).to(torch.int32)
        Hd, Wd, yd = H.to(dev), W.to(dev), y.to(dev)
        outs = {"G": torch.empty(wl.V, wl.d, dtype=torch.float32, device=dev),
                "loss": torch.empty(wl.T, dtype=torch.float32, device=dev)}

        from zeroth_order_transformer_dust_b200.parallel import allreduce_weight_grad

        def step():
            ctx.head_grad(Hd, Wd, yd, K=wl.K, sigma=wl.sigma, S=wl.S, seed=wl.seed,
                          token_offset=t_off, out=outs, asynchronous=True)
            allreduce_weight_grad(outs["G"])   # G_W of all ranks' tokens (no-op at N = 1)
    elif wl.seq_len:
        inp = synth.make_attn_inputs(wl)
        tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        X = torch.from_numpy(inp["X"]).to(tdt).to(dev)
        Qd, Kd, Vd, Ed = (torch.from_numpy(inp[k]).to(dev) for k in ("Q", "K", "V", "E"))
        D = wl.n_heads * wl.head_dim
        outs = {"G": torch.empty(D, wl.d, dtype=torch.float32, device=dev)}
        which = wl.variant[-1]

        def step():
            ctx.attn_grad(X, Qd, Kd, Vd, Ed, seq_len=wl.seq_len, n_heads=wl.n_heads,
                          which=which, K=wl.K, sigma=wl.sigma, seed=wl.seed, token_offset=t_off,
                          out=outs)
            from zeroth_order_transformer_dust_b200.parallel import allreduce_weight_grad
            allreduce_weight_grad(outs["G"])
    else:
        inp = synth.make_mlp_inputs(wl)
        X, Wu, Wdn, Wh = (torch.from_numpy(inp[k]).to(torch.bfloat16).to(dev)
                          for k in ("X", "W_up", "W_down", "W_head"))
        yd = torch.from_numpy(inp["targets"]).to(torch.int32).to(dev)
        gshape = {"mlp": (wl.d_ff, wl.d), "mlp_down": (wl.d, wl.d_ff)}.get(wl.variant, (wl.d, wl.d))
        outs = {"G": torch.empty(*gshape, dtype=torch.float32, device=dev),
                "loss": torch.empty(wl.T, dtype=torch.float32, device=dev)}

        layer = {"mlp_down": "down", "attn_out": "attn_out"}.get(wl.variant, "up")
        Od = torch.from_numpy(inp["O"]).to(torch.bfloat16).to(dev) if layer == "attn_out" else None

        def step():
            ctx.mlp_grad(X, Wu, Wdn, Wh, yd, K=wl.K, sigma=wl.sigma, seed=wl.seed,
                         token_offset=t_off, out=outs, layer=layer, O=Od)
            from zeroth_order_transformer_dust_b200.parallel import allreduce_weight_grad
            allreduce_weight_grad(outs["G"])

    # L2 flush buffer (larger than the 126 MB L2), written between timed steps
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        step()
    ctx.check()
    _barrier(world)

    ctx.set_stage_timing(True)
    clocks = ClockSampler()
    clocks.start()
    launches0 = ctx.kernel_launches
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    stage_ms = []
    _barrier(world)
    for k in range(args.steps):
        flush.fill_(k & 0xFF)
        ev[k][0].record(stream)
        step()
        ev[k][1].record(stream)
        stage_ms.append(ctx.stage_times())
    _barrier(world)
    clk = _merge_clocks(clocks.stop(), world)
    launches = ctx.kernel_launches - launches0
    ctx.check()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    ms = _max_over_ranks(sum(step_ms) / len(step_ms), world)
    ctx.set_stage_timing(False)

    stages = {}
    for s in stage_ms:
        for k_, v in s.items():
            stages.setdefault(k_, []).append(v)
    stages = {k_: sum(v) / len(v) for k_, v in stages.items()}

    value = world * wl.token_draws / (ms * 1e-3)

    # end to end through the host-buffer C-ABI call (head workloads)
    e2e = None
    if wl.variant == "head" and not args.no_e2e:
        Hp, Wp, yp = H.pin_memory(), W.pin_memory(), y.pin_memory()
        hout = {"G": torch.empty(wl.V, wl.d, dtype=torch.float32).pin_memory(),
                "loss": torch.empty(wl.T, dtype=torch.float32).pin_memory()}
        ctx.head_grad_host(Hp, Wp, yp, K=wl.K, sigma=wl.sigma, S=wl.S, seed=wl.seed,
                           token_offset=t_off, out=hout)
        _barrier(world)
        times = []
        for k in range(max(1, min(args.steps, 3))):
            flush.fill_(k & 0xFF)
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            ctx.head_grad_host(Hp, Wp, yp, K=wl.K, sigma=wl.sigma, S=wl.S, seed=wl.seed,
                               token_offset=t_off, out=hout)
            times.append(time.perf_counter() - t0)
        e_ms = _max_over_ranks(1e3 * sum(times) / len(times), world)
        h2d = Hp.numel() * Hp.element_size() + Wp.numel() * Wp.element_size() + yp.numel() * 4
        d2h = hout["G"].numel() * 4 + hout["loss"].numel() * 4
        e2e = {"value": world * wl.token_draws / (e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms}

    roof = None
    draw_key = "subset_draws" if wl.S > 0 else None
    if wl.variant == "head":
        if wl.S > 0:
            draw_ms = stages.get("subset_draws")
        else:  # one pass, or the reward and g passes where no one-pass plan fits
            draw_ms = stages.get("full_draws") or stages.get("reward", 0) + stages.get("g", 0)
        if draw_ms:
            roof = _alu_roofline(wl, draw_ms, peaks)
            roof["peak_kind"] = peak_kind
            if wl.S > 0 and args.config == PROFILED_SUBSET_WORKLOAD:
                roof["traffic"] = SUBSET_DRAM_BYTES_PER_TOKEN * wl.T
                roof["traffic_basis"] = ("ncu DRAM bytes of a 2048-token launch, scaled by "
                                         "tokens to this launch")
    if wl.seq_len and stages.get("draws"):
        roof = _attn_roofline(wl, stages["draws"], peaks)
        roof["peak_kind"] = peak_kind
    if wl.variant in ("mlp", "mlp_down", "attn_out") and stages.get("perturbed"):
        roof = _mlp_roofline(wl, stages["perturbed"], peaks)
        roof["peak_kind"] = peak_kind
    # the two dense contractions of the head, 2 T d V flops each (G_W: the
    # stage includes H's conversion to fp16, two small kernels)
    gemm_flops = 2.0 * wl.T * wl.d * wl.V
    extra = {}
    if wl.variant == "head":
        gemms = {key: _gemm_report(gemm_flops, stages[key], peaks)
                 for key in ("clean_gemm", "gw_gemm") if stages.get(key)}
        if gemms:
            extra["gemms"] = gemms

    # cos(g, exact gradient) against K, outside the timed region (head workloads at N = 1)
    align = None
    if wl.variant == "head" and world == 1 and not args.no_alignment and wl.K >= 64:
        from zeroth_order_transformer_dust_b200.alignment import cosine_vs_k
        ks = [k for k in (64, 256, 1024, 4096, 16384) if k <= wl.K]
        align = cosine_vs_k(ctx, Hd, Wd, yd, ks=ks, sigma=wl.sigma, S=wl.S, seed=wl.seed)
        torch.cuda.empty_cache()

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(args.config, budget_tokens=args.ref_tokens)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic",
                "config": _config(args, wl, world),
                "stage_ms": stages, "gpu_launches": launches, "e2e": e2e, "roofline": roof,
                "cpu_baseline": cb, "clocks": clk, "alignment": align, **extra}
        print(json.dumps(line), flush=True)
    ctx.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def _launch_ranks(argv, n: int) -> int:
    """Start n ranks of this script on this node (one process per GPU) with
    torch.distributed.run and return its exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="large_subset_bf16")
    ap.add_argument("--impl", default="dust", choices=["dust", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-alignment", action="store_true",
                    help="skip the cosine-versus-K report of the head estimator")
    ap.add_argument("--ref-tokens", type=int, default=0,
                    help="oracle sample size in tokens (default: one per host core, at most 16)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="run only the first N tokens of the workload (profiling slices)")
    args = ap.parse_args(argv)
    world_env = os.environ.get("WORLD_SIZE")
    if world_env is None and args.gpus > 1:
        return _launch_ranks(sys.argv[1:] if argv is None else list(argv), args.gpus)
    if world_env is not None and int(world_env) != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but the launcher started WORLD_SIZE={world_env} ranks",
              file=sys.stderr)
        return 2
    if args.tokens:
        import synth
        wl = synth.CONFIGS[args.config]
        synth.CONFIGS[args.config] = wl.with_(T=min(args.tokens, wl.T))
    if args.impl == "reference":
        return run_reference(args)
    return run_dust(args)


if __name__ == "__main__":
    sys.exit(main())
