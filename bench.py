"""Benchmark of the quantized attention hot path on B200.

One step = the whole path on one batch of synthetic input already resident
in HBM: quantization of Q and K (NVFP4, or FP8 per 128-token tile), per-channel
FP8 quantization of V, and the fused attention forward. The default workload
is the sequence sweep's longest single-GPU point: B=1, H=32, N=131072, d=128,
dense, x20 outlier channels, QK^T in NVFP4 and PV in FP8 (2.8e14 flops a
step). W untimed warm-up steps, then exactly K timed steps bracketed by a
barrier and a device synchronize, timed with CUDA events on the launching
stream; multi-GPU runs take the max over ranks. Rank 0 prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
  python bench.py --sweep     # sequence-length sweep, one JSON line per configuration

Workloads: long_seq_128k_nvfp4 (default), long_seq_128k_fp8, llm_prefill_causal,
video_dense_fp8, video_sta_fp8, tiny_nvfp4.

``--impl reference`` times the CPU oracle (the only other implementation of
this path) on a bounded sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "quantized attention fwd TFLOPS & % of B200 FP4/FP8 peak; quantize HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# nominal dense ratios to bf16 (B200: bf16 2.25, fp8 4.5, fp4 9 PFLOP/s)
FP8_RATIO, FP4_RATIO = 2.0, 4.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def strip_comments(text: str) -> str:
    """C++ source without its // and /* */ comments, trailing blanks and
    empty lines (string and character literals are kept whole)."""
    out, i, n, in_block = [], 0, len(text), False
    line = []
    while i < n:
        c = text[i]
        if in_block:
            if text.startswith("*/", i):
                in_block, i = False, i + 2
            else:
                if c == "\n":
                    out.append("".join(line)); line = []
                i += 1
            continue
        if text.startswith("//", i):
            while i < n and text[i] != "\n":
                i += 1
            continue
        if text.startswith("/*", i):
            in_block, i = True, i + 2
            continue
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            line.append(text[i:j + 1]); i = j + 1
            continue
        if c == "\n":
            out.append("".join(line)); line = []
        else:
            line.append(c)
        i += 1
    out.append("".join(line))
    return "\n".join(ln.rstrip() for ln in out if ln.strip())


def kernel_source_hash() -> str:
    """First 16 hex digits of sha256 over the code of attn_fwd.cu and
    sm100.cuh (comments and blank lines removed): ties a DRAM traffic record
    to the kernel code it was captured on, so that a change of wording in a
    comment does not void it."""
    import hashlib
    h = hashlib.sha256()
    for src in ("attn_fwd.cu", "sm100.cuh"):
        with open(os.path.join(ROOT, "precision_attention_nvfp4_b200", "csrc", src), encoding="utf-8") as f:
            h.update(strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """Per-launch DRAM bytes (read + write) of the attention kernel on this
    workload from the committed ncu record, or None when there is none or the
    kernel sources changed since that capture."""
    path = os.path.join(ROOT, "profiles", "attn_fwd_traffic.txt")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash()
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and not line.startswith("#") and parts[0] == workload and parts[1] == want:
                return float(parts[2])
    return None


def executed_block_pairs(w: workloads.Workload) -> int:
    """128x128 (query block, key block) pairs the kernel computes per head."""
    nblk = (w.N + 127) // 128
    if w.sparse:
        import precision_attention_nvfp4_b200 as fp
        tg = tuple(a // b for a, b in zip(w.video, w.sta_tile))
        return fp.sta_plan(tg, w.sta_tile, w.sta_window).nnz
    return nblk * (nblk + 1) // 2 if w.causal else nblk * nblk


def quant_bytes_one_pass(w: workloads.Workload, pv_format: str = "fp8") -> float:
    """The lower bound of the step's quantization bytes: every bf16 input read
    once and every code and scale written once (the amax passes left out)."""
    n = w.B * w.H * w.N * w.d
    qk = 2 * n * ((2 + 0.5 + 1.0 / 16) if w.qk_format == "nvfp4" else (2 + 1))
    v = n * ((2 + 0.5 + 1.0 / 16) if pv_format == "nvfp4" else (2 + 1))
    return qk + v


def quant_bytes(w: workloads.Workload, pv_format: str = "fp8") -> float:
    """Algorithmic HBM bytes of one step's quantization (two-pass amax)."""
    n = w.B * w.H * w.N * w.d
    if w.qk_format == "nvfp4":
        qk = 2 * n * (2 + 2 + 0.5 + 1.0 / 16)   # amax read + quant read + codes + scales
    else:
        qk = 2 * n * (2 + 1)                    # single pass per 128-token tile
    if pv_format == "nvfp4":
        v = n * (2 + 2 + 0.5 + 1.0 / 16)        # tensor amax pass + quant pass (codes + scales)
    else:
        v = n * (2 + 2 + 1)                     # channel amax pass + quant pass
    return qk + v


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons (every 100 ms, with a
    host timestamp per sample) from before the warm-up to the end of the
    timed region; stop() summarises the samples inside the timed window."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.samples = []  # (host time, csv line)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        # wait for the first sample (3 s at most) so that nvidia-smi's
        # start-up falls before the warm-up: inside a short timed region it
        # once coincided with steps ten times their usual length
        t_end = time.time() + 3.0
        while not self.samples and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self, t0: float, t1: float):
        """Summary of the samples taken between host times t0 and t1 (the
        timed region); when that window holds none (a region shorter than the
        sampling period), of all samples since start()."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)  # let the sample that straddles t1 arrive
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        inside = [ln for t, ln in self.samples if t0 <= t <= t1]
        window = "timed region"
        if not inside:
            inside = [ln for _, ln in self.samples]
            window = "warm-up and timed region (timed region shorter than the 100 ms sampling period)"
        sm, mx, power, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in inside:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
                power.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "sm_mhz_min": min(sm) if sm else None, "power_w_max": max(power) if power else None,
                "reasons": sorted(reasons), "samples": len(sm), "window": window}


def oracle_sample(w: workloads.Workload, q, k, v, heads, row_sets, budget_s: float = 0.0, exact: bool = False,
                  cache=None):
    """Run the oracle (as it stands) on a bounded sample of the workload.

    heads: (batch*head) indices; row_sets: arrays of query rows, each within
    one 128-row block. q, k, v are the full CPU bf16 tensors, in the order the
    kernel computes in (tile-major for sliding-tile workloads). The oracle
    quantizes each sampled head once (its K and V serve every query row), then
    runs the attention rows. With budget_s > 0 the sample stops after the
    first row set that ends past the budget. With exact, each sampled row set
    also runs through unquantized fp64 attention (untimed) for the cosine.
    cache (a dict) keeps each head's quantized operands across calls; a head
    found there is not quantized (nor timed) again.

    Returns a dict: flops, attn_s, quant_s (seconds for the sampled heads'
    quantization), done [(head, rows)], out {(head, i): oracle rows}, exact
    {(head, i): fp64 rows}."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import parity
    from oracle import attention as oatt
    kb = None
    if w.sparse:
        from oracle import sta
        kb = sta.block_lists(w.video, w.sta_tile, w.sta_window)
    B, H, N, d = q.shape
    res = {"flops": 0.0, "attn_s": 0.0, "quant_s": 0.0, "done": [], "out": {}, "exact": {}}
    t_start = time.perf_counter()
    for h in heads:
        if cache is not None and h in cache:
            qh, kh, vh = cache[h]
        else:
            t0 = time.perf_counter()
            qh, kh, vh = parity.oracle_operands(q, k, v, w.qk_format, [h])
            res["quant_s"] += time.perf_counter() - t0
            if cache is not None:
                cache[h] = (qh, kh, vh)
        for i, rows in enumerate(row_sets):
            t0 = time.perf_counter()
            o, _ = oatt.attention_rows(qh[0], kh[0], vh[0], rows, causal=w.causal, key_blocks=kb)
            res["attn_s"] += time.perf_counter() - t0
            if kb is not None:
                keys = np.full(len(rows), 128 * len(kb[int(rows[0]) // 128]))
            else:
                keys = (rows + 1) if w.causal else np.full(len(rows), N)
            res["flops"] += float(np.sum(4.0 * keys * d))
            res["done"].append((h, rows))
            res["out"][(h, i)] = o
            if exact:
                qe, ke, ve = (t.reshape(B * H, N, d)[h].double().numpy() for t in (q, k, v))
                res["exact"][(h, i)], _ = oatt.attention_rows(qe, ke, ve, rows, causal=w.causal, key_blocks=kb,
                                                              quantize_p=False)
            if budget_s > 0 and time.perf_counter() - t_start > budget_s:
                return res
    return res


def sample_rows(w: workloads.Workload, qblocks, target_flops: float = 2e9):
    """Query rows per sampled block: as many of the block's first rows as make
    about target_flops of oracle work (8 to 128 rows)."""
    keys = w.N if not w.causal else max(1, w.N // 2)
    n = int(min(128, max(8, target_flops / (4.0 * keys * w.d))))
    return [np.arange(qb * 128, min(w.N, qb * 128 + n)) for qb in qblocks]


def oracle_rate(res, N: int) -> float:
    """Oracle TFLOPS on a sample: the attention rows' flops over their time
    plus the sampled rows' share of the per-head quantization time (each
    head's quantization serves all N of its rows)."""
    rows = sum(len(r) for _, r in res["done"])
    heads = len({h for h, _ in res["done"]})
    t = res["attn_s"] + res["quant_s"] * rows / (heads * N)
    return res["flops"] / t / 1e12


def cosine(a: np.ndarray, b: np.ndarray) -> float:
    a, b = a.astype(np.float64).ravel(), b.astype(np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def run_reference(args, w):
    """CPU oracle arm: each step a bounded sample of the workload (about 2e9
    flops of attention rows of one head), on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    q, k, v = workloads.make_qkv(w, heads=1, batch=1)
    nblk = (w.N + 127) // 128
    rows = sample_rows(w, [nblk - 1])
    # one quantization of the head serves every step (as the inputs of the
    # native arm stay resident); its time is charged per row sampled
    tot = {"flops": 0.0, "attn_s": 0.0, "quant_s": 0.0, "done": []}
    cache = {}
    quant_s = oracle_sample(w, q, k, v, [0], rows, cache=cache)["quant_s"]
    for _ in range(args.warmup):
        oracle_sample(w, q, k, v, [0], rows, cache=cache)
    for _ in range(args.steps):
        r = oracle_sample(w, q, k, v, [0], rows, cache=cache)
        for key in ("flops", "attn_s"):
            tot[key] += r[key]
        tot["done"] += r["done"]
    tot["quant_s"] = quant_s
    value = oracle_rate(tot, w.N)
    # per step: the sampled rows' attention plus their share of the quantization
    step_s = tot["flops"] / args.steps / (value * 1e12)
    sample = (f"{len(rows[0])} query rows of block {nblk - 1} of one head of {w.name} per step (fp64 numpy "
              f"oracle; the head's quantization, {quant_s:.1f} s, charged per row: it serves all {w.N} rows)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * step_s,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(w),
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": host_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def choose_peak(peaks: dict, clk: dict, timed_s: float, qk: str, pv: str):
    """Tensor peak of the attention kernel (TFLOP/s) for its MMA dtypes.

    The measured bf16 figure times the nominal FP8 / FP4 ratios; both MMAs do
    2d flops per score, so a mixed path takes the harmonic mean. The
    sustained bf16 figure was measured under the power cap at a lowered SM
    clock; it applies to a timed region of a second or more that itself ran
    capped or below the maximum clock. A shorter region, or one whose clock
    record shows the maximum clock and no power cap, takes the burst figure
    (measured at the maximum clock). Returns (peak, burst peak, bf16 figure
    used, sustained?, capped?)."""
    capped = bool("sw_power_cap" in clk.get("reasons", []) or
                  (clk.get("sm_mhz") is not None and clk.get("sm_max_mhz") and
                   clk["sm_mhz"] < 0.95 * clk["sm_max_mhz"]))
    sustained = timed_s >= 1.0 and capped and "bf16_tflops_sustained" in peaks
    bf16 = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    p8, p4 = bf16 * FP8_RATIO, bf16 * FP4_RATIO
    p_qk = p4 if qk == "nvfp4" else p8
    p_pv = p4 if pv == "nvfp4" else p8
    peak = 2.0 / (1.0 / p_qk + 1.0 / p_pv)
    return peak, peak * peaks["bf16_tflops"] / bf16, bf16, sustained, capped


# Softmax cycles per 128x128 block and SM, at the split of the exponentials
# between MUFU and the FMA-pipe polynomial where the two balance (5 of 16 exp2
# pairs on the polynomial): MUFU 16,384 * 11/16 / 16 = 704, issue slots ~725
# (about 2,900 warp instructions of softmax work at one a clock per
# sub-partition). The larger binds. This is a bound of the work, not of the
# kernel's own split (4 of 16, which measured faster).
SOFTMAX_CYCLES_PER_BLOCK = 725.0


def alu_roofline(w: workloads.Workload, achieved_tflops: float, peaks: dict) -> dict:
    """The attention kernel against its ALU-side bound: the exponentials of
    a 128x128 block take SOFTMAX_CYCLES_PER_BLOCK cycles of an SM whatever d
    is, so the bound in TFLOP/s is 4*128*128*d flops per block over that
    time on every SM at the maximum clock."""
    mhz = peaks.get("sm_max_mhz", 1965.0)
    peak = 4.0 * 128 * 128 * w.d * 148 * mhz * 1e6 / SOFTMAX_CYCLES_PER_BLOCK / 1e12
    return {"bound": "alu", "achieved": achieved_tflops, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved_tflops / peak,
            "peak_source": f"derived: {SOFTMAX_CYCLES_PER_BLOCK:.0f} cycles of softmax work per 128x128 block "
                           f"and SM (MUFU ex2 and issue counts), 148 SMs at {mhz:.0f} MHz"}


def rank_env():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 if absent)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(dist, x: float, device) -> float:
    """Max of a per-rank time over all ranks (identity without a process group)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(per_rank_flops: float, world: int, ms_per_step: float) -> float:
    """Whole-job TFLOPS: every rank runs one batch (weak scaling), time = max over ranks."""
    return world * per_rank_flops / (ms_per_step * 1e-3) / 1e12


def config_dict(w):
    c = {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
         "qk": w.qk_format, "pv": "e4m3", "sparse": w.sparse,
         "l2": "inputs larger than L2 (bf16 Q,K,V of the step exceed 126 MB)"}
    if w.sparse:
        c["tokens"] = ("raster (time-major) bf16 in and out; the tile-major permutation runs inside the "
                       "quantize kernels and the attention epilogue")
    if w != workloads.get(w.name):
        c["reduced"] = f"B={w.B} H={w.H} instead of the workload's own (a profiler-sized case)"
    return c


def time_cuda(fn, min_runs: int = 5, budget_ms: float = 1500.0) -> float:
    """Median device time (ms) of fn() over enough runs to fill about budget_ms
    (at least min_runs), after 3 warm-up calls."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    fn()
    e1.record()
    torch.cuda.synchronize()
    one = e0.elapsed_time(e1)
    runs = max(min_runs, min(50, int(budget_ms / max(one, 1e-3))))
    times = []
    for _ in range(runs):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    return float(np.median(times))


def run_sweep(args):
    """Sequence sweep: N in 1K..128K, H = 32, B*H*N = 2^22, d in {64, 128},
    causal and not, NVFP4 QK + FP8 PV against all-FP8. Inputs are drawn on the
    device from a seeded CUDA generator (~N(0,1), four x20 outlier channels per
    head shared by Q and K); every N views the same buffers. One JSON line per
    configuration: attention time, dense-equivalent and executed TFLOPS, the
    fraction of the tensor peak, and the quantization bandwidth."""
    import precision_attention_nvfp4_b200 as fp
    torch.cuda.set_device(0)
    peaks, peak_src = load_peaks()
    bf16 = peaks.get("bf16_tflops", 1590.0)
    p8, p4 = bf16 * FP8_RATIO, bf16 * FP4_RATIO
    gen = torch.Generator(device="cuda").manual_seed(5)
    tokens = 1 << 22
    for d in (64, 128):
        qf = torch.randn(tokens, d, device="cuda", generator=gen)
        kf = torch.randn(tokens, d, device="cuda", generator=gen)
        vf = torch.randn(tokens, d, device="cuda", generator=gen)
        for N in (1024, 4096, 16384, 32768, 65536, 131072):
            B = tokens // (32 * N)
            q = qf.view(B, 32, N, d).clone()
            k = kf.view(B, 32, N, d).clone()
            ch = torch.randperm(d, device="cuda", generator=gen)[:4]
            q[..., ch] *= 20.0
            k[..., ch] *= 20.0
            q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
            v = vf.view(B, 32, N, d).to(torch.bfloat16)
            vq = fp.quantize_fp8(v, "channel")
            for fmt in ("nvfp4", "fp8"):
                if fmt == "nvfp4":
                    qq, kq = fp.quantize_nvfp4(q), fp.quantize_nvfp4(k)
                    quant = lambda: (fp.quantize_nvfp4(q), fp.quantize_nvfp4(k))
                    qbytes = 2 * q.numel() * (2 + 2 + 0.5 + 1 / 16)
                else:
                    qq, kq = fp.quantize_fp8(q, "tile128"), fp.quantize_fp8(k, "tile128")
                    quant = lambda: (fp.quantize_fp8(q, "tile128"), fp.quantize_fp8(k, "tile128"))
                    qbytes = 2 * q.numel() * (2 + 1)
                q_ms = time_cuda(quant)
                for causal in (False, True):
                    out, lse = fp.attention_fwd(qq, kq, vq, causal=causal)
                    ms = time_cuda(lambda: fp.attention_fwd(qq, kq, vq, causal=causal, out=out, lse=lse))
                    err = fp.device_error()
                    w = workloads.Workload("sweep", B=B, H=32, N=N, d=d, causal=causal, qk_format=fmt, seed=5)
                    flops = w.dense_flops()
                    exec_flops = 4.0 * 128 * 128 * d * executed_block_pairs(w) * B * 32
                    peak = 2.0 / (1.0 / p4 + 1.0 / p8) if fmt == "nvfp4" else p8
                    tf = flops / (ms * 1e-3) / 1e12
                    order = None
                    if causal:
                        plan = fp.causal_plan(B * 32, N, d, fmt, "fp8",
                                              sm_count=torch.cuda.get_device_properties(0).multi_processor_count)
                        order = ("pairs" if plan["pairs_per_head"] else
                                 f"groups of {plan['heads_per_group']}" if plan["heads_per_group"] < B * 32
                                 else "longest first")
                    print(json.dumps({
                        "sweep": True, "N": N, "B": B, "H": 32, "d": d, "causal": causal, "qk": fmt,
                        "causal_order": order,
                        "attn_ms": ms, "tflops_dense_eq": tf,
                        "tflops_executed": exec_flops / (ms * 1e-3) / 1e12,
                        "frac_of_peak": tf / peak, "peak_tflops": peak,
                        "peak_source": f"{peak_src} bf16 burst {bf16} x nominal fp8 2x / fp4 4x",
                        "quant_qk_ms": q_ms, "quant_qk_gbs": qbytes / (q_ms * 1e-3) / 1e9,
                        "device_error": err}), flush=True)
            del q, k, v, vq
        del qf, kf, vf
        torch.cuda.empty_cache()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_seq_128k_nvfp4", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3, help="timed end-to-end calls (0: no e2e leg)")
    ap.add_argument("--heads", type=int, default=0,
                    help="run the workload with this many heads (B=1) instead of its own B*H: a smaller "
                         "case of the same kernels for profiler captures; the line says so in config")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--pv-format", default="fp8", choices=["fp8", "nvfp4"],
                    help="P and V in E4M3 (default) or both in NVFP4 with P V on FP4 tensor cores")
    ap.add_argument("--rescale-threshold", type=float, default=0.0,
                    help="conditional softmax rescale threshold tau (log2 units); 0 = exact running max")
    args = ap.parse_args()
    if args.sweep:
        return run_sweep(args)
    w = workloads.get(args.workload)
    if args.heads > 0:
        w = w.scaled(B=1, H=args.heads)
    if args.impl == "reference":
        return run_reference(args, w)

    import precision_attention_nvfp4_b200 as fp
    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier(device_ids=[local])

    def rank_max(x: float) -> float:
        return max_over_ranks(dist, x, "cuda")

    # weak scaling: every rank runs one full batch of the workload. Video
    # tokens of the sliding-tile workload stay in raster order: the fused
    # path permutes them inside the kernels.
    mask, video = None, None
    if w.sparse:
        tg = tuple(a // b for a, b in zip(w.video, w.sta_tile))
        mask = fp.sta_plan(tg, w.sta_tile, w.sta_window).to("cuda")
        video = fp.VideoLayout(w.video, w.sta_tile)
    if w.device_draw:
        q, k, v = workloads.make_qkv(w, device="cuda")
        q_h, k_h, v_h = q.cpu(), k.cpu(), v.cpu()
    else:
        q_h, k_h, v_h = workloads.make_qkv(w, tile_major=video is None)
        q, k, v = q_h.cuda(), k_h.cuda(), v_h.cuda()
    stream = torch.cuda.current_stream()

    def step(ev_pair=None):
        if args.pv_format == "fp8":
            # Q, K and V in four fused launches
            qq, kq, vq = fp.quantize_qkv(q, k, v, w.qk_format, video=video)
        else:
            if w.qk_format == "nvfp4":
                qq, kq = fp.quantize_nvfp4(q, video=video), fp.quantize_nvfp4(k, video=video)
            else:
                qq, kq = fp.quantize_fp8(q, "tile128", video=video), fp.quantize_fp8(k, "tile128", video=video)
            vq = fp.quantize_nvfp4_v(v, video=video)
        if ev_pair is not None:
            ev_pair[0].record(stream)
        out, lse = fp.attention_fwd(qq, kq, vq, causal=w.causal, tile_mask=mask, video=video,
                                    rescale_threshold=args.rescale_threshold)
        if ev_pair is not None:
            ev_pair[1].record(stream)
        return out

    # clocks are sampled from before the warm-up; the summary keeps the
    # samples inside the timed region
    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert fp.device_error() == 0

    attn_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t_host0 = time.time()
    start.record(stream)
    for i in range(args.steps):
        out = step(attn_events[i])
    end.record(stream)
    torch.cuda.synchronize()
    t_host1 = time.time()
    barrier()
    clk = clocks.stop(t_host0, t_host1)
    ms_total = start.elapsed_time(end)
    ms_total = rank_max(ms_total)
    attn_ms = float(np.mean([a.elapsed_time(b) for a, b in attn_events]))
    attn_ms = rank_max(attn_ms)
    err = fp.device_error()
    out_last = out.float().cpu() if rank == 0 else None

    pairs = executed_block_pairs(w)
    exec_flops = 4.0 * 128 * 128 * w.d * pairs * w.B * w.H
    # Algorithmic flops: 4*B*H*N^2*d, halved under the causal mask; under the
    # sliding-tile mask only the allowed (tile, tile) token pairs, which the
    # mask makes whole 128x128 blocks, so exactly the executed blocks.
    flops = exec_flops if w.sparse else w.dense_flops()
    ms_step = ms_total / args.steps
    value = aggregate_value(flops, world, ms_step)
    peaks, peak_src = load_peaks()
    timed_s = ms_total * 1e-3
    peak, peak_burst, bf16, sustained, capped = choose_peak(peaks, clk, timed_s, w.qk_format, args.pv_format)
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12
    quant_ms = ms_step - attn_ms
    quant_gbs = quant_bytes(w, args.pv_format) / (quant_ms * 1e-3) / 1e9

    # end to end through the public API: pinned host bf16 in, host bf16 out
    e2e = None
    if args.e2e_steps > 0 and (rank == 0 or world > 1):
        qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
        out_h = torch.empty(q_h.shape, dtype=torch.bfloat16, pin_memory=True)
        lse_h = torch.empty(q_h.shape[:3], dtype=torch.float32, pin_memory=True)
        fp.attention(qp, kp, vp, qk_format=w.qk_format, causal=w.causal, tile_mask=mask, out_host=out_h,
                     lse_host=lse_h, video=video, rescale_threshold=args.rescale_threshold,
                     pv_format=args.pv_format)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        e0.record(stream)
        for _ in range(args.e2e_steps):
            fp.attention(qp, kp, vp, qk_format=w.qk_format, causal=w.causal, tile_mask=mask, out_host=out_h,
                         lse_host=lse_h, video=video, rescale_threshold=args.rescale_threshold,
                         pv_format=args.pv_format)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = rank_max(e0.elapsed_time(e1) / args.e2e_steps)
        h2d = 3 * q_h.numel() * 2
        d2h = out_h.numel() * 2 + lse_h.numel() * 4
        e2e = {"value": world * flops / (e_ms * 1e-3) / 1e12, "unit": "TFLOPS", "ms_per_step": e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
        if w.qk_format == "nvfp4" and args.pv_format == "fp8":
            # the static-amax form: a caller's Q/K amax (here the inputs' own,
            # so the bits are those of the dynamic call) lets each group of
            # heads be quantized as it lands
            amax = (fp.tensor_amax(q), fp.tensor_amax(k))
            torch.cuda.synchronize()
            e0.record(stream)
            for _ in range(args.e2e_steps):
                fp.attention(qp, kp, vp, qk_format=w.qk_format, causal=w.causal, tile_mask=mask, out_host=out_h,
                             lse_host=lse_h, video=video, rescale_threshold=args.rescale_threshold,
                             pv_format=args.pv_format, qk_amax=amax)
            e1.record(stream)
            torch.cuda.synchronize()
            s_ms = rank_max(e0.elapsed_time(e1) / args.e2e_steps)
            e2e["caller_amax"] = {"value": world * flops / (s_ms * 1e-3) / 1e12, "unit": "TFLOPS",
                                  "ms_per_step": s_ms,
                                  "note": "attention(..., qk_amax=(amax Q, amax K)) from the caller, same copies"}

    cpu, accuracy = None, None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # a bounded oracle sample: query rows of four blocks spread over the
        # sequence, of one head (two for short sequences); the same rows also
        # give the accuracy figures against the kernel and against exact
        # (unquantized fp64) attention
        nblk = (w.N + 127) // 128
        bh = w.B * w.H
        heads = [bh // 2] if w.N > 16384 else [0, bh - 1]
        qblocks = sorted({0, nblk // 3, (2 * nblk) // 3, nblk - 1})
        if w.sparse:
            qo, ko, vo = workloads.make_qkv(w)     # tile-major, the order the kernel computes in
        else:
            qo, ko, vo = q_h, k_h, v_h
        rows = sample_rows(w, qblocks)
        res = oracle_sample(w, qo, ko, vo, heads, rows, budget_s=30.0, exact=True)
        rate = oracle_rate(res, w.N)
        nrows = sum(len(r) for _, r in res["done"])
        cpu = {"value": rate, "unit": "TFLOPS", "cores": host_cores(), "kind": "oracle",
               "sample": f"{nrows} query rows of {w.name}: heads {heads}, blocks {qblocks}, the first "
                         f"{len(rows[0])} rows of each (fp64 numpy oracle; {res['attn_s']:.1f} s of attention "
                         f"rows plus the heads' quantization, {res['quant_s']:.1f} s, charged per row)"}
        # accuracy on the same rows: kernel output (raster order for video
        # layouts is undone by the same permutation the oracle input used)
        og = out_last.reshape(bh, w.N, w.d)
        if video is not None:
            perm = workloads.video_tile_major_perm(w.video, w.sta_tile)
            og = og[:, perm]
        ks, os_, ex = [], [], []
        for i, (h, r) in enumerate(res["done"]):
            ks.append(og[h, torch.from_numpy(r)].numpy())
            os_.append(res["out"][(h, i % len(rows))])
            ex.append(res["exact"][(h, i % len(rows))])
        ks, os_, ex = (np.concatenate(x) for x in (ks, os_, ex))
        accuracy = {"rows": nrows, "cos_vs_exact_kernel": cosine(ks, ex), "cos_vs_exact_oracle": cosine(os_, ex),
                    "kernel_vs_oracle_rel_l2": float(np.linalg.norm(ks - os_) / np.linalg.norm(os_)),
                    "kernel_vs_oracle_max_abs": float(np.abs(ks - os_).max())}

    # Our kernels per step. FP8 V: the fused quantizer (zero, amax, convert, finalize) and the
    # attention kernel. NVFP4 V: Q/K NVFP4 zero + amax + quantize + finalize each (or one FP8
    # kernel each), V zero + amax + quantize + finalize, attention.
    if args.pv_format == "fp8":
        launches_per_step = 4 + 1
    else:
        launches_per_step = (8 if w.qk_format == "nvfp4" else 2) + 4 + 1
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e2m1/e4m3 MMA, f32 accumulate", "data": "synthetic",
            "config": dict(config_dict(w), **({"rescale_threshold": args.rescale_threshold}
                                              if args.rescale_threshold else {}),
                           **({"pv": "nvfp4"} if args.pv_format == "nvfp4" else {})),
            "attn_ms": attn_ms, "attn_tflops_algorithmic": attn_tflops,
            "attn_tflops_dense_eq": w.dense_flops() / (attn_ms * 1e-3) / 1e12,
            "attn_tflops_executed": exec_flops / (attn_ms * 1e-3) / 1e12,
            "quant_ms": quant_ms, "quant_gbs": quant_gbs, "quant_frac_hbm": quant_gbs / peaks["hbm_gbs"],
            "quant_one_pass_bound_ms": quant_bytes_one_pass(w, args.pv_format) / (peaks["hbm_gbs"] * 1e9) * 1e3,
            "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": attn_tflops / peak, "frac_of_burst_peak": attn_tflops / peak_burst,
                         "traffic": profiled_traffic(w.name) if args.pv_format == "fp8" and
                         not args.rescale_threshold else None,
                         "frac_of_sustained_peak": attn_tflops / (peak * peaks.get("bf16_tflops_sustained", bf16) / bf16),
                         "peak_source": f"{peak_src} bf16 {'sustained' if sustained else 'burst'} {bf16} "
                                        f"(timed region {timed_s:.2f} s, median SM clock {clk.get('sm_mhz')} MHz, "
                                        f"{'power-capped or below max clock' if capped else 'max clock, no power cap'})"
                                        f" "
                                        f"x nominal fp8 2x / fp4 4x; QK "
                                        f"{'fp4' if w.qk_format == 'nvfp4' else 'fp8'}, PV "
                                        f"{'fp4' if args.pv_format == 'nvfp4' else 'fp8'}, harmonic mean"},
            "alu_roofline": alu_roofline(w, attn_tflops, peaks),
            "accuracy": accuracy, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps, "clocks": clk, "device_error": err,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
