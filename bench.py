#!/usr/bin/env python
"""Benchmark of the Stem prefill hot path on B200 (one JSON line on rank 0).

Workload (default): one attention layer of a 128K-token prefill shaped like
Qwen3-8B — 1 x 131072 tokens, 32 query / 8 KV heads, head_dim 128, bf16,
keep-ratio 0.25, mu 0.7, beta 0.2, 1 sink + 2 window blocks, 128-token blocks,
scoring stride 8 — on synthetic inputs (N(0,1) queries/keys, the first four
keys pushed along the mean query, log-normal value norms).

A step is one pass of the whole path: stem_score (value-norm bonus +
anti-diagonal scoring + block max-pool) -> stem_select (position-decay budget
+ top-k CSR lists) -> stem_bsa_fwd (block-sparse attention), timed with CUDA
events on the launching stream.  Inputs (Q alone is 1.07 GB) exceed the
126 MB L2, so no flush is needed between steps.

value = (scoring FLOPs + attention FLOPs of the selected blocks) summed over
ranks / max-over-ranks step time, in TFLOP/s.  Each rank runs an independent
layer (weak scaling, no collective on the data path).

`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload instead (there is no other implementation of this method to run).
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "128K prefill attn ms & effective TFLOPS (1×B200, ρ=0.25) vs dense; % of roofline"
UNIT = "TFLOP/s (scoring + selected-block attention FLOPs per second)"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "bsa_kernel_traffic.txt")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long128k")
    ap.add_argument("--dtype", choices=["bf16", "fp8"], default=None,
                    help="override the workload's arithmetic type (same shapes and distributions)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="skip the e4m3 attention timing of the default mode")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="bounded oracle sample, seconds")
    ap.add_argument("--mode", choices=["default", "sweep", "fp8stack", "quality", "variants", "once"], default="default",
                    help="sweep: latency vs kept-block density (64K, mu=1); fp8stack: the 36-layer fp8 varlen stack; "
                         "quality: reconstruction error against dense attention (32K); "
                         "variants: the 128K step with the standardized bonus, KV-group-shared lists and 64-token blocks; "
                         "once: one untimed step of --workload (the command profilers wrap)")
    ap.add_argument("--layers", type=int, default=36, help="layers of the fp8 stack")
    ap.add_argument("--block-size", type=int, choices=[64, 128], default=None,
                    help="block size of the workload (default: the workload's, 128)")
    ap.add_argument("--separate-select", action="store_true",
                    help="mode once: stem_score then stem_select as two calls (stem_score_select runs the same "
                         "two kernels unless --fused-select)")
    ap.add_argument("--fused-select", action="store_true",
                    help="mode once: stem_score_select with select_mode 1 (the scoring kernel selects its rows)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------- distributed plumbing
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def dist_init(backend: str):
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def dist_barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def dist_max(x: float, device="cpu") -> float:
    import torch
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return x


def dist_sum(x: float, device="cpu") -> float:
    import torch
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        return float(t.item())
    return x


def dist_done():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.device_id = device_id
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.device_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 8:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        smax = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[4 + k].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def gpu_device_id(torch) -> str:
    """nvidia-smi -i argument of the current device: the physical index from
    CUDA_VISIBLE_DEVICES when it lists indices, else the PCI bus id."""
    cur = torch.cuda.current_device()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x.strip() for x in vis.split(",") if x.strip()]
    if ids and all(x.isdigit() for x in ids) and cur < len(ids):
        return ids[cur]
    props = torch.cuda.get_device_properties(cur)
    try:
        return "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
    except AttributeError:
        return str(cur)


def load_peaks():
    try:
        pk = json.load(open(PEAKS_FILE))
        return pk, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


def bsa_traffic_per_launch(workload: str):
    """dram bytes per launch of the attention kernel from the committed ncu
    summary, valid only for the workload it was captured on and while the
    kernel source is the one that was profiled."""
    try:
        rec, other = {}, {}
        for line in open(TRAFFIC_FILE):
            if not line.strip() or line.startswith("#"):
                continue
            key, val = line.split(None, 1)
            if key == "bytes_per_launch":  # another workload: "bytes_per_launch <workload> <bytes>"
                name, nbytes = val.split()
                other[name] = float(nbytes)
            else:
                rec[key] = val
        src = open(os.path.join(ROOT, "block_sparse_attention_stem_b200", "csrc", "k_bsa.cu"), "rb").read()
        if rec.get("source_sha256", "").strip() != hashlib.sha256(src).hexdigest():
            return None
        if rec.get("workload", "").strip() == workload:
            return float(rec["bytes_per_launch_full_workload"])
        return other.get(workload)
    except (OSError, ValueError, KeyError):
        return None


def measure_gemm_peaks(torch, n: int = 8192, reps: int = 10) -> dict:
    """Burst dense-GEMM throughput on this GPU, measured in this run: e4m3 x
    e4m3 -> bf16 through torch._scaled_mm (per-tensor scales) and bf16 x bf16
    through torch.matmul, n^3 each, best of `reps` single launches after 3
    warm-ups, CUDA events on the current stream.  2 n^3 FLOPs per launch."""
    dev = torch.device("cuda", torch.cuda.current_device())
    gen = torch.Generator(dev).manual_seed(7)
    a = torch.randn(n, n, device=dev, generator=gen, dtype=torch.float32)
    bt = torch.randn(n, n, device=dev, generator=gen, dtype=torch.float32)
    res = {"n": n, "reps": reps, "how": "best of %d launches of an %d^3 GEMM, CUDA events" % (reps, n)}
    flops = 2.0 * n ** 3

    def best(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        return flops / (min(ts) * 1e-3) / 1e12

    try:
        a8 = (a / 8).to(torch.float8_e4m3fn)
        b8 = (bt / 8).to(torch.float8_e4m3fn)
        one = torch.ones((), device=dev, dtype=torch.float32)
        res["fp8_e4m3_tflops"] = round(best(lambda: torch._scaled_mm(a8, b8.t(), scale_a=one, scale_b=one,
                                                                     out_dtype=torch.bfloat16)), 1)
        del a8, b8
    except Exception as e:  # noqa: BLE001  (reported, not hidden)
        res["fp8_e4m3_tflops"] = None
        res["fp8_error"] = repr(e)[:200]
    ab, bb = a.to(torch.bfloat16), bt.to(torch.bfloat16)
    res["bf16_tflops"] = round(best(lambda: torch.matmul(ab, bb)), 1)
    del a, bt, ab, bb
    torch.cuda.empty_cache()
    return res


def bench_workload(I, args):
    """The named workload, with its arithmetic type overridden by --dtype and
    its block size by --block-size."""
    over = {}
    if args.dtype:
        over["dtype"] = args.dtype
    if getattr(args, "block_size", None):
        over["block_size"] = args.block_size
    return I.workload(args.workload, **over)


def describe(w) -> dict:
    return {
        "workload": (f"{w.name}: {len(w.seqlens)} x {w.seqlens if len(w.seqlens) > 1 else w.seqlens[0]} tokens, "
                     f"{w.num_q_heads} Q / {w.num_kv_heads} KV heads, d={w.head_dim}, {w.dtype}, "
                     f"rho={w.keep_ratio}, mu={w.mu}, beta={w.beta}, sink {w.sink_blocks}, window "
                     f"{w.window_blocks}, block {w.block_size}, stride {w.stride}"),
        "seq_len": max(w.seqlens),
        "total_tokens": w.total_tokens,
        "num_q_heads": w.num_q_heads,
        "num_kv_heads": w.num_kv_heads,
        "l2": "inputs larger than L2 (Q alone %.2f GB > 126 MB); no flush" % (
            w.total_tokens * w.num_q_heads * w.head_dim * (2 if w.dtype == "bf16" else 1) / 1e9),
    }


# ---------------------------------------------------------------- oracle sample (CPU)
def oracle_sample(w, host_inp, seconds: float, rows_hint=None):
    """Run the fp64 oracle (score row -> budget -> select -> attention row) on
    (query head, query block) rows of the workload until `seconds` of CPU work
    are done.  Returns (flops, seconds, rows)."""
    import numpy as np
    from block_sparse_attention_stem_b200 import inputs as I
    from oracle import stem_oracle as O

    p = O.Params(**w.params())
    L = w.seqlens[0]
    nb = math.ceil(L / 128)
    G = w.num_q_heads // w.num_kv_heads
    heads = sorted({h for h in (0, G, 2 * G + 1) if h < w.num_q_heads})
    order = rows_hint or [(h, i) for i in list(range(nb - 1, -1, -max(1, nb // 128))) for h in heads]
    cache = {}

    def head(h):
        if h not in cache:
            def sl(t, c):
                x = t[:L, c:c + 1].contiguous()
                if w.dtype == "bf16":
                    return O.dequant(I.raw_bits(x), "bf16")
                sc = host_inp[{"q": "q_scale", "k": "k_scale", "v": "v_scale"}[n]][c:c + 1].numpy()
                return O.dequant(I.raw_bits(x), "fp8", sc)
            hk = h // G
            n = "q"; qh = sl(host_inp["q"], h)
            n = "k"; kh = sl(host_inp["k"], hk)
            n = "v"; vh = sl(host_inp["v"], hk)
            cache[h] = (qh, kh, vh)
        return cache[h]

    flops = 0.0
    spent = 0.0
    done = []
    for (h, i) in order:
        qh, kh, vh = head(h)
        t0 = time.perf_counter()
        srow = O.block_score_row(qh, kh, vh, i, p)
        b = O.tpd_budget(i, nb, p)
        sel = O.select_row(srow, i, b, p.sink_blocks, p.window_blocks)
        rp = np.zeros(nb + 1, dtype=np.int64)
        rp[i + 1:] = len(sel)
        O.bsa(qh, kh, vh, [0, L], rp, np.array(sel), p, rows_subset=[(0, i)])
        spent += time.perf_counter() - t0
        qi = min(128, L - 128 * i)
        flops += (i + 1) * (128 // p.stride) ** 2 * 2 * p.stride * 128  # scoring of the row
        flops += 4 * 128 * ((len(sel) - 1) * qi * 128 + qi * (qi + 1) / 2)  # attention of the row
        done.append((h, i))
        if spent >= seconds:
            break
    return flops, spent, done


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [x.get("num_threads") for x in threadpool_info() if x.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:  # noqa: BLE001
        pass
    return len(os.sched_getaffinity(0))


# ---------------------------------------------------------------- our implementation
def run_ours(args):
    import torch

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
    dist_init("nccl" if world > 1 else "gloo")
    dev = torch.device("cuda", torch.cuda.current_device())

    from block_sparse_attention_stem_b200 import binding as b
    from block_sparse_attention_stem_b200 import inputs as I

    w = bench_workload(I, args)
    seed = w.seed + 1000 * rank  # independent layer per rank
    inp = I.make_inputs(w, seed=seed, device="cuda")
    torch.cuda.synchronize()
    qkv = b.make_qkv(inp["q"], inp["k"], inp["v"], w.cu_seqlens(), q_scale=inp["q_scale"], k_scale=inp["k_scale"],
                     v_scale=inp["v_scale"], cu_seqlens_dev=inp["cu_seqlens"])
    params = b.make_params(**w.params())
    pl = b.stem_plan(qkv, params)
    T, hq, hkv = w.total_tokens, w.num_q_heads, w.num_kv_heads
    scores = torch.empty(hq, pl.nb_total, pl.nb_max, dtype=torch.float32, device=dev)
    vbonus = torch.empty(hkv, pl.nb_total, dtype=torch.float32, device=dev)
    budgets = torch.empty(pl.num_rows, dtype=torch.int32, device=dev)
    row_ptr = torch.empty(pl.num_rows + 1, dtype=torch.int32, device=dev)
    col_idx = torch.empty(pl.nnz, dtype=torch.int32, device=dev)
    out = torch.empty(T, hq, 128, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(hq, T, dtype=torch.float32, device=dev)
    ws = torch.empty(pl.ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev):
        # scoring and selection (stem_score_select: the scoring kernel, then
        # the selection kernel), then the attention; ev[1] = ev[2] marks the boundary
        ev[0].record(stream)
        b.stem_score_select(qkv, params, scores, vbonus, budgets, row_ptr, col_idx, ws, stream)
        ev[1].record(stream)
        ev[2].record(stream)
        b.stem_bsa_fwd(qkv, params, row_ptr, col_idx, out, lse, ws, stream)
        ev[3].record(stream)

    mk = lambda: [torch.cuda.Event(enable_timing=True) for _ in range(4)]  # noqa: E731
    for _ in range(args.warmup):
        step(mk())
    torch.cuda.synchronize()
    status = b.stem_read_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {b.stem_status_string(status)}")

    gemm_peaks = measure_gemm_peaks(torch)
    for _ in range(2):  # back on the step's own kernels before timing
        step(mk())
    torch.cuda.synchronize()

    sampler = ClockSampler(gpu_device_id(torch))
    evs = [mk() for _ in range(args.steps)]
    dist_barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.25)  # let the sampler take its first reading
    for k in range(args.steps):
        step(evs[k])
    torch.cuda.synchronize()
    dist_barrier()
    clocks = sampler.stop()
    status = b.stem_read_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status after timing: {b.stem_status_string(status)}")

    total_ms = evs[0][0].elapsed_time(evs[-1][3])
    score_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    select_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    bsa_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / args.steps
    step_ms_local = total_ms / args.steps
    step_ms = dist_max(step_ms_local, device=dev)
    flops_rank = pl.score_flops + pl.attn_flops
    flops_all = dist_sum(flops_rank, device=dev)
    value = flops_all / (step_ms * 1e-3) / 1e12

    # dense comparator: the same attention kernel with every causal block listed
    dense_rows = torch.arange(pl.num_rows, dtype=torch.int64)
    nb = pl.nb_total
    i_of_row = dense_rows % nb  # one sequence
    counts = (i_of_row + 1).to(torch.int32)
    drp = torch.zeros(pl.num_rows + 1, dtype=torch.int32)
    drp[1:] = torch.cumsum(counts, 0).to(torch.int32)
    dci = torch.cat([torch.arange(int(c), dtype=torch.int32) for c in counts[:nb]]).repeat(hq)
    drp, dci = drp.to(dev), dci.to(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b.stem_bsa_fwd(qkv, params, drp, dci, out, lse, ws, stream)
    e0.record(stream)
    nd = 3
    for _ in range(nd):
        b.stem_bsa_fwd(qkv, params, drp, dci, out, lse, ws, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    dense_ms = e0.elapsed_time(e1) / nd
    del drp, dci

    peaks, peak_kind = load_peaks()
    peak_bf16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_bf16_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    # the fp8 peak: this run's e4m3 GEMM, else the nominal 2x of the bf16 figure
    if gemm_peaks.get("fp8_e4m3_tflops"):
        peak_fp8 = float(gemm_peaks["fp8_e4m3_tflops"])
        fp8_src = "fp8 e4m3 GEMM measured in this run (torch._scaled_mm %d^3, best of %d)" % (
            gemm_peaks["n"], gemm_peaks["reps"])
    else:
        peak_fp8 = 2.0 * peak_bf16
        fp8_src = f"{peak_kind} bf16_tflops x2 (nominal fp8 ratio; the e4m3 GEMM probe failed)"
    # the e4m3 attention runs Q.K^T in e4m3 and P.V in f16 (half of its
    # FLOPs each), so it cannot beat F / (F/2/P8 + F/2/P16)
    mixed_bound = 2.0 * peak_fp8 * peak_bf16 / (peak_fp8 + peak_bf16)

    # the same workload in e4m3 (the fp8 attention path): its own lists, the
    # attention kernel timed alone, against the fp8 peak (2 x bf16, nominal)
    fp8_attn = None
    if w.dtype == "bf16" and not args.no_fp8:
        w8 = I.workload(w.name, dtype="fp8", block_size=w.block_size)
        inp8 = I.make_inputs(w8, seed=seed, device="cuda")
        qkv8 = b.make_qkv(inp8["q"], inp8["k"], inp8["v"], w8.cu_seqlens(), q_scale=inp8["q_scale"],
                          k_scale=inp8["k_scale"], v_scale=inp8["v_scale"], cu_seqlens_dev=inp8["cu_seqlens"])
        params8 = b.make_params(**w8.params())
        pl8 = b.stem_plan(qkv8, params8)
        ws8 = torch.empty(pl8.ws_bytes, dtype=torch.uint8, device=dev)
        b.stem_score_select(qkv8, params8, scores, vbonus, budgets, row_ptr, col_idx, ws8, stream)
        for _ in range(2):
            b.stem_bsa_fwd(qkv8, params8, row_ptr, col_idx, out, lse, ws8, stream)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n8 = 5
        f0.record(stream)
        for _ in range(n8):
            b.stem_bsa_fwd(qkv8, params8, row_ptr, col_idx, out, lse, ws8, stream)
        f1.record(stream)
        torch.cuda.synchronize()
        if b.stem_read_device_status(ws8) != 0:
            raise RuntimeError("device status after the fp8 attention timing")
        ms8 = f0.elapsed_time(f1) / n8
        ach8 = pl8.attn_flops / (ms8 * 1e-3) / 1e12
        fp8_attn = {"workload": w8.name + " in e4m3 (per-head scales), its own block lists",
                    "ms_per_launch": round(ms8, 4), "achieved": round(ach8, 2), "peak": peak_fp8,
                    "unit": "TFLOP/s", "frac": round(ach8 / peak_fp8, 4), "peak_source": fp8_src,
                    "design_bound": round(mixed_bound, 1),
                    "design_bound_frac_of_peak": round(mixed_bound / peak_fp8, 4),
                    "frac_of_design_bound": round(ach8 / mixed_bound, 4),
                    "design_bound_note": "Q.K^T in e4m3 at the fp8 peak, P.V in f16 at the measured bf16 burst "
                                         "peak, half of the FLOPs each",
                    "note": "includes the per-call widening of V to f16 (P.V runs in f16)"}
        del inp8, qkv8, ws8

    # end to end through the public API with host buffers: every step copies
    # the inputs from page-locked host memory, runs the path and copies O and
    # LSE back (stem_prefill_host, which overlaps the copies with compute)
    e2e = None
    if not args.no_e2e:
        hq_t = inp["q"].cpu().pin_memory()
        hk_t = inp["k"].cpu().pin_memory()
        hv_t = inp["v"].cpu().pin_memory()
        h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h_lse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        pws = torch.empty(pl.ws_prefill_bytes, dtype=torch.uint8, device=dev)
        dq, dk, dv = torch.empty_like(inp["q"]), torch.empty_like(inp["k"]), torch.empty_like(inp["v"])
        qkv2 = b.make_qkv(dq, dk, dv, w.cu_seqlens(), q_scale=inp["q_scale"], k_scale=inp["k_scale"],
                          v_scale=inp["v_scale"], cu_seqlens_dev=inp["cu_seqlens"])

        def e2e_step():
            # host inputs -> device, the whole path, results -> host: one call
            # that overlaps the transfers of one KV-head group with the
            # computation of another
            b.stem_prefill_host(qkv2, params, hq_t, hk_t, hv_t, h_out, h_lse, out, lse, pws, stream)

        e2e_step()
        torch.cuda.synchronize()
        ke = max(2, min(args.steps, 5))
        dist_barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(ke):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = dist_max(a0.elapsed_time(a1) / ke, device=dev)
        e2e = {"value": round(flops_all / (e2e_ms * 1e-3) / 1e12, 3), "unit": UNIT,
               "ms_per_step": round(e2e_ms, 3),
               "h2d_bytes_per_step": int(hq_t.numel() * hq_t.element_size() + hk_t.numel() * hk_t.element_size()
                                         + hv_t.numel() * hv_t.element_size()),
               "d2h_bytes_per_step": int(h_out.numel() * h_out.element_size() + h_lse.numel() * 4),
               "steps": ke, "api": "stem_prefill_host"}
        del pws, dq, dk, dv

    achieved = pl.attn_flops / (bsa_ms * 1e-3) / 1e12
    traffic_key = w.name if w.dtype == I.workload(w.name).dtype else f"{w.name}:{w.dtype}"
    if w.block_size != I.workload(w.name).block_size:
        traffic_key += f":b{w.block_size}"
    traffic = bsa_traffic_per_launch(traffic_key)
    if w.dtype == "fp8":
        roofline = {"bound": "tensor", "kernel": "bsa_kernel", "achieved": round(achieved, 2), "peak": peak_fp8,
                    "unit": "TFLOP/s", "frac": round(achieved / peak_fp8, 4), "peak_source": fp8_src,
                    "design_bound": round(mixed_bound, 1), "frac_of_design_bound": round(achieved / mixed_bound, 4)}
    else:
        roofline = {"bound": "tensor", "kernel": "bsa_kernel", "achieved": round(achieved, 2), "peak": peak_bf16,
                    "unit": "TFLOP/s", "frac": round(achieved / peak_bf16, 4),
                    "peak_source": f"{peak_kind} bf16_tflops (burst) of MEASURED_PEAKS.json",
                    "peak_sustained": peak_bf16_sus, "frac_sustained": round(achieved / peak_bf16_sus, 4),
                    "peak_sustained_source": f"{peak_kind} bf16_tflops_sustained of MEASURED_PEAKS.json"}
    roofline.update({
        "traffic": traffic,
        "traffic_source": ((f"{os.path.relpath(TRAFFIC_FILE, ROOT)} (stored: an earlier ncu capture of this "
                            f"kernel source on this workload, not measured in this run)") if traffic is not None
                           else "none stored for this kernel source and workload"),
        "flops_per_launch": pl.attn_flops, "ms_per_launch": round(bsa_ms, 4)})

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
        fl, sec, rows = oracle_sample(w, host, args.cpu_seconds)
        cpu = {"value": round(fl / sec / 1e12, 6), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": (f"{len(rows)} (query head, query block) rows of this workload, longest blocks first "
                          f"(first {rows[:3]}...): fp64 block-score row, budget, top-k, attention row; "
                          f"{sec:.1f} s, {fl / 1e9:.1f} GFLOP")}

    # per launch batch of up to 8 sequences: v-norm, budgets, scoring, the
    # selection pass and attention (the selection runs in the scoring kernel
    # only with select_mode 1, which the step does not use)
    fused = params.select_mode == 1 and w.list_mode == 0 and pl.nb_max <= 5888
    # (fp8: plus one V widening pass per attention call)
    launches_per_step = ((4 if fused else 5) * math.ceil(len([L for L in w.seqlens if L > 0]) / 8)
                         + (1 if w.dtype == "fp8" else 0))
    res = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded, device RNG)",
        "config": describe(w),
        "stages_ms": {"score_select": round(score_ms + select_ms, 3), "bsa": round(bsa_ms, 3)},
        "dense_bsa_ms": round(dense_ms, 3), "speedup_vs_dense": round(dense_ms / step_ms, 3),
        "density_blocks": round(pl.nnz_per_head / sum(
            math.ceil(L / 128) * (math.ceil(L / 128) + 1) / 2 for L in w.seqlens), 4),
        "attn_tflops_selected": round(achieved, 2),
        "dense_equiv_tflops": round(pl.dense_attn_flops / (step_ms * 1e-3) / 1e12, 2),
        "roofline": roofline, "fp8_attention": fp8_attn, "gemm_peaks_this_run": gemm_peaks,
        "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
        "gpu_launches": launches_per_step * args.steps,
    }
    dist_barrier()
    if rank == 0:
        print(json.dumps(res), flush=True)
    dist_done()


# ---------------------------------------------------------------- reference arm (the oracle)
def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import torch
    from block_sparse_attention_stem_b200 import inputs as I

    w = bench_workload(I, args)
    inp = I.make_inputs(w, device="cuda" if torch.cuda.is_available() else "cpu")
    host = {k: (None if v is None else v.cpu()) for k, v in inp.items()}
    per_step = max(1.0, min(args.cpu_seconds, 120.0 / max(1, args.steps)))  # the whole run stays near 2 min
    for _ in range(args.warmup):
        oracle_sample(w, host, per_step / 4)
    fl_tot, sec_tot, rows_tot = 0.0, 0.0, 0
    for _ in range(args.steps):
        fl, sec, rows = oracle_sample(w, host, per_step)
        fl_tot += fl
        sec_tot += sec
        rows_tot += len(rows)
    value = fl_tot / sec_tot / 1e12
    ms = sec_tot / args.steps * 1e3
    res = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, device RNG)",
        "config": describe(w),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{rows_tot} (query head, query block) rows over {args.steps} steps, "
                                   f"about {per_step:.0f} s each"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(res), flush=True)


# ---------------------------------------------------------------- extra modes (one GPU)
def _time_prefill(b, qkv, params, pl, dev, steps, warmup, stages=None):
    """Mean CUDA-event time (ms) of the three stages and of the attention
    stage alone over `steps` runs after `warmup`."""
    import torch
    stream = torch.cuda.current_stream()
    T, hq, hkv = qkv.total_tokens, qkv.q.shape[1], qkv.k.shape[1]
    scores = torch.empty(hq, pl.nb_total, pl.nb_max, dtype=torch.float32, device=dev)
    vbonus = torch.empty(hkv, pl.nb_total, dtype=torch.float32, device=dev)
    budgets = torch.empty(pl.num_rows, dtype=torch.int32, device=dev)
    row_ptr = torch.empty(pl.num_rows + 1, dtype=torch.int32, device=dev)
    col_idx = torch.empty(max(pl.nnz, 1), dtype=torch.int32, device=dev)
    out = torch.empty(T, hq, 128, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(hq, T, dtype=torch.float32, device=dev)
    ws = torch.empty(pl.ws_bytes, dtype=torch.uint8, device=dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps + warmup)]
    for k in range(steps + warmup):
        ev[k][0].record(stream)
        b.stem_score(qkv, params, scores, vbonus, ws, stream)
        ev[k][1].record(stream)
        b.stem_select(qkv, params, scores, budgets, row_ptr, col_idx, ws, stream)
        ev[k][2].record(stream)
        b.stem_bsa_fwd(qkv, params, row_ptr, col_idx, out, lse, ws, stream)
        ev[k][3].record(stream)
    torch.cuda.synchronize()
    status = b.stem_read_device_status(ws)
    if status != 0:
        raise RuntimeError(b.stem_status_string(status))
    tot = sum(e[0].elapsed_time(e[3]) for e in ev[warmup:]) / steps
    bsa = sum(e[2].elapsed_time(e[3]) for e in ev[warmup:]) / steps
    if stages is not None:
        stages["score"] = sum(e[0].elapsed_time(e[1]) for e in ev[warmup:]) / steps
        stages["select"] = sum(e[1].elapsed_time(e[2]) for e in ev[warmup:]) / steps
        stages["bsa"] = bsa
    return tot, bsa


def run_sweep(args):
    """Latency against kept-block density on the 64K workload with a uniform
    budget (mu = 1), rho in {1, 0.5, 0.25, 0.2, 0.1}; the pages report the
    sparse operator's latency as close to linear in density."""
    import numpy as np
    import torch
    from block_sparse_attention_stem_b200 import binding as b
    from block_sparse_attention_stem_b200 import inputs as I
    dev = torch.device("cuda", 0)
    w0 = I.workload("sweep64k")
    inp = I.make_inputs(w0, device="cuda")
    rows = []
    sampler = ClockSampler(gpu_device_id(torch))
    sampler.start()
    for rho in (1.0, 0.5, 0.25, 0.2, 0.1):
        w = I.workload("sweep64k", keep_ratio=rho)
        qkv = b.make_qkv(inp["q"], inp["k"], inp["v"], w.cu_seqlens(), cu_seqlens_dev=inp["cu_seqlens"])
        params = b.make_params(**w.params())
        pl = b.stem_plan(qkv, params)
        tot, bsa = _time_prefill(b, qkv, params, pl, dev, args.steps, args.warmup)
        dens = pl.nnz_per_head / sum(math.ceil(L / 128) * (math.ceil(L / 128) + 1) / 2 for L in w.seqlens)
        rows.append(dict(rho=rho, density=round(dens, 4), ms=round(tot, 3), bsa_ms=round(bsa, 3),
                         attn_tflops=round(pl.attn_flops / (bsa * 1e-3) / 1e12, 1)))
    clocks = sampler.stop()
    d = np.array([r["density"] for r in rows])
    fits = {}
    for key in ("ms", "bsa_ms"):
        y = np.array([r[key] for r in rows])
        A = np.vstack([d, np.ones_like(d)]).T
        (a, c), *_ = np.linalg.lstsq(A, y, rcond=None)
        dev_rel = np.abs(A @ np.array([a, c]) - y) / y
        fits[key] = dict(slope_ms_per_density=round(float(a), 3), intercept_ms=round(float(c), 3),
                         max_rel_deviation=round(float(dev_rel.max()), 4))
    res = {"metric": "latency vs kept-block density (64K, mu=1)", "unit": "ms", "higher_is_better": False,
           "points": rows, "linear_fit": fits, "steps": args.steps, "warmup": args.warmup,
           "config": describe(w0), "clocks": clocks, "dtype": "bf16", "data": "synthetic (seeded, device RNG)"}
    print(json.dumps(res), flush=True)


def run_quality(args):
    """How much of dense attention the selected blocks reproduce, on the 32K
    workload: relative Frobenius error of O against dense attention (the same
    kernel over every causal block) and the softmax mass the selection keeps,
    mean over rows of exp(lse_sparse - lse_dense).  Compares the output-aware
    metric (beta = 0.2) with the routing score alone (beta = 0), and the
    position-decay budget (mu = 0.7) with a uniform one (mu = 1) at the same
    kept-block count, on two input structures: i.i.d. Q and K (attention close
    to uniform) and the block-topic structure of the input generator
    (attention concentrated on the blocks of the query's topic, block-varying
    value magnitudes).  Synthetic inputs: a check of the method's direction,
    not an accuracy benchmark."""
    import torch
    from block_sparse_attention_stem_b200 import binding as b
    from block_sparse_attention_stem_b200 import inputs as I
    results = []
    for structure in ("iid", "topics"):
        w0 = I.workload("qwen32k", structure=structure)
        inp = I.make_inputs(w0, device="cuda")
        cu = w0.cu_seqlens()
        qkv = b.make_qkv(inp["q"], inp["k"], inp["v"], cu, cu_seqlens_dev=inp["cu_seqlens"])
        nb = math.ceil(w0.seqlens[0] / 128)
        hq = w0.num_q_heads
        # dense reference: every causal block listed
        counts = torch.arange(1, nb + 1, dtype=torch.int64).repeat(hq)
        drp = torch.zeros(hq * nb + 1, dtype=torch.int32)
        drp[1:] = torch.cumsum(counts, 0).to(torch.int32)
        dci = torch.cat([torch.arange(c, dtype=torch.int32) for c in range(1, nb + 1)]).repeat(hq)
        params0 = b.make_params(**w0.params())
        o_dense, l_dense, _ = b.stem_bsa_fwd(qkv, params0, drp.cuda(), dci.cuda())
        o_dense = o_dense.float()
        nrm = torch.linalg.vector_norm(o_dense).item()

        def nnz_of(**kw):
            return b.stem_plan(qkv, b.make_params(**dict(w0.params(), **kw))).nnz_per_head

        target = nnz_of(mu=0.7, keep_ratio=w0.keep_ratio)
        lo, hi = 0.01, 1.0  # uniform-budget keep ratio with the same kept-block count
        for _ in range(40):
            mid = 0.5 * (lo + hi)
            lo, hi = (mid, hi) if nnz_of(mu=1.0, keep_ratio=mid) < target else (lo, mid)
        rho_eq = hi
        causal = nb * (nb + 1) // 2
        points = []
        for label, kw in (("stem: OAM beta 0.2, TPD mu 0.7", dict(beta=0.2, mu=0.7)),
                          ("routing score only: beta 0, mu 0.7", dict(beta=0.0, mu=0.7)),
                          ("OAM beta 0.2, uniform budget mu 1 (same kept blocks)",
                           dict(beta=0.2, mu=1.0, keep_ratio=rho_eq)),
                          ("routing score only, uniform budget", dict(beta=0.0, mu=1.0, keep_ratio=rho_eq)),
                          ("standardized bonus beta 0.2, mu 0.7", dict(beta=0.2, mu=0.7, bonus_mode=1)),
                          ("KV-group-shared lists, beta 0.2, mu 0.7", dict(beta=0.2, mu=0.7, list_mode=1))):
            params = b.make_params(**dict(w0.params(), **kw))
            out, lse, _, _, ws = b.stem_prefill(qkv, params, return_lists=False)
            torch.cuda.synchronize()
            assert b.stem_read_device_status(ws) == 0
            err = torch.linalg.vector_norm(out.float() - o_dense).item() / nrm
            mass = torch.exp(lse - l_dense).mean().item()
            pl = b.stem_plan(qkv, params)
            points.append(dict(selection=label, density=round(pl.nnz_per_head / causal, 4),
                               rel_error_vs_dense=round(err, 5), softmax_mass_kept=round(mass, 5), **kw))
        results.append({"inputs": structure, "points": points})
        del inp, qkv, o_dense, l_dense
        torch.cuda.empty_cache()
    res = {"metric": "attention reconstruction vs dense (32K, synthetic)", "unit": "relative Frobenius error",
           "higher_is_better": False, "results": results, "config": describe(I.workload("qwen32k")),
           "dtype": "bf16", "data": "synthetic (seeded, device RNG)"}
    print(json.dumps(res), flush=True)


def run_variants(args):
    """The step on the 128K workload with the selection variants beside the
    default: the standardized value bonus (bonus_mode 1), KV-group-shared
    block lists (list_mode 1) and 64-token blocks (block_size 64, 2048 blocks
    per row); ms per stage and attention TFLOP/s."""
    import torch
    from block_sparse_attention_stem_b200 import binding as b
    from block_sparse_attention_stem_b200 import inputs as I
    dev = torch.device("cuda", 0)
    w0 = I.workload("long128k")
    inp = I.make_inputs(w0, device="cuda")
    qkv = b.make_qkv(inp["q"], inp["k"], inp["v"], w0.cu_seqlens(), cu_seqlens_dev=inp["cu_seqlens"])
    rows = []
    sampler = ClockSampler(gpu_device_id(torch))
    sampler.start()
    for label, kw in (("default (log bonus, per-head lists)", {}),
                      ("standardized bonus (bonus_mode 1)", dict(bonus_mode=1)),
                      ("KV-group-shared lists (list_mode 1)", dict(list_mode=1)),
                      ("64-token blocks (block_size 64)", dict(block_size=64))):
        params = b.make_params(**dict(w0.params(), **kw))
        pl = b.stem_plan(qkv, params)
        st = {}
        tot, bsa = _time_prefill(b, qkv, params, pl, dev, args.steps, args.warmup, stages=st)
        rows.append(dict(variant=label, ms=round(tot, 3), stages_ms={k: round(v, 3) for k, v in st.items()},
                         attn_tflops=round(pl.attn_flops / (bsa * 1e-3) / 1e12, 1), **kw))
    # the default lists with K/V in a page pool (128-token pages in a random
    # order) against the packed layout: attention alone
    params = b.make_params(**w0.params())
    pl = b.stem_plan(qkv, params)
    _, _, rp, ci, _ = b.stem_prefill(qkv, params)
    ps = 128
    npg = w0.total_tokens // ps
    perm = torch.randperm(npg, generator=torch.Generator().manual_seed(5)).cuda()
    kp = torch.empty(npg, ps, w0.num_kv_heads, 128, dtype=inp["k"].dtype, device=dev)
    vp = torch.empty_like(kp)
    kp[perm] = inp["k"].view(npg, ps, w0.num_kv_heads, 128)
    vp[perm] = inp["v"].view(npg, ps, w0.num_kv_heads, 128)
    kv = b.paged_kv(kp, vp, perm.to(torch.int32).view(1, npg).contiguous(), ps)
    out = torch.empty(w0.total_tokens, w0.num_q_heads, 128, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(w0.num_q_heads, w0.total_tokens, dtype=torch.float32, device=dev)
    ws = torch.empty(pl.ws_bytes, dtype=torch.uint8, device=dev)
    for paged in (False, True):
        for _ in range(args.warmup):
            (b.stem_bsa_fwd_paged(qkv, kv, params, rp, ci, out, lse, ws) if paged
             else b.stem_bsa_fwd(qkv, params, rp, ci, out, lse, ws))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            (b.stem_bsa_fwd_paged(qkv, kv, params, rp, ci, out, lse, ws) if paged
             else b.stem_bsa_fwd(qkv, params, rp, ci, out, lse, ws))
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        rows.append(dict(variant=("attention over paged K/V (128-token pages, shuffled)" if paged
                                  else "attention over packed K/V"), ms=round(ms, 3),
                         attn_tflops=round(pl.attn_flops / (ms * 1e-3) / 1e12, 1)))
    clocks = sampler.stop()
    res = {"metric": "128K step per selection variant", "unit": "ms", "higher_is_better": False, "points": rows,
           "steps": args.steps, "warmup": args.warmup, "config": describe(w0), "clocks": clocks, "dtype": "bf16",
           "data": "synthetic (seeded, device RNG)"}
    print(json.dumps(res), flush=True)


def run_fp8stack(args):
    """The fp8 varlen stack: 4 packed sequences {8192, 16384, 40960, 98304},
    e4m3 inputs with per-head scales, one independently seeded layer per step
    (mu = 1 for the first 5 layers, 0.7 after), prefill timed per layer."""
    import torch
    from block_sparse_attention_stem_b200 import binding as b
    from block_sparse_attention_stem_b200 import inputs as I
    dev = torch.device("cuda", 0)
    per_layer = []
    flops = 0.0
    sampler = ClockSampler(gpu_device_id(torch))
    sampler.start()
    for layer in range(args.layers):
        w = I.workload("fp8_varlen", mu=I.fp8_layer_mu(layer), seed=4000 + layer)
        inp = I.make_inputs(w, device="cuda")
        qkv = b.make_qkv(inp["q"], inp["k"], inp["v"], w.cu_seqlens(), q_scale=inp["q_scale"],
                         k_scale=inp["k_scale"], v_scale=inp["v_scale"], cu_seqlens_dev=inp["cu_seqlens"])
        params = b.make_params(**w.params())
        pl = b.stem_plan(qkv, params)
        tot, bsa = _time_prefill(b, qkv, params, pl, dev, max(1, args.steps // 4), 1)
        per_layer.append(dict(layer=layer, mu=w.mu, ms=round(tot, 3), bsa_ms=round(bsa, 3)))
        flops += pl.score_flops + pl.attn_flops
        del inp, qkv
    clocks = sampler.stop()
    total_ms = sum(x["ms"] for x in per_layer)
    res = {"metric": "fp8 varlen 36-layer stack prefill", "value": round(flops / (total_ms * 1e-3) / 1e12, 2),
           "unit": UNIT, "total_ms": round(total_ms, 2), "layers": per_layer, "dtype": "e4m3",
           "config": {"workload": "fp8_varlen: 4 seqs {8192,16384,40960,98304}, 32 Q / 8 KV heads, e4m3, "
                                  "rho 0.25, mu 1.0 (layers 0-4) / 0.7, sink 4, window 4"},
           "clocks": clocks, "data": "synthetic (seeded, device RNG)"}
    print(json.dumps(res), flush=True)


def launch_ranks(args, argv) -> int | None:
    """--gpus N against the launcher's world size.  Under torchrun (WORLD_SIZE
    set) the two must agree.  Without a launcher and N > 1, start N ranks on
    this node through torch.distributed.run (127.0.0.1 rendezvous) and return
    its exit code; None means: run this process as the only rank."""
    world = os.environ.get("WORLD_SIZE")
    if world is not None:
        if int(world) != args.gpus:
            raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch one rank per GPU")
        return None
    if args.gpus <= 1:
        return None
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__),
           *(sys.argv[1:] if argv is None else argv)]
    return subprocess.run(cmd).returncode


def run_once(args):
    """One step of the workload (stem_score_select, then stem_bsa_fwd) and
    nothing else: the smallest program that launches each of the step's
    kernels once, for profilers.  Prints the device status."""
    import torch
    from block_sparse_attention_stem_b200 import binding as b
    from block_sparse_attention_stem_b200 import inputs as I
    w = bench_workload(I, args)
    inp = I.make_inputs(w, device="cuda")
    qkv = b.make_qkv(inp["q"], inp["k"], inp["v"], w.cu_seqlens(), q_scale=inp["q_scale"], k_scale=inp["k_scale"],
                     v_scale=inp["v_scale"], cu_seqlens_dev=inp["cu_seqlens"])
    params = b.make_params(**w.params(), select_mode=1 if args.fused_select else 0)
    if args.separate_select:
        scores, _, ws = b.stem_score(qkv, params)
        budgets, row_ptr, col_idx, _ = b.stem_select(qkv, params, scores, ws=ws)
    else:
        scores, budgets, row_ptr, col_idx, ws = b.stem_score_select(qkv, params)
    out, lse, _ = b.stem_bsa_fwd(qkv, params, row_ptr, col_idx, ws=ws)
    torch.cuda.synchronize()
    print(json.dumps({"mode": "once", "workload": w.name, "dtype": w.dtype,
                      "status": b.stem_status_string(b.stem_read_device_status(ws))}), flush=True)


def main(argv=None):
    args = parse_args(argv)
    rc = launch_ranks(args, argv)
    if rc is not None:
        sys.exit(rc)
    if args.impl == "reference":
        run_reference(args)
    elif args.mode == "sweep":
        run_sweep(args)
    elif args.mode == "quality":
        run_quality(args)
    elif args.mode == "variants":
        run_variants(args)
    elif args.mode == "fp8stack":
        run_fp8stack(args)
    elif args.mode == "once":
        run_once(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
