"""Benchmark: one step = top-p routing + longest-first ordering + block-sparse
attention forward over one synthetic video-latent-like input (B1 H40 N32760
d128, block 128, p 0.9), with the inputs resident in HBM.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload NAME]

Prints one JSON line (rank 0).  Under torchrun every rank runs its own input
(weak scaling, no data-path collective); time is the max over ranks.

Metric: effective TFLOP/s = 4 * block^2 * d * (selected blocks) / time, the
work of the selected key blocks counted as full tiles.  ``value`` uses the
whole step (routing + ordering + attention); ``roofline`` reports the
attention call alone against the measured bf16 tensor peak.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "effective TFLOP/s & tensor-pipe % of peak (sparse attn fwd, p=0.9); routing ms"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ROUTE_KERNELS_PER_CALL = 4      # pool, select, CSR scan, CSR scatter
FWD_KERNELS_PER_CALL = 3        # head ranks, row order, attention


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = ("top_routed_block_b200/csrc/attn_fwd.cu", "top_routed_block_b200/csrc/ptx_sm100.cuh",
                  "top_routed_block_b200/csrc/common.cuh")
TRAFFIC_RECORD = "profiles/dram_traffic_video_dit.json"


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload: str):
    """DRAM bytes per attention launch from the committed ncu record (JSON), if it
    was taken on this workload with the current kernel source; else None."""
    p = os.path.join(ROOT, TRAFFIC_RECORD)
    try:
        with open(p) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("workload") != workload or rec.get("kernel_source_sha256") != kernel_source_hash():
        return None
    try:
        return float(rec["dram_bytes_read"]) + float(rec["dram_bytes_write"])
    except (KeyError, TypeError, ValueError):
        return None


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def eff_flops(nnz: int, w: W.Workload) -> float:
    return 4.0 * w.bs * w.bs * w.d * float(nnz)


class ClockSampler:
    """nvidia-smi clock/throttle samples taken during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.out,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # the timed region can be short: begin it only once the sampler reports
        t0 = time.time()
        while time.time() - t0 < 5.0 and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def gpu_selector(dev) -> str:
    """nvidia-smi -i argument for this device (its UUID when torch exposes it)."""
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        if u:
            return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        pass
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        return vis.split(",")[dev.index or 0].strip()
    return str(dev.index or 0)


def dist_setup(n_gpus: int):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    """Largest value over the ranks (the step time of the slowest replica)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_rank_step: float, world: int, steps: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank runs its own replica of the workload (weak scaling)."""
    return world * flops_per_rank_step * steps / (max_ms * 1e-3) / 1e12


def replica_seed(w: W.Workload, rank: int) -> int:
    """Each rank draws its own input of the same shape."""
    return w.seed + rank


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------- CPU oracle

def oracle_route_timed(w: W.Workload, Q, K):
    """The oracle's full fp64 routing of the workload and its wall time (s)."""
    import oracle
    t0 = time.perf_counter()
    r = oracle.route(Q, K, w.p, w.bs, nthreads=oracle.default_threads())
    return r, time.perf_counter() - t0


def oracle_sample(w: W.Workload, Q, K, V, budget_s: float, seed: int = 7, routed=None):
    """Times the oracle on a bounded sample: full routing (or a routing already timed,
    ``routed`` = (result, seconds)), then whole query blocks (128 rows each) drawn at
    random until the time budget is spent; the routing time is prorated to the
    sampled share of the query blocks."""
    import oracle
    threads = oracle.default_threads()
    r, t_route = routed if routed is not None else oracle_route_timed(w, Q, K)
    counts = r.counts
    rng = np.random.default_rng(seed)
    items = rng.permutation(w.rows)
    done_flops = 0.0
    t_attn = 0.0
    n_items = 0
    for row in items:
        if t_attn >= budget_s:
            break
        bh, qb = divmod(int(row), w.nb)
        t_lo, t_hi = qb * w.bs, min(w.N, (qb + 1) * w.bs)
        toks = bh * w.N + np.arange(t_lo, t_hi, dtype=np.int64)
        t1 = time.perf_counter()
        oracle.attn_rows(Q, K, V, w.bs, w.causal, r.row_ptr, r.col_idx, toks, nthreads=threads)
        t_attn += time.perf_counter() - t1
        done_flops += eff_flops(int(counts[row]), w)
        n_items += 1
    frac = n_items / w.rows
    total_t = t_attn + t_route * frac
    return {
        "value": done_flops / total_t / 1e12,
        "unit": UNIT,
        "cores": threads,
        "cpu_model": cpu_model(),
        "kind": "oracle",
        "sample": (f"{w.name}: full fp64 routing ({t_route:.2f} s, prorated by {frac:.4f}) + {n_items} of "
                   f"{w.rows} query blocks of attention ({t_attn:.1f} s)"),
        "route_s_full": t_route,
    }


def run_reference(args, w, rank, world):
    if rank != 0:
        return
    Q, K, V = W.generate(w)
    for _ in range(args.warmup):
        pass  # the oracle has no warm-up state
    vals = []
    cb = None
    # the whole run stays near a minute and a half of oracle time for any --steps:
    # the routing is timed once and prorated in every step's sample
    routed = oracle_route_timed(w, Q, K)
    per_step = min(2.0, max(0.05, 90.0 / max(1, args.steps)))
    for s in range(args.steps):
        cb = oracle_sample(w, Q, K, V, budget_s=per_step, seed=1000 + s, routed=routed)
        vals.append(cb["value"])
    v = float(np.mean(vals))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "block": w.bs, "p": w.p,
                       "causal": w.causal, "l2": "inputs larger than L2"},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cb["cores"], "cpu_model": cb["cpu_model"],
                             "kind": "oracle", "sample": cb["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ GPU (ours)

# Workloads timed beside the headline one, each for a few steps in the same run.
CONFIG_SET = ("tiny", "dense", "dense_causal", "long_video", "video_dit_bs64", "sweep_d64_s1_p0.9",
              "sweep_d64_s05_8_p0.9", "sweep_d128_s1_p0.9", "sweep_d128_s05_8_p0.9")


def causal_block_csr(w: W.Workload, dev):
    """The dense causal block mask (every key block kb <= qb of every head), the mask a
    causal workload runs on (the pages define no causal top-p routing)."""
    import torch
    nb = w.nb
    counts = torch.arange(1, nb + 1, dtype=torch.int64, device=dev).repeat(w.B * w.H)
    row_ptr = torch.zeros(counts.numel() + 1, dtype=torch.int64, device=dev)
    row_ptr[1:] = torch.cumsum(counts, 0)
    tri = torch.tril_indices(nb, nb, device=dev)[1].to(torch.int32)      # row-major lower triangle: columns
    col_idx = tri.repeat(w.B * w.H)
    return row_ptr.to(torch.int32), col_idx.contiguous()


def time_config(w: W.Workload, dev, stream, steps: int, burst: float) -> dict:
    """Routing and attention of one more workload, timed like the headline one (CUDA events
    per call on the launching stream, after 3 warm-up steps)."""
    import torch

    import top_routed_block_b200 as fv
    Qh, Kh, Vh = W.generate(w)
    dQ, dK, dV = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev) for a in (Qh, Kh, Vh))
    del Qh, Kh, Vh
    plan = fv.FvattnPlan(w.B, w.H, w.N, w.d, w.bs, device=dev)
    rp = ci = None
    if w.causal:
        rp, ci = causal_block_csr(w, dev)

    def route():
        if not w.causal:
            plan.run_route(dQ, dK, w.p, stream=stream)

    def fwd():
        plan.run_fwd(dQ, dK, dV, w.causal, row_ptr=rp, col_idx=ci, stream=stream)

    for _ in range(3):
        route()
        fwd()
    plan.check()
    nnz = int((rp if w.causal else plan.route.row_ptr)[-1].item())
    flops = eff_flops(nnz, w)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    torch.cuda.synchronize(dev)
    for e0, e1, e2 in ev:
        e0.record(stream)
        route()
        e1.record(stream)
        fwd()
        e2.record(stream)
    torch.cuda.synchronize(dev)
    plan.check()
    r_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in ev)
    a_ms = statistics.mean(b.elapsed_time(c) for _, b, c in ev)
    out = {"B": w.B, "H": w.H, "N": w.N, "d": w.d, "block": w.bs, "p": w.p, "causal": w.causal,
           "nnz_blocks": nnz, "density": nnz / (w.B * w.H * w.nb * w.nb), "steps": steps,
           "attn_ms": a_ms, "attn_tflops": flops / (a_ms * 1e-3) / 1e12,
           "attn_frac_of_burst": flops / (a_ms * 1e-3) / 1e12 / burst,
           "route_ms": None if w.causal else r_ms,
           "route_frac": None if w.causal else r_ms / (r_ms + a_ms),
           "step_tflops": flops / ((a_ms + (0.0 if w.causal else r_ms)) * 1e-3) / 1e12}
    del dQ, dK, dV, plan
    torch.cuda.empty_cache()
    return out


def run_ours(args, w, rank, world, local):
    import torch

    import top_routed_block_b200 as fv
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    Qh, Kh, Vh = W.generate(w, seed=replica_seed(w, rank))

    def pinned(a):
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
        return t.pin_memory()
    hQ, hK, hV = pinned(Qh), pinned(Kh), pinned(Vh)
    dQ, dK, dV = (h.to(dev, non_blocking=True) for h in (hQ, hK, hV))
    torch.cuda.synchronize(dev)
    plan = fv.FvattnPlan(w.B, w.H, w.N, w.d, w.bs, device=dev)
    stream = torch.cuda.current_stream(dev)

    # causal workloads run on the dense lower-triangle block mask, without routing
    mask = causal_block_csr(w, dev) if w.causal else None

    def route():
        if mask is None:
            plan.run_route(dQ, dK, w.p, stream=stream)

    def fwd():
        plan.run_fwd(dQ, dK, dV, w.causal, row_ptr=None if mask is None else mask[0],
                     col_idx=None if mask is None else mask[1], stream=stream)

    def mask_csr():
        return (plan.route.row_ptr, plan.route.col_idx) if mask is None else mask

    for _ in range(max(3, args.warmup)):
        route()
        fwd()
    plan.check()
    nnz = int(mask_csr()[0][-1].item())
    flops = eff_flops(nnz, w)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(gpu_selector(dev))
    barrier(world)
    torch.cuda.synchronize(dev)
    sampler.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        e0, e1, e2 = ev[s]
        e0.record(stream)
        route()
        e1.record(stream)
        fwd()
        e2.record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = sampler.stop()
    plan.check()
    total_ms = t_start.elapsed_time(t_end)
    route_ms = [a.elapsed_time(b) for a, b, _ in ev]
    fwd_ms = [b.elapsed_time(c) for _, b, c in ev]
    total_ms_max = max_over_ranks(total_ms, world)
    ms_per_step = total_ms_max / args.steps
    value = job_throughput(flops, world, args.steps, total_ms_max)
    attn_ms = statistics.mean(fwd_ms)
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12
    r_ms = statistics.mean(route_ms)
    step_ms = [a + b for a, b in zip(route_ms, fwd_ms)]
    timing = {"step_ms_mean": statistics.mean(step_ms), "step_ms_median": statistics.median(step_ms),
              "attn_ms_median": statistics.median(fwd_ms), "route_ms_median": statistics.median(route_ms),
              "note": "per-step CUDA events on the launching stream (routing call, attention call); the line's "
                      "ms_per_step is the whole timed region / steps, max over ranks"}

    # end to end through the host-buffer entry point
    hO = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16).pin_memory()
    hL = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()
    fv.fvattn_attention_host(hQ, hK, hV, w.p, w.bs, w.causal, plan=plan, dQ=dQ, dK=dK, dV=dV, hO=hO, hLSE=hL,
                             stream=stream)
    e2e_steps = max(1, min(args.steps, 5))
    barrier(world)
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        fv.fvattn_attention_host(hQ, hK, hV, w.p, w.bs, w.causal, plan=plan, dQ=dQ, dK=dK, dV=dV, hO=hO, hLSE=hL,
                                 stream=stream)
    b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(a.elapsed_time(b), world) / e2e_steps
    elem = w.B * w.H * w.N * w.d
    h2d = 3 * elem * 2
    d2h = elem * 2 + w.B * w.H * w.N * 4 + 8

    # Load balance over the SMs (outside the timed region): busy time of every CTA of the
    # persistent grid, with the head-major longest-first queue and with rows in index order.
    # The host-buffer path above routed chunk by chunk into the plan: route the whole batch again.
    route()
    balance = {}
    for name, natural in (("lpt", False), ("natural", True)):
        runs = []
        for _ in range(3):
            a.record(stream)
            _, _, st, busy = fv.fvattn_sparse_fwd_profiled(dQ, dK, dV, *mask_csr(), w.bs,
                                                           w.causal, natural_order=natural, stream=stream, O=plan.O,
                                                           LSE=plan.LSE, workspace=plan.fwd_ws,
                                                           dev_status=plan.status[1:2])
            b.record(stream)
            torch.cuda.synchronize(dev)
            fv.check_status(st, "fvattn_sparse_fwd_profiled")
            t = busy.double().cpu().numpy()
            runs.append((a.elapsed_time(b), float(t.max() / t.mean()), float(t.max() * 1e-6), int(t.size)))
        ms_, lif, mx, g = sorted(runs)[1]  # the median run by time
        balance[name] = {"lif": lif, "call_ms": ms_, "max_cta_busy_ms": mx, "ctas": g}

    # Backward (outside the timed region): gradients of the same attention for a random dO.
    bwd = None
    if w.bs == 128:
        fwd()
        gen = torch.Generator(device=dev).manual_seed(1234)
        dO = torch.randn(dQ.shape, device=dev, dtype=torch.float32, generator=gen).to(torch.bfloat16)
        ws_b = torch.empty(fv.fvattn_bwd_workspace_bytes(w.B, w.H, w.N, w.bs), dtype=torch.uint8, device=dev)
        gQ, gK, gV = torch.empty_like(dQ), torch.empty_like(dQ), torch.empty_like(dQ)
        st_b = torch.zeros(1, dtype=torch.int32, device=dev)

        def bwd_call():
            fv.fvattn_sparse_bwd(dQ, dK, dV, plan.O, plan.LSE, dO, *mask_csr(), w.bs,
                                 w.causal, stream=stream, dQ=gQ, dK=gK, dV=gV, workspace=ws_b, dev_status=st_b)
        for _ in range(2):
            bwd_call()
        torch.cuda.synchronize(dev)
        fv.check_status(st_b, "fvattn_sparse_bwd")
        reps = 5
        a.record(stream)
        for _ in range(reps):
            bwd_call()
        b.record(stream)
        torch.cuda.synchronize(dev)
        fv.check_status(st_b, "fvattn_sparse_bwd")
        bwd_ms = a.elapsed_time(b) / reps
        bwd = {"ms": bwd_ms, "tflops_effective": 2.5 * flops / (bwd_ms * 1e-3) / 1e12,
               "note": "effective = 2.5 x the forward's 4*block^2*d*nnz (five block GEMMs); the kernels run seven "
                       "(S and dP are recomputed in both the dQ and the dK/dV pass); mean of 5 calls after 2, "
                       "outside the timed region"}
        del gQ, gK, gV, ws_b, dO

    # FP8 variant (outside the timed step): e4m3 block quantization of Q, K and V, then
    # the e4m3 forward on the same mask
    fp8 = None
    if w.d == 128 and not args.no_fp8:
        q8 = [fv.fvattn_quant_e4m3(x, w.bs, stream=stream) for x in (dQ, dK, dV)]
        O8 = torch.empty_like(dQ)
        L8 = torch.empty_like(plan.LSE)
        st8 = torch.zeros(1, dtype=torch.int32, device=dev)

        def quant_call():
            for x, (c, e) in zip((dQ, dK, dV), q8):
                fv.fvattn_quant_e4m3(x, w.bs, stream=stream, out=c, scale_exp=e)

        def fp8_call():
            fv.fvattn_sparse_fwd_fp8(q8[0][0], q8[1][0], q8[2][0], q8[0][1], q8[1][1], q8[2][1], *mask_csr(), w.bs,
                                     w.causal, stream=stream, O=O8, LSE=L8, workspace=plan.fwd_ws, dev_status=st8)
        fwd()
        for _ in range(3):
            quant_call()
            fp8_call()
        torch.cuda.synchronize(dev)
        fv.check_status(st8, "fvattn_sparse_fwd_fp8")
        reps = max(5, min(args.steps, 20))
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
        for e0, e1, e2 in evs:
            e0.record(stream)
            quant_call()
            e1.record(stream)
            fp8_call()
            e2.record(stream)
        torch.cuda.synchronize(dev)
        fv.check_status(st8, "fvattn_sparse_fwd_fp8")
        q_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in evs)
        a8_ms = statistics.mean(b.elapsed_time(c) for _, b, c in evs)
        diff = (O8.float() - plan.O.float()).abs()
        fp8_peak = 2.0 * float(load_peaks()[0]["bf16_tflops"])
        fp8 = {"attn_ms": a8_ms, "attn_tflops": flops / (a8_ms * 1e-3) / 1e12,
               "frac_of_fp8_peak": flops / (a8_ms * 1e-3) / 1e12 / fp8_peak, "fp8_peak": fp8_peak,
               "speedup_vs_bf16_attn": attn_ms / a8_ms, "quant_ms": q_ms,
               "o_vs_bf16_path": {"max_abs": diff.max().item(), "mean_abs": diff.mean().item()},
               "note": "attention on e4m3 Q, K, V with power-of-two block scales (fvattn_sparse_fwd_fp8) on the "
                       "routing mask of the bf16 step; quant = three fvattn_quant_e4m3 calls; fp8_peak = measured "
                       "bf16 burst peak x 2 (the nominal e4m3/bf16 tensor ratio); o_vs_bf16_path compares with "
                       "the bf16 forward's O (the e4m3 rounding of the inputs included); mean of the timed "
                       "calls, outside the timed step"}
        del q8, O8, L8
        torch.cuda.empty_cache()

    # Slack-aware augmentation (outside the timed step): the routed mask plus, on the
    # SMs the list schedule leaves with slack, their rows' next routing candidates;
    # the attention timed on both masks
    sasa = None
    if not w.causal and not args.no_sasa:
        sms_n = torch.cuda.get_device_properties(dev).multi_processor_count
        sres = fv.fvattn_route_sasa(dQ, dK, w.p, w.bs, sms_n, stream=stream)
        torch.cuda.synchronize(dev)
        fv.check_status(sres.dev_status, "fvattn_route_sasa")
        reps = 5
        a.record(stream)
        for _ in range(reps):
            fv.fvattn_route_sasa(dQ, dK, w.p, w.bs, sms_n, stream=stream, out=sres)
        b.record(stream)
        torch.cuda.synchronize(dev)
        sasa_route_ms = a.elapsed_time(b) / reps

        # the two masks timed alternately, call by call, so that clock drift falls on both
        plan.run_route(dQ, dK, w.p, stream=stream)
        masks = [(plan.route.row_ptr, plan.route.col_idx), (sres.row_ptr, sres.col_idx)]
        for rp_, ci_ in masks:
            plan.run_fwd(dQ, dK, dV, w.causal, row_ptr=rp_, col_idx=ci_, stream=stream)
        per = [[], []]
        for _ in range(2 * reps):
            for k_, (rp_, ci_) in enumerate(masks):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                plan.run_fwd(dQ, dK, dV, w.causal, row_ptr=rp_, col_idx=ci_, stream=stream)
                e1.record(stream)
                per[k_].append((e0, e1))
        torch.cuda.synchronize(dev)
        plan.check()
        base_ms = statistics.median(x.elapsed_time(y) for x, y in per[0])
        aug_ms = statistics.median(x.elapsed_time(y) for x, y in per[1])
        added = sres.added.double()
        mass = sres.added_mass
        sasa = {"machines": sms_n, "blocks_added": int(added.sum().item()),
                "rows_touched": int((added > 0).sum().item()), "rows": int(added.numel()),
                "added_mass_mean_per_row": float(mass.mean().item()), "added_mass_max": float(mass.max().item()),
                "route_plus_plan_ms": sasa_route_ms, "route_ms": r_ms,
                "attn_ms_routed_mask": base_ms, "attn_ms_augmented_mask": aug_ms,
                "attn_time_change": aug_ms / base_ms - 1.0,
                "note": "fvattn_route_sasa: the routed rows list-scheduled over the SMs in the attention's queue "
                        "order, each SM's slack below the makespan filled with its rows' next-highest-probability "
                        "unselected blocks; attention timed on the routed and on the augmented mask, alternately "
                        "call by call (medians of 10 calls each, outside the timed step)"}

    peaks, peak_src = load_peaks()
    configs = None
    if world == 1 and not args.no_configs:
        # the other workloads, measured in the same run under their own clock record
        del hO, hL
        torch.cuda.empty_cache()
        cfg_sampler = ClockSampler(gpu_selector(dev))
        cfg_sampler.start()
        configs = {name: time_config(W.ALL[name], dev, stream, args.config_steps, float(peaks["bf16_tflops"]))
                   for name in CONFIG_SET if name != w.name}
        configs["clocks"] = cfg_sampler.stop()
        configs["note"] = ("each workload: 3 warm-up steps, then per-call CUDA events over config_steps steps; "
                           "attn = the fvattn_sparse_fwd call, route = the fvattn_route call; the causal "
                           "workload runs on the dense lower-triangle block mask, without routing")
    if rank != 0:
        return
    peak = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained", peak))
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(w, Qh, Kh, Vh, budget_s=args.cpu_budget)
        cpu.pop("route_s_full", None)
    rp_np = mask_csr()[0].cpu().numpy().astype(np.int64)
    counts = (rp_np[w.nb::w.nb] - rp_np[0:-1:w.nb])
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "block": w.bs, "p": w.p,
                   "causal": w.causal, "nnz_blocks": nnz, "density": nnz / (w.B * w.H * w.nb * w.nb),
                   "l2": "inputs larger than L2 (each of Q, K, V is %d MB)" % (elem * 2 // 10**6),
                   "parallelism": f"replicas x{world}"},
        "attn_tflops": attn_tflops, "attn_ms": attn_ms, "route_ms": r_ms, "timing": timing,
        "route_frac": r_ms / (r_ms + attn_ms),
        "tensor_frac_of_sustained_peak": attn_tflops / sustained,
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": attn_tflops / peak, "traffic": recorded_traffic(w.name),
                     "frac_of_sustained": attn_tflops / sustained,
                     "peak_source": f"{peak_src} bf16_tflops (burst: the timed region is well under a second "
                                    f"of back-to-back steps); frac_of_sustained divides by bf16_tflops_sustained",
                     "note": "achieved = 4*block^2*d*nnz / mean CUDA-event time of the fvattn_sparse_fwd call "
                             "(its 3 small ordering kernels included)"},
        "route_roofline": {"bound": "hbm", "pool_bytes": 2 * elem * 2,
                           "achieved_gbs_whole_route": 2 * elem * 2 / (r_ms * 1e-3) / 1e9,
                           "peak": float(peaks["hbm_gbs"]), "unit": "GB/s"},
        "head_counts": {"min": int(counts.min()), "max": int(counts.max()), "mean": float(counts.mean()),
                        "density_histogram": {"edges": [round(x, 1) for x in np.linspace(0.0, 1.0, 11)],
                                              "heads": np.histogram(counts / float(w.nb * w.nb), bins=10,
                                                                    range=(0.0, 1.0))[0].tolist()}},
        "load_balance": dict(balance, note="LIF = max / mean busy time over the CTAs of the persistent grid "
                                           "(global timer, one call each); lpt = the head-major longest-first "
                                           "queue fvattn_sparse_fwd uses, natural = rows in index order"),
        "bwd": None if bwd is None else dict(bwd, frac_of_burst=bwd["tflops_effective"] / peak,
                                              frac_of_sustained=bwd["tflops_effective"] / sustained),
        "mufu": {"exp_per_s": float(nnz) * w.bs * w.bs / (attn_ms * 1e-3),
                 "ceiling_at_max_clock": 16.0 * sms * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6,
                 "frac": float(nnz) * w.bs * w.bs / (attn_ms * 1e-3)
                         / (16.0 * sms * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6),
                 "note": "one exp2 per selected score (full tiles); ceiling = 16 per clock per SM"},
        "e2e": {"value": flops / (e2e_ms * 1e-3) / 1e12 * world, "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * (ROUTE_KERNELS_PER_CALL + FWD_KERNELS_PER_CALL),
        "clocks": clocks,
        "cpu_baseline": cpu,
        "configs": configs,
        "fp8": fp8,
        "sasa": sasa,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=W.VIDEO.name, choices=sorted(W.ALL))
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the other workloads' timings")
    ap.add_argument("--no-fp8", action="store_true", help="skip the e4m3 forward's timing")
    ap.add_argument("--no-sasa", action="store_true", help="skip the slack-aware augmentation's timing")
    ap.add_argument("--config-steps", type=int, default=10)
    args = ap.parse_args()
    w = W.ALL[args.workload]
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        run_reference(args, w, rank, world)
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        run_ours(args, w, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
