"""Absorbed-MLA decode throughput on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config v3] [--impl reference]

A step is one pass of the per-token hot path over one batch of synthetic,
seeded input: plan + attend + combine (mla_decode) and the per-head
up-projection (mla_up_proj).  Query formation and weight absorption are
setup (once per model / once per token before the layer's attention) and are
not timed.  Inputs are resident in HBM; the step rotates over enough copies
of its inputs (>= 3x the 126 MB L2) that every step reads its cache from HBM.
Each step is replayed from a CUDA graph captured per input copy.  The
attend kernel's own duration comes from event nodes around it, captured in
a second graph per copy that replaces the plain one for the last timed step
of that copy: an event node between two kernels turns their programmatic
(overlapping) launch into a plain dependency, so the other timed steps run
without it, as a caller's step does.

value = algorithmic TFLOP/s of the whole job (all ranks) over the timed
steps; the roofline object rates the attend kernel against the measured
HBM / bf16 peaks.  Multi-GPU runs are weak scaling: every rank decodes its
own batch of the same shape (independent sequences, no data-path
collective); the timing is the max over ranks.

--impl reference times the fp64 CPU oracle (the non-absorbed definition) on
a bounded sample of the same workload per step, on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from mla_latent_kv_23_b200 import synth  # noqa: E402

METRIC = "MLA decode TFLOP/s, HBM GB/s, % of B200 roofline (V3 shape, bf16, 1 GPU)"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
PROFILE_DIR = os.path.join(ROOT, "profiles")
KERNEL_SOURCES = ["decode_sm100.cu", "sm100_ptx.cuh", "schedule.cuh", "internal.h"]


# ----------------------------------------------------------------------------
# algorithmic work (what the method must move / compute; no padding, no partials)
# ----------------------------------------------------------------------------
def decode_work(w: synth.Workload, seqlens) -> dict:
    L = np.asarray(seqlens, dtype=np.int64)
    rows = w.B * w.s_q * w.n_h
    cache_bytes = int(L.sum()) * w.width * 2
    io_bytes = rows * (w.width * 2 + w.d_c * 2 + 4)
    pairs = sum(int(l) - w.s_q + 1 + r for l in L for r in range(w.s_q))   # unmasked (row, token)
    flops = 2 * w.n_h * (w.width + w.d_c) * pairs
    return dict(bytes=cache_bytes + io_bytes, cache_bytes=cache_bytes, flops=flops)


def up_proj_work(w: synth.Workload) -> dict:
    T = w.B * w.s_q
    return dict(bytes=w.n_h * w.d_v * w.d_c * 2 + T * w.n_h * (w.d_c + w.d_v) * 2,
                flops=2 * T * w.n_h * w.d_v * w.d_c)


def load_peaks() -> tuple[dict, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"]))), "measured"
    return dict(FALLBACK_PEAKS, bf16_tflops_sustained=1400.0), "fallback"


def code_only(text: str) -> str:
    """Source text without comments, trailing blanks and empty lines: a
    change to comments alone leaves the compiled kernel and its hash as they
    were."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(code_only(open(os.path.join(ROOT, "mla_latent_kv_23_b200", "csrc", f)).read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """dram bytes per attend launch from the committed ncu summary, if it was
    taken on the current kernel source; else None."""
    path = os.path.join(PROFILE_DIR, f"decode_sm100_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_h = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    m_t = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_h or not m_t or m_h.group(1) != kernel_hash():
        return None
    return float(m_t.group(1))


# ----------------------------------------------------------------------------
# clocks during the timed region (NVML, polled from a thread)
# ----------------------------------------------------------------------------
class ClockSampler:
    REASONS = {"gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
               "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period_s: float = 0.0005):
        self.samples = []
        self.period = period_s
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)
        self._stop = threading.Event()
        self._mark = None

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def mark(self, t0, t1):
        self._mark = (t0, t1)

    def stop(self) -> dict:
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "")}
        self._stop.set()
        self.t.join()
        t0, t1 = self._mark
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed region"
        if len(inside) < 3:   # a short timed region: add the soak replays right before it
            inside = [s for s in self.samples if t0 - 0.1 <= s[0] <= t1]
            window = "timed region + up to 0.1 s of identical untimed replays just before it"
        busy = [s for s in inside if not (s[2] & self.REASONS["gpu_idle"])] or inside
        reasons = sorted({n for s in busy for n, bit in self.REASONS.items()
                          if s[2] & bit and n != "gpu_idle"})
        return {"sm_mhz": statistics.median([s[1] for s in busy]) if busy else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(busy),
                "window": window}


# ----------------------------------------------------------------------------
# the oracle on host cores (cpu_baseline / reference arm)
# ----------------------------------------------------------------------------
def oracle_sample(w: synth.Workload, inp: dict, budget_s: float, picks_per_step: int = 1):
    """Times the expanded fp64 oracle on (sequence, row, head) picks until
    budget_s elapses.  Returns (tflops, seconds, n_picks, threads)."""
    from oracle import mla_oracle as orc
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        threads = os.cpu_count()
    rng = np.random.default_rng(123)
    flops = 0
    n = 0
    t0 = time.perf_counter()
    while True:
        b = int(rng.integers(w.B))
        i = int(rng.integers(w.n_h))
        picks = [(b, r, i) for r in range(w.s_q)]
        orc.decode_expanded(inp, w, picks)
        L = int(inp["seqlens"][b])
        flops += sum(2 * (w.width + w.d_c) * (L - w.s_q + 1 + r) for r in range(w.s_q))
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s and n >= picks_per_step:
            break
    return flops / el / 1e12, el, n, threads


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = synth.draw(w)
    times = []
    flops_total = 0.0
    for k in range(args.warmup + args.steps):
        tf, el, n, threads = oracle_sample(w, inp, budget_s=0.0)
        if k >= args.warmup:
            times.append(el)
            flops_total += tf * 1e12 * el
    total = sum(times)
    value = flops_total / total / 1e12
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": workload_config(w, "oracle: one (sequence, head) pick per step"),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": "per step: the expanded fp64 oracle on one seeded (sequence, head) "
                                       "pick, all query rows, full context length"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(w, l2_note):
    return {"workload": f"{w.name}: DeepSeek-V3-shaped MLA decode layer (n_h={w.n_h}, d_c={w.d_c}, "
                        f"d_R={w.d_R}, d_v={w.d_v}), B={w.B}, "
                        + (f"L={w.seqlens[0]}" if w.seqlens else f"L~U{w.len_range}")
                        + f", s_q={w.s_q}, page={w.page_size}, bf16 cache/weights, fp32 accumulate",
            "B": w.B, "seq_len": int(w.seqlens[0]) if w.seqlens else None, "s_q": w.s_q,
            "n_h": w.n_h, "d_c": w.d_c, "d_R": w.d_R, "page_size": w.page_size,
            "softmax_scale": w.softmax_scale, "l2": l2_note,
            "step": "mla_decode_step (plan + attend + combine fused into the up-projection; "
                    "with a bf16 u: mla_decode + mla_up_proj)",
            "graphs": "CUDA graphs: the steps over the rotating input copies captured back to "
                      "back in one graph; the last copy-count steps replay one-step graphs "
                      "with events around the attend kernel"}


# ----------------------------------------------------------------------------
# the CUDA path
# ----------------------------------------------------------------------------
def run_gpu(args, w):
    import torch
    import torch.distributed as dist

    from mla_latent_kv_23_b200 import mla

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    mla.lib()

    # ---- inputs (the same seeded batch shape on every rank; seed offset by rank)
    wr = w.with_(seed=w.seed + 1000 * rank) if rank else w
    inp = synth.draw(wr)
    tdt = torch.bfloat16
    udt = torch.float32 if args.u_dtype == "fp32" else torch.bfloat16
    from mla_latent_kv_23_b200.device_inputs import absorb_and_query
    q0, W_QK = absorb_and_query(wr, inp, dev)
    del W_QK
    cache_bytes = inp["num_pages"] * w.page_size * w.width * 2
    step_in_bytes = cache_bytes + q0.numel() * 2 + w.n_h * w.d_v * w.d_c * 2  # + W^UV
    R = max(2, math.ceil(3 * L2_BYTES / step_in_bytes))
    caches = [torch.from_numpy(inp["cache"]).to(dev).to(tdt)]
    for _ in range(R - 1):
        caches.append(caches[0].clone())
    qs = [q0] + [q0.clone() for _ in range(R - 1)]
    bt = torch.from_numpy(inp["block_table"]).to(dev)
    sl = torch.from_numpy(inp["seqlens"]).to(dev)
    W_UV = torch.from_numpy(inp["W_UV"]).to(dev).to(tdt)
    # the weights rotate with the inputs: a decode loop reads another layer's W^UV
    # between two uses of one layer's, so no step finds them in L2 from the last
    W_UVs = [W_UV] + [W_UV.clone() for _ in range(R - 1)]
    T = w.B * w.s_q
    u = torch.empty((w.B, w.s_q, w.n_h, w.d_c), dtype=udt, device=dev)
    lse = torch.empty((w.B, w.s_q, w.n_h), dtype=torch.float32, device=dev)
    o = torch.empty((T, w.n_h, w.d_v), dtype=tdt, device=dev)
    params = [mla.decode_params(qs[i], caches[i], bt, sl, u, lse, w.page_size, w.d_R,
                                w.softmax_scale, args.splits) for i in range(R)]
    ws = torch.empty(mla.mla_decode_workspace_size(params[0]), dtype=torch.uint8, device=dev)
    tc, chunks = mla.mla_decode_kernel_info(params[0])
    if not tc:
        raise RuntimeError("the tensor-core decode kernel was not selected for this workload")

    fused = args.u_dtype == "fp32"

    def step(i, ev=None):
        # the caller's step: plan, attend and (with an fp32 u) the combine
        # fused into the up-projection, chained by programmatic dependent
        # launch (mla_decode_step); with a bf16 u, mla_decode then
        # mla_up_proj.  With events, the stages are called one by one so that
        # the attend kernel alone sits between the two event nodes.
        p = params[i % R]
        if ev is None:
            if fused:
                mla.mla_decode_step(p, W_UVs[i % R], o, ws)
                return
            mla.mla_decode(p, ws)
        else:
            ev[2].record()
            mla.mla_decode_plan(p, ws)
            ev[0].record()
            mla.mla_decode_attend(p, ws)
            ev[1].record()
            mla.mla_decode_combine(p, ws)
            ev[3].record()
        mla.mla_up_proj(u.view(T, w.n_h, w.d_c), W_UVs[i % R], o)

    # direct launches once (initialises the library, checks flags)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for i in range(R):
            step(i)
    stream.synchronize()
    mla.mla_check_device_errors(stream)

    # one plain graph per input copy, and one with event nodes around the
    # attend kernel that the last timed step of each copy replays instead
    graphs, timed_graphs, evs = [], [], []
    for i in range(R):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(i)
        graphs.append(g)
        g = torch.cuda.CUDAGraph()
        # [0, 1] around the attend kernel, [2, 3] around plan + attend + combine
        ev = tuple(torch.cuda.Event(enable_timing=True, external=True) for _ in range(4))
        with torch.cuda.graph(g, stream=stream):
            step(i, ev)
        timed_graphs.append(g)
        evs.append(ev)
    # the R copies' steps back to back in one graph: the steps of a decode
    # loop captured together, so consecutive steps are not separated by a
    # graph launch each
    chain = torch.cuda.CUDAGraph()
    with torch.cuda.graph(chain, stream=stream):
        for i in range(R):
            step(i)
    torch.cuda.synchronize(dev)
    # timed step k replays copy (warmup + k) % R; the last min(R, steps) steps
    # carry the event nodes, one per copy
    n_ev = min(R, args.steps)
    ev_copies = [(args.warmup + k) % R for k in range(args.steps - n_ev, args.steps)]

    sampler = ClockSampler(local)
    sampler.start()
    with torch.cuda.stream(stream):
        for k in range(args.warmup):
            graphs[k % R].replay()
        for g in timed_graphs:  # first launches (graph upload) stay out of the timed region
            g.replay()
        chain.replay()
    stream.synchronize()
    # untimed soak of the same replays (~50 ms) so that the clock sampler has
    # readings of the loaded GPU right up to the timed region
    soak_until = time.perf_counter() + 0.05
    with torch.cuda.stream(stream):
        k = 0
        while time.perf_counter() < soak_until:
            for _ in range(16):
                graphs[k % R].replay()
                k += 1
            stream.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wall0 = time.perf_counter()
    with torch.cuda.stream(stream):
        t_start.record()
        k = 0
        while k < args.steps:
            i = (args.warmup + k) % R
            if k >= args.steps - n_ev:
                timed_graphs[i].replay()
                k += 1
            elif i == 0 and k + R <= args.steps - n_ev:
                chain.replay()  # steps k .. k + R - 1 on copies 0 .. R - 1
                k += R
            else:
                graphs[i].replay()
                k += 1
        t_end.record()
    stream.synchronize()
    wall1 = time.perf_counter()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.mark(wall0, wall1)
    clocks = sampler.stop()
    mla.mla_check_device_errors(stream)
    ms_total = t_start.elapsed_time(t_end)
    attend_ms = statistics.fmean(evs[i][0].elapsed_time(evs[i][1]) for i in ev_copies)
    decode_ms = statistics.fmean(evs[i][2].elapsed_time(evs[i][3]) for i in ev_copies)
    hdr = ws[:64 * 4].view(torch.int32).cpu().tolist()  # the plan's header (workspace)

    t = torch.tensor([ms_total], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_total = float(t.item())
    ms_step = ms_total / args.steps

    dw = decode_work(w, inp["seqlens"])
    uw = up_proj_work(w)
    step_flops = dw["flops"] + uw["flops"]
    step_bytes = dw["bytes"] + uw["bytes"]
    value = world * step_flops / (ms_step * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    t_hbm = dw["bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_tc = dw["flops"] / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    if bound == "hbm":
        achieved = dw["bytes"] / (attend_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        achieved = dw["flops"] / (attend_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = profiled_traffic(w.name)
    roof["peak_source"] = peak_src + (" (hbm_gbs copy)" if bound == "hbm" else " (bf16_tflops burst)")
    roof["kernel"] = "decode_sm100_kernel (mla_decode_attend)"
    roof["launch_us"] = attend_ms * 1e3
    roof["samples"] = n_ev
    roof["roofline_us"] = max(t_hbm, t_tc) * 1e6
    roof["alg_bytes_per_launch"] = dw["bytes"]
    roof["alg_flops_per_launch"] = dw["flops"]
    # the decode stage alone (plan + attend + combine, staged calls with
    # events around them), against the same roofline
    decode_stage = {"us": decode_ms * 1e3, "frac": max(t_hbm, t_tc) / (decode_ms * 1e-3),
                    "calls": "mla_decode_plan + mla_decode_attend + mla_decode_combine"}

    # ---- end to end through the public API with host buffers (pinned)
    e2e = run_e2e(args, w, inp, q0, bt, sl, W_UV, dev, stream, mla, step_flops, world) \
        if args.e2e_steps > 0 else None

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and args.cpu_seconds > 0:
            tf, el, n, threads = oracle_sample(wr, inp, budget_s=args.cpu_seconds)
            cpu = {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                   "sample": f"expanded fp64 oracle on {n} seeded (sequence, head) picks of this "
                             f"workload (full context each), {el:.1f} s of host time"}
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic: seeded N(0,1) latent cache and RoPE keys; q from random h "
                        "through the absorbed weights",
                "config": workload_config(w, f"rotating {R} input copies "
                                             f"({R * step_in_bytes / 2**20:.0f} MiB > 3x L2)"),
                "us_per_step": ms_step * 1e3,
                "hbm_gbs": world * step_bytes / (ms_step * 1e-3) / 1e9,
                "decode_roofline_frac_step": max(t_hbm, t_tc) * 1e3 / ms_step,
                "kv_chunks": chunks, "kv_chunks_used": int(hdr[6]),
                "kv_cut": "aligned to sequences" if int(hdr[5]) else "cost line",
                "decode_stage": decode_stage,
                "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": (3 if fused else 4) * (args.steps - n_ev) + 4 * n_ev, "clocks": clocks}
        print(json.dumps(line), flush=True)
    graphs.clear()
    timed_graphs.clear()
    del chain
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return line


def run_e2e(args, w, inp, q0, bt, sl, W_UV, dev, stream, mla, step_flops, world):
    import torch
    import torch.distributed as dist
    tdt = torch.bfloat16
    T = w.B * w.s_q
    h_cache = torch.from_numpy(inp["cache"]).to(tdt).pin_memory()
    h_q = q0.cpu().pin_memory()
    h_bt = torch.from_numpy(inp["block_table"]).pin_memory()
    h_sl = torch.from_numpy(inp["seqlens"]).pin_memory()
    h_o = torch.empty((T, w.n_h, w.d_v), dtype=tdt).pin_memory()
    h_lse = torch.empty((w.B, w.s_q, w.n_h), dtype=torch.float32).pin_memory()
    d_cache = torch.empty(h_cache.shape, dtype=tdt, device=dev)
    d_q = torch.empty(h_q.shape, dtype=tdt, device=dev)
    d_bt = torch.empty(h_bt.shape, dtype=torch.int32, device=dev)
    d_sl = torch.empty(h_sl.shape, dtype=torch.int32, device=dev)
    u = torch.empty((w.B, w.s_q, w.n_h, w.d_c), dtype=torch.float32 if args.u_dtype == "fp32"
                    else tdt, device=dev)
    lse = torch.empty((w.B, w.s_q, w.n_h), dtype=torch.float32, device=dev)
    o = torch.empty((T, w.n_h, w.d_v), dtype=tdt, device=dev)
    p = mla.decode_params(d_q, d_cache, d_bt, d_sl, u, lse, w.page_size, w.d_R, w.softmax_scale,
                          args.splits)
    ws = torch.empty(mla.mla_decode_workspace_size(p), dtype=torch.uint8, device=dev)
    h2d = sum(t.numel() * t.element_size() for t in (h_cache, h_q, h_bt, h_sl))
    d2h = h_o.numel() * h_o.element_size() + h_lse.numel() * 4

    def one():
        d_cache.copy_(h_cache, non_blocking=True)
        d_q.copy_(h_q, non_blocking=True)
        d_bt.copy_(h_bt, non_blocking=True)
        d_sl.copy_(h_sl, non_blocking=True)
        if args.u_dtype == "fp32":
            mla.mla_decode_step(p, W_UV, o, ws)
        else:
            mla.mla_decode(p, ws)
            mla.mla_up_proj(u.view(T, w.n_h, w.d_c), W_UV, o)
        h_o.copy_(o, non_blocking=True)
        h_lse.copy_(lse, non_blocking=True)

    steps = max(3, min(args.steps, args.e2e_steps))
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            one()
    stream.synchronize()
    if world > 1:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record()
        for _ in range(steps):
            one()
        b.record()
    stream.synchronize()
    ms = a.elapsed_time(b) / steps
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms = float(t.item())
    mla.mla_check_device_errors(stream)
    return {"value": world * step_flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "steps": steps, "api": "mla_decode_step (C ABI via ctypes), pinned host buffers"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="v3", choices=["v3", "ragged", "mtp", "long"])
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="host time for the oracle baseline (0 = skip)")
    ap.add_argument("--e2e-steps", type=int, default=20,
                    help="steps of the end-to-end (host buffers) measurement (0 = skip)")
    ap.add_argument("--splits", type=int, default=0,
                    help="KV chunks the batch is cut into (0: the library's automatic count)")
    ap.add_argument("--u-dtype", default="fp32", choices=["fp32", "bf16"],
                    help="type of the decode's u (fp32: the precision the parity tests hold "
                         "every workload to)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = synth.config(args.config)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
