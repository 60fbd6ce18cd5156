"""Benchmark of the RoM projection block forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--no-cpu-baseline]

One step = one pass of the whole block over one batch of synthetic input:
route -> dispatch -> Conv+Gate grouped GEMM (+ gate combine for top-k > 1)
-> Out grouped GEMM (+ slot sum for top-k > 1); for the Swimba decode
workload: route -> dispatch -> routed in-projection. Inputs are resident in
HBM when the timed region starts. Between timed steps the L2 is flushed (a
256 MiB write, outside the step's events), except where the step's inputs
(tokens and weights) exceed twice the L2: then every step streams them from
HBM anyway, and a flush would only add the write-back of its own dirty lines
to the next step. `config["l2"]` says which. Each step is timed with CUDA
events on the launching stream; the dominant kernel is bracketed by its own
events for the roofline. Under torchrun every rank runs an independent
replica on its own GPU (the block needs no collective in the forward); the
reported time is the max over ranks and `value` counts all ranks' tokens.

`--impl reference` times the CPU oracle (the float64 numpy definition) on a
bounded sample of the same workload on the host cores; under torchrun only
rank 0 runs it.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_projections_b200.inputs import WORKLOADS, bf16_bits, make_workload_inputs  # noqa

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
L2_BYTES = 126 * 10**6  # B200 L2


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


def strip_c_comments(src):
    """C / C++ / CUDA source without its comments, trailing blanks and blank
    lines; string and character literals are kept as written."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (ln.rstrip() for ln in "".join(out).splitlines())
    return "\n".join(ln for ln in lines if ln)


def csrc_digest(root=ROOT):
    """sha256 over the CUDA sources and the C header with their comments
    removed (identifies the kernels: a comment edit leaves it unchanged)."""
    import glob
    import hashlib
    h = hashlib.sha256()
    files = sorted(glob.glob(os.path.join(root, "mixture_experts_projections_b200", "csrc", "*.cu*")))
    files.append(os.path.join(root, "include", "rom.h"))
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, encoding="utf-8") as fh:
            h.update(strip_c_comments(fh.read()).encode())
    return h.hexdigest()


def profiled_traffic(workload):
    """DRAM bytes per launch of the dominant kernel from profiles/traffic.json,
    if that ncu capture was taken on exactly these kernel sources, else None."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    ent = t.get(workload)
    if not ent or ent.get("csrc_sha256") != csrc_digest():
        return None
    return ent.get("dram_bytes_per_launch")


def block_flops(wl):
    R = wl.T * wl.k
    if wl.kind == "inproj":
        return {"inproj": 2.0 * R * wl.Dm * wl.De}
    f = {"conv_gate": 4.0 * R * wl.Dm * wl.De, "out": 2.0 * R * wl.De * wl.Dm}
    if wl.backward:  # dgrad (Out, In+Gate) and wgrad (Out, In+Gate): twice the forward
        f["backward"] = 2.0 * (f["conv_gate"] + f["out"])
    return f


def inproj_bytes(wl, n_experts_hit):
    """Algorithmic HBM bytes of the routed in-projection: the weights of the
    experts that received tokens, x in, the output out (bf16)."""
    return n_experts_hit * wl.Dm * wl.De * 2 + wl.T * wl.Dm * 2 + wl.T * wl.De * 2


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        return summarize_clocks(self.lines)


THROTTLE_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


def summarize_clocks(lines):
    """Median SM clock, the largest max clock and the throttle reasons seen
    Active in `nvidia-smi --query-gpu=<ClockSampler.FIELDS> --format=csv,
    noheader,nounits` lines; lines that do not parse are skipped."""
    sm, smax, reasons = [], [], set()
    for ln in lines:
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            smax.append(float(parts[2]))
        except ValueError:
            continue
        for n, v in zip(THROTTLE_REASONS, parts[5:9]):
            if v.lower().startswith("active"):
                reasons.add(n)
    return {"sm_mhz": float(np.median(sm)) if sm else None,
            "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
            "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def oracle_sample_run(wl, inp, tokens):
    """One call of the CPU oracle on the given tokens; returns seconds."""
    from oracle import rom_oracle as orc
    t0 = time.perf_counter()
    if wl.kind == "inproj":
        orc.inproj_forward(inp["x"], inp["w_r"], inp["w"], k=wl.k, tokens=tokens)
    else:
        orc.block_forward(inp["x"], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"],
                          k=wl.k, bias=inp["bias"], renorm=wl.renorm, tokens=tokens)
    return time.perf_counter() - t0


def cpu_baseline(wl, inp, budget_s=15.0):
    """Time the oracle on a growing token sample until it takes ~budget_s."""
    n = 16
    rng = np.random.default_rng(0)
    while True:
        toks = np.sort(rng.choice(wl.T, size=min(n, wl.T), replace=False))
        dt = oracle_sample_run(wl, inp, toks)
        if dt >= budget_s / 3 or n >= wl.T:
            break
        n = min(wl.T, n * 4)
    return {"value": len(toks) / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{len(toks)} of {wl.T} tokens of {wl.name} (float64 numpy oracle), "
                      f"{dt:.1f} s"}


# ------------------------------------------------------------------ GPU arm


def to_dev(torch, a, bf16):
    if bf16:
        return torch.from_numpy(bf16_bits(a).view(np.int16).copy()).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def max_over_ranks(values, device, world):
    """Elementwise maximum of per-rank timings (ms totals) over all ranks of the
    default process group: a multi-rank step lasts as long as its slowest
    rank. Every rank calls it, in the same order."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_tokens_per_s(tokens_per_rank, world, step_ms):
    """Whole-job throughput of replicas: every rank processes its own batch of
    `tokens_per_rank` tokens in a step that lasts `step_ms` (max over ranks)."""
    return tokens_per_rank * world / (step_ms / 1e3)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from mixture_experts_projections_b200 import rom

    torch.cuda.set_device(local_rank)
    rom.load_library()
    wl = WORKLOADS[args.workload]
    bf16 = wl.dtype == "bf16"
    inp = make_workload_inputs(wl, seed=0)
    stream = torch.cuda.current_stream()
    x = to_dev(torch, inp["x"], bf16)
    w_r = to_dev(torch, inp["w_r"], False)
    bias = None if inp.get("bias") is None else to_dev(torch, inp["bias"], False)
    if wl.kind == "inproj":
        w = to_dev(torch, inp["w"], bf16).transpose(1, 2).contiguous()
        bufs = rom.RoutingBuffers(wl.T, wl.Dm, wl.E, wl.k, x.dtype, x.device)
        out = torch.empty((wl.T, wl.De), dtype=x.dtype, device=x.device)
        slots = (torch.empty((wl.T * wl.k, wl.De), dtype=torch.float32, device=x.device)
                 if wl.k > 1 else None)
    else:
        ws = {n: to_dev(torch, inp[n], bf16).transpose(1, 2).contiguous()
              for n in ("w_conv", "w_gate", "w_out")}
        bufs = rom.BlockBuffers(wl.T, wl.Dm, wl.De, wl.E, wl.k, x.dtype, x.device)
    del inp["x"]
    # inputs of one step: the tokens and every weight the step reads
    in_bytes = x.numel() * x.element_size() + w_r.numel() * w_r.element_size()
    if wl.kind == "inproj":
        in_bytes += w.numel() * w.element_size()
    else:
        in_bytes += sum(t.numel() * t.element_size() for t in ws.values())
    if wl.backward:
        in_bytes += x.numel() * x.element_size()  # dO, same shape as X
    flush_l2 = in_bytes < 2 * L2_BYTES
    flush = (torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=x.device)
             if flush_l2 else None)
    l2_note = ("flushed before every timed step (256 MiB write)" if flush_l2 else
               f"not flushed: the step's inputs ({in_bytes / 1e6:.0f} MB) exceed twice the L2 "
               f"({L2_BYTES / 1e6:.0f} MB) and are streamed from HBM every step")

    def do_flush():
        if flush is not None:
            flush.zero_()
    R = wl.T * wl.k
    dt = rom.ROM_BF16 if bf16 else rom.ROM_F32

    # The step as three phases: route + dispatch, the dominant projection
    # (Conv+Gate, or the in-projection), and the rest.
    if wl.kind == "inproj":
        def ph_route():
            rom.route_and_dispatch(x, w_r, bias, wl.E, wl.k, wl.renorm, bufs)

        def ph_p0():
            rom.rom_expert_proj(rom.ROM_PROJ_INPROJ, bufs.x_sorted[:R], w, None, wl.E, wl.k,
                                bufs.offsets, bufs.sorted_slot, bufs.topk_w,
                                out if wl.k == 1 else slots)

        def ph_p1():
            if wl.k > 1:
                rom.rom_combine(rom.ROM_COMBINE_SUM, dt, slots, wl.T, wl.k, wl.De, None, out)
        out_t = out
        counts_t = bufs.counts
    else:
        rb = bufs.routing

        def ph_route():
            rom.route_and_dispatch(x, w_r, bias, wl.E, wl.k, wl.renorm, rb)

        def ph_p0():
            rom.rom_expert_proj(rom.ROM_PROJ_CONV_GATE, rb.x_sorted[:R], ws["w_conv"],
                                ws["w_gate"], wl.E, wl.k, rb.offsets, rb.sorted_slot, rb.topk_w,
                                bufs.h_sorted if wl.k == 1 else bufs.uz)

        def ph_p1():
            if wl.k == 1:
                rom.rom_expert_proj(rom.ROM_PROJ_OUT, bufs.h_sorted[:R], ws["w_out"], None, wl.E,
                                    1, rb.offsets, rb.sorted_slot, rb.topk_w, bufs.out)
            else:
                rom.rom_combine(rom.ROM_COMBINE_GATE, dt, bufs.uz, wl.T, wl.k, wl.De,
                                rb.slot_pos, bufs.h_sorted)
                rom.rom_expert_proj(rom.ROM_PROJ_OUT, bufs.h_sorted[:R], ws["w_out"], None,
                                    wl.E, wl.k, rb.offsets, rb.sorted_slot, rb.topk_w,
                                    bufs.o_slots)
                rom.rom_combine(rom.ROM_COMBINE_SUM, dt, bufs.o_slots, wl.T, wl.k, wl.Dm, None,
                                bufs.out)
        out_t = bufs.out
        counts_t = rb.counts
    phases = [ph_route, ph_p0, ph_p1]
    if wl.backward:
        dout = to_dev(torch, inp["dout"], bf16)
        bwd_bufs = rom.BackwardBuffers(wl.T, wl.Dm, wl.De, wl.E, wl.k, x.device)

        def ph_bwd():
            rom.block_backward(bufs, dout, w_r, ws["w_conv"], ws["w_gate"], ws["w_out"],
                               renorm=wl.renorm, bufs=bwd_bufs)
        phases.append(ph_bwd)

    def step():
        for ph in phases:
            ph()
        return out_t

    # our kernels per step: router + dispatch (+ the memset of counts, not ours),
    # the projection(s) and, for top-k > 1, the combines
    if wl.kind == "inproj":
        launches_per_step = 3 + (1 if wl.k > 1 else 0)
    else:
        launches_per_step = 4 + (2 if wl.k > 1 else 0) + (7 if wl.backward else 0)

    for _ in range(args.warmup):
        do_flush()
        step()
    torch.cuda.synchronize()
    if rom.rom_get_status() != 0:
        raise RuntimeError("device status word reports an error after warm-up")

    # The step captured once as one CUDA graph (the launch sequence of the
    # library is static: its kernels read the expert counts on the device),
    # and each phase once more on its own for the per-phase breakdown.
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        step()
    graphs = []
    for ph in phases:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            ph()
        graphs.append(g)
    torch.cuda.synchronize()

    def timed_loop(run_phase, n):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(phases) + 1)]
               for _ in range(n)]
        for i in range(n):
            do_flush()
            torch.cuda._sleep(200_000)  # GPU-side head start so that the host stays ahead
            evs[i][0].record(stream)
            for j in range(len(phases)):
                run_phase(j)
                evs[i][j + 1].record(stream)
        torch.cuda.synchronize()
        return np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(len(phases))]
                         for i in range(n)])

    def timed_steps(n):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
        for i in range(n):
            do_flush()
            torch.cuda._sleep(200_000)  # GPU-side head start so that the host stays ahead
            evs[i][0].record(stream)
            g_step.replay()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        return np.array([evs[i][0].elapsed_time(evs[i][1]) for i in range(n)])

    for _ in range(2):  # graph warm-up
        timed_loop(lambda j: graphs[j].replay(), 1)
        timed_steps(1)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    step_ms = timed_steps(args.steps)
    ph_ms = timed_loop(lambda j: graphs[j].replay(), args.steps)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    eager_ms = timed_loop(lambda j: phases[j](), args.steps)
    t_total_ms = float(step_ms.sum())
    part_names = ["route_dispatch", "proj0", "proj1", "backward"][:len(phases)]
    part_ms = {n: float(ph_ms[:, j].mean()) for j, n in enumerate(part_names)}
    # The dominant kernel alone (one eager launch between two events, the
    # host ahead of the GPU): no graph-launch latency in its duration.
    part_ms_eager = {n: float(eager_ms[:, j].mean()) for j, n in enumerate(part_names)}

    # ---------------------------------------------- e2e through host buffers
    # The public host-buffer call: inputs in pinned host memory, result copied
    # back, copies inside the timed region. Forward-only workloads go through
    # rom.HostPipeline (chunks over 3 streams: copies overlap the kernels);
    # the forward + backward step copies x in and O out around one step.
    h_x = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
    h_x.copy_(x)
    h_out = torch.empty(out_t.shape, dtype=out_t.dtype, pin_memory=True)
    pipe = None
    if not wl.backward:
        pipe = rom.HostPipeline(wl.T, wl.Dm, wl.De, wl.E, wl.k, x.dtype, x.device,
                                De=None if wl.kind == "inproj" else wl.De)

    def e2e_call():
        if pipe is None:
            x.copy_(h_x, non_blocking=True)
            o = step()
            h_out.copy_(o, non_blocking=True)
        elif wl.kind == "inproj":
            pipe.inproj_forward(h_x, w_r, w, h_out, renorm=wl.renorm, bias=bias)
        else:
            pipe.block_forward(h_x, w_r, bias, ws["w_conv"], ws["w_gate"], ws["w_out"], h_out,
                               renorm=wl.renorm)

    e2e_ms = []
    for i in range(args.warmup + args.steps):
        do_flush()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        e2e_call()
        s1.record(stream)
        s1.synchronize()
        if i >= args.warmup:
            e2e_ms.append(s0.elapsed_time(s1))
    e2e_total = float(np.sum(e2e_ms))
    del graphs, g_step

    t_total_ms, e2e_total = max_over_ranks([t_total_ms, e2e_total], x.device, world)
    res = dict(wl=wl, step_ms=t_total_ms / args.steps, part_ms=part_ms,
               part_ms_eager=part_ms_eager,
               eager_ms=float(eager_ms.sum()) / args.steps,
               e2e_ms=e2e_total / args.steps, clocks=clk, launches=launches_per_step * args.steps,
               counts=counts_t.cpu().numpy(), x_bytes=x.numel() * x.element_size(), l2=l2_note,
               out_bytes=out_t.numel() * out_t.element_size())
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill_16k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token count (smaller profiling cases)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.tokens is not None:
        import dataclasses
        WORKLOADS[args.workload] = dataclasses.replace(WORKLOADS[args.workload], T=args.tokens)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = WORKLOADS[args.workload]
    flops = block_flops(wl)
    metric = (f"tokens/s and TFLOPS (% bf16 peak) for RoM projection block "
              f"{'fwd+bwd' if wl.backward else 'fwd'}, {world} B200")
    config = {"workload": wl.name, "tokens": wl.T, "d_model": wl.Dm,
              ("d_out" if wl.kind == "inproj" else "d_inner"): wl.De, "experts": wl.E,
              "top_k": wl.k, "renorm": wl.renorm, "parallelism": f"replicas x{world}",
              "l2": "flushed before every timed step (256 MiB write)"}

    if args.impl == "reference":
        if rank != 0:
            return
        inp = make_workload_inputs(wl, seed=0)
        rng = np.random.default_rng(1)
        n = 64 if wl.kind == "block" else wl.T
        times = []
        for i in range(args.warmup + args.steps):
            toks = np.sort(rng.choice(wl.T, size=min(n, wl.T), replace=False))
            dt = oracle_sample_run(wl, inp, toks)
            if i >= args.warmup:
                times.append(dt)
        t = float(np.sum(times))
        val = len(toks) * args.steps / t
        config["l2"] = "n/a (host CPU run)"
        line = {"impl": "reference", "metric": metric, "value": val, "unit": "tokens/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": config,
                "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": blas_threads(),
                                 "kind": "oracle",
                                 "sample": f"{min(n, wl.T)} random tokens of {wl.T} per step"},
                "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    res = run_ours(args, rank, world, local_rank)
    if rank == 0:
        config["l2"] = res["l2"]
        peaks, src = load_peaks()
        step_s = res["step_ms"] / 1e3
        value = job_tokens_per_s(wl.T, world, res["step_ms"])
        tot_flops = sum(flops.values())
        if wl.kind == "inproj":
            n_hit = int(np.count_nonzero(res["counts"]))
            t_k = res["part_ms_eager"]["proj0"] / 1e3
            ach = inproj_bytes(wl, n_hit) / t_k / 1e9
            roof = {"bound": "hbm", "kernel": "rom_expert_proj(INPROJ)", "achieved": ach,
                    "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
                    "traffic": profiled_traffic(wl.name), "peak_source": f"{src} hbm_gbs"}
        else:
            t_k = res["part_ms_eager"]["proj0"] / 1e3
            ach = flops["conv_gate"] / t_k / 1e12
            pk = peaks["bf16_tflops"]
            roof = {"bound": "tensor", "kernel": "rom_expert_proj(CONV_GATE)", "achieved": ach,
                    "peak": pk, "unit": "TFLOP/s", "frac": ach / pk,
                    "traffic": profiled_traffic(wl.name),
                    "peak_source": f"{src} bf16_tflops (burst)"}
        line = {"metric": metric, "value": value, "unit": "tokens/s", "n_gpus": world,
                "csrc_sha256": csrc_digest(),
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["step_ms"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic",
                "config": config, "roofline": roof,
                "block_tflops": tot_flops / step_s / 1e12,
                "block_frac_of_bf16_peak": tot_flops / step_s / 1e12 / peaks["bf16_tflops"],
                "kernels_ms": res["part_ms"], "kernels_ms_eager": res["part_ms_eager"],
                "eager_ms_per_step": res["eager_ms"],
                "step": "forward + backward" if wl.backward else "forward",
                "timing": "step: the whole step replayed as one CUDA graph between two CUDA "
                          "events on the launching stream (max over ranks); kernels_ms: each "
                          "phase replayed as its own graph; roofline kernel: eager launch "
                          "between two events",
                "e2e": {"value": job_tokens_per_s(wl.T, world, res["e2e_ms"]), "unit": "tokens/s",
                        "h2d_bytes_per_step": res["x_bytes"], "d2h_bytes_per_step": res["out_bytes"]},
                "gpu_launches": res["launches"], "clocks": res["clocks"],
                "expert_load": (res["counts"] / max(1, res["counts"].sum())).round(4).tolist()}
        if not args.no_cpu_baseline and world == 1:
            inp = make_workload_inputs(wl, seed=0)
            line["cpu_baseline"] = cpu_baseline(wl, inp)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
