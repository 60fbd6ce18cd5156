"""Benchmark of the RoM projection block forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--no-cpu-baseline]

One step = one pass of the whole block over one batch of synthetic input:
route -> dispatch -> Conv+Gate grouped GEMM (+ gate combine for top-k > 1)
-> Out grouped GEMM (+ slot sum for top-k > 1); for the Swimba decode
workload: route -> routed in-projection (a decode batch of at most 64 tokens
needs no dispatch). Inputs are resident in
HBM when the timed region starts. Between timed steps the L2 is flushed (a
256 MiB write, outside the step's events), except where the step's inputs
(tokens and weights) exceed twice the L2: then every step streams them from
HBM anyway, and a flush would only add the write-back of its own dirty lines
to the next step. The line's "l2" key says which. Each step is timed with CUDA
events on the launching stream; the dominant kernel is bracketed by its own
events for the roofline. Under torchrun every rank runs an independent
replica on its own GPU (the block needs no collective in the forward); the
reported time is the max over ranks and `value` counts all ranks' tokens.

A single-GPU run also times the other configurations of the block (decode
in-projection, top-2 forward + backward, load-imbalanced, tiny float32, and
the independently routed and RoM (Gate, Out) projection variants at the
prefill shape, and the prefill block with the dense core between the
projections, its x and dt projections shared or expertized) and reports them
under "workloads"; `--no-extra` skips them.

`--impl reference` times the CPU oracle (the float64 numpy definition) on the
host cores, on the whole workload per step when that fits about two minutes
(else a random token sample); under torchrun only rank 0 runs it.

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
    if wl.kind == "variant":
        # Conv and Gate as two projections (dense ones over the T tokens), then Out
        rows_conv = wl.T if wl.variant == "gate_out" else R
        return {"conv": 2.0 * rows_conv * wl.Dm * wl.De, "gate": 2.0 * R * wl.Dm * wl.De,
                "out": 2.0 * R * wl.De * wl.Dm}
    f = {"conv_gate": 4.0 * R * wl.Dm * wl.De, "out": 2.0 * R * wl.De * wl.Dm}
    if wl.backward:  # dgrad (Out, In+Gate) and wgrad (Out, In+Gate): twice the forward
        f["backward"] = 2.0 * (f["conv_gate"] + f["out"])
    return f


def inproj_bytes(wl, n_experts_hit):
    """Algorithmic HBM bytes of the routed in-projection: the weights of the
    experts that received tokens, x in, the output out (bf16)."""
    return n_experts_hit * wl.Dm * wl.De * 2 + wl.T * wl.Dm * 2 + wl.T * wl.De * 2


def variant_spec(wl, inp):
    """Routers (None: dense) and weighting of the projections of a variant
    workload: which router drives which projection."""
    if wl.variant == "independent":
        return ({"conv": inp["w_r"], "gate": inp["w_r_gate"], "out": inp["w_r_out"]},
                {"conv": True, "gate": True, "out": True})
    if wl.variant == "gate_out":
        return ({"conv": None, "gate": inp["w_r"], "out": inp["w_r"]},
                {"conv": False, "gate": False, "out": True})
    raise ValueError(wl.variant)


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
# NVML clock-event reason bits (nvml.h) of the reasons above
NVML_REASON_BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40,
                    "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}


_NVML = {}


def nvml_device(gpu_index):
    """(pynvml, handle) of a GPU, NVML initialised once per process (its
    first call is slow), or None without NVML."""
    if gpu_index not in _NVML:
        try:
            import pynvml
            if not _NVML:
                pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            # the first queries of a device are slow: made here, before any timed region
            pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
            (getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None)
             or pynvml.nvmlDeviceGetCurrentClocksThrottleReasons)(h)
            _NVML[gpu_index] = (pynvml, h)
        except Exception:  # noqa: BLE001
            _NVML[gpu_index] = None
    return _NVML[gpu_index]


class NvmlSampler:
    """SM clock and clock-event reasons read through NVML every `period_s`
    seconds around the timed steps and phases: a short workload's timed
    region spans only a sample or two of nvidia-smi's 100 ms loop, which then
    mostly sees the idle moments around it."""

    def __init__(self, gpu_index, period_s=0.0005):
        self.gpu = gpu_index
        self.period = period_s
        self.samples = []  # (sm MHz, reason bits)
        self.stop_evt = threading.Event()
        self.thread = None

    def start(self):
        dev = nvml_device(self.gpu)
        if dev is None:
            return
        pynvml, h = dev
        reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons

        def run():
            while not self.stop_evt.is_set():
                try:
                    self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                         int(reasons(h))))
                except Exception:  # noqa: BLE001
                    pass
                self.stop_evt.wait(self.period)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_evt.set()
        self.thread.join(timeout=2)
        return summarize_nvml(self.samples, self.period)


def summarize_nvml(samples, period_s):
    """Median and lowest SM clock and the throttle reasons (of
    THROTTLE_REASONS) active in any of the (MHz, NVML reason bits) samples."""
    if not samples:
        return {"samples": 0}
    mhz = [float(m) for m, _ in samples]
    bits = 0
    for _, b in samples:
        bits |= b
    return {"samples": len(samples), "period_ms": period_s * 1e3,
            "sm_mhz": float(np.median(mhz)), "sm_mhz_min": min(mhz),
            "reasons": sorted(n for n, b in NVML_REASON_BITS.items() if bits & b)}


def merge_clocks(smi, fast):
    """The reported clocks: nvidia-smi's summary, with the median SM clock
    and the reasons of the NVML samples taken during the timed steps when
    there are enough of them (their summary is kept under "nvml")."""
    out = dict(smi)
    if fast and fast.get("samples", 0) >= 3:
        out["sm_mhz"] = fast["sm_mhz"]
        out["reasons"] = sorted(set(smi.get("reasons") or []) | set(fast["reasons"]))
        out["nvml"] = fast
    return out


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
    elif wl.kind == "variant":
        routers, weighted = variant_spec(wl, inp)
        w_conv = inp["w_conv"][:1] if routers["conv"] is None else inp["w_conv"]
        orc.variant_block_forward(inp["x"], w_conv, inp["w_gate"], inp["w_out"], wl.k, routers,
                                  weighted, renorm=wl.renorm, tokens=tokens)
    elif wl.core:
        # The core mixes tokens over time, so a sample of n tokens is the
        # first n of the batch (whole sequences, or a prefix of the first
        # one): their outputs are those of the whole workload.
        L = wl.seq_len or wl.T
        n = wl.T if tokens is None else len(tokens)
        n = (n // L) * L if n >= L else n
        orc.block_forward(inp["x"][:n], inp["w_r"], inp["w_conv"], inp["w_gate"], inp["w_out"],
                          k=wl.k, bias=inp["bias"], renorm=wl.renorm, core=inp["core"],
                          seq_len=min(n, L))
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


def build_workload(torch, rom, wl, inp):
    """Device inputs of one workload and its step as phases.

    Returns a dict: phases [(name, fn)], dominant (fn, "flop"|"byte" work
    function of the routing counts), out (result tensor), counts (expert
    counts of the main routing), x, in_bytes (a step's inputs), launches
    (our kernels per step), e2e (the public host-buffer call or None).
    """
    bf16 = wl.dtype == "bf16"
    x = to_dev(torch, inp["x"], bf16)
    w_r = to_dev(torch, inp["w_r"], False)
    bias = None if inp.get("bias") is None else to_dev(torch, inp["bias"], False)
    R = wl.T * wl.k
    dt = rom.ROM_BF16 if bf16 else rom.ROM_F32
    flops = block_flops(wl)
    in_bytes = x.numel() * x.element_size() + w_r.numel() * w_r.element_size()
    res = {"x": x}
    if wl.kind == "inproj":
        w = to_dev(torch, inp["w"], bf16).transpose(1, 2).contiguous()
        in_bytes += w.numel() * w.element_size()
        bufs = rom.RoutingBuffers(wl.T, wl.Dm, wl.E, wl.k, x.dtype, x.device)
        out = torch.empty((wl.T, wl.De), dtype=x.dtype, device=x.device)
        slots = (torch.empty((R, wl.De), dtype=torch.float32, device=x.device)
                 if wl.k > 1 else None)

        # a decode-sized batch takes the projection without a dispatch, over
        # the weights in the tile-major layout (packed once, here)
        dense = bf16 and wl.T <= rom.DENSE_SMALL_MAX_TOKENS
        w_tiled = rom.pack_expert_weights(w) if dense else None

        def ph_route():
            if dense:
                # no dispatch follows: neither counts nor chunk histograms
                rom.rom_route(x, w_r, bias, wl.k, wl.renorm, bufs.topk_idx, bufs.topk_w, None,
                              None)
            else:
                rom.route_and_dispatch(x, w_r, bias, wl.E, wl.k, wl.renorm, bufs)

        def ph_p0():
            if dense:
                rom.rom_expert_proj_dense(rom.ROM_PROJ_INPROJ, x, w_tiled, wl.E, wl.k,
                                          bufs.topk_idx, bufs.topk_w,
                                          out if wl.k == 1 else slots, tiled=True)
            else:
                rom.rom_expert_proj(rom.ROM_PROJ_INPROJ, bufs.x_sorted[:R], w, None, wl.E, wl.k,
                                    bufs.offsets, bufs.sorted_slot, bufs.topk_w,
                                    out if wl.k == 1 else slots)

        def ph_p1():
            if wl.k > 1:
                rom.rom_combine(rom.ROM_COMBINE_SUM, dt, slots, wl.T, wl.k, wl.De, None, out)
        res.update(phases=[("route" if dense else "route_dispatch", ph_route), ("proj0", ph_p0),
                           ("proj1", ph_p1)],
                   dominant=(ph_p0, "byte",
                             lambda counts: inproj_bytes(wl, int(np.count_nonzero(counts)))),
                   out=out,
                   counts=((lambda: torch.bincount(bufs.topk_idx.reshape(-1).long(),
                                                   minlength=wl.E).int())
                           if dense else bufs.counts),
                   launches=(2 if dense else 3) + (1 if wl.k > 1 else 0))
        pipe = rom.HostPipeline(wl.T, wl.Dm, wl.De, wl.E, wl.k, x.dtype, x.device)
        res["e2e"] = (pipe, lambda hx, ho: pipe.inproj_forward(hx, w_r, w, ho, renorm=wl.renorm,
                                                                bias=bias, w_tiled=w_tiled))
    elif wl.kind == "variant":
        routers, weighted = variant_spec(wl, inp)
        d_r = {}
        for n, r in routers.items():  # the same array -> one device tensor (shared routing)
            if r is not None and id(r) not in d_r:
                d_r[id(r)] = w_r if r is inp["w_r"] else to_dev(torch, r, False)
        d_routers = {n: (None if r is None else d_r[id(r)]) for n, r in routers.items()}
        ws = {n: to_dev(torch, inp[n][:1] if (routers[p] is None) else inp[n], bf16)
              .transpose(1, 2).contiguous()
              for n, p in (("w_conv", "conv"), ("w_gate", "gate"), ("w_out", "out"))}
        in_bytes += sum(t.numel() * t.element_size() for t in ws.values())
        in_bytes += sum(t.numel() * t.element_size() for t in d_r.values() if t is not w_r)
        bufs = rom.VariantBuffers(wl.T, wl.Dm, wl.De, wl.k, x.dtype, x.device)
        args = (x, d_routers, weighted, ws["w_conv"], ws["w_gate"], ws["w_out"], wl.k)

        def phase(names):
            return lambda: rom.variant_block_forward(*args, renorm=wl.renorm, bias=bias,
                                                     bufs=bufs, phases=names)
        phase(("route", "project", "output"))()  # makes the routing buffers
        rb_c = bufs.routings[id(d_routers["conv"])] if d_routers["conv"] is not None else None

        def dominant():  # the Conv projection alone
            if rb_c is None:
                rom.rom_expert_proj(rom.ROM_PROJ_SLOTS, x, ws["w_conv"], None, 1, 1, None, None,
                                    None, bufs.uz[:wl.T])
            else:
                rom.rom_expert_proj(rom.ROM_PROJ_SLOTS, rb_c.x_sorted[:R], ws["w_conv"], None,
                                    wl.E, wl.k, rb_c.offsets, rb_c.sorted_slot,
                                    rb_c.topk_w if weighted["conv"] else None, bufs.uz[:R])
        n_routings = len(d_r)
        main_rb = bufs.routings[id(w_r)]
        res.update(phases=[("route_dispatch", phase(("route",))),
                           ("proj0", phase(("project",))), ("proj1", phase(("output",)))],
                   dominant=(dominant, "flop", lambda counts: flops["conv"]),
                   out=bufs.out, counts=main_rb.counts,
                   launches=2 * n_routings + 2 + 2 + (1 if wl.k > 1 else 0))
        res["e2e"] = None
    elif wl.core:
        # the block with the dense core between the projections (top-1)
        assert wl.k == 1
        ws = {n: to_dev(torch, inp[n], bf16).transpose(1, 2).contiguous()
              for n in ("w_conv", "w_gate", "w_out")}
        in_bytes += sum(t.numel() * t.element_size() for t in ws.values())
        core = rom.CoreParams(inp["core"], x.device)
        L = wl.seq_len or wl.T
        bufs = rom.BlockBuffers(wl.T, wl.Dm, wl.De, wl.E, wl.k, x.dtype, x.device, core, L)
        rb = bufs.routing
        flat = bufs.uz.view(2 * R, wl.De)

        def ph_route():
            rom.route_and_dispatch(x, w_r, bias, wl.E, wl.k, wl.renorm, rb)

        def ph_p0():
            rom.rom_expert_proj(rom.ROM_PROJ_CONV_GATE_SLOTS, rb.x_sorted[:R], ws["w_conv"],
                                ws["w_gate"], wl.E, wl.k, rb.offsets, rb.sorted_slot, rb.topk_w,
                                bufs.uz)

        def ph_core():
            rom.rom_ssm_core(flat[:wl.T], L, core, flat[:wl.T], bufs.core_ws, routing=rb)

        def ph_p1():
            rom.rom_combine(rom.ROM_COMBINE_GATE_DENSE, dt, flat, wl.T, 1, wl.De, rb.slot_pos,
                            bufs.h_sorted)
            rom.rom_expert_proj(rom.ROM_PROJ_OUT, bufs.h_sorted[:R], ws["w_out"], None, wl.E, 1,
                                rb.offsets, rb.sorted_slot, rb.topk_w, bufs.out)
        res.update(phases=[("route_dispatch", ph_route), ("proj0", ph_p0), ("core", ph_core),
                           ("proj1", ph_p1)],
                   dominant=(ph_p0, "flop", lambda counts: flops["conv_gate"]),
                   out=bufs.out, counts=rb.counts,
                   launches=4 + 7 + 1 + (2 if wl.core_routed else 0))
        res["e2e"] = None
    else:
        ws = {n: to_dev(torch, inp[n], bf16).transpose(1, 2).contiguous()
              for n in ("w_conv", "w_gate", "w_out")}
        in_bytes += sum(t.numel() * t.element_size() for t in ws.values())
        bufs = rom.BlockBuffers(wl.T, wl.Dm, wl.De, wl.E, wl.k, x.dtype, x.device)
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
        phases = [("route_dispatch", ph_route), ("proj0", ph_p0), ("proj1", ph_p1)]
        if wl.backward:
            dout = to_dev(torch, inp["dout"], bf16)
            in_bytes += dout.numel() * dout.element_size()
            bwd_bufs = rom.BackwardBuffers(wl.T, wl.Dm, wl.De, wl.E, wl.k, x.device)
            # Data parallel over ranks: every rank trains on its own tokens and
            # the weight gradients (experts and router) are summed over all.
            import torch.distributed as dist
            dp = dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1
            grad_sync = rom.GradientAllReduce() if dp else None

            def ph_bwd():
                rom.block_backward(bufs, dout, w_r, ws["w_conv"], ws["w_gate"], ws["w_out"],
                                   renorm=wl.renorm, bufs=bwd_bufs, x=x, bias=bias,
                                   grad_sync=grad_sync)
            phases.append(("backward", ph_bwd))
            # NCCL collectives are not captured into CUDA graphs here: the
            # data-parallel step is timed as eager launches
            res["eager_only"] = dp
        res.update(phases=phases, dominant=(ph_p0, "flop", lambda counts: flops["conv_gate"]),
                   out=bufs.out, counts=rb.counts,
                   launches=4 + (2 if wl.k > 1 else 0) + (8 if wl.backward else 0))
        if wl.backward:
            res["e2e"] = None  # host copies around one step (below)
        else:
            pipe = rom.HostPipeline(wl.T, wl.Dm, wl.De, wl.E, wl.k, x.dtype, x.device, De=wl.De)
            res["e2e"] = (pipe, lambda hx, ho: pipe.block_forward(
                hx, w_r, bias, ws["w_conv"], ws["w_gate"], ws["w_out"], ho, renorm=wl.renorm))
    res["in_bytes"] = in_bytes
    return res


def measure(args, wl, world, local_rank, with_e2e):
    """Times one workload on this rank's GPU; returns the per-rank figures."""
    import torch
    import torch.distributed as dist

    from mixture_experts_projections_b200 import rom

    inp = make_workload_inputs(wl, seed=0)
    stream = torch.cuda.current_stream()
    b = build_workload(torch, rom, wl, inp)
    del inp
    x, out_t = b["x"], b["out"]
    phases = [f for _, f in b["phases"]]
    names = [n for n, _ in b["phases"]]
    flush_l2 = b["in_bytes"] < 2 * L2_BYTES
    flush = (torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=x.device)
             if flush_l2 else None)
    l2_note = ("flushed before every timed step (256 MiB write)" if flush_l2 else
               f"not flushed: the step's inputs ({b['in_bytes'] / 1e6:.0f} MB) exceed twice the "
               f"L2 ({L2_BYTES / 1e6:.0f} MB) and are streamed from HBM every step")

    def do_flush():
        if flush is not None:
            flush.zero_()

    def step():
        for ph in phases:
            ph()

    for _ in range(args.warmup):
        do_flush()
        step()
    torch.cuda.synchronize()
    if rom.rom_get_status() != 0:
        raise RuntimeError(f"{wl.name}: device status word reports an error after warm-up")

    # The step captured once as one CUDA graph (the library's launch sequence
    # is static: its kernels read the expert counts on the device), and each
    # phase once more on its own for the per-phase breakdown. A step with a
    # collective (data-parallel backward) runs as eager launches instead.
    class _Eager:
        def __init__(self, fn):
            self.replay = fn
    if b.get("eager_only"):
        g_step = _Eager(step)
        graphs = [_Eager(ph) for ph in phases]
    else:
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

    def timed_loop(run_phase, n, count):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(count + 1)]
               for _ in range(n)]
        for i in range(n):
            do_flush()
            torch.cuda._sleep(200_000)  # GPU-side head start so that the host stays ahead
            evs[i][0].record(stream)
            for j in range(count):
                run_phase(j)
                evs[i][j + 1].record(stream)
        torch.cuda.synchronize()
        return np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(count)]
                         for i in range(n)])

    for _ in range(2):  # graph warm-up
        timed_loop(lambda j: graphs[j].replay(), 1, len(phases))
        timed_loop(lambda j: g_step.replay(), 1, 1)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    clocks.start()
    nvml_device(local_rank)  # NVML's slow first call before the timed region
    time.sleep(0.3)
    fast = NvmlSampler(local_rank)
    fast.start()
    step_ms = timed_loop(lambda j: g_step.replay(), args.steps, 1)[:, 0]
    ph_ms = timed_loop(lambda j: graphs[j].replay(), args.steps, len(phases))
    fast_clk = fast.stop()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = merge_clocks(clocks.stop(), fast_clk)
    eager_ms = timed_loop(lambda j: phases[j](), args.steps, len(phases))
    # The dominant kernel alone: one eager launch between two events, the
    # host ahead of the GPU (no graph-launch latency in its duration).
    dom_fn, dom_kind, dom_work = b["dominant"]
    dom_ms = timed_loop(lambda j: dom_fn(), args.steps, 1)[:, 0]
    counts = (b["counts"]() if callable(b["counts"]) else b["counts"]).cpu().numpy()
    t_total_ms = float(step_ms.sum())

    # ---------------------------------------------- e2e through host buffers
    # The public host-buffer call: inputs in pinned host memory, result copied
    # back, copies inside the timed region. Forward-only workloads go through
    # rom.HostPipeline (chunks staged over copy-in, kernel and copy-out streams);
    # the others copy x in and O out around one step.
    e2e_total = 0.0
    if with_e2e:
        h_x = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
        h_x.copy_(x)
        h_out = torch.empty(out_t.shape, dtype=out_t.dtype, pin_memory=True)

        def e2e_call():
            if b["e2e"] is None:
                x.copy_(h_x, non_blocking=True)
                step()
                h_out.copy_(out_t, non_blocking=True)
            else:
                b["e2e"][1](h_x, h_out)

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
    return dict(wl=wl, step_ms=t_total_ms / args.steps,
                part_ms={n: float(ph_ms[:, j].mean()) for j, n in enumerate(names)},
                part_ms_eager={n: float(eager_ms[:, j].mean()) for j, n in enumerate(names)},
                eager_ms=float(eager_ms.sum()) / args.steps, dominant_ms=float(dom_ms.mean()),
                dominant_kind=dom_kind, dominant_work=float(dom_work(counts)),
                e2e_ms=e2e_total / args.steps, clocks=clk, launches=b["launches"] * args.steps,
                counts=counts, x_bytes=x.numel() * x.element_size(), l2=l2_note,
                out_bytes=out_t.numel() * out_t.element_size())


def roofline(res, peaks, src):
    """Roofline of the dominant kernel: algorithmic work per launch over its
    eager-launch duration, against the measured peak."""
    wl = res["wl"]
    t_k = res["dominant_ms"] / 1e3
    if res["dominant_kind"] == "byte":
        ach = res["dominant_work"] / t_k / 1e9
        kern = ("rom_expert_proj_dense(INPROJ)" if wl.T <= 64 and wl.dtype == "bf16"
                else "rom_expert_proj(INPROJ)")
        return {"bound": "hbm", "kernel": kern, "achieved": ach,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
                "traffic": profiled_traffic(wl.name), "peak_source": f"{src} hbm_gbs"}
    ach = res["dominant_work"] / t_k / 1e12
    pk = peaks["bf16_tflops"]
    kern = "rom_expert_proj(SLOTS, Conv)" if wl.kind == "variant" else "rom_expert_proj(CONV_GATE)"
    out = {"bound": "tensor", "kernel": kern, "achieved": ach, "peak": pk, "unit": "TFLOP/s",
           "frac": ach / pk, "traffic": profiled_traffic(wl.name),
           "peak_source": f"{src} bf16_tflops (burst)"}
    # Under the power cap (a long step of GEMMs) the burst peak is out of
    # reach; the measured sustained figure is given beside it.
    sus = peaks.get("bf16_tflops_sustained")
    if sus and "sw_power_cap" in (res.get("clocks") or {}).get("reasons", []):
        out["sustained"] = {"peak": sus, "frac": ach / sus,
                            "peak_source": f"{src} bf16_tflops_sustained"}
    return out


def workload_config(wl, world):
    from mixture_experts_projections_b200 import rom
    return {"workload": wl.name, "tokens": wl.T, "d_model": wl.Dm,
            ("d_out" if wl.kind == "inproj" else "d_inner"): wl.De, "experts": wl.E,
            "top_k": wl.k, "renorm": wl.renorm, "parallelism": f"replicas x{world}",
            **({"projections": wl.variant} if wl.kind == "variant" else {}),
            **({"weights": "tile-major (rom_pack_expert_weights, once, before timing)"}
               if wl.kind == "inproj" and wl.dtype == "bf16" and wl.T <= rom.DENSE_SMALL_MAX_TOKENS
               else {})}


SM_COUNT = 148
SFU_PER_SM_CLK = 16  # special-function results (exp2, log2, ...) per SM per clock


def core_roofline(res, wl):
    """The core's state updates (one exp(delta A) per token, channel and
    state: T * d_inner * N) per second over the whole core phase (the
    convolution, the x and dt projections and the scan), against the
    special-function unit's exp2 rate: 148 SMs x 16 results per clock x the
    highest SM clock seen."""
    from mixture_experts_projections_b200.inputs import CORE_STATE
    t_s = res["part_ms"]["core"] / 1e3
    mhz = res["clocks"].get("sm_max_mhz") or 1965.0
    peak = SM_COUNT * SFU_PER_SM_CLK * mhz * 1e6 / 1e9
    ach = wl.T * wl.De * CORE_STATE / t_s / 1e9
    return {"bound": "alu", "unit": "G exp2/s", "achieved": ach, "peak": peak,
            "frac": ach / peak, "kernel": "rom_ssm_core (whole phase)"}


def phase_figures(wl, part_ms, hbm_gbs, world):
    """Figures of single phases: the route + dispatch phase's HBM rate (the
    router reads X once, the dispatch reads and writes the R = T*k routed
    rows: algorithmic bytes / the phase's device time, against the measured
    HBM copy rate), and for a training step the forward's token rate (its
    phases' device times summed)."""
    out = {}
    elt = 2 if wl.dtype == "bf16" else 4
    if "route_dispatch" in part_ms and part_ms["route_dispatch"] > 0:
        routings = 3 if wl.kind == "variant" and wl.variant == "independent" else 1
        nbytes = routings * (wl.T * wl.Dm * elt + 2 * wl.T * wl.k * wl.Dm * elt)
        gbs = nbytes / (part_ms["route_dispatch"] / 1e3) / 1e9
        out["route_dispatch_hbm"] = {"bytes": nbytes, "achieved_gbs": gbs,
                                     "frac": gbs / hbm_gbs}
    if wl.backward:
        fwd_ms = sum(v for n, v in part_ms.items() if n != "backward")
        out["forward_tokens_per_s"] = job_tokens_per_s(wl.T, world, fwd_ms)
    return out


def summary_entry(res, peaks, src, world):
    """Per-workload figures of the extra workloads of one bench run."""
    wl = res["wl"]
    tot = sum(block_flops(wl).values())
    step_s = res["step_ms"] / 1e3
    extra = {"core_roofline": core_roofline(res, wl)} if wl.core else {}
    return {**extra, "config": workload_config(wl, world), "l2": res["l2"],
            "step": "forward + backward" if wl.backward else "forward",
            "ms_per_step": res["step_ms"], "tokens_per_s": job_tokens_per_s(wl.T, world,
                                                                            res["step_ms"]),
            "block_tflops": tot / step_s / 1e12, "roofline": roofline(res, peaks, src),
            **phase_figures(wl, res["part_ms"], peaks["hbm_gbs"], world),
            "kernels_ms": res["part_ms"], "kernels_ms_eager": res["part_ms_eager"],
            "clocks": res["clocks"], "gpu_launches": res["launches"],
            "expert_load": (res["counts"] / max(1, res["counts"].sum())).round(4).tolist()}


def reference_arm(args, wl, metric, config, world):
    """The CPU oracle, as it stands, on the host cores (rank 0 only): each
    step evaluates a token sample of the workload, the whole workload when
    its estimated time fits the run's budget (about two minutes)."""
    inp = make_workload_inputs(wl, seed=0)
    rng = np.random.default_rng(1)
    n_steps = args.warmup + args.steps
    budget_s = 120.0
    probe = np.sort(rng.choice(wl.T, size=min(wl.T, 4096), replace=False))
    per_tok = oracle_sample_run(wl, inp, probe) / len(probe)
    # the whole workload when it fits (a large batch costs less per token
    # than the probe), else the sample that fills the budget
    if per_tok * wl.T * n_steps <= 1.5 * budget_s:
        n = wl.T
    else:
        n = int(min(wl.T, max(16, budget_s / n_steps / max(per_tok, 1e-9))))
    times = []
    for i in range(n_steps):
        toks = np.sort(rng.choice(wl.T, size=n, replace=False)) if n < wl.T else None
        dt = oracle_sample_run(wl, inp, toks)
        if i >= args.warmup:
            times.append(dt)
    t = float(np.sum(times))
    val = n * args.steps / t
    sample = (f"all {wl.T} tokens of {wl.name} per step" if n >= wl.T else
              f"{n} random tokens of the {wl.T} of {wl.name} per step")
    return {"impl": "reference", "metric": metric, "value": val, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "l2": "n/a (host CPU run)",
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": blas_threads(),
                             "kind": "oracle", "sample": sample + " (float64 numpy oracle)"},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# Workloads timed next to the headline in a single-GPU run: the other
# configurations of the block, each reported under "workloads".
EXTRA_WORKLOADS = ["decode_swimba_inproj", "top2_fwd_bwd", "imbalanced_8x4096", "tiny_fp32",
                   "independent_moe_16k", "rom_gate_out_16k", "prefill_16k_core",
                   "prefill_16k_core_dtx"]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill_16k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time the headline workload only (no other configurations)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token count (smaller profiling cases)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.tokens is not None:
        import dataclasses
        w0 = WORKLOADS[args.workload]
        WORKLOADS[args.workload] = dataclasses.replace(
            w0, T=args.tokens, seq_len=min(w0.seq_len, args.tokens) if w0.seq_len else 0)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = WORKLOADS[args.workload]
    metric = (f"tokens/s and TFLOPS (% bf16 peak) for RoM projection block "
              f"{'fwd+bwd' if wl.backward else 'fwd'}, {world} B200")
    config = workload_config(wl, world)

    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(reference_arm(args, wl, metric, config, world)), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    torch.cuda.set_device(local_rank)
    from mixture_experts_projections_b200 import rom
    rom.load_library()
    res = measure(args, wl, world, local_rank, with_e2e=True)
    extra = {}
    if world == 1 and not args.no_extra and args.tokens is None:
        for name in EXTRA_WORKLOADS:
            if name != wl.name:
                extra[name] = measure(args, WORKLOADS[name], world, local_rank, with_e2e=False)
    if rank == 0:
        peaks, src = load_peaks()
        step_s = res["step_ms"] / 1e3
        tot_flops = sum(block_flops(wl).values())
        line = {"metric": metric, "value": job_tokens_per_s(wl.T, world, res["step_ms"]),
                "unit": "tokens/s", "n_gpus": world, "csrc_sha256": csrc_digest(),
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["step_ms"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if wl.dtype == "bf16" else "f32", "data": "synthetic",
                "config": config, "l2": res["l2"], "roofline": roofline(res, peaks, src),
                "block_tflops": tot_flops / step_s / 1e12,
                "block_frac_of_bf16_peak": tot_flops / step_s / 1e12 / peaks["bf16_tflops"],
                **phase_figures(wl, res["part_ms"], peaks["hbm_gbs"], world),
                "kernels_ms": res["part_ms"], "kernels_ms_eager": res["part_ms_eager"],
                "eager_ms_per_step": res["eager_ms"],
                "step": "forward + backward" if wl.backward else "forward",
                "timing": "step: the whole step replayed as one CUDA graph between two CUDA "
                          "events on the launching stream (max over ranks); kernels_ms: each "
                          "phase replayed as its own graph; roofline kernel: eager launch "
                          "between two events",
                "e2e": {"value": job_tokens_per_s(wl.T, world, res["e2e_ms"]),
                        "unit": "tokens/s", "h2d_bytes_per_step": res["x_bytes"],
                        "d2h_bytes_per_step": res["out_bytes"]},
                "gpu_launches": res["launches"], "clocks": res["clocks"],
                "expert_load": (res["counts"] / max(1, res["counts"].sum())).round(4).tolist()}
        if extra:
            line["workloads"] = {n: summary_entry(r, peaks, src, world) for n, r in extra.items()}
        if not args.no_cpu_baseline and world == 1:
            inp = make_workload_inputs(wl, seed=0)
            line["cpu_baseline"] = cpu_baseline(wl, inp)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
