#!/usr/bin/env python
"""Throughput of the routed-MoE FFN layer forward on B200, through the C ABI.

One step = the whole hot path on one batch: route -> (budget) -> dispatch ->
expert gate/up GEMM + SwiGLU -> expert down GEMM + weighted scatter ->
combine.  `value` times moe_forward (one C call) replayed as a CUDA graph
between two events; the per-kernel breakdown replays the same launches as
separate stage entry points with an event between stages, on the launching
stream.  Inputs are resident in HBM; L2 is flushed (a 256 MB write) before
every replay, outside the timed events.

Prints ONE JSON line (rank 0).  `value` = tokens/s over all ranks; `e2e` =
the same metric through moe_forward with host buffers (pinned H2D of x and
logits, D2H of the output inside the timed region); `roofline` = the
slowest kernel against the measured HBM or bf16 tensor peak;
`cpu_baseline` = the CPU oracle on the host cores (rank 0, N = 1).

Multi-GPU: one process per GPU (torchrun); each rank runs an independent
replica of the workload (the layer has no exchange step with all experts
resident), the time is the max over ranks, scaling is weak.

`--impl reference` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import math
import os
import re
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s (bf16) + % of tcgen05 peak or HBM roofline, 1 B200"
FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------ workloads --
def workload_from_args(args):
    from routed_expert_ffn_renorm_b200 import workloads as W
    cfg = W.WORKLOADS[args.workload]
    kw = {}
    if args.T is not None:
        kw["T"] = args.T
    if args.alpha is not None:
        kw["zipf_alpha"] = args.alpha
    if args.budget is not None:
        kw["budget"] = args.budget
    if args.topp is not None:
        kw["topp"] = args.topp
    if args.router_proj:
        kw["router_proj"] = True
    if args.E is not None:
        kw["E"] = args.E
    return cfg.with_(**kw) if kw else cfg


def workload_desc(cfg) -> dict:
    d = {"workload": cfg.label, "tokens": cfg.T, "hidden": cfg.H, "n_routed_experts": cfg.E,
         "moe_intermediate_size": cfg.I, "num_experts_per_tok": cfg.k, "shared_intermediate_size": cfg.Is,
         "norm_topk": cfg.norm_topk, "budget": cfg.budget, "topp": cfg.topp, "router_proj": cfg.router_proj,
         "zipf_alpha": cfg.zipf_alpha,
         "seed": cfg.seed,
         "l2": "flushed between timed steps (256 MB write, outside the timed events)"}
    return d


# -------------------------------------------------------- accounting --
def stage_work(cfg, counts, wfmt: str = "bf16"):
    """Algorithmic flops and HBM bytes per launch of each stage.

    Bytes count what a kernel must move at least once: the touched experts'
    weights (2 bytes a weight in bf16; 1 + 1/32 in MXFP8 and 1/2 + 1/16 in
    NVFP4: a code and its share of a block scale), its input activations and
    its output; flops are 2 per MAC."""
    H, I, Is, T, k, E = cfg.H, cfg.I, cfg.Is, cfg.T, cfg.k, cfg.E
    wb = {"bf16": 2.0, "mxfp8": 1.0 + 1.0 / 32, "nvfp4": 0.5 + 1.0 / 16}[wfmt]
    touched = int(sum(1 for c in counts if c > 0))
    slots = int(sum(counts))
    sh = 1 if Is else 0
    gate_up = dict(
        flops=4 * H * I * slots + 4 * H * Is * T,
        bytes=touched * 2 * I * H * wb + sh * 2 * Is * H * wb + slots * H * 2 + sh * T * H * 2 + (slots * I + T * Is) * 2)
    down = dict(
        flops=2 * H * I * slots + 2 * H * Is * T,
        bytes=touched * H * I * wb + sh * H * Is * wb + (slots * I + T * Is) * 2 + (slots + sh * T) * H * 2)
    ffn = dict(flops=gate_up["flops"] + down["flops"],
               bytes=touched * 3 * H * I * wb + sh * 3 * H * Is * wb + slots * H * 2 + sh * T * H * 2
               + (slots + sh * T) * H * 2)
    route = dict(flops=0, bytes=T * E * 4 + T * k * 8 + sh * (T * H * 2 + H * 2 + T * 4))
    proj = cfg.router_proj
    router_proj = dict(flops=2 * T * E * H if proj else 0, bytes=(T * H * 2 + E * H * 2 + T * E * 4) if proj else 0)
    budget = dict(flops=0, bytes=(T * k * 8 * 2) if cfg.budget else 0)
    dispatch = dict(flops=0, bytes=T * k * 4 * 3 + slots * H * 2 * 2)
    combine = dict(flops=0, bytes=(slots + sh * T) * H * 2 + T * H * 2)
    layer = dict(flops=gate_up["flops"] + down["flops"] + router_proj["flops"],
                 bytes=touched * 3 * H * I * wb + sh * (3 * H * Is * wb + H * 2) + 2 * T * H * 2
                 + (E * H * 2 if proj else T * E * 4))
    return dict(router_proj=router_proj, route=route, budget=budget, dispatch=dispatch, gate_up=gate_up, down=down,
                ffn=ffn, combine=combine, layer=layer, touched=touched, slots=slots)


def launches_forward(cfg) -> int:
    """Our kernel launches in one moe_forward call."""
    Tk = cfg.T * cfg.k
    ffn = 1 if (Tk + cfg.E - 1) // cfg.E < 128 else 2  # fused, or gate/up + down once the mean group >= 128
    if cfg.budget and Tk <= 8192 and cfg.T * cfg.E <= 16384:
        return int(cfg.router_proj) + 1 + ffn + 1  # [projection], fused front end, FFN, combine
    return launches_stages(cfg)


def launches_stages(cfg) -> int:
    """Our kernel launches of the stage entry points called one by one."""
    Tk = cfg.T * cfg.k
    ffn = 1 if (Tk + cfg.E - 1) // cfg.E < 128 else 2
    budget = (1 if Tk <= 8192 else 2) if cfg.budget else 0  # one block, or partial sums + select
    dispatch = 1 if Tk <= 8192 else 4  # sort + gather, or histogram + scan + scatter + gather
    return int(cfg.router_proj) + 1 + budget + dispatch + ffn + 1


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def code_hash(text: str) -> str:
    """sha256 prefix of C++/CUDA source with its comments and blank lines
    removed: what a recorded measurement depends on."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    lines = [ln.rstrip() for ln in text.splitlines() if ln.strip()]
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()[:16]


def kernel_source_hash() -> str:  # the grouped FFN kernel's code
    with open(os.path.join(ROOT, "routed_expert_ffn_renorm_b200", "csrc", "ffn_gemm.cu")) as f:
        return code_hash(f.read())


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from an ncu capture recorded under profiles/,
    if it was taken on the current kernel source for this workload."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("bytes_per_launch")


def roofline(stage: str, work: dict, ms: float, peaks: dict, peak_kind: str, long_run: bool, traffic):
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    w = work[stage]
    if w["flops"] and w["flops"] / max(w["bytes"], 1) > ridge:
        peak = peaks["bf16_tflops_sustained" if long_run else "bf16_tflops"]
        achieved = w["flops"] / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": traffic, "kernel": stage, "peak_source": f"{peak_kind} bf16 "
                + ("sustained" if long_run else "burst"), "algorithmic_flops": w["flops"],
                "algorithmic_bytes": w["bytes"]}
    achieved = w["bytes"] / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "kernel": stage,
            "peak_source": f"{peak_kind} HBM copy", "algorithmic_flops": w["flops"], "algorithmic_bytes": w["bytes"]}


# ------------------------------------------------------------ clocks --
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (reads only)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, device, period_s: float = 0.002):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self._nv = pynvml
            try:  # NVML numbers GPUs without CUDA_VISIBLE_DEVICES: match by PCI id
                pr = torch.cuda.get_device_properties(device)
                bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device.index or 0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as e:  # NVML missing: report that, do not guess
            self.error = repr(e)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self) -> dict:
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "")}
        s = sorted(self.samples)
        med = s[len(s) // 2] if s else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(s)}


# ------------------------------------------------------- distributed --
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, device) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and getattr(device, "type", "cpu") == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate_tokens_per_s(tokens_per_rank: int, steps: int, max_total_ms: float, world: int) -> float:
    """Whole-job tokens/s: every rank processes tokens_per_rank per step."""
    return world * tokens_per_rank * steps / (max_total_ms * 1e-3)


# ------------------------------------------------------- CPU oracle --
def sample_order(T: int):
    """Seeded order in which token rows enter the CPU sample (spread over the batch)."""
    import numpy as np
    return np.random.default_rng(0).permutation(T).astype(np.int32)


def oracle_rows_per_s(cfg, inp_host, target_s: float, max_rows: int, repeat: bool = False):
    """Time the oracle on a bounded sample of rows (the first n of
    sample_order).  Routing, budget and dispatch run over the whole batch; the
    FFN and combine over the sample.  With `repeat`, a batch whose every row
    fits well inside target_s is run again until about target_s has passed.
    Returns (rows/s, rows, passes, seconds, threads)."""
    import oracle
    x, logits, wg, wu, wd, shared = inp_host
    nthreads = oracle.max_threads()
    order = sample_order(cfg.T)
    max_rows = min(max_rows, cfg.T)

    def run(nrows):
        t0 = time.perf_counter()
        oracle.forward(x, logits, wg, wu, wd, k=cfg.k, norm_topk=cfg.norm_topk, budget=cfg.budget, topp=cfg.topp,
                       rows=order[:nrows], nthreads=nthreads, I=cfg.I, **shared)
        return time.perf_counter() - t0

    n = min(2, max_rows)
    dt = run(n)
    n2 = int(min(max_rows, max(n, n * target_s / max(dt, 1e-6))))
    if n2 > n:
        n, dt = n2, run(n2)
    passes = 1
    if repeat and n == max_rows and 2 * dt < target_s:
        passes = int(target_s / max(dt, 1e-6))
        dt = sum(run(n) for _ in range(passes))
    return n * passes / dt, n, passes, dt, nthreads


def host_inputs(cfg, inp, max_rows: int, wfmt: str = "bf16"):
    """Host copies for the oracle: x, logits, and the weights -- all experts
    when they fit in 2 GB, else only the experts the first max_rows sample
    rows route to (routing after the budget is a subset of routing before).
    MXFP8 / NVFP4: every expert matrix as the oracle's MXFP8 / NVFP4 weights
    (quantised by the oracle, once, before any timing; NVFP4's matrix scales
    go to the oracle as its output factors)."""
    import numpy as np
    import oracle
    from routed_expert_ffn_renorm_b200 import workloads as W
    scaled = {}  # NVFP4: matrix name -> {expert: matrix scale}

    def bits(t, name=None, e=None):
        if wfmt == "bf16":
            return W.bf16_bits(t)
        if wfmt == "mxfp8":
            return oracle.mxfp8_weights(W.bf16_bits(t))
        v, st = oracle.nvfp4_weights(W.bf16_bits(t))
        scaled.setdefault(name, {})[e] = float(st)
        return v
    x = W.bf16_bits(inp.x)
    if cfg.router_proj:  # the projection's logits, computed once before the timed oracle runs
        logits = oracle.router_logits(x, W.bf16_bits(inp.w_router))
    else:
        logits = inp.logits.float().cpu().numpy()
    if 3 * cfg.E * cfg.H * cfg.I * 2 <= (2 << 30) and wfmt == "bf16":
        wg, wu, wd = W.bf16_bits(inp.w_gate), W.bf16_bits(inp.w_up), W.bf16_bits(inp.w_down)
    else:
        idx, _ = oracle.route(logits, cfg.k, cfg.norm_topk)
        need = sorted(set(idx[sample_order(cfg.T)[:max_rows]].ravel().tolist()))
        wg = {e: bits(inp.w_gate[e], "g", e) for e in need}
        wu = {e: bits(inp.w_up[e], "u", e) for e in need}
        wd = {e: bits(inp.w_down[e], "d", e) for e in need}
    shared = {}
    if cfg.Is:
        shared = dict(ws_gate=bits(inp.ws_gate, "sg", 0), ws_up=bits(inp.ws_up, "su", 0),
                      ws_down=bits(inp.ws_down, "sd", 0), ws_gvec=W.bf16_bits(inp.ws_gvec))
    if wfmt == "nvfp4":
        sc = np.ones((cfg.E, 3))
        for j, name in enumerate("gud"):
            for e, v in scaled.get(name, {}).items():
                sc[e, j] = v
        shared["scales"] = sc
        if cfg.Is:
            shared["shared_scales"] = np.array([scaled["sg"][0], scaled["su"][0], scaled["sd"][0]])
    return x, logits, wg, wu, wd, shared


def cpu_max_rows(cfg, wfmt: str = "bf16") -> int:
    """Largest CPU sample: the whole batch for small layers, 16 rows when the
    expert weights do not fit a 2 GB host copy; with MXFP8 or NVFP4 weights
    (which the oracle quantises itself, about a second per expert matrix) 2
    rows."""
    if wfmt != "bf16":
        return min(cfg.T, 2)
    return cfg.T if 3 * cfg.E * cfg.H * cfg.I * 2 <= (2 << 30) else min(cfg.T, 16)


# ------------------------------------------------------------- our arm --
def run_ours(args, cfg):
    import torch
    import torch.distributed as dist
    import routed_expert_ffn_renorm_b200 as moe
    from routed_expert_ffn_renorm_b200 import workloads as W

    world, rank, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lib = moe.load_library()

    inp = W.make_inputs(cfg, device=dev)
    c = moe.MoEConfig(cfg.H, cfg.E, cfg.I, cfg.k, cfg.Is, cfg.norm_topk, cfg.budget, cfg.topp)
    T, k, E, H = cfg.T, cfg.k, cfg.E, cfg.H
    ws = torch.zeros(moe.workspace_bytes(c, T), dtype=torch.uint8, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    tw = torch.empty((T, k), dtype=torch.float32, device=dev)
    sgate = torch.empty(T, dtype=torch.float32, device=dev)
    keff = torch.empty(T, dtype=torch.int32, device=dev)
    kept = torch.empty(E, dtype=torch.uint8, device=dev)
    nd = torch.empty(1, dtype=torch.int32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    slot_pos = torch.empty(T * k, dtype=torch.int32, device=dev)
    x_perm = torch.empty((T * k, H), dtype=torch.bfloat16, device=dev)
    ybuf = torch.empty((T, k + 1, H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    # prebuilt C arguments: the timed loop makes plain C calls
    P = ctypes.c_void_p
    pc = ctypes.byref(c._c())
    wts = moe.MoEWeights(inp.w_gate, inp.w_up, inp.w_down, inp.ws_gate, inp.ws_up, inp.ws_down, inp.ws_gvec,
                         inp.w_router)
    fmt = args.weights
    if fmt != "bf16":  # the weight pack step, once, before anything is timed
        wts = moe.pack_mxfp8(wts) if fmt == "mxfp8" else moe.pack_nvfp4(wts)
        torch.cuda.synchronize(dev)
    wts_c = wts._c()
    pw = ctypes.byref(wts_c)
    sfx = "" if fmt == "bf16" else "_" + fmt
    ffn_fn = getattr(lib, "moe_expert_ffn" + sfx)
    fwd_fn = getattr(lib, "moe_forward" + sfx)
    fwd_py = getattr(moe, "moe_forward" + sfx)
    p = {n: P(t.data_ptr()) for n, t in dict(idx=idx, tw=tw, sgate=sgate, keff=keff, kept=kept, nd=nd,
                                                counts=counts, offsets=offsets, perm=perm, slot_pos=slot_pos,
                                                x_perm=x_perm, ybuf=ybuf, out=out, ws=ws, x=inp.x,
                                                logits=inp.logits).items()}
    gvec = P(inp.ws_gvec.data_ptr()) if cfg.Is else None
    sg = p["sgate"] if cfg.Is else None
    wsb = ws.numel()

    def chk(name, rc):
        if rc != 0:
            raise moe.MoEError(name, rc, lib.moe_error_string(rc).decode())

    stages = (["router_proj"] if cfg.router_proj else []) + ["route", "budget", "dispatch", "ffn", "combine"]
    NEV = len(stages) + 1
    pr = int(cfg.router_proj)  # event index shift
    wr = P(inp.w_router.data_ptr()) if cfg.router_proj else None

    def step(ev):
        sp = P(torch.cuda.current_stream(dev).cuda_stream)  # the capture stream while capturing
        st = torch.cuda.current_stream(dev)
        ev[0].record(st)
        if cfg.router_proj:  # the logits buffer then holds the projection's logits
            chk("moe_router_logits", lib.moe_router_logits(pc, T, p["x"], wr, p["logits"], p["ws"], wsb, sp))
            ev[1].record(st)
        chk("moe_route", lib.moe_route(pc, T, p["logits"], p["x"] if cfg.Is else None, gvec, p["idx"], p["tw"], sg,
                                       p["keff"], sp))
        ev[pr + 1].record(st)
        if cfg.budget:
            chk("moe_budget", lib.moe_budget(pc, T, p["idx"], p["tw"], p["keff"], p["kept"], p["nd"], p["ws"], wsb, sp))
        ev[pr + 2].record(st)
        chk("moe_dispatch", lib.moe_dispatch(pc, T, p["idx"], p["keff"], p["x"], p["counts"], p["offsets"], p["perm"],
                                             p["slot_pos"], p["x_perm"], p["ws"], wsb, sp))
        ev[pr + 3].record(st)
        chk("moe_expert_ffn", ffn_fn(pc, T, p["x"], p["x_perm"], p["offsets"], p["perm"], p["tw"], sg, pw,
                                     p["ybuf"], p["ws"], wsb, sp))
        ev[pr + 4].record(st)
        chk("moe_combine", lib.moe_combine(pc, T, p["ybuf"], p["keff"], p["out"], sp))
        ev[pr + 5].record(st)

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.graph(g, stream=side):
            fn()
        stream.wait_stream(side)
        return g

    moe.status_clear(ws)
    mk = lambda ext=False: [torch.cuda.Event(enable_timing=True, external=ext) for _ in range(NEV)]  # noqa: E731
    for _ in range(args.warmup):
        flush.zero_()
        step(mk())
    torch.cuda.synchronize(dev)
    status = moe.status_read(ws)
    if status:
        raise RuntimeError(f"device status {status} after warm-up")
    counts_h = counts.cpu().tolist()
    work = stage_work(cfg, counts_h, args.weights)

    # ---- eager launches (diagnostic): K steps back to back from the host
    evs = [mk() for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.zero_()
        step(evs[i])
    torch.cuda.synchronize(dev)
    eager_ms = sum(e[0].elapsed_time(e[NEV - 1]) for e in evs) / args.steps

    # ---- timed region.  Each step replays two CUDA graphs on device-resident
    # inputs, with an L2 flush before each:
    #   fwd:    one moe_forward call between two timing events -> `value`;
    #   stages: the same launches as separate entry-point calls with an
    #           event between stages -> per-kernel durations (roofline).
    # Events are graph nodes, so host launch overhead is outside them; the
    # per-step synchronisation and the flushes are outside the events too.
    aux_c = moe._Aux()
    for n_, t_ in dict(topk_idx=idx, topk_w=tw, keff=keff, expert_kept=kept, n_dropped=nd, counts=counts,
                       offsets=offsets, perm=perm, slot_pos=slot_pos).items():
        setattr(aux_c, n_, P(t_.data_ptr()))
    if cfg.Is:
        aux_c.sgate = P(sgate.data_ptr())

    def fwd_step(e0, e1):
        st = torch.cuda.current_stream(dev)
        e0.record(st)
        chk("moe_forward", fwd_fn(pc, T, p["x"], None if cfg.router_proj else p["logits"], pw, p["out"],
                                  ctypes.byref(aux_c), p["ws"], wsb, P(st.cuda_stream)))
        e1.record(st)

    fev = mk(ext=True)[:2]
    fwd_graph = capture(lambda: fwd_step(*fev))
    gev = mk(ext=True)
    stage_graph = capture(lambda: step(gev))
    for _ in range(args.warmup):
        flush.zero_()
        fwd_graph.replay()
        flush.zero_()
        stage_graph.replay()
    torch.cuda.synchronize(dev)
    stage_sum = {s: 0.0 for s in stages}
    step_sum = 0.0
    staged_sum = 0.0
    barrier(dev)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev)
    t_host0 = time.perf_counter()
    with sampler:
        for i in range(args.steps):
            flush.zero_()
            fwd_graph.replay()
            fev[1].synchronize()
            step_sum += fev[0].elapsed_time(fev[1])
            flush.zero_()
            stage_graph.replay()
            gev[NEV - 1].synchronize()
            for j, sname in enumerate(stages):
                stage_sum[sname] += gev[j].elapsed_time(gev[j + 1])
            staged_sum += gev[0].elapsed_time(gev[NEV - 1])
        torch.cuda.synchronize(dev)
    host_s = time.perf_counter() - t_host0
    barrier(dev)
    per_stage = {s: v / args.steps for s, v in stage_sum.items()}
    step_ms = step_sum / args.steps
    total_ms = max_over_ranks(step_sum, dev)
    status = moe.status_read(ws)
    if status:
        raise RuntimeError(f"device status {status} after timing")
    value = aggregate_tokens_per_s(T, args.steps, total_ms, world)
    del fwd_graph, stage_graph

    # ---- end to end through moe_forward with host buffers (one graph:
    # pinned H2D of x and logits, the layer, D2H of the output)
    e2e = None
    if not args.no_e2e:
        xh = torch.empty((T, H), dtype=torch.bfloat16, pin_memory=True)
        lh = torch.empty((T, E), dtype=torch.float32, pin_memory=True)
        oh = torch.empty((T, H), dtype=torch.bfloat16, pin_memory=True)
        xh.copy_(inp.x)
        lh.copy_(inp.logits)
        xd = torch.empty_like(inp.x)
        ld = torch.empty_like(inp.logits)
        e0, e1 = mk(ext=True)[:2]

        def e2e_step():
            st = torch.cuda.current_stream(dev)
            e0.record(st)
            xd.copy_(xh, non_blocking=True)
            if not cfg.router_proj:  # else the layer computes its logits from x
                ld.copy_(lh, non_blocking=True)
            fwd_py(c, xd, None if cfg.router_proj else ld, wts, out, ws, stream=st)
            oh.copy_(out, non_blocking=True)
            e1.record(st)

        e2e_step()
        torch.cuda.synchronize(dev)
        eg = capture(e2e_step)
        for _ in range(args.warmup):
            flush.zero_()
            eg.replay()
        torch.cuda.synchronize(dev)
        e2e_sum = 0.0
        barrier(dev)
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            flush.zero_()
            eg.replay()
            e1.synchronize()
            e2e_sum += e0.elapsed_time(e1)
        torch.cuda.synchronize(dev)
        barrier(dev)
        e2e_ms = max_over_ranks(e2e_sum, dev)
        e2e = {"value": aggregate_tokens_per_s(T, args.steps, e2e_ms, world), "unit": "tokens/s",
               "h2d_bytes_per_step": T * H * 2 + (0 if cfg.router_proj else T * E * 4), "d2h_bytes_per_step": T * H * 2,
               "ms_per_step": e2e_ms / args.steps, "api": "moe_forward (one CUDA graph per step with the copies)"}
        if not torch.equal(oh.to(dev), out):
            raise RuntimeError("e2e output copy mismatch")
        del eg

    peaks, peak_kind = load_peaks()
    dom = max(stages, key=lambda s: per_stage[s])
    # the sustained peak applies to a kernel timed inside a long run, or whenever
    # the power cap held the clocks down during the timed region
    long_run = (total_ms * 1e-3) > 1.0 or "sw_power_cap" in sampler.summary().get("reasons", [])
    rl = roofline(dom, work, per_stage[dom], peaks, peak_kind, long_run,
                  recorded_traffic(dom, cfg.label + ("" if fmt == "bf16" else ":" + fmt)))
    layer_bw = work["layer"]["bytes"] / (step_ms * 1e-3) / 1e9
    layer_tf = work["layer"]["flops"] / (step_ms * 1e-3) / 1e12

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        mr = cpu_max_rows(cfg, args.weights)
        hi = host_inputs(cfg, inp, mr, args.weights)
        rps, nrows, passes, secs, thr = oracle_rows_per_s(cfg, hi, args.cpu_seconds, mr, repeat=True)
        cpu = {"value": rps, "unit": "tokens/s", "cores": thr, "kind": "oracle",
               "sample": f"{nrows} of {T} tokens of {cfg.label}: routing, budget and dispatch over all {T} tokens, "
                         f"expert FFN + combine (fp64 accumulate) for the sample; {passes} pass(es), {secs:.1f} s"}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,0.02) bf16 x and weights, N(0,1) fp32 router logits + Zipf popularity bias"
                + {"bf16": "",
                   "mxfp8": "; expert weights packed to MXFP8 (E4M3 codes + UE8M0 scales per 32) by the library's "
                            "quantiser",
                   "nvfp4": "; expert weights packed to NVFP4 (E2M1 codes + E4M3 scales per 16 + an fp32 scale per "
                            "matrix) by the library's quantiser"}[fmt],
        "config": {**workload_desc(cfg), "expert_weights": args.weights,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": rl, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": (launches_forward(cfg) + launches_stages(cfg)) * args.steps,
        "clocks": sampler.summary(),
        "stages_ms": per_stage,
        "stages_GB_per_s": {sn: work[sn]["bytes"] / (per_stage[sn] * 1e-3) / 1e9 for sn in stages
                            if work[sn]["bytes"] and per_stage[sn] > 0},
        **({"router_proj_roofline": roofline("router_proj", work, per_stage["router_proj"], peaks, peak_kind,
                                             long_run, None)} if cfg.router_proj else {}),
        "layer": {"touched_experts": work["touched"], "kept_slots": work["slots"],
                  "algorithmic_bytes": work["layer"]["bytes"], "algorithmic_flops": work["layer"]["flops"],
                  "GB_per_s": layer_bw, "TFLOP_per_s": layer_tf,
                  "hbm_frac": layer_bw / peaks["hbm_gbs"]},
        "host_s": host_s,
        "eager_ms_per_step": eager_ms,
        "staged_ms_per_step": staged_sum / args.steps,
        "timing": "value: CUDA-graph replay of moe_forward between two event nodes; stages_ms and roofline: a "
                  "second graph of the stage entry points with an event node between stages; both replayed every "
                  "step, L2 flushed before each, per-step sync outside the events",
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------ reference arm --
def run_reference(args, cfg):
    import torch
    from routed_expert_ffn_renorm_b200 import workloads as W
    world, rank, _ = dist_env()
    if rank != 0:
        return
    inp = W.make_inputs(cfg, device="cuda" if torch.cuda.is_available() and cfg.E * cfg.I * cfg.H > (1 << 28)
                        else "cpu")
    mr = cpu_max_rows(cfg, args.weights)
    hi = host_inputs(cfg, inp, mr, args.weights)
    per_step = min(5.0, 150.0 / max(args.steps + args.warmup, 1))  # whole run within a few minutes
    rps, nrows, _, secs, thr = oracle_rows_per_s(cfg, hi, per_step, mr)
    import oracle
    x, logits, wg, wu, wd, shared = hi
    rows = sample_order(cfg.T)[:nrows]

    def one():
        oracle.forward(x, logits, wg, wu, wd, k=cfg.k, norm_topk=cfg.norm_topk, budget=cfg.budget, topp=cfg.topp, rows=rows,
                       nthreads=thr, I=cfg.I, **shared)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = time.perf_counter() - t0
    value = nrows * args.steps / dt
    sample = f"{nrows} of {cfg.T} tokens of {cfg.label} per step: routing, budget and dispatch over all tokens, " \
             f"expert FFN + combine for the sample"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (same seeded inputs as the GPU arm)",
            "config": {**workload_desc(cfg), "expert_weights": args.weights, "parallelism": "CPU oracle, rank 0"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": thr, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="large_256e",
                    help="named workload (default: the 256-expert top-8 layer, T = 16384, the largest one-GPU "
                         "configuration); drafter_16x1024 / drafter_512x512 / budget_s32 / tiny for the others")
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--alpha", type=float, default=None)
    ap.add_argument("--budget", type=int, default=None)
    ap.add_argument("--topp", type=float, default=None, help="per-token top-p trim (0 = off)")
    ap.add_argument("--E", type=int, default=None,
                    help="override the number of routed experts (a scaled stand-in of a workload for ncu captures)")
    ap.add_argument("--router-proj", action="store_true",
                    help="compute the logits with the router projection x . W_r^T inside the layer")
    ap.add_argument("--weights", choices=["bf16", "mxfp8", "nvfp4"], default="bf16",
                    help="expert weight format: bf16; MXFP8 (E4M3 codes + a power-of-two scale per 32 weights, "
                         "converted to bf16 on chip; half the weight bytes); NVFP4 (E2M1 codes + an E4M3 scale per "
                         "16 weights + an fp32 scale per matrix; a quarter of the weight bytes)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, _, _ = dist_env()
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")
    cfg = workload_from_args(args)
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
