#!/usr/bin/env python
"""Benchmark of the SSD chunked-scan forward on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                [--workload NAME] [--path auto|simt|fused]

One step = one ssd_fwd call, the whole forward path over one batch of the
workload with its inputs resident in HBM: on the fused family (the default
for bf16) segment_state and fused_scan (which chains the cuts); on the chunked
families chunk_cumsum, chunk_state, state_passing and chunk_scan. The default workload is the Mamba-2-2.7B-shaped layer (batch 4, T 4096,
80 heads, P 64, N 128, Q 256, bf16 in / fp32 state). Its inputs (~360 MB) are
larger than L2, so no flush runs between steps. Prints one JSON line on rank 0.

Under torchrun every rank runs the same per-GPU workload (weak scaling: the
(batch, head) units are independent; no data-path collective), the timed
region is bracketed by barriers and the time is the max over ranks.

--impl reference times the CPU fp64 oracle on the host cores on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "SSD fwd tokens·heads/s and TFLOP/s at 2.7B-layer shape; % BF16 tensor peak"
UNIT = "tokens·heads/s"
DEFAULT_WORKLOAD = "mamba2_2p7b_layer"


# --------------------------------------------------------------------------- #
# Algorithmic work (the per-unit figures of the design notes)
# --------------------------------------------------------------------------- #

def algorithmic_flops(w, q=None) -> float:
    """F = b * C_n * [H (Q(Q+1) P + 4 Q N P) + G Q(Q+1) N]: the masked quadratic
    term and C B^T on the lower triangle, the chunk state and the state read-out,
    at the workload's chunk Q (the primary count) or at block length q (the
    fused kernels work in 128-token tiles, whose masked work is that of q = 128)."""
    Q = w.chunk if q is None else q
    cn = w.seqlen / Q
    N, P = w.dstate, w.headdim
    return w.batch * cn * (w.nheads * (Q * (Q + 1) * P + 4 * Q * N * P) + w.ngroups * Q * (Q + 1) * N)


def _esize(w):
    return 2 if w.dtype == "bf16" else 4


def algorithmic_bytes(w) -> float:
    """Minimum I/O of the forward: X, Y, B, C, log a, D, seq_idx, init and final states."""
    e = _esize(w)
    b, T, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    by = 2 * b * T * H * P * e + 2 * b * T * G * N * e + b * T * H * 4
    if w.has_D != "none":
        by += H * 4
    if w.varlen != "none":
        by += b * T * 4
    nseq = w.nseq if w.varlen != "none" else 1
    if w.has_init:
        by += b * nseq * H * N * P * 4
    by += b * nseq * H * N * P * 4  # final states are returned
    return by


def fused_plan(w, wt):
    """The fused path's work ranges for tiles-per-range wt: (nwork, cut_tokens,
    ncuts). cut_tokens: tokens x head pairs that segment_state walks (the last
    piece of every range that ends inside its row); ncuts: ranges that start
    inside a row (each needs one incoming state per head of its pair)."""
    b, T, H = w.batch, w.seqlen, w.nheads
    npairs, nt = H // 2, -(-T // 128)
    total = b * npairs * nt
    nwork = -(-total // wt)
    cut_tokens = ncuts = 0
    for i in range(nwork):
        fb, fe = i * wt, min((i + 1) * wt, total)
        r = (fe - 1) // nt
        s0, s1 = 128 * max(fb - r * nt, 0), min(128 * (fe - r * nt), T)
        if s1 < T:
            cut_tokens += s1 - s0
        if fb % nt:
            ncuts += 1
    return nwork, cut_tokens, ncuts


def kernel_model(w, wt=None):
    """Algorithmic bytes and flops per launch of each kernel.

    Chunked path (chunk Q):
      chunk_cumsum  reads log a, writes cs.
      chunk_state   reads X, B, cs; writes one fp32 state per (b, chunk, h);
                    2 Q N P flops per (b, chunk, h).
      state_passing reads the states and cs, writes the incoming states and the
                    final states; 2 N P flops per (b, chunk, h).
      chunk_scan    reads X, B, C, cs, D and the incoming states; writes Y;
                    Q(Q+1)P + 2QNP flops per (b, chunk, h) + Q(Q+1)N per (b, chunk, g).
    Fused path (work ranges of wt tiles of 128 over the (batch row, head pair)
    rows; see fused_plan):
      segment_state   reads X, B, log a of the last piece of every range that
                      ends inside a row; writes one fp32 state and one decay per
                      such range and head; 2 N P flops per token and head walked.
      segment_passing (the step entry point; ssd_fwd folds it into fused_scan)
                      reads those states and decays, writes one incoming state
                      per range start inside a row and head; 2 N P flops each.
      fused_scan      reads X, B, C, log a, D and the initial states; writes Y
                      and the final states (the algorithmic bytes: the range
                      states it also reads at each cut are a state spill, which
                      the count leaves out); per (b, tile, h) 128*129 P +
                      4*128 N P flops, per (b, tile, g) 128*129 N.
    """
    e = _esize(w)
    b, T, H, P, N, G, Q = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups, w.chunk
    cn = T // Q
    st = b * cn * H * N * P * 4
    xb = b * T * H * P * e
    bcb = b * T * G * N * e
    csb = b * T * H * 4
    nseq = w.nseq if w.varlen != "none" else 1
    fin = b * nseq * H * N * P * 4
    init = fin if w.has_init else 0
    out = {
        "chunk_cumsum": dict(bytes=2 * csb, flops=b * T * H),
        "chunk_state": dict(bytes=xb + bcb + csb + st, flops=b * cn * H * 2 * Q * N * P),
        "state_passing": dict(bytes=2 * st + csb / Q + fin + init, flops=b * cn * H * 2 * N * P),
        "chunk_scan": dict(bytes=2 * xb + 2 * bcb + csb + st + init,
                           flops=b * cn * (H * (Q * (Q + 1) * P + 2 * Q * N * P) + G * Q * (Q + 1) * N)),
    }
    if wt:
        nwork, cut_tokens, ncuts = fused_plan(w, wt)
        ntile = -(-T // 128)
        st2 = 2 * N * P * 4  # the two heads of a pair
        walked = cut_tokens * 2  # token x head
        out.update({
            "segment_state": dict(bytes=walked * (P * e + 4) + cut_tokens * N * e + ncuts * (st2 + 8),
                                  flops=walked * 2 * N * P),
            "segment_passing": dict(bytes=ncuts * (2 * st2 + 8), flops=ncuts * 2 * 2 * N * P),
            "fused_scan": dict(bytes=2 * xb + 2 * bcb + csb + (H * 4 if w.has_D != "none" else 0) + init + fin,
                               flops=b * ntile * (H * (128 * 129 * P + 4 * 128 * N * P) + G * 128 * 129 * N)),
        })
    return out


def profiled_traffic(kernel):
    """dram bytes read + written per launch of `kernel`, from the committed ncu
    summary of the fused path (profiles/fused_path_mamba2_2p7b_layer.json), or
    None when that capture was taken on another version of the kernel source
    (or covers no such kernel)."""
    import hashlib
    prof = os.path.join(ROOT, "profiles", "fused_path_mamba2_2p7b_layer.json")
    if not os.path.exists(prof):
        return None
    with open(prof) as f:
        rec = json.load(f)
    src = os.path.join(ROOT, rec.get("kernel_source", ""))
    if not os.path.isfile(src):
        return None
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest()[: len(rec["sha256_prefix"])] != rec["sha256_prefix"]:
            return None
    v = rec.get("dram_bytes_per_launch", {}).get(kernel)
    return int(v) if v is not None else None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return dict(hbm_gbs=float(pk["hbm_gbs"]), bf16_tflops=float(pk["bf16_tflops"]),
                    bf16_tflops_sustained=float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# --------------------------------------------------------------------------- #
# Clock sampling during the timed region
# --------------------------------------------------------------------------- #

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- #
# Distributed helpers (also exercised by the CPU gloo tests)
# --------------------------------------------------------------------------- #

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(value: float, device=None) -> float:
    """Max over ranks of a scalar (a control-plane reduction, not a data path)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank: float, seconds_per_rank: float, device=None):
    """Whole-job throughput: units of all ranks / the slowest rank's time."""
    import torch.distributed as dist
    ws = dist.get_world_size() if dist.is_available() and dist.is_initialized() else 1
    t = reduce_max(seconds_per_rank, device)
    return units_per_rank * ws / t, t


# --------------------------------------------------------------------------- #
# CPU oracle leg
# --------------------------------------------------------------------------- #

def cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), or the platform string."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def oracle_sample(w, inputs, budget_s: float = 12.0, threads: int = 0, outputs=None):
    """Time the oracle on whole (batch row, head) pairs of the workload, one
    batch row and `cores` heads per call (cores = threads, or every host core
    when threads is 0), until about budget_s seconds of CPU work or the whole
    workload; return (token·heads/s, cores, sample, seconds). With `outputs` (a
    list), each call's (batch row, heads, Y) is appended to it."""
    import oracle
    cores = threads if threads > 0 else max(1, oracle.max_threads())
    done, t_total = 0, 0.0
    for b in range(w.batch):
        for h0 in range(0, w.nheads, cores):
            if t_total >= budget_s:
                break
            hs = slice(h0, min(w.nheads, h0 + cores))
            X = inputs["X"][b:b + 1, :, hs]
            la = inputs["log_a"][b:b + 1, :, hs]
            D = None if inputs["D"] is None else inputs["D"][hs]
            init = None if inputs["init_states"] is None else inputs["init_states"][b:b + 1, :, hs]
            seq = None if inputs["seq_idx"] is None else inputs["seq_idx"][b:b + 1]
            if w.ngroups != 1:
                raise NotImplementedError("oracle sampling assumes one group")
            t0 = time.perf_counter()
            Yr, _ = oracle.ssd_reference(X, la, inputs["B"][b:b + 1], inputs["C"][b:b + 1], D, init, seq,
                                         nseq=inputs["nseq"], nthreads=cores)
            t_total += time.perf_counter() - t0
            if outputs is not None:
                outputs.append((b, hs, Yr))
            done += X.shape[2]
    return done * w.seqlen / t_total, cores, f"{done} (batch row, head) pairs x {w.seqlen} tokens of {w.name}", t_total


# --------------------------------------------------------------------------- #
# Reference arm: the oracle as the timed CPU program
# --------------------------------------------------------------------------- #

def run_reference(args, w):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    inputs = make_inputs(w)
    import oracle
    cores = oracle.max_threads()
    hs = list(range(min(w.nheads, max(1, cores))))
    X = inputs["X"][:1, :, hs]
    la = inputs["log_a"][:1, :, hs]
    D = None if inputs["D"] is None else inputs["D"][hs]
    init = None if inputs["init_states"] is None else inputs["init_states"][:1, :, hs]
    seq = None if inputs["seq_idx"] is None else inputs["seq_idx"][:1]
    step = lambda: oracle.ssd_reference(X, la, inputs["B"][:1], inputs["C"][:1], D, init, seq,
                                        nseq=inputs["nseq"], nthreads=cores)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    units = len(hs) * w.seqlen
    value = units * args.steps / dt
    sample = f"1 batch row x {len(hs)} heads x {w.seqlen} tokens of {w.name} per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, args),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def family(ssd, p, path):
    """Kernel family ssd_fwd runs for problem p under the requested path."""
    if path in ("simt", "fused"):
        return path
    return "fused" if ssd.path_supported(p, "fused") else "simt"


def workload_config(w, args):
    nseq = w.nseq if w.varlen != "none" else 1
    return {"workload": w.name, "batch": w.batch, "seq_len": w.seqlen, "nheads": w.nheads, "headdim": w.headdim,
            "dstate": w.dstate, "ngroups": w.ngroups, "chunk": w.chunk, "nseq": nseq,
            "parallelism": f"dp{args.gpus}" if args.gpus > 1 else "single",
            "l2": "inputs larger than L2, no flush" if algorithmic_bytes(w) > 126e6 else "L2 flushed between steps"}


# --------------------------------------------------------------------------- #
# Our arm
# --------------------------------------------------------------------------- #

def run_ours(args, w):
    import torch
    import torch.distributed as dist
    ws, rank, local = dist_env()
    if args.gpus > 1 and ws != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={ws}: launch with torchrun")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import mamba_ssd_layer_chunked_b200 as ssd

    inputs = make_inputs(w)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def dev_t(a, dt=torch.float32):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dt).to(dev)

    X, la, B, C = dev_t(inputs["X"], tdt), dev_t(inputs["log_a"]), dev_t(inputs["B"], tdt), dev_t(inputs["C"], tdt)
    D, init = dev_t(inputs["D"]), dev_t(inputs["init_states"])
    seq = None if inputs["seq_idx"] is None else torch.from_numpy(inputs["seq_idx"]).to(dev)
    nseq = inputs["nseq"] if seq is not None else None
    p = ssd.problem_from(X, B, w.chunk, inputs["nseq"], args.path)
    Y = torch.empty_like(X)
    b, T, H, P = X.shape
    N = B.shape[3]
    F = torch.empty((b, inputs["nseq"], H, N, P), dtype=torch.float32, device=dev)
    wsp = torch.empty(ssd.workspace_bytes(p), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ssd.ssd_fwd(X, la, B, C, w.chunk, D=D, init_states=init, seq_idx=seq, nseq=nseq, path=args.path,
                    out=Y, final_out=F, workspace=wsp)

    def barrier():
        if ws > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize(dev)

    # the clock sampler starts first, so that the warm-up steps run right before
    # the timed ones (an idle GPU lowers its clocks; the first timed step would
    # pay for the ramp)
    clocks = ClockSampler(local) if rank == 0 and not args.no_clocks else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    for _ in range(args.warmup):
        step()
    evs_step = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    barrier()
    evs_step[0].record(stream)
    for i in range(args.steps):
        step()
        evs_step[i + 1].record(stream)
    barrier()
    t_dev = evs_step[0].elapsed_time(evs_step[-1]) / 1e3
    step_ms = sorted(evs_step[i].elapsed_time(evs_step[i + 1]) for i in range(args.steps))
    pct = lambda q: step_ms[min(len(step_ms) - 1, int(round(q * (len(step_ms) - 1))))]
    units = w.tokens_heads * args.steps
    value, t_max = aggregate(units, t_dev, dev if ws > 1 else None)
    ms_per_step = t_max / args.steps * 1e3

    # per-kernel durations: the kernels of the path ssd_fwd runs, launched one by
    # one through their C-ABI entry points, events between them on the stream
    import ctypes
    lib = ssd.lib()
    fam = family(ssd, p, args.path)
    sp = ctypes.c_void_p(stream.cuda_stream)
    vp = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    pr = ctypes.byref(p)
    wt = nwork = None
    if fam == "fused":
        wt = ssd.fused_work_tiles(p)
        nwork = ssd.fused_work_count(p, wt)
        stb = nwork * 2 * N * P * 4
        al = lambda x: (x + 255) // 256 * 256
        wloc = wsp[:stb].view(torch.float32)
        wdec = wsp[2 * al(stb): 2 * al(stb) + nwork * 2 * 4].view(torch.float32)
        cuts = nwork > 1 and wt % -(-T // 128) != 0
        names, launches = [], []
        if cuts:  # the launches of ssd_fwd: segment_state, then the scan chaining the cuts itself
            names.append("segment_state")
            launches.append(
                lambda: lib.ssd_segment_state(pr, wt, vp(X), vp(la), vp(B), vp(seq), vp(wloc), vp(wdec), sp))
        names.append("fused_scan")
        launches.append(lambda: lib.ssd_fused_scan_chained(pr, wt, vp(X), vp(la), vp(B), vp(C), vp(D),
                                                           vp(wloc) if cuts else None, vp(wdec) if cuts else None,
                                                           vp(init), vp(seq), vp(Y), vp(F), sp))
    else:
        pk = ssd.problem_from(X, B, w.chunk, inputs["nseq"], "simt")
        pr = ctypes.byref(pk)
        nc = -(-T // w.chunk)
        cs = wsp[: b * nc * w.chunk * H * 4].view(torch.float32)
        off = (b * nc * w.chunk * H * 4 + 255) // 256 * 256
        states = wsp[off: off + b * nc * H * N * P * 4].view(torch.float32)
        names = ["chunk_cumsum", "chunk_state", "state_passing", "chunk_scan"]
        launches = [
            lambda: lib.ssd_chunk_cumsum(pr, vp(la), vp(cs), sp),
            lambda: lib.ssd_chunk_state(pr, vp(X), vp(B), vp(cs), vp(seq), vp(states), vp(F), sp),
            lambda: lib.ssd_state_passing(pr, vp(cs), vp(states), vp(states), vp(init), vp(seq), vp(F), sp),
            lambda: lib.ssd_chunk_scan(pr, vp(X), vp(B), vp(C), vp(cs), vp(D), vp(states), vp(init), vp(seq), vp(Y),
                                       sp),
        ]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(launches) + 1)] for _ in range(args.steps)]
    for i in range(args.steps):
        evs[i][0].record(stream)
        for j, fn in enumerate(launches):
            rc = fn()
            if rc != 0:
                raise RuntimeError(f"{names[j]} failed: {ssd.status_string(rc)}")
            evs[i][j + 1].record(stream)
    torch.cuda.synchronize(dev)
    per_kernel = {n: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps)) / 1e3
                  for j, n in enumerate(names)}
    clk = clocks.stop() if clocks else None

    # end to end through the public call on pinned HOST buffers: every step copies
    # its inputs host -> device, runs ssd_fwd and copies Y and the final states
    # back; the copies of neighbouring steps overlap the compute on their own
    # streams (double-buffered device tensors; PCIe carries both directions at once)
    host = dict(X=X.cpu().pin_memory(), la=la.cpu().pin_memory(), B=B.cpu().pin_memory(), C=C.cpu().pin_memory(),
                D=None if D is None else D.cpu().pin_memory(),
                init=None if init is None else init.cpu().pin_memory(),
                seq=None if seq is None else seq.cpu().pin_memory())
    h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
    d2h = Y.numel() * Y.element_size() + F.numel() * F.element_size()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    dbuf = [{k: (None if t is None else torch.empty(t.shape, dtype=t.dtype, device=dev)) for k, t in host.items()}
            for _ in range(2)]
    obuf = [(torch.empty_like(Y), torch.empty_like(F)) for _ in range(2)]
    hout = [(torch.empty(Y.shape, dtype=Y.dtype, pin_memory=True), torch.empty(F.shape, dtype=F.dtype, pin_memory=True))
            for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n):
        for i in range(n):
            j = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_c[j])  # step i-2 has read buffer j
                for k, t in host.items():
                    if t is not None:
                        dbuf[j][k].copy_(t, non_blocking=True)
                ev_in[j].record(s_in)
            stream.wait_event(ev_in[j])
            if i >= 2:
                stream.wait_event(ev_out[j])  # step i-2's outputs have left buffer j
            g_ = dbuf[j]
            ssd.ssd_fwd(g_["X"], g_["la"], g_["B"], g_["C"], w.chunk, D=g_["D"], init_states=g_["init"],
                        seq_idx=g_["seq"], nseq=nseq, path=args.path, out=obuf[j][0], final_out=obuf[j][1],
                        workspace=wsp, stream=stream)
            ev_c[j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c[j])
                hout[j][0].copy_(obuf[j][0], non_blocking=True)
                hout[j][1].copy_(obuf[j][1], non_blocking=True)
                ev_out[j].record(s_out)

    e2e_steps(2)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    e2e_steps(args.steps)
    s_in.wait_stream(s_out)
    s_in.wait_stream(stream)
    e1.record(s_in)
    barrier()
    e2e_value, _ = aggregate(units, e0.elapsed_time(e1) / 1e3, dev if ws > 1 else None)

    # roofline of the dominant kernel
    model = kernel_model(w, wt)
    dom = max(per_kernel, key=per_kernel.get)
    peaks = load_peaks()
    km = model[dom]
    ai = km["flops"] / km["bytes"]
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if ai < ridge:
        achieved = km["bytes"] / per_kernel[dom] / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        achieved = km["flops"] / per_kernel[dom] / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = profiled_traffic(dom)
    roof["kernel"] = dom
    roof["peak_source"] = peaks["source"]

    step_s = t_max / args.steps
    flops = algorithmic_flops(w)
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic", "config": workload_config(w, args),
        "tflops": flops * ws / step_s / 1e12,
        "pct_bf16_peak": flops / step_s / 1e12 / peaks["bf16_tflops"],
        "tflops_note": "algorithmic count at the workload's chunk Q; tflops_at_tile128 counts the masked work "
                       "of the 128-token tiles the fused kernels compute in",
        "tflops_at_tile128": algorithmic_flops(w, 128) * ws / step_s / 1e12,
        "pct_bf16_peak_at_tile128": algorithmic_flops(w, 128) / step_s / 1e12 / peaks["bf16_tflops"],
        "step_ms": {"median": statistics.median(step_ms), "p10": pct(0.1), "p90": pct(0.9),
                    "note": "rank 0, CUDA events between consecutive steps"},
        "pct_hbm": algorithmic_bytes(w) / step_s / 1e9 / peaks["hbm_gbs"],
        "path": fam,
        "work_tiles": wt,
        "work_ranges": nwork,
        "per_kernel_us": {k: v * 1e6 for k, v in per_kernel.items()},
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": len(launches) * args.steps,
        "clocks": clk,
    }
    result["parity"] = None
    if rank == 0 and not args.no_cpu_baseline:
        outs = []
        v, cores, sample, secs = oracle_sample(w, inputs, budget_s=args.cpu_budget, outputs=outs)
        # parity of the timed output on the rows the oracle computed: max|dY| / max|Y_ref|
        err = scale = 0.0
        for b_, hs, Yr in outs:
            Yg = Y[b_:b_ + 1, :, hs].float().cpu().numpy().astype(np.float64)
            err = max(err, float(np.max(np.abs(Yg - Yr))))
            scale = max(scale, float(np.max(np.abs(Yr))))
        result["parity"] = {"max_abs_err_over_max_abs_y": err / scale if scale else 0.0,
                            "tau": 2e-2 if w.dtype == "bf16" else 1e-5, "rows": sample}
        v1, _, sample1, secs1 = oracle_sample(w, inputs, budget_s=max(1.0, args.cpu_budget / 4), threads=1)
        result["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                                  "seconds": secs, "cpu_model": cpu_model(),
                                  "one_core": {"value": v1, "sample": sample1, "seconds": secs1}}
    if rank == 0:
        print(json.dumps(result), flush=True)
    if ws > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return 0


def _device_inputs(w, dev):
    import torch
    inputs = make_inputs(w)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def dev_t(a, dt=torch.float32):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dt).to(dev)

    g = dict(X=dev_t(inputs["X"], tdt), la=dev_t(inputs["log_a"]), B=dev_t(inputs["B"], tdt),
             C=dev_t(inputs["C"], tdt), D=dev_t(inputs["D"]), init=dev_t(inputs["init_states"]),
             seq=None if inputs["seq_idx"] is None else torch.from_numpy(inputs["seq_idx"]).to(dev),
             nseq=inputs["nseq"])
    return inputs, g


def _time_device(fn, steps, warmup, stream):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3 / steps


def _time_graph(fn, steps, warmup, stream):
    """Device time per call of fn replayed from a CUDA graph (no host launch
    cost in the timed region); the eager timing when capture is not possible."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="relaxed"):
            fn()
    except Exception:  # capture refused: fall back to eager launches
        return _time_device(fn, steps, warmup, stream), False
    g.replay()
    torch.cuda.synchronize()
    s_ = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_)
    for _ in range(steps):
        g.replay()
    e1.record(s_)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3 / steps, True


def run_sweep(args):
    """--mode sweep: ssd_fwd on every workload (device time, inputs resident),
    one JSON line each: tokens*heads/s, TFLOP/s and the fractions of the
    measured bf16 and HBM peaks. Not the headline line."""
    import torch
    import mamba_ssd_layer_chunked_b200 as ssd
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)
    for name in sorted(WORKLOADS):
        w = WORKLOADS[name]
        _, g = _device_inputs(w, dev)
        seq = g["seq"]
        p = ssd.problem_from(g["X"], g["B"], w.chunk, g["nseq"], args.path)
        wsp = torch.empty(ssd.workspace_bytes(p), dtype=torch.uint8, device=dev)
        Y = torch.empty_like(g["X"])
        F = torch.empty((w.batch, g["nseq"], w.nheads, w.dstate, w.headdim), dtype=torch.float32, device=dev)
        fn = lambda: ssd.ssd_fwd(g["X"], g["la"], g["B"], g["C"], w.chunk, D=g["D"], init_states=g["init"],
                                 seq_idx=seq, nseq=g["nseq"] if seq is not None else None, path=args.path,
                                 out=Y, final_out=F, workspace=wsp)
        t = _time_device(fn, args.steps, args.warmup, stream)
        flops, byts = algorithmic_flops(w), algorithmic_bytes(w)
        print(json.dumps({"mode": "sweep", "workload": name, "path": family(ssd, p, args.path),
                          "tokens_heads_per_s": w.tokens_heads / t, "ms_per_step": t * 1e3,
                          "tflops": flops / t / 1e12, "pct_bf16_peak": flops / t / 1e12 / peaks["bf16_tflops"],
                          "pct_hbm": byts / t / 1e9 / peaks["hbm_gbs"], "peak_source": peaks["source"],
                          "steps": args.steps, "warmup": args.warmup}), flush=True)
        del g, wsp, Y, F
        torch.cuda.empty_cache()
    return 0


def run_decode(args, w):
    """--mode decode: ssd_decode_step over --decode-batch sequences with the
    workload's heads, state and dtype (state cache larger than L2). Bytes per
    step: the state read and written (2 * b * H * N * P * 4) plus x, y, B, C,
    log a. One JSON line, not the headline."""
    import torch
    import mamba_ssd_layer_chunked_b200 as ssd
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    b, H, P, N, G = args.decode_batch, w.nheads, w.headdim, w.dstate, w.ngroups
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    gen = torch.Generator(device=dev).manual_seed(7)
    x = torch.randn(b, H, P, device=dev, generator=gen).to(tdt)
    Bm = (torch.randn(b, G, N, device=dev, generator=gen) / N ** 0.5).to(tdt)
    Cm = (torch.randn(b, G, N, device=dev, generator=gen) / N ** 0.5).to(tdt)
    la = -torch.rand(b, H, device=dev, generator=gen) * 0.1
    state = torch.randn(b, H, N, P, device=dev, generator=gen)
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream(dev)
    t = _time_device(lambda: ssd.decode_step(x, la, Bm, Cm, state, out=y), args.steps, args.warmup, stream)
    e = 2 if w.dtype == "bf16" else 4
    byts = 2 * b * H * N * P * 4 + 2 * b * H * P * e + 2 * b * G * N * e + b * H * 4
    peaks = load_peaks()
    print(json.dumps({"mode": "decode", "metric": "SSD decode step tokens·heads/s", "workload": w.name,
                      "decode_batch": b, "value": b * H / t, "unit": "tokens·heads/s", "us_per_step": t * 1e6,
                      "roofline": {"bound": "hbm", "achieved": byts / t / 1e9, "peak": peaks["hbm_gbs"],
                                   "unit": "GB/s", "frac": byts / t / 1e9 / peaks["hbm_gbs"]},
                      "steps": args.steps, "warmup": args.warmup, "dtype": w.dtype}), flush=True)
    return 0


def run_discretize(args, w):
    """--mode discretize: ssd_discretize over the workload's (b, T, H, P) (the step
    before the scan: softplus step size, log a = delta A, X = delta x). Bytes per
    step: x read and X written (P e each per token x head), dt read and log a
    written (4 each). One JSON line, not the headline."""
    import torch
    import mamba_ssd_layer_chunked_b200 as ssd
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    b, T, H, P = w.batch, w.seqlen, w.nheads, w.headdim
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    gen = torch.Generator(device=dev).manual_seed(11)
    dt = torch.randn(b, T, H, device=dev, generator=gen) - 3
    A = -torch.rand(H, device=dev, generator=gen) * 16
    bias = torch.randn(H, device=dev, generator=gen) * 0.1
    x = torch.randn(b, T, H, P, device=dev, generator=gen).to(tdt)
    X = torch.empty_like(x)
    la = torch.empty(b, T, H, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        flush.zero_()  # inputs of one step fit in L2: flush between steps, timed separately below
        ssd.discretize(dt, A, x, dt_bias=bias, out=(la, X))

    t_all = _time_device(step, args.steps, args.warmup, stream)
    t_flush = _time_device(lambda: flush.zero_(), args.steps, args.warmup, stream)
    t = max(t_all - t_flush, 1e-9)
    e = 2 if w.dtype == "bf16" else 4
    byts = b * T * H * (2 * P * e + 8)
    peaks = load_peaks()
    print(json.dumps({"mode": "discretize", "metric": "discretisation tokens·heads/s", "workload": w.name,
                      "value": b * T * H / t, "unit": "tokens·heads/s", "us_per_step": t * 1e6,
                      "roofline": {"bound": "hbm", "achieved": byts / t / 1e9, "peak": peaks["hbm_gbs"],
                                   "unit": "GB/s", "frac": byts / t / 1e9 / peaks["hbm_gbs"]},
                      "l2": "flushed between steps (flush time subtracted)", "steps": args.steps,
                      "warmup": args.warmup, "dtype": w.dtype}), flush=True)
    return 0


def run_sp(args, w):
    """--mode sp: the sequence-parallel forward (every batch row's tokens in R
    consecutive segments). Under torchrun (WORLD_SIZE > 1) it runs over NCCL,
    one segment per rank, timed on the device as the max over ranks. On one
    GPU it emulates R = --sp-ranks ranks one after another: it times each
    rank's summary, combine and forward on its segment (the exchanged
    summaries are those of the real segments) and reports the slowest rank's
    sum next to the whole-sequence forward; the exchange itself (an all-gather
    of R x (b H N P + b H) fp32 + b x 2 int32 per rank, and the final-state sum)
    is not timed there. One JSON line, not the headline."""
    import torch
    import mamba_ssd_layer_chunked_b200 as ssd
    from mamba_ssd_layer_chunked_b200.sp import ssd_fwd_sp, torch_collectives
    world, rank, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    _, g = _device_inputs(w, dev)
    stream = torch.cuda.current_stream(dev)
    seq, nseq = g["seq"], g["nseq"]
    nseq_arg = nseq if seq is not None else None
    T = w.seqlen
    R = world if world > 1 else args.sp_ranks
    bounds = [T * r // R for r in range(R + 1)]
    seg = lambda t, r: None if t is None else t[:, bounds[r]:bounds[r + 1]].contiguous()
    b, H, N, P = w.batch, w.nheads, w.dstate, w.headdim
    xbytes = R * (b * H * N * P * 4 + b * H * 4 + b * 2 * 4)
    if world > 1:
        r = rank
        X, la, B, C, sq = (seg(g[k], r) for k in ("X", "la", "B", "C", "seq"))
        ag, ar = torch_collectives()
        fn = lambda: ssd_fwd_sp(X, la, B, C, w.chunk, rank=r, all_gather=ag, all_reduce_sum=ar, D=g["D"],
                                init_states=g["init"], seq_idx=sq, nseq=nseq_arg)
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        t = reduce_max(e0.elapsed_time(e1) / 1e3 / args.steps)
        if rank == 0:
            print(json.dumps({"mode": "sp", "workload": w.name, "ranks": R, "emulated": False,
                              "value": w.tokens_heads / t, "unit": "tokens·heads/s", "ms_per_step": t * 1e3,
                              "exchange_bytes_per_rank": xbytes, "scaling": "strong",
                              "steps": args.steps, "warmup": args.warmup}), flush=True)
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
        return 0
    graphs = True
    def timed(fn):
        nonlocal graphs
        t, ok = _time_graph(fn, args.steps, args.warmup, stream)
        graphs = graphs and ok
        return t
    t_full = timed(lambda: ssd.ssd_fwd(g["X"], g["la"], g["B"], g["C"], w.chunk, D=g["D"], init_states=g["init"],
                                       seq_idx=seq, nseq=nseq_arg))
    parts = [{k: seg(g[k], r) for k in ("X", "la", "B", "C", "seq")} for r in range(R)]
    sums = [ssd.sp_summary(q["X"], q["la"], q["B"], seq_idx=q["seq"], nseq=nseq) for q in parts]
    g_loc, g_dec, g_ids = (torch.stack([s_[i] for s_ in sums]) for i in range(3))
    per_rank = []
    for r, q in enumerate(parts):
        init_local = ssd.sp_combine(q["X"], q["B"], g_loc, g_dec, g_ids, r, init_states=g["init"], nseq=nseq)
        t_sum = timed(lambda: ssd.sp_summary(q["X"], q["la"], q["B"], seq_idx=q["seq"], nseq=nseq))
        t_comb = timed(lambda: ssd.sp_combine(q["X"], q["B"], g_loc, g_dec, g_ids, r, init_states=g["init"],
                                              nseq=nseq))
        t_fwd = timed(lambda: ssd.ssd_fwd(q["X"], q["la"], q["B"], q["C"], w.chunk, D=g["D"],
                                          init_states=init_local, seq_idx=q["seq"], nseq=nseq_arg))
        per_rank.append((t_sum, t_comb, t_fwd))
    slow = max(per_rank, key=sum)
    t_rank = sum(slow)
    print(json.dumps({"mode": "sp", "workload": w.name, "ranks": R, "emulated": True, "cuda_graphs": graphs,
                      "ms_full_one_gpu": t_full * 1e3, "ms_slowest_rank": t_rank * 1e3,
                      "slowest_rank_ms": {"summary": slow[0] * 1e3, "combine": slow[1] * 1e3, "forward": slow[2] * 1e3},
                      "speedup_without_exchange": t_full / t_rank, "exchange_bytes_per_rank": xbytes,
                      "steps": args.steps, "warmup": args.warmup}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "fused"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--mode", choices=["scan", "sweep", "decode", "sp", "discretize"], default="scan",
                    help="scan: the headline line (default); sweep: every workload; decode: the decode step; "
                         "sp: the sequence-parallel forward; discretize: the discretisation step")
    ap.add_argument("--decode-batch", type=int, default=64)
    ap.add_argument("--sp-ranks", type=int, default=4, help="ranks emulated on one GPU by --mode sp")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.mode == "sweep":
        return run_sweep(args)
    if args.mode == "decode":
        return run_decode(args, w)
    if args.mode == "discretize":
        return run_discretize(args, w)
    if args.mode == "sp":
        return run_sp(args, WORKLOADS["long16k_N128"] if args.workload == DEFAULT_WORKLOAD else w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
