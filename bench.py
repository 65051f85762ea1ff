#!/usr/bin/env python
"""Throughput of the fused folded selective scan (aux init + conv + scan + gate) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload stage4_t49] [--impl sfm|reference]

One step = one fused forward (aux init -> conv+SiLU -> Delta -> folded scan with reset
-> D skip -> SiLU(z) gate) over one batch of the workload, with B1 from the look-up
table.  Prints one JSON line on rank 0.

* value: elements (B*D*L) per second over all ranks, inputs resident in HBM; K launches
  timed with CUDA events on the launch stream between a barrier + synchronize on both
  sides, max over ranks.  Inputs rotate over several sets whose total exceeds 2x L2.
* e2e: the same metric through the public Python API with each step's inputs copied
  host->device from pinned memory and the output read back device->host; two device
  buffer sets on three streams let one step's upload overlap the previous step's kernel
  and readback.
* roofline: the kernel is bound by its transcendental arithmetic (MUFU), not by HBM;
  the ALU peak is derived from unit counts and the SM clock; the HBM
  fraction is reported next to it.
* cpu_baseline: the fp64 CPU oracle on a bounded sample of the same workload.
Multi-GPU: one process per GPU (torchrun), each rank runs its own shard of a global batch
(weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
SMS = 148
MUFU_PER_CLK_SM = 16      # ex2/lg2/rcp lanes per clock per SM (measured on B200)
FP32_PER_CLK_SM = 128     # FP32 FMA lanes per clock per SM
METRIC = "folded scan+conv elems/s (B*D*L) and HBM GB/s as % of peak, T=49/196"


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", default="stage4_t49")
    p.add_argument("--impl", default="sfm", choices=["sfm", "reference"])
    p.add_argument("--no-extra", action="store_true",
                   help="skip the T=196 and ragged lines and the CPU baseline")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-baseline sample budget")
    return p.parse_args(argv)


# ----------------------------------------------------------------------------- host logic (CPU-testable)

def shard_range(global_batch: int, world: int, rank: int, fold: int = 1):
    """Samples [lo, hi) of a global batch owned by `rank`: whole fold groups, contiguous."""
    groups = global_batch // fold
    lo_g = groups * rank // world
    hi_g = groups * (rank + 1) // world
    return lo_g * fold, hi_g * fold


def algorithmic_bytes(B, D, T, L, N, K, in_size, out_size):
    """Bytes the fused forward must move at least: read x [B,D,T], dt and z [B,D,L],
    B and C [B,N,L], the fp32 parameters; write y [B,D,L]."""
    acts = B * D * T * in_size + 2 * B * D * L * in_size + 2 * B * N * L * in_size
    params = D * (N + 3 + K) * 4
    return acts + params + B * D * L * out_size


POLY_EXP2_FMA_OPS = 8      # FMA-pipe lane-ops of one polynomial exp2 (Cody-Waite + degree 5)


def alu_ops_per_element(N, K):
    """(transcendental functions, fp32 ops) per element of the fused forward.
    Transcendentals: N decays exp(Delta*A_n); softplus (an exp and a log); the two SiLUs
    (one sigmoid each).  FP32: 4 per state (Delta*A, B*Delta*u, state update, read-out),
    the conv (K taps + bias), Delta*u, the D skip, the gate, and about 6 around the
    transcendentals."""
    return N + 4, 4 * N + K + 12


def alu_clk_per_element(N, K):
    """Least SM clocks per element on the two pipes that can do the work: each
    transcendental goes either to the MUFU (16 lanes/clk/SM) or, as a polynomial of
    POLY_EXP2_FMA_OPS lane-ops, to the FMA pipe (128 lanes/clk/SM) that also carries the
    fp32 work; the best split balances the two pipes."""
    E, F = alu_ops_per_element(N, K)
    c = POLY_EXP2_FMA_OPS
    m = (F + c * E) / (FP32_PER_CLK_SM / MUFU_PER_CLK_SM + c)  # transcendentals left on the MUFU
    m = min(max(m, 0.0), E)
    return max(m / MUFU_PER_CLK_SM, (F + c * (E - m)) / FP32_PER_CLK_SM)


def alu_peak_elems(N, K, sm_mhz, sms=SMS):
    return sms * sm_mhz * 1e6 / alu_clk_per_element(N, K)


def mufu_only_peak_elems(N, K, sm_mhz, sms=SMS):
    E, F = alu_ops_per_element(N, K)
    return sms * sm_mhz * 1e6 / max(E / MUFU_PER_CLK_SM, F / FP32_PER_CLK_SM)


# the sources that decide the benchmark kernel and its launch shape
FWD_SOURCES = ("sfm_fwd.cu", "sfm_device.cuh", "sfm_internal.h", "sfm_api.cu", "sfm_lut.inc")


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_scan_sfm_b200", "csrc")
    for f in FWD_SOURCES:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on the
    current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))
    except (OSError, ValueError):
        return None
    r = rec.get(workload)
    if not r or r.get("kernel_source_hash") != kernel_source_hash():
        return None
    return r.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid=None):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits", "-lms", "100"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], cap=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        pmax = max(r["power"] for r in rows)
        load = [r for r in rows if r["power"] >= 0.5 * pmax] or rows
        sms = sorted(r["sm"] for r in load)
        reasons = []
        for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                          ("cap", "sw_power_cap")):
            if any(r[key].lower() == "active" for r in load):
                reasons.append(name)
        return {"sm_mhz": sms[len(sms) // 2], "sm_max_mhz": max(r["smax"] for r in rows), "reasons": reasons,
                "samples": len(load), "power_w_max": pmax}


# ----------------------------------------------------------------------------- CPU oracle baseline

def cpu_baseline(workload, budget_s, seed=0):
    """The oracle (fp64, all host cores by sample) on a bounded sample of the workload."""
    import oracle
    from selective_scan_sfm_b200 import synth
    w = dict(synth.WORKLOADS[workload])
    cores = os.cpu_count() or 1
    w1 = dict(w, B=1)
    d = synth.make_inputs(**w1, seed=seed)
    f = lambda t: t.double().numpy()
    args = lambda dd: (f(dd["x"]), f(dd["dt"]), f(dd["z"]), f(dd["Bm"]), f(dd["Cm"]), f(dd["A"]), f(dd["Dskip"]),
                       f(dd["dt_bias"]), f(dd["conv_w"]), f(dd["conv_b"]))
    t0 = time.perf_counter()
    oracle.mixer_layer(*args(d), aux_init_in=True, threads=1)
    one = time.perf_counter() - t0
    nb = int(max(cores, min(w["B"], round(budget_s * cores / max(one, 1e-6)))))
    nb = max(1, min(nb, w["B"]))
    d = synth.make_inputs(**dict(w, B=nb), seed=seed)
    t0 = time.perf_counter()
    oracle.mixer_layer(*args(d), aux_init_in=True, threads=cores)
    dt = time.perf_counter() - t0
    L = w["T"] + 2
    el = nb * w["D"] * L
    return {"value": el / dt, "unit": "elems/s", "cores": min(cores, nb), "kind": "oracle",
            "sample": "%d of %d samples of %s (%d elements), fp64, %.1f s" % (nb, w["B"], workload, el, dt)}


def run_reference(args, world, rank):
    """--impl reference: the oracle timed on the host cores, rank 0 only."""
    if rank != 0:
        return
    from selective_scan_sfm_b200 import synth
    import oracle
    w = synth.WORKLOADS[args.workload]
    cores = os.cpu_count() or 1
    total_budget = 150.0
    per_step = total_budget / max(1, args.steps + args.warmup)
    f = lambda t: t.double().numpy()
    d1 = synth.make_inputs(**dict(w, B=1), seed=0)
    t0 = time.perf_counter()
    oracle.mixer_layer(f(d1["x"]), f(d1["dt"]), f(d1["z"]), f(d1["Bm"]), f(d1["Cm"]), f(d1["A"]), f(d1["Dskip"]),
                       f(d1["dt_bias"]), f(d1["conv_w"]), f(d1["conv_b"]), aux_init_in=True, threads=1)
    one = time.perf_counter() - t0
    nb = max(1, min(w["B"], int(per_step * cores / max(one, 1e-6))))
    d = synth.make_inputs(**dict(w, B=nb), seed=0)
    a = tuple(f(d[k]) for k in ("x", "dt", "z", "Bm", "Cm", "A", "Dskip", "dt_bias", "conv_w", "conv_b"))
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.mixer_layer(*a, aux_init_in=True, threads=cores)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    L = w["T"] + 2
    el = nb * w["D"] * L
    tot = sum(times)
    value = el * len(times) / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "elems/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "B": w["B"], "D": w["D"], "T": w["T"], "L": L, "N": w["N"],
                   "io_dtype": w["dtype"]},
        "cpu_baseline": {"value": value, "unit": "elems/s", "cores": min(cores, nb), "kind": "oracle",
                         "sample": "%d of %d samples per step (%d elements), fp64" % (nb, w["B"], el)},
        "e2e": {"value": value, "unit": "elems/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU measurement

def measure(workload, steps, warmup, world, rank, device, seed_base=0, with_e2e=True):
    import torch
    from selective_scan_sfm_b200 import _abi, sfm_choose_variant, sfm_selective_scan_fold, synth
    from selective_scan_sfm_b200 import _scan_args  # noqa: F401  (argument marshalling of the binding)

    w = synth.WORKLOADS[workload]
    B, D, T, N, K = w["B"], w["D"], w["T"], w["N"], w["K"]
    L = T + 2
    io = synth.torch_dtype(w["dtype"])
    esz = 2 if w["dtype"] == "bf16" else 4
    var = sfm_choose_variant(B, T, D, N)
    set_bytes = algorithmic_bytes(B, D, T, L, N, K, esz, esz)
    nsets = max(2, math.ceil(2 * L2_BYTES / set_bytes) + 1)
    sets = []
    for i in range(nsets):
        d = synth.make_inputs(**w, seed=seed_base + 17 * i)
        dc = {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
        dc["y"] = torch.empty(B, D, L, dtype=io, device=device)
        sets.append(dc)
    stream = torch.cuda.current_stream(device)
    sp = ctypes.c_void_p(stream.cuda_stream)
    lib = _abi.lib()
    cargs = []
    from selective_scan_sfm_b200 import _scan_args as mk
    for dc in sets:
        a, _ = mk(dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], dc["z"], dc["Dskip"], dc["dt_bias"], dc["conv_w"],
                  dc["conv_b"], dc["y"], None, 0, None, True, True, False, None, 0, 0, 0)
        cargs.append(a)

    def launch(i):
        rc = lib.sfm_selective_scan_fold(ctypes.byref(cargs[i % nsets]), sp)
        if rc != 0:
            raise RuntimeError(_abi.status_string(rc))

    for i in range(warmup):
        launch(i)
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    t_start.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        launch(i)
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    total_ms = t_start.elapsed_time(t_end)
    launch_ms = sorted(e0.elapsed_time(e1) for e0, e1 in ev)
    avg_launch_ms = sum(launch_ms) / len(launch_ms)
    res = dict(total_ms=total_ms, avg_launch_ms=avg_launch_ms, median_launch_ms=launch_ms[len(launch_ms) // 2],
               elements=B * D * L, bytes=set_bytes, variant=var, nsets=nsets, set_bytes=set_bytes, w=w, L=L)

    if with_e2e:
        # the public API with host buffers: pinned H2D of the step's inputs, D2H of y.  Two
        # device buffer sets on three streams: step i+1's H2D overlaps step i's kernel and
        # D2H (PCIe carries both directions at once); each step still copies its own inputs
        # in and its own output out inside the timed region.
        host = synth.make_inputs(**w, seed=seed_base + 999)
        pin = {k: host[k].pin_memory() for k in ("x", "dt", "z", "Bm", "Cm")}
        par = {k: host[k].to(device) for k in ("A", "Dskip", "dt_bias", "conv_w", "conv_b")}
        dev = [{k: torch.empty_like(pin[k], device=device) for k in pin} for _ in range(2)]
        yd = [torch.empty(B, D, L, dtype=io, device=device) for _ in range(2)]
        yh = [torch.empty(B, D, L, dtype=io).pin_memory() for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in pin.values())
        d2h = yh[0].numel() * yh[0].element_size()
        s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev = lambda: torch.cuda.Event()
        in_done, run_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        used = [False, False]

        def e2e_step(i):
            j = i % 2
            with torch.cuda.stream(s_in):
                if used[j]:
                    s_in.wait_event(run_done[j])   # the kernel two steps back has read dev[j]
                for k in pin:
                    dev[j][k].copy_(pin[k], non_blocking=True)
                in_done[j].record(s_in)
            stream.wait_event(in_done[j])
            if used[j]:
                stream.wait_event(out_done[j])     # yd[j] has been read out
            sfm_selective_scan_fold(dev[j]["x"], dev[j]["dt"], dev[j]["Bm"], dev[j]["Cm"], par["A"], z=dev[j]["z"],
                                    Dskip=par["Dskip"], dt_bias=par["dt_bias"], conv_w=par["conv_w"],
                                    conv_b=par["conv_b"], y=yd[j], aux_init=True)
            run_done[j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(run_done[j])
                yh[j].copy_(yd[j], non_blocking=True)
                out_done[j].record(s_out)
            used[j] = True

        def drain():  # the launch stream waits for every copy in flight
            for j in range(2):
                if used[j]:
                    stream.wait_event(out_done[j])

        e2e_steps = max(3, min(steps, 20))
        for i in range(3):
            e2e_step(i)
        drain()
        torch.cuda.synchronize(device)
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(e2e_steps):
            e2e_step(i)
        drain()
        e1.record(stream)
        torch.cuda.synchronize(device)
        if world > 1:
            torch.distributed.barrier()
        res.update(e2e_ms=e0.elapsed_time(e1), e2e_steps=e2e_steps, h2d=h2d, d2h=d2h)
    return res


def ragged_algorithmic_bytes(S, D, Lt, N, K, in_size, out_size, aux=True):
    """Bytes the ragged fused forward must move at least: x [D, Lt-2S], dt and z [D, Lt],
    B and C [N, Lt], the offsets, the fp32 parameters; write y [D, Lt]."""
    Lx = Lt - 2 * S if aux else Lt
    acts = D * Lx * in_size + 2 * D * Lt * in_size + 2 * N * Lt * in_size
    return acts + 4 * (S + 1) + D * (N + 3 + K) * 4 + D * Lt * out_size


def _time_launches(launch, nsets, steps, warmup, world, device, stream):
    import torch
    for i in range(warmup):
        launch(i)
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        launch(i)
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    return t0.elapsed_time(t1), sum(a.elapsed_time(b) for a, b in ev) / steps


def measure_ragged(steps, warmup, world, rank, device, seed_base=0, workload="ragged_t49_196"):
    """The ragged forward on packed samples of unequal length, and, for comparison, the
    fixed-layout forward on the same samples padded to the longest one (useful elements
    counted in both)."""
    import torch
    from selective_scan_sfm_b200 import _abi, _scan_args, _varlen_args, synth

    w = synth.WORKLOADS[workload]
    S, D, N, K = w["S"], w["D"], w["N"], w["K"]
    lens = synth.ragged_lengths(S, w["T_lo"], w["T_hi"], seed=seed_base)
    Lt = sum(lens)
    esz = 2 if w["dtype"] == "bf16" else 4
    set_bytes = ragged_algorithmic_bytes(S, D, Lt, N, K, esz, esz)
    nsets = max(2, math.ceil(2 * L2_BYTES / set_bytes) + 1)
    stream = torch.cuda.current_stream(device)
    sp = ctypes.c_void_p(stream.cuda_stream)
    lib = _abi.lib()
    keep, cargs = [], []
    for i in range(nsets):
        d = synth.make_ragged_inputs(lens, D=D, N=N, K=K, dtype=w["dtype"], seed=seed_base + 31 * i)
        dc = {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
        a, y = _varlen_args(dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], dc["cu_seqlens"], dc["z"], dc["Dskip"],
                            dc["dt_bias"], dc["conv_w"], dc["conv_b"], None, None, 0, None, True, True, False, None)
        keep.append((dc, y))
        cargs.append((a, ctypes.c_void_p(dc["cu_seqlens"].data_ptr())))

    def launch(i):
        a, cu = cargs[i % nsets]
        rc = lib.sfm_selective_scan_fold_varlen(ctypes.byref(a), cu, sp)
        if rc != 0:
            raise RuntimeError(_abi.status_string(rc))

    total_ms, launch_ms = _time_launches(launch, nsets, steps, warmup, world, device, stream)
    del keep, cargs
    # the same samples padded to the longest one, fixed [S, D, Tmax + 2] layout
    Tmax = max(lens) - 2
    pb = synth.make_inputs(B=S, D=D, T=Tmax, N=N, K=K, dtype=w["dtype"], seed=seed_base + 7)
    pbytes = algorithmic_bytes(S, D, Tmax, Tmax + 2, N, K, esz, esz)
    psets = max(2, math.ceil(2 * L2_BYTES / pbytes) + 1)
    pkeep, pargs = [], []
    for i in range(psets):
        dc = {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in pb.items()}
        a, y = _scan_args(dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], dc["z"], dc["Dskip"], dc["dt_bias"],
                          dc["conv_w"], dc["conv_b"], None, None, 0, None, True, True, False, None, 0, 0, 0)
        pkeep.append((dc, y))
        pargs.append(a)

    def launch_padded(i):
        rc = lib.sfm_selective_scan_fold(ctypes.byref(pargs[i % psets]), sp)
        if rc != 0:
            raise RuntimeError(_abi.status_string(rc))

    ptotal_ms, plaunch_ms = _time_launches(launch_padded, psets, steps, warmup, world, device, stream)
    return dict(total_ms=total_ms, avg_launch_ms=launch_ms, elements=D * Lt, bytes=set_bytes, w=w, lens=lens,
                padded_total_ms=ptotal_ms, padded_launch_ms=plaunch_ms, padded_elements=S * D * (Tmax + 2))


def measure_proj(steps, warmup, world, device, workload="stage4_t49", seed=0):
    """The projections around the scan at a workload's shape, each a tcgen05 GEMM timed on
    its own: in_proj (tokens [B*L, D/2] -> x, z [B,D,L]), x_proj (u [B*L, D] -> dt_low
    token-major [B*L, R], B and C [B,N,L]) and dt_proj (dt_low -> dt [B,D,L]), with
    d_model = D/2 and R = ceil(D/16) (the Mamba defaults; the pages fix neither)."""
    import torch
    from selective_scan_sfm_b200 import _abi, _proj_args, synth

    w = synth.WORKLOADS[workload]
    B, D, L, N = w["B"], w["D"], w["T"] + 2, w["N"]
    C, R = D // 2, -(-D // 16)
    R = -(-R // 8) * 8  # a multiple of 8 (16-byte rows for the tensor maps)
    Ntok = B * L
    g = torch.Generator().manual_seed(seed)
    bf = torch.bfloat16
    mk = lambda *sh, scale=1.0: (scale * torch.randn(*sh, generator=g)).to(bf).to(device)
    tok, u = mk(Ntok, C), mk(Ntok, D)
    W_in, W_x, W_dt = mk(2 * D, C, scale=C ** -0.5), mk(R + 2 * N, D, scale=D ** -0.5), mk(D, R, scale=R ** -0.5)
    dt_low = mk(Ntok, R)
    gemms = {
        "in_proj": (_proj_args(W_in, tok, L, D, False, bf, None, None, 0)[0], 2.0 * Ntok * C * 2 * D),
        "x_proj_bc": (_proj_args(W_x[R:].contiguous(), u, L, N, False, bf, None, None, 0)[0], 2.0 * Ntok * D * 2 * N),
        "x_proj_dt": (_proj_args(W_x[:R].contiguous(), u, L, None, True, bf, None, None, 0)[0], 2.0 * Ntok * D * R),
        "dt_proj": (_proj_args(W_dt, dt_low, L, D, False, bf, None, None, 0)[0], 2.0 * Ntok * R * D),
    }
    keep = (tok, u, W_in, W_x, W_dt, dt_low)  # noqa: F841  (the args point into these)
    lib = _abi.lib()
    stream = torch.cuda.current_stream(device)
    sp = ctypes.c_void_p(stream.cuda_stream)
    out = {}
    for name, (a, flops) in gemms.items():
        def launch(i, a=a):
            rc = lib.sfm_proj_gemm(ctypes.byref(a), sp)
            if rc != 0:
                raise RuntimeError(_abi.status_string(rc))
        _, ms = _time_launches(launch, 1, steps, warmup, world, device, stream)
        out[name] = dict(ms=ms, flops=flops)
    out["shape"] = dict(B=B, L=L, d_model=C, D=D, N=N, R=R)
    return out


def measure_bwd(steps, warmup, world, device, workload="chain4_stage3", seed_base=0):
    """The backward of the whole mixer layer (aux init, conv + SiLU, folded scan, gate,
    swap) at a workload's layer shape, timed alone over rotating input sets."""
    import torch
    from selective_scan_sfm_b200 import _abi, _mixer_bwd_args, synth

    w = synth.WORKLOADS[workload]
    B, D, T, N, K = w["B"], w["D"], w["T"], w["N"], w["K"]
    L = T + 2
    esz = 2 if w["dtype"] == "bf16" else 4
    # inputs read (x, dt, z, B, C, dout) and fp32 gradients written (dx, ddt, dz, dB, dC)
    set_bytes = B * D * (T + 3 * L) * esz + 2 * B * N * L * esz + B * D * (T + 2 * L) * 4 + 2 * B * N * L * 4
    nsets = max(2, math.ceil(2 * L2_BYTES / set_bytes) + 1)
    stream = torch.cuda.current_stream(device)
    sp = ctypes.c_void_p(stream.cuda_stream)
    lib = _abi.lib()
    keep, cargs = [], []
    for i in range(nsets):
        d = synth.make_inputs(**w, seed=seed_base + 13 * i)
        dc = {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
        dout = synth.make_dout(B, D, L, seed=seed_base + i).to(device)
        a, g, grads, ws = _mixer_bwd_args(dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], dout, dc["z"], dc["Dskip"],
                                          dc["dt_bias"], dc["conv_w"], dc["conv_b"], None, True, True, True, None)
        keep.append((dc, dout, grads, ws))
        cargs.append((a, g, ctypes.c_void_p(ws.data_ptr()), ws.numel()))

    def launch(i):
        a, g, wp, wn = cargs[i % nsets]
        rc = lib.sfm_mixer_bwd(ctypes.byref(a), ctypes.byref(g), wp, wn, sp)
        if rc != 0:
            raise RuntimeError(_abi.status_string(rc))

    total_ms, _ = _time_launches(launch, nsets, steps, warmup, world, device, stream)
    return dict(ms=total_ms / steps, elements=B * D * L, bytes=set_bytes, workspace=cargs[0][3], w=w)


def max_over_ranks(v, world, device):
    if world == 1:
        return v
    import torch
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if world > 1:
            import torch
            torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=600))
        try:
            run_reference(args, world, rank)
        finally:
            if world > 1:
                torch.distributed.destroy_process_group()
        return

    import torch
    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    from selective_scan_sfm_b200 import _abi
    _abi.lib()
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(device).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        uuid = None

    # main workload: rank r owns samples [r*B, (r+1)*B) of a global batch of world*B
    clocks = ClockSampler(uuid)
    clocks.start()
    res = measure(args.workload, args.steps, args.warmup, world, rank, device, seed_base=1000 * rank)
    ck = clocks.stop()
    t_ms = max_over_ranks(res["total_ms"], world, device)
    launch_ms = max_over_ranks(res["avg_launch_ms"], world, device)
    e2e_ms = max_over_ranks(res["e2e_ms"], world, device)
    w, L = res["w"], res["L"]
    el = res["elements"]
    value = world * el * args.steps / (t_ms * 1e-3)
    e2e_value = world * el * res["e2e_steps"] / (e2e_ms * 1e-3)

    extra = {}
    if not args.no_extra and args.workload != "stage3_t196":
        r2 = measure("stage3_t196", args.steps, args.warmup, world, rank, device, seed_base=1000 * rank + 5,
                     with_e2e=False)
        t2 = max_over_ranks(r2["total_ms"], world, device)
        l2 = max_over_ranks(r2["avg_launch_ms"], world, device)
        w2 = r2["w"]
        extra = {"workload": "stage3_t196", "value": world * r2["elements"] * args.steps / (t2 * 1e-3),
                 "unit": "elems/s", "ms_per_step": t2 / args.steps,
                 "hbm": {"achieved": r2["bytes"] / (l2 * 1e-3) / 1e9, "unit": "GB/s"},
                 "alu_frac": (r2["elements"] / (l2 * 1e-3)) / alu_peak_elems(w2["N"], w2["K"], 1965.0),
                 "B1": r2["variant"]["B1"]}

    ragged = {}
    if not args.no_extra:
        rr = measure_ragged(args.steps, args.warmup, world, rank, device, seed_base=1000 * rank)
        tr = max_over_ranks(rr["total_ms"], world, device)
        lr = max_over_ranks(rr["avg_launch_ms"], world, device)
        tp = max_over_ranks(rr["padded_total_ms"], world, device)
        wr = rr["w"]
        ragged = {"workload": "ragged_t49_196", "value": world * rr["elements"] * args.steps / (tr * 1e-3),
                  "unit": "elems/s", "ms_per_step": tr / args.steps,
                  "samples": wr["S"], "tokens": "T_s uniform on {%d..%d} + 2 aux, %d packed positions per rank"
                  % (wr["T_lo"], wr["T_hi"], rr["elements"] // wr["D"]),
                  "hbm": {"achieved": rr["bytes"] / (lr * 1e-3) / 1e9, "unit": "GB/s"},
                  "alu_frac": (rr["elements"] / (lr * 1e-3)) / alu_peak_elems(wr["N"], wr["K"], 1965.0),
                  "padded_fixed": {"value": world * rr["elements"] * args.steps / (tp * 1e-3), "unit": "elems/s",
                                   "note": "useful elements/s of the fixed-layout forward on the same samples "
                                           "padded to the longest (%d of %d elements useful)"
                                           % (rr["elements"], rr["padded_elements"])}}

    bwd = {}
    if not args.no_extra:
        rb = measure_bwd(args.steps, args.warmup, world, device, seed_base=1000 * rank)
        bms = max_over_ranks(rb["ms"], world, device)
        bwd = {"workload": "chain4_stage3 layer (B=64, D=640, T=196+2, N=16, bf16): sfm_mixer_bwd, all gradients",
               "value": world * rb["elements"] / (bms * 1e-3), "unit": "elems/s", "ms_per_step": bms,
               "hbm": {"achieved": rb["bytes"] / (bms * 1e-3) / 1e9, "unit": "GB/s",
                       "note": "inputs read and fp32 gradients written once; the %.0f MB workspace "
                               "(the forward states the reverse sweep reads back) not counted"
                               % (rb["workspace"] / 1e6)}}

    proj = {}
    if not args.no_extra:
        pr = measure_proj(args.steps, args.warmup, world, device)
        proj = {k: v for k, v in pr.items()}
        for k in ("in_proj", "x_proj_bc", "x_proj_dt", "dt_proj"):
            proj[k]["ms"] = max_over_ranks(proj[k]["ms"], world, device)

    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        hbm_peak, peak_src = float(peaks["hbm_gbs"]), "measured"
    except (OSError, ValueError, KeyError):
        hbm_peak, peak_src = 6650.0, "fallback"
    sm_max = float(peaks.get("sm_max_mhz", 1965.0)) if peaks else 1965.0
    hbm_achieved = res["bytes"] / (launch_ms * 1e-3) / 1e9
    elem_rate = el / (launch_ms * 1e-3)
    alu_peak = alu_peak_elems(w["N"], w["K"], sm_max)
    if extra:
        extra["hbm"].update(peak=hbm_peak, frac=extra["hbm"]["achieved"] / hbm_peak)
    if ragged:
        ragged["hbm"].update(peak=hbm_peak, frac=ragged["hbm"]["achieved"] / hbm_peak)
    cpu = None
    if not args.no_extra and world == 1:
        cpu = cpu_baseline(args.workload, args.cpu_seconds)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "elems/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": args.workload, "B": w["B"], "D": w["D"], "T": w["T"], "L": L, "N": w["N"],
                   "K": w["K"], "io_dtype": w["dtype"], "B1": res["variant"]["B1"],
                   "d_tile": res["variant"]["d_tile"], "chunk": res["variant"]["chunk"],
                   "l2": "inputs rotate over %d sets of %.0f MB (%.0f MB > 2x L2)" % (
                       res["nsets"], res["set_bytes"] / 1e6, res["nsets"] * res["set_bytes"] / 1e6),
                   "parallelism": "dp%d (independent shards)" % world},
        "roofline": {"bound": "alu", "achieved": elem_rate / 1e9, "peak": alu_peak / 1e9, "unit": "Gelem/s",
                     "frac": elem_rate / alu_peak, "traffic": recorded_traffic(args.workload),
                     "peak_basis": "%d MUFU + %d FP32 lanes/clk/SM x %d SMs x %.0f MHz; %d transcendentals and "
                                   "%d fp32 ops per element, a transcendental costing 1 MUFU lane or %d FMA-pipe "
                                   "lane-ops, best split" % ((MUFU_PER_CLK_SM, FP32_PER_CLK_SM, SMS, sm_max)
                                                             + alu_ops_per_element(w["N"], w["K"])
                                                             + (POLY_EXP2_FMA_OPS,)),
                     "peak_mufu_only": mufu_only_peak_elems(w["N"], w["K"], sm_max) / 1e9},
        "hbm": {"achieved": hbm_achieved, "peak": hbm_peak, "unit": "GB/s", "frac": hbm_achieved / hbm_peak,
                "peak_source": peak_src, "algorithmic_bytes_per_launch": res["bytes"]},
        "kernel_ms": launch_ms,
        "e2e": {"value": e2e_value, "unit": "elems/s", "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"],
                "schedule": "two device buffer sets; H2D, kernel and D2H on three streams, so step i+1's "
                            "H2D overlaps step i's kernel and D2H"},
        "gpu_launches": args.steps,  # timed region of the main workload: one kernel per step
        "clocks": ck,
    }
    if extra:
        line["t196"] = extra
    if ragged:
        line["ragged"] = ragged
    if bwd:
        bwd["hbm"].update(peak=hbm_peak, frac=bwd["hbm"]["achieved"] / hbm_peak)
        line["bwd"] = bwd
    if proj:
        bf_peak = float(peaks.get("bf16_tflops", 1590.0)) if peaks else 1590.0
        bf_sus = float(peaks.get("bf16_tflops_sustained", 1400.0)) if peaks else 1400.0
        pj = {"workload": "stage4_t49 projections (tcgen05 GEMMs, bf16 in, fp32 accumulate, bf16 out)",
              "shape": proj["shape"], "peak_tflops": bf_peak, "peak_tflops_sustained": bf_sus,
              "peak_source": "measured" if peaks else "fallback"}
        for k in ("in_proj", "x_proj_bc", "x_proj_dt", "dt_proj"):
            tf = proj[k]["flops"] / (proj[k]["ms"] * 1e-3) / 1e12
            pj[k] = {"ms": proj[k]["ms"], "tflops": tf, "frac": tf / bf_peak}
        line["proj"] = pj
    if cpu:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
