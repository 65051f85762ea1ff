"""Builds the adaptive-B1 look-up table from a sweep on the GPU it runs on.

    python -m selective_scan_sfm_b200.lut_sweep [--quick] [--write] [--json out.json]

For every shape of the grid (T, B, D, N) it times the fused forward for each candidate
launch shape -- B2 samples per folded row (B1 = B / B2), channels per CTA, tokens staged
per step -- and keeps the fastest.  --write rewrites csrc/sfm_lut.inc (rebuild libsfm
afterwards).  Timing: CUDA events around repeated launches on rotating input sets whose
total exceeds twice the L2, median of the repeats.  The full table of timings (the
folded-versus-unfolded comparison included) goes to --json.
"""
from __future__ import annotations

import argparse
import ctypes
import itertools
import json
import math
import os

import torch

from . import _abi, _scan_args, synth

L2_BYTES = 126 * 1024 * 1024
PKG = os.path.dirname(os.path.abspath(__file__))
LUT = os.path.join(PKG, "csrc", "sfm_lut.inc")

# (T, B, D, N): the shapes the table is keyed on -- stage-3/4 token counts of MambaVision
# at 224^2 and their neighbours, the batch sizes of training and inference, and widths
GRID_FULL = ([(49, B, D, 16) for B in (16, 64, 128, 256, 512) for D in (640, 1280)] +
             [(196, B, D, 16) for B in (8, 32, 64, 128, 256) for D in (320, 640)] +
             [(784, B, D, 16) for B in (4, 16, 32) for D in (160, 320)] +
             [(49, 4, 16, 8)])
GRID_QUICK = [(49, 256, 1280, 16), (196, 128, 640, 16), (784, 16, 320, 16), (196, 64, 640, 16), (49, 4, 16, 8)]


def divisors_upto(B, cap):
    return [v for v in (1, 2, 4, 8, 16, 32) if v <= cap and B % v == 0]


LANE_TOKENS = 16  # tokens per lane per chunk in the library's lanes mode


def candidates(B, T, D, N=16):
    """(B2, d_tile, chunk, lanes, chans_per_thread): one thread per channel or two side by
    side (lanes = 1) with whole-sample or chunked staging, and, for longer samples, P lanes
    per channel (chunk = 16 P: each lane scans 16 tokens of a chunk)."""
    L = T + 2
    out = []
    tiles = [t for t in (32, 64, 128) if t <= max(32, ((D + 31) // 32) * 32)]
    chunks = sorted(set([c for c in (16, 24, 32, 56, 64, 128) if c < L] + [((L + 7) // 8) * 8 if L <= 256 else 0]) - {0})
    cpts = (1, 2) if (8 < N <= 16 and D % 2 == 0) else (1,)
    for B2, dt, ch, cpt in itertools.product(divisors_upto(B, 32), tiles, chunks, cpts):
        if cpt == 2 and B2 > 4:
            continue
        out.append((B2, dt, ch, 1, cpt))
    if L >= 100:
        for B2, P, threads in itertools.product(divisors_upto(B, 4), (2, 4, 8, 16, 32), (64, 128, 256)):
            if threads // P >= 1 and LANE_TOKENS * P <= 4 * L:
                out.append((B2, threads // P, LANE_TOKENS * P, P, 1))
    return out


def time_variant(sets, lib, stream, B2, d_tile, chunk, reps, exp2_split=0, lanes=1, cpt=1):
    args = []
    for s in sets:
        a = s["args"]
        a.B1, a.d_tile, a.chunk, a.exp2_split, a.lanes = s["B"] // B2, d_tile, chunk, exp2_split, lanes
        a.chans_per_thread = cpt
        args.append(ctypes.byref(a))
    sp = ctypes.c_void_p(stream.cuda_stream)
    for i in range(3):
        if lib.sfm_selective_scan_fold(args[i % len(args)], sp) != 0:
            return None
    torch.cuda.synchronize()
    times = []
    for r in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        lib.sfm_selective_scan_fold(args[r % len(args)], sp)
        e1.record(stream)
        times.append((e0, e1))
    torch.cuda.synchronize()
    ms = sorted(a.elapsed_time(b) for a, b in times)
    return ms[len(ms) // 2]


def sweep(grid, reps=15, log=print):
    lib = _abi.lib()
    stream = torch.cuda.current_stream()
    results = []
    for (T, B, D, N) in grid:
        dtype = "f32" if N == 8 and D == 16 else "bf16"
        w = dict(B=B, D=D, T=T, N=N, K=4, dtype=dtype)
        esz = 2 if dtype == "bf16" else 4
        set_bytes = B * D * (3 * (T + 2) + T) * esz
        nsets = max(2, min(6, math.ceil(2 * L2_BYTES / max(set_bytes, 1)) + 1))
        sets = []
        for i in range(nsets):
            d = synth.make_inputs(**w, seed=100 + i)
            dc = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
            y = torch.empty(B, D, T + 2, dtype=dc["dt"].dtype, device="cuda")
            a, _ = _scan_args(dc["x"], dc["dt"], dc["Bm"], dc["Cm"], dc["A"], dc["z"], dc["Dskip"], dc["dt_bias"],
                              dc["conv_w"], dc["conv_b"], y, None, 0, None, True, True, False, None, 0, 0, 0)
            sets.append(dict(args=a, keep=(dc, y), B=B))
        rows = []
        split0 = 3 if N == 16 else 1  # stage 1 at two FMA-pipe exp2 pairs (N = 16)
        for (B2, dtile, ch, P, cpt) in candidates(B, T, D, N):
            ms = time_variant(sets, lib, stream, B2, dtile, ch, reps, split0, P, cpt)
            if ms is None:
                continue
            rows.append(dict(B2=B2, d_tile=dtile, chunk=ch, lanes=P, cpt=cpt, exp2_pairs=split0 - 1, ms=ms,
                             gelem_s=B * D * (T + 2) / ms / 1e6))
        rows.sort(key=lambda r: r["ms"])
        if N == 16 and rows[0]["lanes"] == 1:  # stage 2: the exp2 split for the best launch shape
            b0 = rows[0]
            for split in (1, 2, 4):
                ms = time_variant(sets, lib, stream, b0["B2"], b0["d_tile"], b0["chunk"], reps, split, 1, b0["cpt"])
                if ms is not None:
                    rows.append(dict(b0, exp2_pairs=split - 1, ms=ms, gelem_s=B * D * (T + 2) / ms / 1e6))
            rows.sort(key=lambda r: r["ms"])
        best = rows[0]
        unfolded = min((r for r in rows if r["B2"] == 1), key=lambda r: r["ms"])
        res = dict(T=T, B=B, D=D, N=N, dtype=dtype, best=best, best_unfolded=unfolded, all=rows)
        results.append(res)
        log("T=%4d B=%4d D=%5d N=%2d best B2=%2d lanes=%2d cpt=%d d_tile=%3d chunk=%3d exp2_pairs=%d %.4f ms "
            "(%.1f Gelem/s); best unfolded %.4f ms -> folding speedup %.3f" % (
                T, B, D, N, best["B2"], best["lanes"], best["cpt"], best["d_tile"], best["chunk"], best["exp2_pairs"],
                best["ms"], best["gelem_s"], unfolded["ms"], unfolded["ms"] / best["ms"]))
        del sets
        torch.cuda.empty_cache()
    return results


def write_lut(results, path=LUT, gpu=None):
    gpu = gpu or results[0].get("gpu") or torch.cuda.get_device_name()
    lines = ["// sfm_lut.inc -- adaptive-B1 look-up table: launch choices measured on B200.",
             "// Written by selective_scan_sfm_b200/lut_sweep.py from a sweep over B, T, D and N on %s;" % gpu,
             "// each row is the fastest measured variant for that shape.",
             "// Columns: T, B, D, N, B2, lanes, d_tile, chunk, exp2_pairs, chans_per_thread."]
    for r in results:
        b = r["best"]
        lines.append("{%d, %d, %d, %d, %d, %d, %d, %d, %d, %d}," % (
            r["T"], r["B"], r["D"], r["N"], b["B2"], b["lanes"], b["d_tile"], b["chunk"], b["exp2_pairs"],
            b.get("cpt", 1)))
    open(path, "w").write("\n".join(lines) + "\n")


def merge(base, newer):
    """The rows of `base` with those of the same (T, B, D, N) replaced by `newer`'s, in base order."""
    key = lambda r: (r["T"], r["B"], r["D"], r["N"])
    fresh = {key(r): r for r in newer}
    out = [fresh.pop(key(r), r) for r in base]
    return out + list(fresh.values())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--quick", action="store_true")
    ap.add_argument("--write", action="store_true")
    ap.add_argument("--json", default=None)
    ap.add_argument("--reps", type=int, default=15)
    ap.add_argument("--from-json", default=None, help="rewrite the table from a saved sweep (no GPU needed)")
    ap.add_argument("--T", type=int, default=None, help="sweep only the shapes of this patch-token count")
    ap.add_argument("--merge", default=None,
                    help="a saved full sweep whose rows for the swept shapes are replaced before writing")
    a = ap.parse_args()
    if a.from_json:
        rows = json.load(open(a.from_json))
        if a.merge:
            rows = merge(json.load(open(a.merge)), rows)
        write_lut(rows)
        return
    grid = GRID_QUICK if a.quick else GRID_FULL
    if a.T is not None:
        grid = [g for g in grid if g[0] == a.T]
    res = sweep(grid, reps=a.reps)
    for r in res:
        r["gpu"] = torch.cuda.get_device_name()
    if a.json:
        json.dump(res, open(a.json, "w"), indent=1)
    if a.write:
        write_lut(merge(json.load(open(a.merge)), res) if a.merge else res)


if __name__ == "__main__":
    main()
