"""Benchmark of the tile-hybrid (dense / 2:4) Wanda-masked linear layer on B200.

One step = one pass of the whole hot path over one batch of synthetic input,
for every weight matrix of the workload, in four phases:
  1. column sums of squares of each distinct calibration set (patch_colsq);
  2. Wanda scores / 2:4 codes / tile loss / tile map per matrix
     (patch_score_mask, reusing the column sums of the matrix's input);
  3. pack per matrix (patch_pack);
  4. hybrid GEMM for every matrix and every token count, largest M first
     (patch_hybrid_gemm).
Default workload: the full Llama-7B-shaped decoder block (q, k, v, o
4096x4096; gate, up 11008x4096; down 4096x11008), 128x128 tiles, Wanda masks
from 128 x 2048 = 262144 calibration tokens per distinct layer input, the 60 %
of tiles with the least pruned-score loss 2:4 (30 % target sparsity), GEMMs at
M in {4096, 512, 64, 8, 1}.

Metric: effective TFLOP/s of the step's hybrid GEMMs = sum over the GEMMs of
2*M*N*K (dense-equivalent) / the device time of the GEMM phase.  Tokens/s per
token count M = M / the time of that M's GEMMs over all the matrices.  The
column-norm, mask and pack phases are timed and reported beside it
(`phases_ms`); `ms_per_step` is the whole step.  Also reported: the roofline
of the kernel with the largest share of device time, isolated GEMM timings
over the 2:4-tile fraction (speedup over the same kernel with an all-dense
map), the decode GEMV in a CUDA graph, the end-to-end time through host
buffers, and the CPU oracle on a bounded sample.

Launch: ``python bench.py [--gpus N --steps K --warmup W]``; for N > 1 under
``torch.distributed.run`` one rank per GPU, each rank running the step on its
own independent matrices (weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_gemm_wanda_b200 import inputs  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# The oracle's bounded sample (CPU baseline and reference arm alike): the
# first 128 rows (one band) of every matrix, the first 16384 tokens of every
# calibration set, every token count.
ORACLE_ROWS = 128
ORACLE_CALIB_TOKENS = 16384


# ----------------------------------------------------------------- utilities
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
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
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        top = max(sm)
        loaded = [s for s in sm if s >= 0.5 * top] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "samples": len(sm), "reasons": sorted(reasons)}


class L2Flusher:
    def __init__(self, nbytes: int = 512 << 20):
        self.buf = torch.empty(nbytes // 4, dtype=torch.int32, device="cuda")

    def __call__(self):
        self.buf.fill_(1)


def max_over_ranks(value: float, device) -> float:
    """The largest value over all ranks (the job's time is its slowest rank's)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


# ----------------------------------------------------------------- workload
def make_tensors(wl, rank: int, device="cpu", rows=None, calib_tokens=None):
    """Synthetic weights, calibration sets and inputs of a workload (per-rank seed).

    Calibration sets and the GEMM inputs X are keyed by input group: layers
    that read the same activations (q/k/v; gate/up) share one calibration set
    (hence one column norm) and one X per token count.
    `rows` / `calib_tokens` cut a bounded sample (the first rows of every
    matrix, the first tokens of every calibration set: the same values as the
    full draw's)."""
    seed = wl.seed + 1009 * rank
    mats = []
    outl = {}
    calib = {}
    group_x = {}
    for mi, m in enumerate(wl.matrices):
        if m.K not in outl:
            outl[m.K] = inputs.outlier_channels(m.K, seed, wl.outlier_count)
        g = m.input_group
        if wl.calib_tokens and g not in calib:
            T = min(wl.calib_tokens, calib_tokens or wl.calib_tokens)
            buf = torch.empty((T, m.K), dtype=torch.bfloat16,
                              pin_memory=device != "cpu" and torch.cuda.is_available())
            inputs.activations_chunked(T, m.K, seed, outl[m.K], role=10 * len(calib), out=buf)
            calib[g] = buf.to(device)
        w = inputs.weight(m.N, m.K, seed + 17 * (mi + 1))
        if rows is not None:
            w = w[:rows].contiguous()
        if g not in group_x:
            gi = len(group_x)
            group_x[g] = {M: inputs.activations(M, m.K, seed, outl[m.K], role=1 + gi * 100 + M).to(device)
                          for M in wl.tokens}
        mats.append({"name": m.name, "N": w.shape[0], "K": m.K, "group": g, "W": w.to(device),
                     "X": group_x[g]})
    return mats, calib


def units_of(wl, mats):
    """(matrix index, 2:4-tile fraction) pairs of one step: every matrix at the
    workload's fraction; a random-map sweep runs every matrix at every fraction."""
    if wl.map_rule == "random":
        return [(mi, f) for mi in range(len(mats)) for f in wl.fractions]
    return [(mi, wl.fractions[0]) for mi in range(len(mats))]


def random_maps(wl, mats, rank, device):
    """Seeded random tile maps of the random-map workloads, one per unit."""
    maps = {}
    if wl.map_rule != "random":
        return maps
    for mi, f in units_of(wl, mats):
        m = wl.matrices[mi]  # the full matrix's tiles, also for a row sample
        nt = (m.N // wl.tile_n) * (m.K // wl.tile_k)
        maps[(mi, f)] = inputs.random_map(nt, inputs.n_sparse_tiles(f, nt),
                                          wl.seed + 1009 * rank + 31 * mi + int(f * 100)).to(device)
    return maps


def gemm_flops(wl, mats):
    return sum(2.0 * M * mats[mi]["N"] * mats[mi]["K"] for mi, _ in units_of(wl, mats) for M in wl.tokens)


class StepEvents:
    """CUDA events at the phase boundaries of one step (on the launching stream)."""

    def __init__(self):
        self.marks = []

    def mark(self, name):
        e = torch.cuda.Event(enable_timing=True)
        e.record(torch.cuda.current_stream())
        self.marks.append((name, e))

    def spans(self):
        """{name: ms} between consecutive marks (a mark's span runs to the next)."""
        out = {}
        for (name, e0), (_, e1) in zip(self.marks, self.marks[1:]):
            out[name] = out.get(name, 0.0) + e0.elapsed_time(e1)
        return out


def run_step(P, wl, mats, calib, maps, ys, ev: StepEvents | None = None, colsq_calls=None):
    """The hot path once for every unit of the workload.

    Phases in order: column sums of squares per calibration set, masks, packs,
    GEMMs (largest token count first, so that the host has queued the short
    decode calls long before the device reaches them).  `ev` gets a mark at
    every phase boundary and before each token count's GEMMs; `colsq_calls`
    collects (event, event, T, K) around each column-norm call."""
    mark = ev.mark if ev is not None else (lambda name: None)
    units = units_of(wl, mats)
    mark("colsq")
    colsq = {}
    if wl.calib_tokens:
        for g, xc in calib.items():
            if colsq_calls is not None:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(torch.cuda.current_stream())
                colsq[g] = P.patch_colsq(xc)
                e1.record(torch.cuda.current_stream())
                colsq_calls.append((e0, e1, xc.shape[0], xc.shape[1]))
            else:
                colsq[g] = P.patch_colsq(xc)
    mark("mask")
    masks = []
    Mmax = max(wl.tokens)
    for mi, f in units:
        m = mats[mi]
        if wl.calib_tokens:
            r = P.patch_score_mask(m["W"], None, tile_n=wl.tile_n, tile_k=wl.tile_k, fraction=f,
                                   colsq_in=colsq[m["group"]])
        else:
            # random-map workloads: 2:4 patterns from Wanda with the input X as calibration
            r = P.patch_score_mask(m["W"], m["X"][Mmax], tile_n=wl.tile_n, tile_k=wl.tile_k,
                                   map_in=maps[(mi, f)])
        masks.append(r)
    mark("pack")
    # up to eight matrices per call: one host wait for each call's layouts
    pks = []
    for b in range(0, len(units), 8):
        chunk = list(zip(units[b:b + 8], masks[b:b + 8]))
        pks += P.patch_pack_group([mats[mi]["W"] for (mi, _), _ in chunk], [r["meta"] for _, r in chunk],
                                  [r["map"] for _, r in chunk], tile_n=wl.tile_n, tile_k=wl.tile_k)
    # matrices that read the same X (one unit per matrix) share one call
    batches = []
    for (mi, f), pk in zip(units, pks):
        g = mats[mi]["group"] if wl.map_rule != "random" else (mi, f)
        if batches and batches[-1][0] == g:
            batches[-1][1].append((mi, f, pk))
        else:
            batches.append((g, [(mi, f, pk)]))
    for M in sorted(wl.tokens, reverse=True):
        mark(f"gemm_m{M}")
        for _, members in batches:
            x = mats[members[0][0]]["X"][M]
            if len(members) == 1:
                mi, f, pk = members[0]
                P.patch_hybrid_gemm(pk, x, out=ys[(mi, f, M)])
            else:
                P.patch_hybrid_gemm_group([pk for _, _, pk in members], x,
                                          outs=[ys[(mi, f, M)] for mi, f, _ in members])
    mark("end")
    return pks


def close_all(pks):
    for pk in pks:
        pk.close()


def traffic_for(kernel_key: str):
    """dram read+write bytes per launch from the committed ncu summary, if the
    kernel's source is unchanged since the capture; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        d = json.load(fh)
    ent = d.get(kernel_key)
    if not ent:
        return None
    src = os.path.join(ROOT, ent["source"])
    if not os.path.exists(src):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if h != ent.get("source_sha256_16"):
        return None
    return ent


def colsq_bytes(T, K):
    """Algorithmic bytes of one column-norm call: the calibration set read once,
    the 128-token chunk partials written and read back, the sums written."""
    chunks = (T + 127) // 128
    return 2.0 * T * K + 2 * 8.0 * chunks * K + 8.0 * K


# ----------------------------------------------------------- isolated GEMMs
def isolated_gemm(P, wl, W, M, frac_map, X, flush, reps=20, seed=0, nm=(2, 4), fp8=False):
    """Time one GEMM configuration with L2 flushed before every call.  The
    N:M patterns (2:4, or 4:8) are Wanda's with X as calibration; the map is
    seeded random."""
    N, K = W.shape
    nt = (N // wl.tile_n) * (K // wl.tile_k)
    tmap = inputs.random_map(nt, inputs.n_sparse_tiles(frac_map, nt), seed).cuda()
    r = P.patch_score_mask(W, X, tile_n=wl.tile_n, tile_k=wl.tile_k, map_in=tmap, nm=nm)
    if fp8:
        pk = P.patch_pack_fp8(W, r["meta"], r["map"], tile_n=wl.tile_n, tile_k=wl.tile_k)
    else:
        pk = P.patch_pack(W, r["meta"], r["map"], tile_n=wl.tile_n, tile_k=wl.tile_k, nm=nm)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    for _ in range(3):
        P.patch_hybrid_gemm(pk, X, out=Y)
    ts = []
    s = torch.cuda.current_stream()
    for _ in range(reps):
        flush()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s)
        P.patch_hybrid_gemm(pk, X, out=Y)
        e1.record(s)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1))
    status = P.patch_get_status(pk)
    nbytes = pk.packed_bytes
    pk.close()
    if status:
        raise RuntimeError(f"GEMM status {status}")
    return statistics.median(ts), nbytes


def graph_gemm(P, wl, W, M, frac_map, X, calls_per_copy=8, replays=5, seed=0):
    """Per-call time of back-to-back GEMMs captured in one CUDA graph.

    The graph cycles through enough independently packed copies of W that
    their bytes exceed three times the L2 size, so every call streams its
    weights from HBM, as in a decode loop over many layers.
    Returns (ms per call, packed bytes of one copy, copies)."""
    N, K = W.shape
    nt = (N // wl.tile_n) * (K // wl.tile_k)
    tmap = inputs.random_map(nt, inputs.n_sparse_tiles(frac_map, nt), seed).cuda()
    r = P.patch_score_mask(W, X, tile_n=wl.tile_n, tile_k=wl.tile_k, map_in=tmap)
    first = P.patch_pack(W, r["meta"], r["map"], tile_n=wl.tile_n, tile_k=wl.tile_k)
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    copies = max(2, -(-3 * l2 // first.packed_bytes))
    pks = [first] + [P.patch_pack(W, r["meta"], r["map"], tile_n=wl.tile_n, tile_k=wl.tile_k)
                     for _ in range(copies - 1)]
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for pk in pks:  # warm-up outside the capture
            P.patch_hybrid_gemm(pk, X, out=Y)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    n_calls = calls_per_copy * copies
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(n_calls):
            P.patch_hybrid_gemm(pks[i % copies], X, out=Y)
    graph.replay()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    ts = []
    for _ in range(replays):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s)
        graph.replay()
        e1.record(s)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1) / n_calls)
    status = [P.patch_get_status(pk) for pk in pks]
    nbytes = first.packed_bytes
    del graph
    for pk in pks:
        pk.close()
    torch.cuda.synchronize()
    if any(status):
        raise RuntimeError(f"GEMM status {status}")
    return statistics.median(ts), nbytes, copies


def prefill_sweep(P, wl_name, flush, peaks):
    """Isolated prefill GEMMs over the 2:4-tile fraction: the Llama-7B MLP shapes
    at M = 2048 (f in {0, .25, .5, .75, 1}) and the 13B MLP shapes at M = 4096
    (f in {0, .75, 1}), each with its speedup over the all-dense map."""
    wls = inputs.workloads()
    dense_peak = float(peaks["bf16_tflops"])
    out = {}
    for name, fracs in (("llama7b-prefill", (0.0, 0.25, 0.5, 0.75, 1.0)),
                        ("llama13b-prefill", (0.0, 0.75, 1.0))):
        w = wls[name]
        M = w.tokens[0]
        for mi, m in enumerate(w.matrices):
            o = inputs.outlier_channels(m.K, w.seed)
            Wd = inputs.weight(m.N, m.K, w.seed + m.N).cuda()
            Xd = inputs.activations(M, m.K, w.seed, o, role=1).cuda()
            ent = {}
            base = None
            for f in fracs:
                t_ms, _ = isolated_gemm(P, w, Wd, M, f, Xd, flush, seed=w.seed + m.N + int(f * 100))
                fl = 2.0 * M * m.N * m.K
                nt = (m.N // 128) * (m.K // 128)
                s_ach = inputs.n_sparse_tiles(f, nt) / nt / 2.0
                eff = fl / (t_ms * 1e-3) / 1e12
                useful = fl * (1 - s_ach) / (t_ms * 1e-3) / 1e12
                if f == 0.0:
                    base = t_ms
                e = {"us": t_ms * 1e3, "sparsity": s_ach, "effective_tflops": eff,
                     "useful_tflops": useful, "speedup_vs_all_dense": base / t_ms,
                     "useful_frac_of_dense_peak": useful / dense_peak}
                if f == 1.0:
                    e["frac_of_sparse_peak"] = eff / (2.0 * dense_peak)
                ent[f"f{f}"] = e
            out[f"{name} M={M} N={m.N} K={m.K}"] = ent
            del Wd, Xd
    return {"by_shape": out, "dense_peak_tflops": dense_peak,
            "note": "effective = 2MNK / t (dense-equivalent); useful = 2MNK(1-s) / t against the "
                    "burst dense peak (a kernel timed alone); sparse peak = 2 x the dense peak; "
                    "seeded random maps, 2:4 patterns from Wanda with X as calibration; L2 "
                    "flushed before every call"}


def nm48_isolated(P, flush, peaks):
    """4:8 tiles (expanded in shared memory for dense MMAs) against 2:4 and the
    all-dense map on the Llama-7B MLP shape, half the tiles sparse, one call
    after an L2 flush: M = 16 (bound by the compressed weight bytes) and
    M = 2048."""
    w = inputs.workloads()["llama7b-prefill"]
    m = w.matrices[0]
    o = inputs.outlier_channels(m.K, w.seed)
    Wd = inputs.weight(m.N, m.K, w.seed + m.N).cuda()
    hbm = float(peaks["hbm_gbs"])
    out = {}
    for M in (16, 2048):
        Xd = inputs.activations(M, m.K, w.seed, o, role=1).cuda()
        ent = {}
        for name, f, nm, fp8 in (("dense", 0.0, (2, 4), False), ("2:4 f=0.5", 0.5, (2, 4), False),
                                 ("4:8 f=0.5", 0.5, (4, 8), False), ("fp8 dense", 0.0, (2, 4), True),
                                 ("fp8 2:4 f=0.5", 0.5, (2, 4), True), ("fp8 2:4 f=1", 1.0, (2, 4), True)):
            # the same map, the same Wanda ranking; only the pattern / precision differs
            t_ms, nb = isolated_gemm(P, w, Wd, M, f, Xd, flush, seed=w.seed + 5, nm=nm, fp8=fp8)
            e = {"us": t_ms * 1e3, "packed_bytes": nb,
                 "effective_tflops": 2.0 * M * m.N * m.K / (t_ms * 1e-3) / 1e12}
            if M <= 16:
                b = nb + 2 * M * (m.N + m.K)
                e["achieved_gbs"] = b / (t_ms * 1e-3) / 1e9
                e["frac_of_hbm"] = e["achieved_gbs"] / hbm
            ent[name] = e
        out[f"M={M} N={m.N} K={m.K}"] = ent
        del Xd
    return {"by_shape": out,
            "note": "4:8 handles run the one-band kernel whose converter warps expand 4:8 k-steps "
                    "into dense tiles in shared memory (no 4:8 tensor-core mode for 16-bit "
                    "inputs); FP8 handles quantise X per token inside the call and run the "
                    "kind::f8f6f4 kernel (its time includes that quantisation); effective TFLOP/s "
                    "count 2MNK; L2 flushed before every call"}


def fp8_block_gemms(P, wl, mats, calib, flush, reps=5):
    """The block's GEMM phase on FP8 handles: the same least-loss masks and maps
    as the bf16 step, W_eff quantised per output row (patch_pack_fp8), every
    token count, q/k/v and gate/up as grouped calls; device time per token
    count (median of `reps` phases, L2 flushed before each), beside the same
    phase on the bf16 handles."""
    units = units_of(wl, mats)
    if wl.map_rule == "random" or not wl.calib_tokens:
        return None
    colsq = {g: P.patch_colsq(xc) for g, xc in calib.items()}
    masks = [P.patch_score_mask(mats[mi]["W"], None, tile_n=wl.tile_n, tile_k=wl.tile_k, fraction=f,
                                colsq_in=colsq[mats[mi]["group"]]) for mi, f in units]
    out = {}
    for kind in ("bf16", "fp8"):
        if kind == "fp8":
            pks = [P.patch_pack_fp8(mats[mi]["W"], r["meta"], r["map"], tile_n=wl.tile_n, tile_k=wl.tile_k)
                   for (mi, _), r in zip(units, masks)]
        else:
            pks = [P.patch_pack(mats[mi]["W"], r["meta"], r["map"], tile_n=wl.tile_n, tile_k=wl.tile_k)
                   for (mi, _), r in zip(units, masks)]
        batches = []
        for (mi, f), pk in zip(units, pks):
            g = mats[mi]["group"]
            if batches and batches[-1][0] == g:
                batches[-1][1].append((mi, pk))
            else:
                batches.append((g, [(mi, pk)]))
        ys = {(mi, M): torch.empty((M, mats[mi]["N"]), dtype=torch.bfloat16, device="cuda")
              for mi, _ in units for M in wl.tokens}
        res = {}
        for M in sorted(wl.tokens, reverse=True):
            def phase():
                for _, members in batches:
                    x = mats[members[0][0]]["X"][M]
                    if len(members) == 1:
                        P.patch_hybrid_gemm(members[0][1], x, out=ys[(members[0][0], M)])
                    else:
                        P.patch_hybrid_gemm_group([pk for _, pk in members], x,
                                                  outs=[ys[(mi, M)] for mi, _ in members])
            phase()
            ts = []
            for _ in range(reps):
                flush()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                phase()
                e1.record()
                e1.synchronize()
                ts.append(e0.elapsed_time(e1))
            t = statistics.median(ts)
            fl = sum(2.0 * M * mats[mi]["N"] * mats[mi]["K"] for mi, _ in units)
            res[f"m{M}"] = {"ms": t, "effective_tflops": fl / (t * 1e-3) / 1e12}
        status = [P.patch_get_status(pk) for pk in pks]
        packed = sum(pk.packed_bytes for pk in pks)
        close_all(pks)
        if any(status):
            raise RuntimeError(f"GEMM status {status}")
        out[kind] = {"by_m": res, "packed_bytes": packed}
    return {**out, "note": "the block's GEMM phase per token count on bf16 and on FP8 (e4m3) handles "
                           "built from the same masks and maps; FP8 calls quantise X per token "
                           "inside the call; L2 flushed before each phase"}


def tile_shapes_isolated(P, flush, peaks):
    """Finer tiles on the Llama-7B MLP shape at M = 2048: 128x128, 128x64,
    64x128 and 64x64 tiles at f in {0, .5, 1} (seeded random maps).  The GEMM
    runs 128-row bands with 64-column k-steps; a band's k-step runs the 2:4
    MMA when every tile it covers is 2:4, so a 64-row tile is fast only where
    its band partner agrees (M = 64 MMAs run at half the M = 128 rate on this
    GPU, so splitting a band is no faster than running it dense)."""
    import types

    import numpy as np
    w = inputs.workloads()["llama7b-prefill"]
    m = w.matrices[0]
    M = w.tokens[0]
    o = inputs.outlier_channels(m.K, w.seed)
    Wd = inputs.weight(m.N, m.K, w.seed + m.N).cuda()
    Xd = inputs.activations(M, m.K, w.seed, o, role=1).cuda()
    fl = 2.0 * M * m.N * m.K
    out = {}
    base = None
    for tn, tk in ((128, 128), (128, 64), (64, 128), (64, 64)):
        shape = types.SimpleNamespace(tile_n=tn, tile_k=tk)
        ent = {}
        for f in (0.0, 0.5, 1.0):
            seed = w.seed + 7 * tn + tk + int(f * 100)
            t_ms, _ = isolated_gemm(P, shape, Wd, M, f, Xd, flush, seed=seed)
            nt = (m.N // tn) * (m.K // tk)
            bits = np.unpackbits(inputs.random_map(nt, inputs.n_sparse_tiles(f, nt), seed).numpy()
                                 .view(np.uint8), bitorder="little")[:nt].reshape(m.N // tn, m.K // tk)
            # 128-row bands x 64-column k-steps that run the 2:4 MMA
            b = bits.repeat(tn // 64, axis=0).repeat(tk // 64, axis=1)
            run_sparse = float((b[0::2] & b[1::2]).mean())
            if base is None:
                base = t_ms
            ent[f"f{f}"] = {"us": t_ms * 1e3, "effective_tflops": fl / (t_ms * 1e-3) / 1e12,
                            "ksteps_run_sparse": run_sparse, "speedup_vs_128x128_dense": base / t_ms}
        out[f"{tn}x{tk}"] = ent
    del Wd, Xd
    return {"shape": f"M={M} N={m.N} K={m.K}", "by_tile": out,
            "note": "seeded random maps; L2 flushed before every call; ksteps_run_sparse = share "
                    "of (128-row band, 64-column k-step) units whose tiles are all 2:4"}


def graph_gemm_group(P, wl, Ws, M, frac_map, X, calls_per_copy=8, replays=5, seed=0):
    """Per-call time of back-to-back grouped calls (patch_hybrid_gemm_group over
    matrices that read the same X) captured in one CUDA graph, cycling through
    enough packed copies of the group that their bytes exceed three times the
    L2 size.  Returns (ms per grouped call, packed bytes of one group copy)."""
    first = []
    masks = []
    for i, W in enumerate(Ws):
        N, K = W.shape
        nt = (N // wl.tile_n) * (K // wl.tile_k)
        tmap = inputs.random_map(nt, inputs.n_sparse_tiles(frac_map, nt), seed + 7 * i).cuda()
        r = P.patch_score_mask(W, X, tile_n=wl.tile_n, tile_k=wl.tile_k, map_in=tmap)
        masks.append(r)
        first.append(P.patch_pack(W, r["meta"], r["map"], tile_n=wl.tile_n, tile_k=wl.tile_k))
    group_bytes = sum(pk.packed_bytes for pk in first)
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    copies = max(2, -(-3 * l2 // group_bytes))
    groups = [first] + [[P.patch_pack(W, r["meta"], r["map"], tile_n=wl.tile_n, tile_k=wl.tile_k)
                         for W, r in zip(Ws, masks)] for _ in range(copies - 1)]
    Ys = [torch.empty((M, W.shape[0]), dtype=torch.bfloat16, device="cuda") for W in Ws]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for g in groups:  # warm-up outside the capture
            P.patch_hybrid_gemm_group(g, X, outs=Ys)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    n_calls = calls_per_copy * copies
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(n_calls):
            P.patch_hybrid_gemm_group(groups[i % copies], X, outs=Ys)
    graph.replay()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    ts = []
    for _ in range(replays):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s)
        graph.replay()
        e1.record(s)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1) / n_calls)
    status = [P.patch_get_status(pk) for g in groups for pk in g]
    del graph
    for g in groups:
        for pk in g:
            pk.close()
    torch.cuda.synchronize()
    if any(status):
        raise RuntimeError(f"GEMM status {status}")
    return statistics.median(ts), group_bytes


def decode_isolated(P, flush, peaks):
    """The decode GEMV on the Llama-7B decode shapes at M in {1, 4, 16}: one
    CUDA graph of back-to-back calls over copies larger than 3x L2, per call;
    and grouped calls over the matrices of the Llama-7B block that read one X
    (q/k/v: 3 x 4096x4096; gate/up: 2 x 11008x4096) at M in {1, 4, 16, 64}."""
    w = inputs.workloads()["llama7b-decode"]
    hbm = float(peaks["hbm_gbs"])
    out = {}
    for label, N, count in (("q/k/v 3x4096x4096", 4096, 3), ("gate/up 2x11008x4096", 11008, 2)):
        K = 4096
        o = inputs.outlier_channels(K, w.seed)
        Ws = [inputs.weight(N, K, w.seed + N + i).cuda() for i in range(count)]
        for M in tuple(w.tokens) + (64,):
            X = inputs.activations(M, K, w.seed, o, role=1 + M).cuda()
            tg_ms, nbytes = graph_gemm_group(P, w, Ws, M, w.fractions[0], X, seed=M)
            b = nbytes + 2 * M * K + 2 * M * N * count
            out[f"group {label} m{M}"] = {"us_graph": tg_ms * 1e3, "compressed_bytes": b,
                                          "achieved_gbs": b / (tg_ms * 1e-3) / 1e9,
                                          "frac_of_hbm": b / (tg_ms * 1e-3) / 1e9 / hbm}
        del Ws
    for mi, m in enumerate(w.matrices):
        o = inputs.outlier_channels(m.K, w.seed)
        Wd = inputs.weight(m.N, m.K, w.seed + m.N).cuda()
        for M in w.tokens:
            X = inputs.activations(M, m.K, w.seed, o, role=1 + M).cuda()
            tg_ms, nbytes, copies = graph_gemm(P, w, Wd, M, w.fractions[0], X, seed=M)
            b = nbytes + 2 * M * m.K + 2 * M * m.N
            out[f"{m.N}x{m.K} m{M}"] = {"us_graph": tg_ms * 1e3, "compressed_bytes": b,
                                        "achieved_gbs": b / (tg_ms * 1e-3) / 1e9,
                                        "frac_of_hbm": b / (tg_ms * 1e-3) / 1e9 / hbm}
        del Wd
    return {"by_shape": out, "map": "seeded random, half the tiles 2:4 (2:4 patterns from Wanda "
                                     "with X as calibration)",
            "timing": "one CUDA graph of back-to-back calls cycling through packed copies larger "
                      "than 3x L2, per call (a grouped call counts once)",
            "bytes": "packed weight bytes (values + metadata) + X + Y (of every matrix of a group)"}


# -------------------------------------------------------------- CPU oracle
def oracle_sample(wl, reps=1):
    """The oracle as it stands on the bounded sample (ORACLE_ROWS rows of every
    matrix, ORACLE_CALIB_TOKENS tokens of every calibration set, every token
    count), every step of the path.  Returns (seconds of the GEMMs, GEMM flops,
    seconds of everything, description)."""
    import numpy as np
    import oracle
    mats, calib = make_tensors(wl, 0, rows=ORACLE_ROWS, calib_tokens=ORACLE_CALIB_TOKENS)
    maps = random_maps(wl, mats, 0, "cpu")

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    t_all = time.perf_counter()
    t_gemm = 0.0
    flops = 0.0
    Mmax = max(wl.tokens)
    for _ in range(reps):
        colsq = {g: oracle.colsq(bits(x)) for g, x in calib.items()}
        for mi, f in units_of(wl, mats):
            m = mats[mi]
            w = bits(m["W"])
            if wl.calib_tokens:
                s = colsq[m["group"]]
            else:
                s = oracle.colsq(bits(m["X"][Mmax]))
            sc = oracle.wanda_scores(w, s)
            meta = oracle.select_2of4(sc)
            loss = oracle.tile_loss(sc, meta, wl.tile_n, wl.tile_k)
            if wl.map_rule == "random":
                # the sample's rows are the first tile row: its tiles keep
                # their types from the full matrix's map (tiles 0 .. K/tk - 1)
                full = maps[(mi, f)].numpy().view(np.uint32)
                nt = loss.shape[0]
                tmap = np.zeros((nt + 31) // 32, dtype=np.uint32)
                for t in range(nt):
                    if (int(full[t // 32]) >> (t % 32)) & 1:
                        tmap[t // 32] |= np.uint32(1 << (t % 32))
            else:
                tmap = oracle.select_map(loss, oracle.n_sparse(f, loss.shape[0]))
            oracle.pack(w, meta, tmap, wl.tile_n, wl.tile_k)
            weff = oracle.weff(w, meta, tmap, wl.tile_n, wl.tile_k)
            for M in wl.tokens:
                t0 = time.perf_counter()
                oracle.gemm(bits(m["X"][M]), weff)
                t_gemm += time.perf_counter() - t0
                flops += 2.0 * M * m["N"] * m["K"]
    secs = time.perf_counter() - t_all
    desc = (f"first {ORACLE_ROWS} rows of every matrix"
            + (f", first {ORACLE_CALIB_TOKENS} tokens of every calibration set" if wl.calib_tokens
               else "") + f", M in {wl.tokens}, every step (column norms, scores, codes, tile "
            f"loss, map, pack, W_eff, GEMM); value = sample GEMM flops / GEMM seconds")
    return t_gemm, flops, secs, desc


def config_of(wl, world):
    return {"workload": wl.name,
            "matrices": [f"{m.name} {m.N}x{m.K}" for m in wl.matrices],
            "tiles": f"{wl.tile_n}x{wl.tile_k}",
            "fractions_2to4_tiles": wl.fractions,
            "map": "least Wanda tile loss" if wl.map_rule == "loss" else "seeded random",
            "calibration_tokens_per_input": wl.calib_tokens, "tokens": wl.tokens,
            "l2": "flushed (512 MB write) before every timed step, outside its events; the "
                  "calibration sets (2.1-5.8 GB) exceed L2",
            "parallelism": f"independent matrices per rank x{world}"}


METRIC = ("hybrid-sparse GEMM effective TFLOP/s (dense-equivalent 2*M*N*K over the device time "
          "of the step's hybrid GEMMs) & tokens/s, vs sparsity; %roofline")


# --------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama7b-block")
    ap.add_argument("--no-extras", action="store_true", help="skip isolated GEMM / oracle legs")
    ap.add_argument("--case", choices=["gemm", "mask", "pack", "colsq"], default=None,
                    help="run one operation a few times and exit (profiling aid, no JSON)")
    ap.add_argument("--N", type=int, default=11008)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--M", type=int, default=2048)
    ap.add_argument("--T", type=int, default=2048)
    ap.add_argument("--frac", type=float, default=0.5)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--fp8", action="store_true", help="--case gemm: FP8 (e4m3) values in the tiles")
    ap.add_argument("--group", type=int, default=1,
                    help="--case gemm: this many [N, K] matrices reading one X, one grouped call")
    ap.add_argument("--force-kernel", type=int, default=0,
                    help="--case gemm: prefill kernel (library test hook; 0 = the library's choice)")
    args = ap.parse_args()
    if args.case:
        return run_case(args)
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    wl = inputs.workloads()[args.workload]

    if args.impl == "reference":
        return main_reference(args, wl, world, rank)

    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))

    from sparse_gemm_wanda_b200 import patch as P
    P.load_library()

    mats, calib = make_tensors(wl, rank, device="cuda")
    maps = random_maps(wl, mats, rank, "cuda")
    units = units_of(wl, mats)
    ys = {(mi, f, M): torch.empty((M, mats[mi]["N"]), dtype=torch.bfloat16, device="cuda")
          for mi, f in units for M in wl.tokens}
    flops = gemm_flops(wl, mats)
    flush = L2Flusher()
    s = torch.cuda.current_stream()

    for _ in range(args.warmup):
        close_all(run_step(P, wl, mats, calib, maps, ys))
    torch.cuda.synchronize()

    # ------------------------------------------------------------ timed steps
    clocks = ClockSampler(torch.cuda.current_device())
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    steps = []
    colsq_calls = []
    launches0 = P.launch_count()
    for _ in range(args.steps):
        flush()  # between timed steps, outside the events
        ev = StepEvents()
        close_all(run_step(P, wl, mats, calib, maps, ys, ev=ev, colsq_calls=colsq_calls))
        steps.append(ev)
    launches = P.launch_count() - launches0
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()

    spans = [ev.spans() for ev in steps]
    step_ms = [sum(sp.values()) for sp in spans]
    total_ms = max_over_ranks(sum(step_ms), "cuda")
    ms_per_step = total_ms / args.steps
    phase = {k: statistics.fmean(sp[k] for sp in spans) for k in spans[0]}
    gemm_keys = [k for k in phase if k.startswith("gemm_m")]
    gemm_ms = max_over_ranks(sum(phase[k] for k in gemm_keys), "cuda")
    value = flops * world / (gemm_ms * 1e-3) / 1e12
    n_mats = len(units)
    by_m = {}
    for M in wl.tokens:
        t = max_over_ranks(phase[f"gemm_m{M}"], "cuda")
        fl = sum(2.0 * M * mats[mi]["N"] * mats[mi]["K"] for mi, _ in units)
        by_m[f"m{M}"] = {"ms": t, "tokens_per_s": M * world / (t * 1e-3),
                         "effective_tflops": fl * world / (t * 1e-3) / 1e12,
                         "gemms": n_mats}
    tokens_per_s = sum(wl.tokens) * world / (gemm_ms * 1e-3)
    phases_max = {k: max_over_ranks(v, "cuda") for k, v in phase.items()}  # every rank takes part

    peaks, peak_kind = load_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    dense_burst = float(peaks["bf16_tflops"])

    # ---------------------------------------------------- rooflines
    rooflines = {}
    if colsq_calls:
        tot_ms = sum(e0.elapsed_time(e1) for e0, e1, _, _ in colsq_calls)
        tot_b = sum(colsq_bytes(T, K) for _, _, T, K in colsq_calls)
        n = len(colsq_calls)
        ach = tot_b / (tot_ms * 1e-3) / 1e9
        tr = traffic_for("colsq")
        traffic = None
        if tr:
            # captured on a smaller calibration set: scaled by the tokens per call
            tok = statistics.fmean(T for _, _, T, _ in colsq_calls)
            kk = statistics.fmean(T * K for _, _, T, K in colsq_calls) / tok
            traffic = tr["bytes_per_token_column"] * tok * kk
        rooflines["colsq"] = {
            "bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s",
            "frac": ach / hbm_peak, "traffic": traffic,
            "kernel": "colsq_partial_kernel (+ colsq_final_kernel, the in-order fold)",
            "algorithmic_bytes_per_launch": tot_b / n, "launch_us": tot_ms / n * 1e3,
            "share_of_step": phase["colsq"] / ms_per_step,
            "timing": "CUDA events around every patch_colsq call of the timed steps",
            "bytes": "2*T*K calibration read + 16*K*ceil(T/128) chunk partials written and "
                     "re-read + 8*K sums",
            "peak_source": peak_kind}
    big = max(M for M in wl.tokens)
    if big > 16:
        units_fl = sum(2.0 * big * mats[mi]["N"] * mats[mi]["K"] * (1 - f / 2) for mi, f in units)
        t = phase[f"gemm_m{big}"]
        ach = units_fl / (t * 1e-3) / 1e12
        rooflines["gemm_prefill"] = {
            "bound": "tensor", "achieved": ach, "peak": dense_burst, "unit": "TFLOP/s",
            "frac": ach / dense_burst, "traffic": None,
            "kernel": f"hybrid GEMM at M = {big} (two-SM / band-pair kernels)",
            "share_of_step": t / ms_per_step,
            "flops": "useful 2*M*N*K*(1 - f/2) over the step's GEMMs at this M",
            "peak_note": "burst bf16 dense peak (tcgen05 dense and sparse MMAs together)",
            "peak_source": peak_kind}
    dominant = max(rooflines, key=lambda k: rooflines[k]["share_of_step"]) if rooflines else None
    roof = rooflines.get(dominant)

    # ------------------------------------------------------- end to end
    e2e = None
    if not args.no_extras or world > 1:
        gx = {}
        for m in mats:  # one X per input group and token count
            gx.setdefault(m["group"], m["X"])
        host = {"W": [m["W"].cpu().pin_memory() for m in mats],
                "X": {g: {M: x.cpu().pin_memory() for M, x in xs.items()} for g, xs in gx.items()},
                "C": {g: c.cpu().pin_memory() for g, c in calib.items()}}
        h2d = sum(t.numel() * 2 for t in host["W"]) + sum(c.numel() * 2 for c in host["C"].values()) \
            + sum(x.numel() * 2 for d in host["X"].values() for x in d.values())
        hy = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in ys.items()}
        d2h = sum(v.numel() * 2 for v in ys.values())
        e2e_ms = []
        n_e2e = min(args.steps, 5)
        for it in range(args.warmup + n_e2e):
            flush()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(s)
            dx = {g: {M: x.to("cuda", non_blocking=True) for M, x in xs.items()}
                  for g, xs in host["X"].items()}
            dm = [{"name": m["name"], "N": m["N"], "K": m["K"], "group": m["group"],
                   "W": host["W"][mi].to("cuda", non_blocking=True), "X": dx[m["group"]]}
                  for mi, m in enumerate(mats)]
            dc = {g: c.to("cuda", non_blocking=True) for g, c in host["C"].items()}
            close_all(run_step(P, wl, dm, dc, maps, ys))
            for k, v in ys.items():
                hy[k].copy_(v, non_blocking=True)
            e1.record(s)
            e1.synchronize()
            del dm, dc, dx
            if it >= args.warmup:
                e2e_ms.append(e0.elapsed_time(e1))
        e_ms = max_over_ranks(statistics.fmean(e2e_ms), "cuda")
        e2e = {"value": flops * world / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "note": "the step's GEMM flops over the whole end-to-end step: host->device copies "
                       "of W, calibration sets and X from pinned memory, every phase, and the "
                       "device->host copy of every Y, through the binding's public calls"}
        del host, hy

    # --------------------------------------------- isolated measurements
    extras = {}
    # one GPU only: under torchrun the other ranks would wait for rank 0 at the
    # closing barrier for as long as these take
    if not args.no_extras and rank == 0 and world == 1:
        extras["prefill_gemm_isolated"] = prefill_sweep(P, wl.name, flush, peaks)
        extras["decode_gemm_isolated"] = decode_isolated(P, flush, peaks)
        extras["pattern_precision_isolated"] = nm48_isolated(P, flush, peaks)
        extras["tile_shapes_isolated"] = tile_shapes_isolated(P, flush, peaks)
        fb = fp8_block_gemms(P, wl, mats, calib, flush)
        if fb is not None:
            extras["block_gemms_fp8_vs_bf16"] = fb

    cpu = None
    if rank == 0 and world == 1 and not args.no_extras:
        t_gemm, fl, secs, desc = oracle_sample(wl)
        cpu = {"value": fl / t_gemm / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(),
               "kind": "oracle", "sample": f"{desc}; {secs:.1f} s in all, {t_gemm:.1f} s GEMMs"}

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": value,
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_per_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded Llama-shaped weights N(0,0.02); activations N(0,1) with "
                    "1% outlier channels x20)",
            "config": config_of(wl, world),
            "gemm_ms_per_step": gemm_ms,
            "phases_ms": phases_max,
            "tokens_per_s": tokens_per_s,
            "by_m": by_m,
            "e2e": e2e,
            "gpu_launches": launches,
            "roofline": roof,
            "rooflines": rooflines,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        line.update(extras)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_case(args):
    """One operation on seeded inputs, `reps` times (for profiler captures)."""
    from sparse_gemm_wanda_b200 import patch as P
    torch.cuda.set_device(0)
    P.load_library()
    g = torch.Generator().manual_seed(4242)
    if args.case == "colsq":
        Xcal = torch.randn(args.T, args.K, generator=g).to(torch.bfloat16).cuda()
        for _ in range(args.reps):
            P.patch_colsq(Xcal)
        torch.cuda.synchronize()
        print(f"case colsq T={args.T} K={args.K} ok")
        return
    W = (torch.randn(args.N, args.K, generator=g) * 0.02).to(torch.bfloat16).cuda()
    X = torch.randn(args.M, args.K, generator=g).to(torch.bfloat16).cuda()
    Xcal = torch.randn(args.T, args.K, generator=g).to(torch.bfloat16).cuda()
    nt = (args.N // 128) * (args.K // 128)
    tmap = inputs.random_map(nt, int(round(args.frac * nt)), 7).cuda()
    if args.case == "mask":
        for _ in range(args.reps):
            P.patch_score_mask(W, Xcal, fraction=args.frac)
    else:
        r = P.patch_score_mask(W, Xcal, map_in=tmap)
        if args.case == "pack":
            for _ in range(args.reps):
                P.patch_pack(W, r["meta"], r["map"]).close()
        else:
            pack = P.patch_pack_fp8 if args.fp8 else P.patch_pack
            pks = [pack(W, r["meta"], r["map"])]
            for i in range(1, args.group):
                Wi = (torch.randn(args.N, args.K, generator=g) * 0.02).to(torch.bfloat16).cuda()
                ri = P.patch_score_mask(Wi, Xcal, map_in=inputs.random_map(nt, int(round(args.frac * nt)), 7 + i).cuda())
                pks.append(pack(Wi, ri["meta"], ri["map"]))
            P.test_prefill_kernel(args.force_kernel)
            for _ in range(args.reps):
                if args.group > 1:
                    P.patch_hybrid_gemm_group(pks, X)
                else:
                    P.patch_hybrid_gemm(pks[0], X)
            torch.cuda.synchronize()
            for pk in pks:
                assert P.patch_get_status(pk) == 0
                pk.close()
    torch.cuda.synchronize()
    print(f"case {args.case} N={args.N} K={args.K} M={args.M} frac={args.frac}{' fp8' if args.fp8 else ''}"
          f"{f' group={args.group}' if args.group > 1 else ''} ok")


def main_reference(args, wl, world, rank):
    """The oracle as it stands on the host cores, on the bounded sample, per step."""
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(wl)
    tot_g, tot_f, tot_s = 0.0, 0.0, 0.0
    desc = ""
    for _ in range(args.steps):
        t_gemm, fl, secs, desc = oracle_sample(wl)
        tot_g += t_gemm
        tot_f += fl
        tot_s += secs
    v = tot_f / tot_g / 1e12
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": v, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Llama-shaped weights N(0,0.02); activations N(0,1) with "
                "1% outlier channels x20)",
        "config": config_of(wl, world),
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
