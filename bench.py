"""Benchmark of the PATCH hybrid tile-sparse linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload WORKLOAD]
                    [--impl ours|reference]

Default workload ("all"): one JSON line whose `value` is the decode step and
whose blocks time every configuration of the layer this library targets:

* decode (the headline `value`): the 7 LLaMA-2-7B linear layers (q/k/v/o
  4096x4096, gate/up 11008x4096, down 4096x11008), 50% of the 128x128 tiles
  2:4 sparse (exact count, seeded positions), magnitude-top-2 patterns, at
  M = 1, 4 and 16 tokens.  One step = the 21 independent GEMMs over packed
  weights resident in HBM, as one patch_gemm_chain launch (the value; the
  block also times them as 21 separate patch_gemm calls and as a chain of
  calls that wait for each other); the metric is HBM GB/s counting only the
  bytes the layer must move: stored weight bytes (dense tiles 32 KiB, sparse
  tiles 16 KiB values + 2 KiB metadata, 16 B descriptor per tile) + X + Y.
* "prefill": the same 7 shapes at M = 2048, sparse-tile fraction swept over
  {0, 0.25, 0.5, 0.75, 1}; dense-equivalent TFLOP/s (2*M*N*K / time), the
  mixed roofline (dense tiles at the dense peak, sparse tiles at r times it),
  the speedup of every fraction over the same shape packed all-dense, and
  whether throughput rises monotonically with the fraction; the same 35 GEMMs
  also as 5 patch_gemm_group launches (one per fraction).
* "stack": the 32-layer LLaMA-2-7B linear stack (7 projections per layer, 224
  distinct weights, ~9 GB), run sequentially at M = 1 and at M = 8, with the
  non-uniform per-layer sparse-tile fractions (0.1 / 0.7, +0.1 for the MLP);
  GB/s over stored bytes and milliseconds per pass over the stack.
* "llama3_qwen": LLaMA-3-8B and Qwen-2.5-0.5B linears with spatially
  clustered sparse tiles (50%), at M = 1 (GB/s; also as one patch_gemm_chain)
  and M = 512 (TFLOP/s; also as one patch_gemm_group).
* "mma_probe": the dense and 2:4-sparse tensor-core MMA rates (M = 128, 64).
Other workloads: decode_fused (q|k|v and gate|up as one GEMM each),
tile_ablation (mask tile sizes 4..128).  A workload run alone (--workload)
prints its own line; one timed per token count reports its smallest.

Prints one JSON line (rank 0).  --impl reference times the CPU oracle (plain
C, fp64) on a bounded sample of the decode workload on the host cores.
"""
from __future__ import annotations

import argparse
import functools
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

import synth_inputs as si  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
DECODE_MS = (1, 4, 16)
PREFILL_M = 2048
STACK_MS = (1, 8)
LQ_MS = (1, 512)
FRACS = (0.0, 0.25, 0.5, 0.75, 1.0)
DECODE_CONFIG = 2   # seeds of the decode workload
PREFILL_CONFIG = 3  # seeds of the prefill workload
STACK_CONFIG = 4    # seeds of the 32-layer stack
LQ_CONFIG = 5       # seeds of the LLaMA-3-8B / Qwen-2.5-0.5B workload
STACK_LAYERS = 32
BLOCKS = ("decode", "prefill", "stack", "llama3_qwen")  # the default run, in this order


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def measured_traffic(kind, names):
    """DRAM bytes per launch (read + write) of the dominant kernel, from the ncu
    capture summarised in profiles/dram_traffic.json: the mean over this step's
    calls.  None when there is no capture for every call, or when the kernel's
    source has changed since the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(kind)
    if not rec:
        return None
    with open(os.path.join(ROOT, rec["source"]), "rb") as f:
        if hashlib.sha1(f.read()).hexdigest() != rec["sha1"]:
            return None
    per = rec["bytes_per_call"]
    if not all(n in per for n in names):
        return None
    return float(np.mean([per[n] for n in names]))


def stored_bytes(N, K, n_sparse):
    T = (N // 128) * (K // 128)
    return (T - n_sparse) * 32768 + n_sparse * (16384 + 2048) + 16 * T


# ------------------------------------------------------------ clocks


class ClockSampler:
    """nvidia-smi samples (every 20 ms) of the SM clock and throttle reasons.

    The timed region may be shorter than the sampling period, so the summary
    uses the samples from 0.25 s before the region starts (the warm-up, at the
    same load) until it ends."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.samples = []  # (host time, line)
        self.marks = {}

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.monotonic(), line.strip()))

    def wait_first_sample(self, timeout=3.0):
        t0 = time.monotonic()
        while self.proc and not self.samples and time.monotonic() - t0 < timeout:
            time.sleep(0.01)

    def mark(self, name):
        self.marks[name] = time.monotonic()

    def __exit__(self, *exc):
        time.sleep(0.05)
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        t0 = self.marks.get("start", 0.0) - 0.25
        t1 = self.marks.get("end", float("inf")) + 0.03
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, ln in self.samples:
            if not (t0 <= ts <= t1):
                continue
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 6:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, v in zip(names, parts[2:6]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "window": "0.25 s before the timed region to its end"}


# ------------------------------------------------------------ workloads


def is_decode(workload):
    return workload in ("decode", "decode_fused", "stack")


def build_layers(workload, only=None, fracs=None, tokens=None):
    """Inputs of every layer in the workload: list of dicts with the shape, the
    tile bitmap, the sparse-tile fraction, X per token count and either the
    host weight bits and pattern ids ("w", "ids") or the seeds from which the
    weight is drawn on the device ("gen": the 32-layer stack, ~13 GB of bf16
    weights, too large to draw on the host).  `only`, `fracs` and `tokens`
    select a subset (profiling runs); the default is the whole workload."""
    layers = []
    if workload == "decode_fused":
        # q|k|v and gate|up as single GEMMs over row-concatenated weights (the
        # usual fused projections; tiles stay whole), o and down alone; the same
        # weights, tile choices and patterns as the "decode" workload
        ms = tuple(tokens) if tokens else DECODE_MS
        members = {}
        for i, (name, N, K) in enumerate(si.LLAMA2_7B):
            w = si.gen_w(N, K, DECODE_CONFIG, i)
            f = fracs[0] if fracs else 0.5
            members[name] = (i, w, si.tiles_exact(N, K, f, DECODE_CONFIG, i), si.patterns_top2(w), f)
        for name, parts in (("qkv", ("q", "k", "v")), ("o", ("o",)), ("gate_up", ("gate", "up")), ("down", ("down",))):
            if only and name not in only:
                continue
            i0, _, _, _, f = members[parts[0]]
            w = np.concatenate([members[m][1] for m in parts])
            bm = np.concatenate([members[m][2] for m in parts])
            ids = np.concatenate([members[m][3] for m in parts])
            N, K = w.shape
            layers.append(dict(name=name, N=N, K=K, w=w, bm=bm, ids=ids, frac=f,
                               xs={M: si.gen_x(M, K, DECODE_CONFIG, i0) for M in ms}))
    elif workload == "decode":
        ms = tuple(tokens) if tokens else DECODE_MS
        for i, (name, N, K) in enumerate(si.LLAMA2_7B):
            if only and name not in only:
                continue
            w = si.gen_w(N, K, DECODE_CONFIG, i)
            f = fracs[0] if fracs else 0.5
            bm = si.tiles_exact(N, K, f, DECODE_CONFIG, i)
            layers.append(dict(name=name, N=N, K=K, w=w, bm=bm, ids=si.patterns_top2(w), frac=f,
                               xs={M: si.gen_x(M, K, DECODE_CONFIG, i) for M in ms}))
    elif workload == "prefill":
        ms = tuple(tokens) if tokens else (PREFILL_M,)
        for i, (name, N, K) in enumerate(si.LLAMA2_7B):
            if only and name not in only:
                continue
            w = si.gen_w(N, K, PREFILL_CONFIG, i)
            ids = si.patterns_top2(w)
            xs = {M: si.gen_x(M, K, PREFILL_CONFIG, i) for M in ms}
            for f in (fracs or FRACS):
                bm = si.tiles_exact(N, K, f, PREFILL_CONFIG, i)
                layers.append(dict(name=name, N=N, K=K, w=w, bm=bm, ids=ids, frac=f, xs=xs))
    elif workload == "stack":
        ms = tuple(tokens) if tokens else STACK_MS
        for layer in range(STACK_LAYERS):
            for i, (name, N, K) in enumerate(si.LLAMA2_7B):
                if only and name not in only:
                    continue
                idx = 7 * layer + i
                f = si.stack_fraction(layer, name)
                layers.append(dict(name=f"L{layer}.{name}", proj=name, N=N, K=K, gen=(STACK_CONFIG, idx),
                                   bm=si.tiles_exact(N, K, f, STACK_CONFIG, idx), frac=f,
                                   xs={M: si.gen_x(M, K, STACK_CONFIG, idx) for M in ms}))
    elif workload == "llama3_qwen":
        ms = tuple(tokens) if tokens else LQ_MS
        for family, shapes, base in (("llama3", si.LLAMA3_8B, 0), ("qwen", si.QWEN25_05B, 7)):
            for j, (name, N, K) in enumerate(shapes):
                if only and name not in only:
                    continue
                idx = base + j
                w = si.gen_w(N, K, LQ_CONFIG, idx)
                layers.append(dict(name=f"{family}.{name}", N=N, K=K, w=w,
                                   bm=si.tiles_clustered(N, K, 0.5, LQ_CONFIG, idx), ids=si.patterns_top2(w),
                                   frac=0.5, xs={M: si.gen_x(M, K, LQ_CONFIG, idx) for M in ms}))
    else:
        raise ValueError(workload)
    return layers


def calls_of(layers, ms=None):
    """(layer index, M) for every GEMM of one step, in order: for each token
    count, every layer in order (the stack runs all 224 layers at M = 1, then
    all at M = 8)."""
    all_ms = sorted({m for L in layers for m in L["xs"]})
    return [(li, M) for M in all_ms if ms is None or M in ms for li, L in enumerate(layers) if M in L["xs"]]


def shard_layers(layers, rank, world, shard_rows):
    """Column-parallel shard of every layer for `rank` of `world` ranks: its
    contiguous tile rows (shard_rows(bitmap, world): balanced by stored bytes)
    of W, the bitmap and the pattern ids.  Each shard keeps the layer's X; its
    Y is the layer's Y columns [128 b, 128 e)."""
    out = []
    for L in layers:
        b, e = shard_rows(L["bm"], world)[rank]
        S = dict(L, N=(e - b) * 128, bm=L["bm"][b:e], full_N=L["N"], rows=(b, e))
        if "w" in L:
            S.update(w=L["w"][b * 128:e * 128], ids=L["ids"][b * 128:e * 128])
        out.append(S)
    return out


def gather_layout(layers, calls, world, shard_rows):
    """Where each rank's Y shards sit in the buffer that one all-gather moves:
    rank r's Y of call j (M_j x 128 (e - b) bf16) at offset[r][j] elements of
    its segment; every rank's segment is padded to the largest, `seg`."""
    sizes = [[0] * len(calls) for _ in range(world)]
    offset = [[0] * len(calls) for _ in range(world)]
    for r in range(world):
        o = 0
        for j, (li, M) in enumerate(calls):
            b, e = shard_rows(layers[li]["bm"], world)[r]
            offset[r][j], sizes[r][j] = o, M * (e - b) * 128
            o += sizes[r][j]
    seg = max(sum(s_) for s_ in sizes)
    return offset, sizes, seg


def call_bytes(L, M):
    return stored_bytes(L["N"], L["K"], int(L["bm"].sum())) + 2 * M * L["K"] + 2 * M * L["N"]


def call_flops(L, M):
    return 2.0 * M * L["N"] * L["K"]


def call_alg_flops(L, M):
    """FLOPs the tensor cores do: a dense tile 2*M*128*128, a sparse tile half
    of it (its MMAs multiply only the kept half of W)."""
    T = (L["N"] // 128) * (L["K"] // 128)
    ns = int(L["bm"].sum())
    return 2.0 * M * 128 * (128 * (T - ns) + 64 * ns)


def roof_seconds(L, M, P_tflops, ratio):
    """Mixed roofline time of one prefill GEMM: dense tiles at the dense peak P,
    sparse tiles (half the MMA work) at ratio x P."""
    T = (L["N"] // 128) * (L["K"] // 128)
    ns = int(L["bm"].sum())
    return 2.0 * M * 128 * 128 * ((T - ns) / P_tflops + ns / (ratio * P_tflops)) / 1e12


# ------------------------------------------------------------ CPU oracle


def cpu_baseline(workload, budget_s=15.0, min_s=0.0, one_thread=True):
    """Time the CPU oracle on a bounded sample of the workload (same metric):
    passes over the step's calls until `min_s` seconds are spent, stopping
    within a pass once `budget_s` is reached; with `one_thread`, also the same
    oracle on one thread over the sample's first calls.  Prefill calls are
    sampled to 16 of their 2048 token rows."""
    import oracle
    layers = build_layers(workload)
    done_units, spent, what, passes = 0.0, 0.0, [], 0
    sample_rows = (lambda M: np.arange(0, M, M // 16)[:16]) if workload == "prefill" else (lambda M: None)
    while True:
        passes += 1
        for li, M in calls_of(layers):
            L = layers[li]
            x = L["xs"][M]
            t0 = time.perf_counter()
            oracle.hybrid_gemm(x, L["w"], L["bm"], L["ids"], rows=sample_rows(M))
            dt = time.perf_counter() - t0
            spent += dt
            if is_decode(workload):
                done_units += call_bytes(L, M) / 1e9
                if passes == 1:
                    what.append(f"{L['name']}@M={M}")
            else:
                done_units += call_flops(L, 16) / 1e12
                if passes == 1:
                    what.append(f"{L['name']}/f={L['frac']}@16rows")
            if spent >= budget_s:
                break
        if spent >= budget_s or spent >= min_s:
            break
    # the same oracle on one thread, over the first calls of the sample (about a second)
    cores = oracle.num_threads()
    one_units, one_spent = 0.0, 0.0
    oracle.set_num_threads(1)
    try:
        for li, M in (calls_of(layers)[:4] if one_thread else []):
            L = layers[li]
            t0 = time.perf_counter()
            oracle.hybrid_gemm(L["xs"][M], L["w"], L["bm"], L["ids"], rows=sample_rows(M))
            one_spent += time.perf_counter() - t0
            one_units += (call_bytes(L, M) / 1e9) if is_decode(workload) else (call_flops(L, 16) / 1e12)
            if one_spent >= 2.0:
                break
    finally:
        oracle.set_num_threads(cores)
    cpu_model = None
    try:
        with open("/proc/cpuinfo") as f:
            cpu_model = next((ln.split(":", 1)[1].strip() for ln in f if ln.startswith("model name")), None)
    except OSError:
        pass
    return {"value": done_units / spent, "unit": "GB/s" if is_decode(workload) else "TFLOP/s",
            "cores": cores, "kind": "oracle", "seconds": round(spent, 3), "passes": passes,
            "one_thread_value": round(one_units / one_spent, 6) if one_spent > 0 else None, "cpu_model": cpu_model,
            "sample": ("decode GEMMs " if is_decode(workload) else "prefill GEMMs, 16 of 2048 token rows each: ")
            + ", ".join(what[:8]) + (" ..." if len(what) > 8 else "") + f" ({len(what)} calls per pass)"}


# ------------------------------------------------------------ offline steps


def offline_steps(layers, dev, pk, reps=5):
    """HBM throughput of the once-per-model steps on the step's layers: the hard
    mask (argmax of tile and pattern logits, masked W), the packer, and the
    fused path (tile kinds, then a pack that takes the pattern argmax itself)."""
    import torch

    import tile_sparse_gemm_b200 as tsg

    out = {}
    status = tsg.new_status(dev)
    mask_bytes = pack_bytes = fused_bytes = soft_bytes = 0
    mask_ms = pack_ms = fused_ms = soft_ms = 0.0
    for i, L in enumerate(layers):
        N, K = L["N"], L["K"]
        w = torch.from_numpy(L["w"].view(np.int16)).view(torch.bfloat16).to(dev)
        tl = torch.from_numpy(si.gen_tile_logits(N, K, DECODE_CONFIG, i)).to(dev)
        pl = torch.from_numpy(si.gen_pattern_logits(N, K, DECODE_CONFIG, i)).to(dev)
        bm = torch.from_numpy(L["bm"]).to(dev)
        ids = torch.from_numpy(L["ids"]).to(dev)
        ns = int(L["bm"].sum())
        for _ in range(2):
            tsg.patch_hard_mask(w, tl, pl, status=status)
            tsg.patch_pack(w, bm, ids, ns, status=status)
        fbm, fns = tsg.patch_tile_kinds(tl)
        fns = int(fns.item())
        tsg.patch_pack_from_logits(w, fbm, pl, fns, status=status)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        torch.cuda.synchronize()
        e[0].record()
        for _ in range(reps):
            tsg.patch_hard_mask(w, tl, pl, status=status)
        e[1].record()
        for _ in range(reps):
            tsg.patch_pack(w, bm, ids, ns, status=status)
        e[2].record()
        for _ in range(reps):  # fused: tile kinds, then pack with the pattern argmax inside
            tsg.patch_tile_kinds(tl)
            tsg.patch_pack_from_logits(w, fbm, pl, fns, status=status)
        e[3].record()
        # training-time soft mask with noise inputs and the mask output (the noise
        # tensors' contents do not change the work: the logits stand in for them)
        tsg.patch_soft_mask(w, tl, pl, 0.5, tl, pl)  # warm-up (allocates its outputs)
        e4, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e4.record()
        for _ in range(reps):
            tsg.patch_soft_mask(w, tl, pl, 0.5, tl, pl)
        e5.record()
        torch.cuda.synchronize()
        soft_ms += e4.elapsed_time(e5) / reps
        soft_bytes += N * K * (2 + 6 + 6 + 2 + 4) + (N // 128) * (K // 128) * 16
        mask_ms += e[0].elapsed_time(e[1]) / reps
        pack_ms += e[1].elapsed_time(e[2]) / reps
        fused_ms += e[2].elapsed_time(e[3]) / reps
        T = (N // 128) * (K // 128)
        # reads W, the tile logits and the pattern logits of sparse tiles; writes the bitmap and the blobs
        fused_bytes += 2 * N * K + 8 * T + 6 * fns * 128 * 128 + T + stored_bytes(N, K, fns)
        mask_bytes += N * K * (2 + 6 + 2) + N * K // 4 + (N // 128) * (K // 128) * 9
        # reads W (dense tiles whole, sparse tiles whole 16 B rows) + ids of sparse tiles + bitmap; writes the blobs
        pack_bytes += 2 * N * K + ns * 128 * 32 + (N // 128) * (K // 128) + stored_bytes(N, K, ns)
        del w, tl, pl, bm, ids
    code, bits = tsg.patch_read_status(status)
    if code != 0:
        raise RuntimeError(f"offline steps: device status {code} bits {bits}")
    for name, b, ms in (("hard_mask", mask_bytes, mask_ms), ("pack", pack_bytes, pack_ms),
                        ("tile_kinds+pack_from_logits", fused_bytes, fused_ms),
                        ("soft_mask (training forward)", soft_bytes, soft_ms)):
        gbs = b / 1e9 / (ms / 1e3)
        out[name] = {"GB/s": round(gbs, 1), "frac": round(gbs / pk["hbm_gbs"], 4), "ms_total": round(ms, 3),
                     "bytes": int(b), "note": "7 LLaMA-2-7B layers, mean of %d calls each (eager launches)" % reps}
    return out


# ------------------------------------------------------------ gated MLP


def mlp_steps(dev, pk, reps=10):
    """The gated MLP's first half H = silu(X Wg^T) * (X Wu^T) on LLaMA-2-7B's
    gate and up (11008 x 4096, 50% sparse tiles): one fused launch against two
    separate GEMMs, at M = 2048 (prefill) and M = 16 (decode)."""
    import torch

    import tile_sparse_gemm_b200 as tsg

    status = tsg.new_status(dev)
    packed = []
    for i in (4, 5):  # gate, up
        name, N, K = si.LLAMA2_7B[i]
        w = si.gen_w(N, K, PREFILL_CONFIG, i)
        bm = si.tiles_exact(N, K, 0.5, PREFILL_CONFIG, i)
        packed.append(tsg.patch_pack(torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).to(dev),
                                     torch.from_numpy(bm).to(dev), torch.from_numpy(si.patterns_top2(w)).to(dev),
                                     int(bm.sum()), status=status))
    g, u = packed
    out = {}
    for M in (PREFILL_M, 16):
        x = torch.from_numpy(si.gen_x(M, g.K, PREFILL_CONFIG, 4).view(np.int16)).view(torch.bfloat16).to(dev)
        h = torch.empty((M, g.N), dtype=torch.bfloat16, device=dev)
        y1, y2 = torch.empty_like(h), torch.empty_like(h)
        ws = torch.zeros(max(tsg.patch_gemm_workspace_size(M, g), 16), dtype=torch.uint8, device=dev)
        import ctypes
        b = ctypes.c_size_t()
        sg, su = g.struct(), u.struct()
        tsg.lib().patch_gemm_mlp_workspace_size(M, ctypes.byref(sg), ctypes.byref(su), ctypes.byref(b))
        wsm = torch.zeros(max(b.value, 16), dtype=torch.uint8, device=dev)

        def fused():
            tsg.patch_gemm_mlp(x, g, u, H=h, workspace=wsm, status=status)

        def separate():
            tsg.patch_gemm(x, g, Y=y1, workspace=ws, status=status)
            tsg.patch_gemm(x, u, Y=y2, workspace=ws, status=status)

        res = {}
        for name, fn in (("fused", fused), ("two_gemms", separate)):
            for _ in range(3):
                fn()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record()
            for _ in range(reps):
                fn()
            e1.record()
            torch.cuda.synchronize()
            res[name] = e0.elapsed_time(e1) / reps * 1e3  # us
        flops = 2 * 2.0 * M * g.N * g.K
        out[f"M={M}"] = {"fused_us": round(res["fused"], 1), "two_gemms_us": round(res["two_gemms"], 1),
                         "fused_TFLOP/s": round(flops / (res["fused"] * 1e-6) / 1e12, 1),
                         "note": "fused = one prefill launch with silu(gate)*up in the epilogue" if M > 16
                         else "fused = two decode GEMMs + one elementwise launch"}
    code, bits = tsg.patch_read_status(status)
    if code != 0:
        raise RuntimeError(f"gated MLP: device status {code} bits {bits}")
    return out


# ------------------------------------------------------------ GPU arm


def tile_ablation(args):
    """Tile-size ablation ("Ablation Studies", tile size: performance holds
    across learned tile sizes down to 4 x 4, while hardware efficiency needs
    128 x 128 execution tiles).  For each mask tile b and layout (b x b tiles
    sparse at seeded random positions, or as one band of tile rows), half of
    the mask tiles sparse, the product path runs at both execution-tile sizes:
    patch_hard_mask_tiles -> patch_exec_tiles (128 x 128) -> patch_pack of
    W_masked -> patch_gemm, and for b <= 64 patch_exec_tiles64 ->
    patch_pack64 -> patch_gemm64 (64 x 64 execution tiles, M = 64 MMAs).
    Each is timed at M = 1 (decode) and M = 2048 (prefill) against the same
    layer packed all-dense in the 128 x 128 format (and, for the 64 x 64 rows,
    also in its own format).  Weights rotate over copies that exceed L2."""
    import torch

    import tile_sparse_gemm_b200 as tsg
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    status = tsg.new_status(dev)
    shapes = [(n, N, K) for n, N, K in si.LLAMA2_7B if n in ("q", "gate")]
    sizes = [128, 64, 32, 16, 8, 4]
    l2_bytes = 126e6

    def copies_of(pw):
        n = max(2, int(np.ceil(3 * l2_bytes / pw.stored_bytes)))
        return [pw] + [type(pw)(pw.N, pw.K, pw.n_sparse, pw.values.clone(), pw.meta.clone(), pw.desc.clone())
                       for _ in range(n - 1)]

    def time_us(packs, M, reps):
        K, N = packs[0].K, packs[0].N
        is64 = isinstance(packs[0], tsg.PackedWeight64)
        gemm = tsg.patch_gemm64 if is64 else tsg.patch_gemm
        need = (tsg.patch_gemm64_workspace_size if is64 else tsg.patch_gemm_workspace_size)(M, packs[0])
        x = torch.randn(M, K, device=dev).to(torch.bfloat16)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        ws = torch.zeros(max(need, 16), dtype=torch.uint8, device=dev)
        for i in range(len(packs)):
            gemm(x, packs[i], Y=y, workspace=ws, status=status)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for r in range(reps):
            gemm(x, packs[r % len(packs)], Y=y, workspace=ws, status=status)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e3 / reps

    def paired(packs, dense_packs, M, reps, rounds=5):
        """Medians over alternating rounds of (this layer, the all-dense layer)."""
        a, d = [], []
        for _ in range(rounds):
            d.append(time_us(dense_packs, M, reps))
            a.append(time_us(packs, M, reps))
        return statistics.median(a), statistics.median(d)

    runs = (("decode", 1, 2000), ("prefill", 2048, 200))
    rows = []
    warm = torch.empty(2**28, dtype=torch.uint8, device=dev)
    t_end = time.time() + 1.0
    while time.time() < t_end:  # bring the clocks up before the first timing
        warm.add_(1)
        torch.cuda.synchronize()
    del warm
    for idx, (name, N, K) in enumerate(shapes):
        w_np = si.gen_w(N, K, 2, idx)
        ids = si.patterns_top2(w_np)
        pl_np = np.zeros((N, K // 4, 6), np.float32)
        np.put_along_axis(pl_np, ids[..., None].astype(np.int64), 1.0, axis=2)  # magnitude top-2 as logits
        w = torch.from_numpy(w_np.view(np.int16)).view(torch.bfloat16).to(dev)
        pl = torch.from_numpy(pl_np).to(dev)
        del pl_np
        pid_dev = torch.from_numpy(ids).to(dev)
        dense = tsg.patch_pack(w, torch.zeros((N // 128, K // 128), dtype=torch.uint8, device=dev), pid_dev, 0,
                               status=status)
        dense_packs = copies_of(dense)
        dense_bytes = dense.stored_bytes
        dense64_packs = copies_of(tsg.patch_pack64(w, torch.zeros((N // 64, K // 64), dtype=torch.uint8,
                                                                   device=dev), pid_dev, 0, status=status))
        base_all = {"decode": [], "prefill": []}
        base64 = {kind: paired(dense64_packs, dense_packs, M, reps)[0] for kind, M, reps in runs}
        for clustered in (False, True):
            for b in sizes:
                kinds = si.mask_tiles(N, K, b, 0.5, clustered, 2, idx)
                tl = torch.from_numpy(si.choice_logits(kinds)).to(dev)
                wm, bm, pid = tsg.patch_hard_mask_tiles(w, tl, pl, b, status=status)
                layouts = [(128, tsg.patch_exec_tiles, tsg.patch_pack)]
                if b <= 64:
                    layouts.append((64, tsg.patch_exec_tiles64, tsg.patch_pack64))
                for E, exec_fn, pack_fn in layouts:
                    ex, n_dev = exec_fn(bm, N, K, b)
                    pw = pack_fn(wm, ex, pid, int(n_dev.item()), status=status)
                    packs = copies_of(pw)
                    t, base = {}, {}
                    for kind, M, reps in runs:
                        t[kind], base[kind] = paired(packs, dense_packs, M, reps)
                        base_all[kind].append(base[kind])
                    row = {"shape": f"{name} {N}x{K}", "mask_tile": b, "exec_tile": E,
                           "layout": "band of tile rows" if clustered else "random",
                           "sparse_mask_tiles": 0.5,
                           "sparse_exec_tiles": round(pw.n_sparse / ((N // E) * (K // E)), 4),
                           "stored_vs_dense": round(pw.stored_bytes / dense_bytes, 4),
                           "decode_us": round(t["decode"], 2),
                           "decode_GBps": round(pw.stored_bytes / t["decode"] / 1e3, 1),
                           "decode_speedup": round(base["decode"] / t["decode"], 3),
                           "prefill_us": round(t["prefill"], 2),
                           "prefill_speedup": round(base["prefill"] / t["prefill"], 3)}
                    if E == 64:  # against the all-dense layer in the 64 x 64 format itself
                        row["decode_speedup_vs_dense64"] = round(base64["decode"] / t["decode"], 3)
                        row["prefill_speedup_vs_dense64"] = round(base64["prefill"] / t["prefill"], 3)
                    rows.append(row)
                    del packs, pw
                del wm
        del dense_packs, dense64_packs
        rows.append({"shape": f"{name} {N}x{K}", "mask_tile": None, "exec_tile": 128, "layout": "all dense",
                     "decode_us": round(statistics.median(base_all["decode"]), 2),
                     "prefill_us": round(statistics.median(base_all["prefill"]), 2)})
        rows.append({"shape": f"{name} {N}x{K}", "mask_tile": None, "exec_tile": 64, "layout": "all dense",
                     "decode_us": round(base64["decode"], 2), "prefill_us": round(base64["prefill"], 2)})
    code, bits = tsg.patch_read_status(status)
    if code != 0:
        raise RuntimeError(f"device status {code} bits {bits}")
    return {"metric": "tile-size ablation: speedup over the all-dense bitmap", "value": None, "unit": "x",
            "n_gpus": 1, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "LLaMA-2-7B q and gate, mask tiles 128..4, half of them sparse, "
                                   "128 x 128 and (b <= 64) 64 x 64 execution tiles",
                       "l2": "weights rotate over copies holding 3x L2", "decode_M": 1, "prefill_M": 2048,
                       "timing": "median of 5 rounds, each timing the all-dense 128 x 128 layer then this one"},
            "mma_probe": mma_rates(dev),
            "rows": rows}


def mma_rates(dev, iters=20000, rounds=3):
    """Tensor-core MMA rate probe (patch_mma_probe_m): dense and 2:4-sparse
    rounds of M = 128 and M = 64, N = 240 MMAs on shared-memory operands, one
    CTA per SM, alternated `rounds` times; the best of each, in
    dense-equivalent TFLOP/s, and their ratios: sparse over dense is the
    sparse half of the prefill path's mixed roofline, M = 64 over M = 128 the
    hardware side of the tile-size trade-off (64 x 64 execution tiles run the
    M = 64 forms)."""
    import torch

    import tile_sparse_gemm_b200 as tsg
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    status = tsg.new_status(dev)
    forms = [(m, sparse) for m in (128, 64) for sparse in (False, True)]
    best = {f: 0.0 for f in forms}
    for m, sparse in forms:  # warm-up (clocks up, code loaded)
        tsg.patch_mma_probe_m(m, sparse, iters // 4, status)
    torch.cuda.synchronize()
    for _ in range(rounds):
        for m, sparse in forms:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            tsg.patch_mma_probe_m(m, sparse, iters, status)
            e1.record()
            torch.cuda.synchronize()
            flops = sms * iters * 4 * 2 * m * 240 * (32 if sparse else 16)
            best[(m, sparse)] = max(best[(m, sparse)], flops / (e0.elapsed_time(e1) * 1e-3) / 1e12)
    code, bits = tsg.patch_read_status(status)
    if code != 0:
        raise RuntimeError(f"mma probe: device status {code} bits {bits}")
    d, sp = best[(128, False)], best[(128, True)]
    d64, sp64 = best[(64, False)], best[(64, True)]
    return {"dense_tflops": round(d, 1), "sparse_tflops": round(sp, 1),
            "sparse_over_dense": round(sp / d, 3),
            "m64": {"dense_tflops": round(d64, 1), "sparse_tflops": round(sp64, 1),
                    "dense_over_m128": round(d64 / d, 3), "sparse_over_m128": round(sp64 / sp, 3)},
            "how": f"patch_mma_probe_m: {sms} CTAs, {iters} rounds of four M=128 (or M=64) N=240 MMAs each "
                   "(dense K=16, sparse K=32 dense-equivalent) on shared-memory operands, best of %d alternating "
                   "runs" % rounds}


def job_times(ms, e2e_ms, world, dev=None):
    """Timed-region and end-to-end times (ms) of the whole job: the maximum over
    ranks, since the job ends when its slowest rank does."""
    if world > 1:
        import torch
        import torch.distributed as dist
        t = torch.tensor([ms, e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms, e2e_ms = float(t[0]), float(t[1])
    return ms, e2e_ms


def job_throughput(per_step_units, steps, world, ms):
    """Whole-job throughput of `world` replicas that each process per_step_units
    per step (weak scaling): all ranks' units over the job's time."""
    return per_step_units * steps * world / (ms / 1e3)


# ------------------------------------------------------------ GPU arm: timed blocks


def pack_layers(layers, dev, status):
    """Pack every layer on the device (weights drawn there for "gen" layers)."""
    import torch

    import tile_sparse_gemm_b200 as tsg
    packed = []
    for L in layers:
        bm = torch.from_numpy(L["bm"]).to(dev)
        if "gen" in L:
            w = si.gen_w_device(L["N"], L["K"], *L["gen"], device=dev)
            ids = si.patterns_top2_torch(w)
        else:
            w = torch.from_numpy(L["w"].view(np.int16)).view(torch.bfloat16).to(dev)
            ids = torch.from_numpy(L["ids"]).to(dev)
        packed.append(tsg.patch_pack(w, bm, ids, int(L["bm"].sum()), status=status))
        del w, ids, bm
    code, bits = tsg.patch_read_status(status)
    if code != 0:
        raise RuntimeError(f"pack: device status {code} bits {bits}")
    return packed


def time_calls(args, layers, packed, calls, dev, world, status, segments=None, chain=False, after=True,
               gather=None, group=False):
    """Device time of K steps of `calls` (each a patch_gemm), and the same steps
    end to end with host buffers.

    The K timed steps are captured once as one CUDA graph (launch-bound small
    kernels); one replay is the timed region, bracketed by a barrier and a
    synchronize, with the SM clock sampled meanwhile.  A second graph of the
    same steps with an (external) event pair around each segment of the step
    (every call, or the ranges in `segments`) gives the split of the step;
    event nodes add a few microseconds each, so it is not used for totals.
    With `chain`, a step is one patch_gemm_chain per segment over the same
    calls; with `after` every call waits for the previous one's completion
    before reading its X (the ordering of separate calls on one stream),
    without it the calls run as the independent GEMMs they are (each X is an
    input of the step, not an earlier call's output).  With `group` (and
    `chain`), a step is one patch_gemm_group per segment instead: the
    independent GEMMs in one launch of the prefill kernel.
    With `gather` (column-parallel shards, one per rank), every step ends with
    one NCCL all-gather of all ranks' Y shards (padded to `gather` elements
    each), and the steps run eagerly (no graph).
    Returns ms (timed region), e2e_ms, seg_ms [K][segments], clocks, bytes moved
    by the end-to-end copies, and the launch count."""
    import torch
    import torch.distributed as dist

    import tile_sparse_gemm_b200 as tsg
    if segments is None:
        segments = [(0, len(calls))] if chain else [(j, j + 1) for j in range(len(calls))]
    # every call's X (and Y) is a view into one device buffer, so that the
    # end-to-end run moves a step's inputs and results with one copy each way
    x_sizes = [M * layers[li]["K"] for li, M in calls]
    y_sizes = [M * layers[li]["N"] for li, M in calls]
    x_all = torch.empty(sum(x_sizes), dtype=torch.bfloat16, device=dev)
    y_all = torch.empty(max(sum(y_sizes), gather or 0), dtype=torch.bfloat16, device=dev)
    gathered = torch.empty(world * gather, dtype=torch.bfloat16, device=dev) if gather else None
    x_sets, y_sets = [x_all, torch.empty_like(x_all)], [y_all, torch.empty_like(y_all)]
    views = []
    for bset in range(2):
        xv, yv, xo, yo = [], [], 0, 0
        for (li, M), xn, yn in zip(calls, x_sizes, y_sizes):  # sizes are multiples of 128: 16-byte aligned views
            xv.append(x_sets[bset][xo:xo + xn].view(M, layers[li]["K"]))
            yv.append(y_sets[bset][yo:yo + yn].view(M, layers[li]["N"]))
            xo += xn
            yo += yn
        views.append((xv, yv))
    for j, (li, M) in enumerate(calls):
        views[0][0][j].copy_(torch.from_numpy(layers[li]["xs"][M].view(np.int16)).view(torch.bfloat16))
    ws_bytes = max(tsg.patch_gemm_workspace_size(M, packed[li]) for li, M in calls)
    chains = None
    if chain and group:  # per buffer set, one group launch per segment
        chains = [{(lo, hi): tsg.Group([(views[b][0][j], packed[calls[j][0]], views[b][1][j])
                                        for j in range(lo, hi)], status) for lo, hi in segments} for b in range(2)]
    elif chain:  # per buffer set, one chain per segment; every call waits for the previous one
        chains = [{(lo, hi): tsg.Chain([(views[b][0][j], packed[calls[j][0]], views[b][1][j], after)
                                        for j in range(lo, hi)]) for lo, hi in segments} for b in range(2)]
        ws_bytes = max([ws_bytes] + [ch.workspace_bytes for ch in chains[0].values()])
    ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=dev)  # zero-filled once, left zeroed by each call
    if chain and not group:
        for per_set in chains:
            for ch in per_set.values():
                ch.workspace, ch.status = ws, status
    stream = torch.cuda.current_stream()

    def run_calls(bset, lo=0, hi=None):
        if gather and hi is None and lo == 0:
            run_calls(bset, 0, len(calls))
            dist.all_gather_into_tensor(gathered, y_sets[bset][:gather])
            return
        if chain:
            for (a, b), ch in chains[bset].items():
                if a >= lo and (hi is None or b <= hi):
                    ch.run()
            return
        xv, yv = views[bset]
        for j in range(lo, len(calls) if hi is None else hi):
            li, M = calls[j]
            tsg.patch_gemm(xv[j], packed[li], Y=yv[j], workspace=ws, status=status)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        run_calls(0)
    torch.cuda.synchronize()
    code, bits = tsg.patch_read_status(status)
    if code != 0:
        raise RuntimeError(f"device status {code} bits {bits} after warm-up")

    def capture(with_events):
        g = torch.cuda.CUDAGraph()
        evs = [[(torch.cuda.Event(enable_timing=True, external=True),
                 torch.cuda.Event(enable_timing=True, external=True)) for _ in segments]
               for _ in range(args.steps)] if with_events else None
        with torch.cuda.graph(g):
            cap = torch.cuda.current_stream()
            for st in range(args.steps):
                if evs:
                    for s, (lo, hi) in enumerate(segments):
                        evs[st][s][0].record(cap)
                        run_calls(0, lo, hi)
                        evs[st][s][1].record(cap)
                else:
                    run_calls(0)
        g.replay()  # untimed: the first replay uploads the graph
        torch.cuda.synchronize()
        return g, evs

    graph = None if (args.no_graph or gather) else capture(False)[0]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clocks:
        clocks.wait_first_sample()
        barrier()
        torch.cuda.synchronize()
        clocks.mark("start")
        t_start.record(stream)
        if graph is not None:
            graph.replay()
        else:
            for _ in range(args.steps):
                run_calls(0)
        t_end.record(stream)
        torch.cuda.synchronize()
        clocks.mark("end")
        barrier()
    ms = t_start.elapsed_time(t_end)
    del graph
    seg_ms = None
    if not (args.no_graph or gather):
        g_ev, ev = capture(True)
        g_ev.replay()
        torch.cuda.synchronize()
        try:
            seg_ms = np.array([[a.elapsed_time(b) for a, b in ev[st]] for st in range(args.steps)])
        except RuntimeError:
            seg_ms = None
        del g_ev
    code, bits = tsg.patch_read_status(status)
    if code != 0:
        raise RuntimeError(f"device status {code} bits {bits} after timing")

    # End to end through the public API with host buffers.  Every step copies its
    # inputs host -> device from pinned memory (one copy) and its results
    # device -> host (one copy).  Two device buffer sets make a three-stage
    # pipeline: while step s computes on set s%2, step s+1's inputs arrive in the
    # other set and step s-1's results leave it, on two copy streams.  One stage
    # (copy in, compute, copy out, joined) is one CUDA graph per set parity.  The
    # timed region runs from before step 0's input copy to after step K-1's
    # result copy; it carries K+1 copies each way for K steps (the first stage's
    # result copy and the last stage's input copy are surplus).
    x_host = x_all.cpu().pin_memory()
    y_host = [torch.empty(y_all.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = x_host.numel() * 2
    d2h = y_host[0].numel() * 2
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def stage(p):
        cur = torch.cuda.current_stream()
        q = 1 - p
        s_in.wait_stream(cur)
        s_out.wait_stream(cur)
        with torch.cuda.stream(s_in):
            x_sets[q].copy_(x_host, non_blocking=True)  # inputs of the next step
        with torch.cuda.stream(s_out):
            y_host[q].copy_(y_sets[q], non_blocking=True)  # results of the previous step
        run_calls(p)
        cur.wait_stream(s_in)
        cur.wait_stream(s_out)

    stage_graphs = None
    if not (args.no_graph or gather):
        stage_graphs = []
        for p in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                stage(p)
            stage_graphs.append(g)

    def run_e2e(n):
        x_sets[0].copy_(x_host, non_blocking=True)
        for st in range(n):
            if stage_graphs is not None:
                stage_graphs[st % 2].replay()
            else:
                stage(st % 2)
        y_host[(n - 1) % 2].copy_(y_sets[(n - 1) % 2], non_blocking=True)

    run_e2e(max(2, args.warmup))
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run_e2e(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    del stage_graphs
    e2e_ms = e0.elapsed_time(e1)
    ms, e2e_ms = job_times(ms, e2e_ms, world, dev)
    # kernels per step: one per patch_gemm call, a plan kernel and a chain kernel per chain launch,
    # or one prefill kernel per group launch
    if chain and group:
        per_step = sum((hi - lo + tsg.GROUP_MAX_CALLS - 1) // tsg.GROUP_MAX_CALLS for lo, hi in segments)
    elif chain:
        per_step = sum(2 * ((hi - lo + tsg.CHAIN_MAX_CALLS - 1) // tsg.CHAIN_MAX_CALLS) for lo, hi in segments)
    else:
        per_step = len(calls)
    return {"ms": ms, "e2e_ms": e2e_ms, "seg_ms": seg_ms, "clocks": clocks.summary(), "h2d": h2d, "d2h": d2h,
            "launches": per_step * args.steps}


def split_of(t, units, steps):
    """Mean time (ms) of each segment, scaled to the event-free step time (the
    event-instrumented split, or in proportion to `units` without it)."""
    step_ms = t["ms"] / steps
    w_ = np.asarray(units, dtype=np.float64)
    split = step_ms * w_ / w_.sum() if t["seg_ms"] is None else t["seg_ms"].mean(axis=0)
    return split * (step_ms / split.sum())


def block_common(args, t, per_step, unit, world):
    value = job_throughput(per_step, args.steps, world, t["ms"])
    return {"value": round(value, 2), "unit": unit, "ms_per_step": round(t["ms"] / args.steps, 4),
            "e2e": {"value": round(job_throughput(per_step, args.steps, world, t["e2e_ms"]), 2), "unit": unit,
                    "h2d_bytes_per_step": t["h2d"], "d2h_bytes_per_step": t["d2h"]},
            "gpu_launches": t["launches"], "clocks": t["clocks"]}


def bytes_block(args, name, layers, calls, t, pk, world, segments=None, seg_names=None, traffic_kind=None,
                chain=False):
    """A GB/s block (decode-sized calls): HBM bytes the calls must move."""
    alg = np.array([call_bytes(layers[li], M) for li, M in calls], dtype=np.float64)
    if segments is None:
        segments = [(j, j + 1) for j in range(len(calls))]
        seg_names = [f"{layers[li]['name']}@M={M}" for li, M in calls]
    kernel = "chain_kernel (patch_gemm_chain)" if chain else "decode_tc_kernel"
    seg_bytes = np.array([alg[lo:hi].sum() for lo, hi in segments])
    split = split_of(t, seg_bytes, args.steps)
    achieved = float(alg.sum() / 1e9 / (split.sum() / 1e3))
    traffic = None
    if traffic_kind == "chain":  # one launch per step: its DRAM bytes, if captured for this workload
        traffic = measured_traffic("chain", ["+".join(f"{layers[li]['name']}@M={M}" for li, M in calls)])
    elif traffic_kind:
        traffic = measured_traffic(traffic_kind, [f"{layers[li]['name']}@M={M}" for li, M in calls])
    out = block_common(args, t, alg.sum() / 1e9, "GB/s", world)
    # a chain launch covers up to 64 calls of a segment, a separate call one
    launches = sum((hi - lo + 63) // 64 for lo, hi in segments) if chain else len(calls)
    out["roofline"] = {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                       "frac": round(achieved / pk["hbm_gbs"], 4),
                       "traffic": None if traffic is None else round(traffic),
                       "traffic_unit": "bytes per launch (DRAM read + write, ncu)",
                       "algorithmic_bytes_per_launch": round(float(alg.sum()) / launches),
                       "kernel": kernel, "peak_source": pk["source"]}
    out["per_segment" if len(segments) != len(calls) else "per_call"] = {
        n: {"us": round(1e3 * split[s], 2), "GB/s": round(seg_bytes[s] / 1e9 / (split[s] / 1e3), 1)}
        for s, n in enumerate(seg_names)}
    return out


def flops_block(args, name, layers, calls, t, pk, world, sparse_ratio=None, traffic_kind=None):
    """A TFLOP/s block (prefill-sized calls): dense-equivalent FLOPs, the mixed
    roofline with sparse tiles at 2x the dense peak (the datasheet ratio) and,
    when measured in this run, at the measured sparse/dense MMA rate ratio."""
    P = pk["bf16_tflops"]
    alg = np.array([call_flops(layers[li], M) for li, M in calls], dtype=np.float64)
    split = split_of(t, alg, args.steps)
    t2 = np.array([roof_seconds(layers[li], M, P, 2.0) for li, M in calls])
    achieved = float(alg.sum() / 1e12 / (split.sum() / 1e3))
    frac = float(t2.sum() / (split.sum() / 1e3))
    traffic = measured_traffic(traffic_kind, [f"{layers[li]['name']}/f={layers[li]['frac']}" for li, M in calls]) \
        if traffic_kind else None
    out = block_common(args, t, alg.sum() / 1e12, "TFLOP/s", world)
    done = np.array([call_alg_flops(layers[li], M) for li, M in calls], dtype=np.float64)
    roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": P, "unit": "TFLOP/s",
            "algorithmic_tflops": round(float(done.sum() / 1e12 / (split.sum() / 1e3)), 1),
            "frac": round(frac, 4), "traffic": None if traffic is None else round(traffic),
            "traffic_unit": "bytes per launch (DRAM read + write, ncu)",
            "frac_of_sustained": round(frac * P / pk["bf16_tflops_sustained"], 4)
            if pk.get("bf16_tflops_sustained") else None,
            "kernel": "prefill_kernel (tcgen05)", "peak_source": pk["source"],
            "note": "frac = mixed roofline time (dense tiles at the dense peak, sparse tiles at 2x it) / measured; "
                    "achieved counts dense-equivalent FLOPs (2 M N K), algorithmic_tflops the FLOPs the tensor "
                    "cores do (a sparse tile half of a dense one)"}
    if sparse_ratio:
        # the same roofline with sparse tiles at the measured sparse/dense MMA rate ratio
        tm = np.array([roof_seconds(layers[li], M, P, sparse_ratio) for li, M in calls])
        roof["sparse_ratio_measured"] = round(sparse_ratio, 3)
        roof["frac_measured_sparse_peak"] = round(float(tm.sum() / (split.sum() / 1e3)), 4)
    out["roofline"] = roof
    out["per_call"] = {f"{layers[li]['name']}/f={layers[li]['frac']}@M={M}":
                       {"us": round(1e3 * split[j], 1), "TFLOP/s": round(alg[j] / 1e12 / (split[j] / 1e3), 1),
                        "algorithmic_TFLOP/s": round(done[j] / 1e12 / (split[j] / 1e3), 1),
                        "roofline_frac": round(t2[j] / (split[j] / 1e3), 3)}
                       for j, (li, M) in enumerate(calls)}
    return out, split


def group_flops_block(args, layers, calls, t, pk, world, segments, seg_names, sparse_ratio=None):
    """A TFLOP/s block for calls timed as patch_gemm_group launches (one per
    segment): the dense-equivalent FLOPs and mixed roofline of flops_block,
    over the whole step and per segment."""
    P = pk["bf16_tflops"]
    alg = np.array([call_flops(layers[li], M) for li, M in calls], dtype=np.float64)
    t2 = np.array([roof_seconds(layers[li], M, P, 2.0) for li, M in calls])
    seg_fl = np.array([alg[lo:hi].sum() for lo, hi in segments])
    split = split_of(t, seg_fl, args.steps)
    out = block_common(args, t, alg.sum() / 1e12, "TFLOP/s", world)
    done = sum(call_alg_flops(layers[li], M) for li, M in calls)
    roof = {"bound": "tensor", "achieved": round(float(alg.sum() / 1e12 / (split.sum() / 1e3)), 1), "peak": P,
            "algorithmic_tflops": round(float(done / 1e12 / (split.sum() / 1e3)), 1),
            "unit": "TFLOP/s", "frac": round(float(t2.sum() / (split.sum() / 1e3)), 4), "traffic": None,
            "kernel": "prefill_kernel (patch_gemm_group)", "peak_source": pk["source"],
            "note": "frac = mixed roofline time (dense tiles at the dense peak, sparse tiles at 2x it) / measured"}
    if sparse_ratio:
        tm = np.array([roof_seconds(layers[li], M, P, sparse_ratio) for li, M in calls])
        roof["sparse_ratio_measured"] = round(sparse_ratio, 3)
        roof["frac_measured_sparse_peak"] = round(float(tm.sum() / (split.sum() / 1e3)), 4)
    out["roofline"] = roof
    if len(segments) > 1:
        out["per_segment"] = {n: {"us": round(1e3 * split[s], 1),
                                  "TFLOP/s": round(seg_fl[s] / 1e12 / (split[s] / 1e3), 1),
                                  "roofline_frac": round(float(t2[lo:hi].sum()) / (split[s] / 1e3), 3)}
                              for s, (n, (lo, hi)) in enumerate(zip(seg_names, segments))}
    return out


def sweep_summary(layers, calls, split):
    """Per shape: TFLOP/s at each sparse-tile fraction, speedup over the same
    shape packed all-dense (f = 0, same kernel), and whether time falls (so
    throughput rises) strictly with every step of the fraction."""
    by = {}
    for j, (li, M) in enumerate(calls):
        L = layers[li]
        by.setdefault(L["name"], []).append((L["frac"], split[j], call_flops(L, M)))
    out, mono_all = {}, True
    for name, rows in by.items():
        rows.sort()
        t0 = rows[0][1] if rows[0][0] == 0.0 else None
        mono = all(b[1] < a[1] for a, b in zip(rows, rows[1:]))
        mono_all &= mono
        out[name] = {"TFLOP/s": [round(fl / 1e12 / (ms / 1e3), 1) for _, ms, fl in rows],
                     "fracs": [f for f, _, _ in rows],
                     "speedup_vs_all_dense": [round(t0 / ms, 3) for _, ms, _ in rows] if t0 else None,
                     "monotonic": mono}
    return out, mono_all


def run_block(args, workload, rank, world, dev, pk, status, sparse_ratio=None):
    """One workload's timed block (see the module docstring)."""
    import torch
    layers = build_layers(workload, args.layers, args.fracs, args.tokens)
    full_layers = layers
    shard = getattr(args, "shard", False) and world > 1 and workload in ("decode", "prefill")
    if shard:
        import tile_sparse_gemm_b200 as tsg
        # decode streams stored bytes, prefill spends tensor-core work: balance each by its own
        by = "bytes" if workload == "decode" else "flops"
        split_rows = functools.partial(tsg.shard_rows, by=by)
        layers = shard_layers(full_layers, rank, world, split_rows)
    packed = pack_layers(layers, dev, status)
    resident = sum(p.stored_bytes for p in packed)
    full = not (args.layers or args.fracs or args.tokens)
    if shard:  # one column-parallel shard per rank, the step's Y shards all-gathered once per step
        calls = calls_of(layers)
        _, _, seg = gather_layout(full_layers, calls, world, split_rows)
        if workload == "decode":  # this rank's shards of the step's independent GEMMs as one chain launch
            t = time_calls(args, layers, packed, calls, dev, world, status, chain=True, after=False, gather=seg)
            out = bytes_block(args, workload, full_layers, calls, t, pk, 1, segments=[(0, len(calls))],
                              seg_names=["step"], chain=True)
            out["metric"] = "hybrid GEMM HBM GB/s over stored bytes (decode, sharded)"
        else:  # this rank's shards as separate patch_gemm calls
            t = time_calls(args, layers, packed, calls, dev, world, status, gather=seg)
            out = flops_block(args, workload, full_layers, calls, t, pk, 1, sparse_ratio)[0]
            out.pop("per_call", None)  # eager steps carry no per-call split
            out["metric"] = "hybrid GEMM TFLOP/s, dense-equivalent (prefill, sharded)"
        out["scaling"] = "strong"
        out["step"] = (f"column-parallel: each of {world} ranks multiplies its tile rows of every layer (balanced by "
                       f"{'stored bytes' if by == 'bytes' else 'tensor-core work'}), then one NCCL all-gather of the "
                       "step's Y shards")
        out["config"] = {"workload": f"LLaMA-2-7B linear layers ({workload}), column-parallel shards",
                         "parallelism": f"column-parallel x{world}", "shard_balance": by}
        del packed
        torch.cuda.synchronize()
        return out
    if workload in ("decode", "decode_fused"):
        calls = calls_of(layers)
        # the step's 21 GEMMs are independent (every X is an input of the step):
        # the headline runs them as one patch_gemm_chain in which none waits for
        # another, so the CTAs split the whole step's panel sequence; beside it the
        # same GEMMs as separate patch_gemm calls (each kernel waits for the one
        # before it) and as a chain whose calls wait for each other
        t = time_calls(args, layers, packed, calls, dev, world, status, chain=True, after=False)
        out = bytes_block(args, workload, layers, calls, t, pk, world, segments=[(0, len(calls))],
                          seg_names=["step"], traffic_kind="chain", chain=True)
        out["metric"] = "hybrid GEMM HBM GB/s over stored bytes (decode" + (
            ", fused q|k|v and gate|up projections)" if workload == "decode_fused" else ")")
        out["step"] = ("the step's GEMMs (independent: every X is an input of the step) as one patch_gemm_chain "
                       "launch in which no call waits for another: the CTAs split the step's whole panel sequence")
        t = time_calls(args, layers, packed, calls, dev, world, status)
        out["separate_calls"] = bytes_block(args, workload, layers, calls, t, pk, world, traffic_kind="decode")
        out["separate_calls"]["step"] = ("one patch_gemm call per GEMM on one stream (programmatic dependent "
                                         "launch: each waits for the previous one before reading its X), "
                                         "captured in one CUDA graph")
        t = time_calls(args, layers, packed, calls, dev, world, status, chain=True, after=True)
        out["chain_dependent"] = bytes_block(args, workload, layers, calls, t, pk, world,
                                             segments=[(0, len(calls))], seg_names=["step"], chain=True)
        out["chain_dependent"]["step"] = ("one patch_gemm_chain launch whose calls each wait for the previous "
                                          "one's completion before reading their X")
        out["config"] = {"workload": f"LLaMA-2-7B linear layers ({workload})",
                         "shapes": [f"{L['name']}:{L['N']}x{L['K']}" for L in layers],
                         "tokens": sorted({M for _, M in calls}),
                         "sparse_tile_fraction": sorted({L["frac"] for L in layers}),
                         "resident_weight_bytes": resident,
                         "l2": f"inputs larger than L2: {resident / 2**20:.0f} MiB of packed weights read in rotation",
                         "parallelism": f"replicas x{world}"}
        if workload == "decode" and full:
            out["offline"] = offline_steps(layers, dev, pk)
    elif workload == "prefill":
        calls = calls_of(layers)
        t = time_calls(args, layers, packed, calls, dev, world, status)
        out, split = flops_block(args, workload, layers, calls, t, pk, world, sparse_ratio, traffic_kind="prefill")
        out["metric"] = "hybrid GEMM TFLOP/s, dense-equivalent (prefill)"
        out["sweep"], out["monotonic"] = sweep_summary(layers, calls, split)
        out["config"] = {"workload": "LLaMA-2-7B linear layers (prefill)",
                         "shapes": [f"{n}:{N}x{K}" for n, N, K in si.LLAMA2_7B],
                         "tokens": sorted({M for _, M in calls}),
                         "sparse_tile_fraction": sorted({L["frac"] for L in layers}),
                         "resident_weight_bytes": resident,
                         "l2": "inputs larger than L2 (X 16-45 MB and W 26-90 MB per call, 35 calls in rotation)"}
        # the same 35 GEMMs, those of one sparse-tile fraction (the 7 shapes) per patch_gemm_group launch
        calls_g = sorted(calls, key=lambda c: layers[c[0]]["frac"])
        fr = [layers[li]["frac"] for li, _ in calls_g]
        seg = [(fr.index(f), len(fr) - fr[::-1].index(f)) for f in sorted(set(fr))]
        tg = time_calls(args, layers, packed, calls_g, dev, world, status, segments=seg, chain=True, group=True)
        out["group"] = dict(
            group_flops_block(args, layers, calls_g, tg, pk, world, seg, [f"f={f}" for f in sorted(set(fr))],
                              sparse_ratio),
            step="the same 35 GEMMs as 5 patch_gemm_group launches, one per sparse-tile fraction over the 7 "
                 "shapes (independent GEMMs whose units share one grid)")
        if full:
            out["gated_mlp"] = mlp_steps(dev, pk)
    elif workload == "stack":
        calls = calls_of(layers)
        segments, names, lo = [], [], 0
        for M in sorted({M for _, M in calls}):
            n = sum(1 for _, m in calls if m == M)
            segments.append((lo, lo + n))
            names.append(f"pass@M={M}")
            lo += n
        t = time_calls(args, layers, packed, calls, dev, world, status, segments=segments)
        out = bytes_block(args, workload, layers, calls, t, pk, world, segments, names)
        out["metric"] = "hybrid GEMM HBM GB/s over stored bytes (32-layer stack, sequential)"
        out["step"] = "one patch_gemm call per layer, in order, captured in one CUDA graph"
        t = time_calls(args, layers, packed, calls, dev, world, status, segments=segments, chain=True)
        ch = bytes_block(args, workload, layers, calls, t, pk, world, segments, names, chain=True)
        out["chain"] = dict(ch, step="per pass (M = 1, then M = 8) patch_gemm_chain over the 224 layers in order, "
                                     "each call waiting for the previous one (64 calls per launch)")
        out["chain"]["ms_per_pass"] = {n: v["us"] / 1e3 for n, v in ch["per_segment"].items()}
        t = time_calls(args, layers, packed, calls, dev, world, status, segments=segments, chain=True, after=False)
        ch = bytes_block(args, workload, layers, calls, t, pk, world, segments, names, chain=True)
        out["chain_independent"] = dict(ch, step="per pass patch_gemm_chain over the 224 layers' GEMMs as the "
                                                 "independent GEMMs they are here (no call waits; each launch's "
                                                 "CTAs split its whole panel sequence)")
        out["chain_independent"]["ms_per_pass"] = {n: v["us"] / 1e3 for n, v in ch["per_segment"].items()}
        out["ms_per_pass"] = {n: v["us"] / 1e3 for n, v in out["per_segment"].items()}
        out["stored_gb_per_pass"] = round(sum(p.stored_bytes for p in packed) / 1e9, 3)
        out["config"] = {"workload": "32-layer LLaMA-2-7B linear stack, 7 projections per layer, run in order",
                         "layers": STACK_LAYERS, "weights": len(layers), "tokens": sorted({M for _, M in calls}),
                         "sparse_tile_fraction": "layers 0-3 and 28-31: attention 0.1, MLP 0.2; "
                                                 "layers 4-27: attention 0.7, MLP 0.8",
                         "weights_drawn": "on the device (torch generator seeded per layer), N(0, 0.02) bf16",
                         "resident_weight_bytes": resident,
                         "l2": f"inputs larger than L2: {resident / 2**30:.1f} GiB of packed weights per pass"}
    elif workload == "llama3_qwen":
        out = {"metric": "LLaMA-3-8B and Qwen-2.5-0.5B linears, clustered 50% sparse tiles",
               "config": {"workload": "LLaMA-3-8B + Qwen-2.5-0.5B linear layers, clustered sparse tiles",
                          "shapes": [f"{L['name']}:{L['N']}x{L['K']}" for L in layers],
                          "sparse_tile_fraction": [0.5], "resident_weight_bytes": resident,
                          "note": "Qwen-2.5-0.5B's layers (0.2-8.7 MB) are latency-bound kernels: judge them on "
                                  "their time, not their bandwidth"}}
        for M in sorted({m for L in layers for m in L["xs"]}):
            calls = calls_of(layers, ms=(M,))
            t = time_calls(args, layers, packed, calls, dev, world, status)
            if M <= 16:
                out[f"M={M}"] = bytes_block(args, workload, layers, calls, t, pk, world)
                # the same GEMMs as the independent GEMMs they are here, in one launch
                seg = [(0, len(calls))]
                t = time_calls(args, layers, packed, calls, dev, world, status, segments=seg, chain=True, after=False)
                ch = bytes_block(args, workload, layers, calls, t, pk, world, seg, [f"M={M}"], chain=True)
                out[f"M={M}"]["chain_independent"] = dict(
                    ch, step="one patch_gemm_chain over the 14 GEMMs as the independent GEMMs they are here "
                             "(no call waits; the CTAs split the launch's whole panel sequence)")
            else:
                out[f"M={M}"] = flops_block(args, workload, layers, calls, t, pk, world, sparse_ratio)[0]
                # the same independent GEMMs in one patch_gemm_group launch
                seg = [(0, len(calls))]
                t = time_calls(args, layers, packed, calls, dev, world, status, segments=seg, chain=True,
                               group=True)
                out[f"M={M}"]["group"] = dict(
                    group_flops_block(args, layers, calls, t, pk, world, seg, [f"M={M}"], sparse_ratio),
                    step=f"one patch_gemm_group over the {len(calls)} GEMMs as the independent GEMMs they are "
                         "(their units share one grid of the prefill kernel)")
    else:
        raise ValueError(workload)
    del packed
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world):
    import torch

    import tile_sparse_gemm_b200 as tsg

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    pk = peaks()
    status = tsg.new_status(dev)
    blocks = BLOCKS if args.workload == "all" else (args.workload,)
    probe = mma_rates(dev) if any(b in ("prefill", "llama3_qwen") for b in blocks) else None
    ratio = probe["sparse_over_dense"] if probe else None
    results = {}
    for b in blocks:
        results[b] = run_block(args, b, rank, world, dev, pk, status, sparse_ratio=ratio)
    head = results[blocks[0]]
    if "value" not in head:  # a per-token-count block alone: its smallest token count is the line's figure
        first = head[min((k for k in head if k.startswith("M=")), key=lambda k: int(k[2:]))]
        head = dict(head, **{k: first[k] for k in ("value", "unit", "ms_per_step", "roofline", "e2e", "clocks",
                                                   "gpu_launches") if k in first},
                    headline=f"M={min(int(k[2:]) for k in head if k.startswith('M='))}")
    out = {"metric": head.pop("metric"), "value": head.pop("value"), "unit": head.pop("unit"), "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": head.pop("ms_per_step"),
           "higher_is_better": True, "scaling": head.pop("scaling", "weak"), "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic"}
    out.update(head)
    if probe:
        out["mma_probe"] = probe
    if args.workload == "all":
        out["config"]["blocks"] = list(BLOCKS)
        for b in blocks[1:]:
            out[b] = results[b]
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="all",
                    choices=["all", "decode", "decode_fused", "prefill", "stack", "llama3_qwen", "tile_ablation"])
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch the timed calls eagerly instead of one CUDA graph")
    ap.add_argument("--layers", nargs="*", help="profiling: only these projections (q k v o gate up down)")
    ap.add_argument("--fracs", nargs="*", type=float, help="profiling: only these sparse-tile fractions")
    ap.add_argument("--tokens", nargs="*", type=int, help="profiling: only these token counts M")
    ap.add_argument("--shard", action="store_true",
                    help="decode or prefill under torchrun: each rank multiplies a column-parallel shard of every layer, "
                         "then one all-gather of Y per step (strong scaling) instead of independent replicas")
    args = ap.parse_args()
    if args.impl == "ours" and args.warmup < 3:
        ap.error("--warmup must be at least 3 (timing rule)")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    # the oracle's sample: the headline's workload (decode), or the named one when it has host weights
    ref_workload = args.workload if args.workload in ("decode", "decode_fused", "prefill") else "decode"

    if args.impl == "reference":
        # the CPU oracle, timed as it stands on the host cores; rank 0 only
        if rank != 0:
            return
        steps = []
        cb = None
        for _ in range(args.warmup):
            cpu_baseline(ref_workload, budget_s=1.0, one_thread=False)
        for _ in range(args.steps):
            cb = cpu_baseline(ref_workload, budget_s=5.0, one_thread=False)
            steps.append(cb["value"])
        value = statistics.median(steps)
        cb = dict(cb, value=round(value, 4))
        print(json.dumps({"impl": "reference", "metric": "hybrid GEMM HBM GB/s over stored bytes (decode)"
                          if is_decode(ref_workload) else "hybrid GEMM TFLOP/s, dense-equivalent (prefill)",
                          "value": round(value, 4), "unit": cb["unit"], "n_gpus": args.gpus, "steps": args.steps,
                          "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                          "dtype": "f64", "data": "synthetic",
                          "config": {"workload": f"LLaMA-2-7B linear layers ({ref_workload})"},
                          "cpu_baseline": cb,
                          "e2e": {"value": round(value, 4), "unit": cb["unit"], "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}))
        return

    if args.workload == "tile_ablation":  # one GPU, rank 0 only
        if rank == 0:
            print(json.dumps(tile_ablation(args)))
        return

    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    out = run_ours(args, rank, world)
    if rank == 0:
        # the oracle's host-core baseline: single-GPU runs only
        if world == 1 and not args.no_cpu_baseline and args.workload in ("all", "decode", "decode_fused", "prefill"):
            out["cpu_baseline"] = cpu_baseline(ref_workload, budget_s=30.0, min_s=10.0)
            if args.workload == "all":
                out["prefill"]["cpu_baseline"] = cpu_baseline("prefill", budget_s=15.0, min_s=5.0)
        print(json.dumps(out))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
