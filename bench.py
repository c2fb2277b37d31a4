#!/usr/bin/env python
"""Benchmark of the 2:4 structured-sparse FP8 hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input.
Default workload (``--workload decode``): the decode-shaped MLP up-projection
W[11008, 4096] (bf16, N(0, 0.02)) with X[M, 4096] (N(0, 1)) for M in
{1, 8, 32, 64}.  Each step

  * prunes, quantises and compresses one layer's weights (weight amax +
    2:4 prune/quantise/compress, written in the GEMM's tile-packed layout:
    ``sp24_prune_compress_packed``), and
  * for each M: quantises X and runs the sparse GEMM against another layer's
    compressed weights: in one launch (``sp24_quantize_gemm_packed``) when
    M * K <= 8192, otherwise as ``fp8_quantize_pertensor`` (one thread-block
    cluster for a decode-sized X) followed by ``sp24_gemm_packed``, which is
    what the fused call does at those sizes too.
The 6:8 workload decomposes into the packed layout
(``slide68_decompose_packed``) and lifts and quantises X instead
(``slide68_lift_gemm_packed``, or ``slide68_lift`` + ``sp24_gemm_packed``).
``--unfused`` keeps the two launches at every M; ``fused_vs_unfused`` in the
output times both forms of each small-M GEMM.

Layers rotate over pools of at least three times the 126 MB L2 (bf16 weight
copies and compressed layers), so every kernel reads weights that were last
touched more than a full L2 ago: inputs larger than L2, no flush needed.

Timing: W warm-up steps, then exactly K steps captured in one CUDA graph and
timed with CUDA events on the launching stream, bracketed by a barrier and
``torch.cuda.synchronize()``; max over ranks.  A second replay of the same K
steps with an event between every call gives the per-kernel durations used
for the roofline.  ``e2e`` repeats the K steps eagerly through the public
API with the step's inputs copied from pinned host memory and the outputs
read back every step.

``--impl reference`` times the CPU oracle instead (a bounded sample per
step), on the same metric.  Multi-GPU (torchrun): every rank runs its own
independent replica of the workload (weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse FP8 GEMM TFLOPS & HBM GB/s vs roofline; speedup over dense FP8"
L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------- workloads
# Algorithmic bytes / flops per call (the minimum traffic each op must move).

def bytes_prune24(n, k):
    return 2 * n * k + n * k // 2 + n * k // 8 + 4


def bytes_quant(m, k):
    return 3 * m * k + 4


def bytes_sparse_gemm(m, n, k):
    return n * k // 2 + n * k // 8 + m * k + 2 * m * n + 8


def bytes_dense_gemm(m, n, k):
    return n * k + m * k + 2 * m * n + 8


def bytes_bf16_sparse_gemm(m, n, k):
    return n * k + n * k // 8 + 2 * m * k + 2 * m * n


def bytes_prune24_fp4(n, k):
    return 2 * n * k + n * k // 4 + n * k // 8 + 4


def bytes_quant_fp4(m, k):
    return 2 * m * k + m * k // 2 + 4


def bytes_sparse_gemm_fp4(m, n, k):
    return n * k // 4 + n * k // 8 + m * k // 2 + 2 * m * n + 8


def bytes_slide68(n, k):
    return 2 * n * k + 3 * n * k // 4 + 3 * n * k // 16 + 4


def bytes_lift(m, k):
    return 2 * m * k + 3 * m * k // 2 + 4


def bytes_fused_gemm(m, n, k, kc):
    """Quantise (or lift) + GEMM in one launch: packed weights, X in bf16, the
    codes written out, Y."""
    return n * kc // 2 + n * kc // 8 + 2 * m * k + m * kc + 2 * m * n + 8


FUSED_MAX_M = 64  # above this the full-grid quantiser launch is faster
FUSED_ONE_LAUNCH = 8192  # X elements up to which the fused call is one launch


WORKLOADS = {
    "decode": dict(cfg=2, n=11008, k=4096, ms=(1, 8, 32, 64), pattern="2:4",
                   name="decode MLP up-proj W[11008,4096], M in {1,8,32,64}, 2:4 FP8 E4M3"),
    "prefill": dict(cfg=3, n=12288, k=4096, ms=(4096,), pattern="2:4",
                    name="prefill fused QKV M4096 N12288 K4096, 2:4 FP8 E4M3"),
    "downproj": dict(cfg=4, n=4096, k=14336, ms=(256,), pattern="2:4",
                     name="MLP down-proj M256 N4096 K14336, 2:4 FP8 E4M3"),
    "slide68": dict(cfg=5, n=4096, k=4096, ms=(64, 2048), pattern="6:8",
                    name="6:8 sliding-window W[4096,4096] K'=6144, M in {64,2048}"),
}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def source_hash(files):
    """Hash of the named kernel sources (under structured_sparse_fp8_b200/csrc)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "structured_sparse_fp8_b200", "csrc")
    for f in files:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def load_traffic():
    """DRAM bytes per launch ("workload:op" -> bytes) from the committed ncu
    summaries, for the entries whose kernel sources are unchanged since the
    capture (an entry whose sources changed is dropped: its traffic is null)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return {}
    d = json.load(open(path))
    out = {}
    for key, e in d.get("entries", {}).items():
        try:
            if source_hash(e["sources"]) == e["source_hash"]:
                out[key] = e["bytes_per_launch"]
        except (OSError, KeyError):
            pass
    return out


def runs_of_equal_names(names):
    """[start, end) index ranges of the maximal runs of consecutive equal
    names: the launches one event pair brackets in the per-kernel timing."""
    runs, i = [], 0
    while i < len(names):
        j = i + 1
        while j < len(names) and names[j] == names[i]:
            j += 1
        runs.append((i, j))
        i = j
    return runs


# ---------------------------------------------------------------- ranks

def max_over_ranks(seconds: float, device=None) -> float:
    """Largest of every rank's measured time (identity on one process)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return seconds
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(step_bytes: int, steps: int, world: int, seconds: float) -> float:
    """Whole-job throughput: the bytes every rank processed over the slowest rank's time."""
    return step_bytes * steps * world / seconds / 1e9


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index, period=0.002):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self.period = period
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - NVML unavailable: report no clocks
            self.nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        for bit, name in self.REASONS.items():
            if r & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:  # noqa: BLE001
                return
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self._stop.set()
            self._t.join()
            try:
                self._sample()
            except Exception:  # noqa: BLE001
                pass

    def summary(self):
        if not self.samples:
            return None
        busy = [s for s in self.samples]
        return {"sm_mhz": float(statistics.median(busy)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(busy)}


# ---------------------------------------------------------------- GPU arm

class GpuWorkload:
    """Device buffers, rotating pools and the step for one workload."""

    def __init__(self, wl, device, unfused=False):
        import torch

        import structured_sparse_fp8_b200 as sp
        from structured_sparse_fp8_b200 import workloads as WL
        self.torch, self.sp, self.wl, self.dev = torch, sp, wl, device
        n, k, ms = wl["n"], wl["k"], wl["ms"]
        self.n, self.k, self.ms = n, k, ms
        self.is68 = wl["pattern"] == "6:8"
        # the fused call where it is one kernel; above that size it runs the
        # same two launches as the separate calls, timed as what they are
        self.fused = {m: (not unfused) and m * self.k <= FUSED_ONE_LAUNCH for m in ms}
        self.kc = k * 3 // 2 if self.is68 else k   # K of the compressed operand
        w_host = WL.weight_bits(wl["cfg"])
        self.w_host_pinned = torch.from_numpy(w_host.view(np.int16)).view(torch.bfloat16).pin_memory()
        w_dev = self.w_host_pinned.to(device)
        wbytes = n * k * 2
        self.R_w = max(2, -(-3 * L2_BYTES // wbytes))
        self.w_pool = [w_dev.clone() for _ in range(self.R_w)]
        comp_bytes = n * self.kc // 2 + n * self.kc // 8
        self.R_g = max(2 * len(ms), -(-3 * L2_BYTES // comp_bytes))
        self.comp_bytes = comp_bytes
        self.R_g = -(-self.R_g // len(ms)) * len(ms)
        self.ws = sp.Workspace(device)
        lib = sp._lib.load()
        # every GEMM this workload times (packed, fused, canonical, BF16, dense),
        # sized once here so that no workspace is allocated inside a graph
        self.ws.get(max(max(lib.sp24_workspace_size(sp._lib.OP_GEMM, m, n, self.kc, 0),
                            lib.sp24_workspace_size(sp._lib.OP_LIFT_GEMM_PACKED if self.is68
                                                    else sp._lib.OP_QUANTIZE_GEMM_PACKED, m, n, k, 0),
                            lib.sp24_workspace_size(sp._lib.OP_GEMM, m, n, k, 1),
                            lib.sp24_workspace_size(sp._lib.OP_GEMM_DENSE, m, n, k, 0)) for m in ms) + 4096)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

        def new_comp():
            return dict(scale=torch.empty((1,), dtype=torch.float32, device=device),
                        packed=torch.empty(n * self.kc // 2 + n * self.kc // 8, dtype=torch.uint8,
                                           device=device))
        self.prune_out = [new_comp() for _ in range(2)]
        self.weight_op(w_dev, self.prune_out[0])
        self.g_pool = []   # the GEMM streams the packed copy only
        for _ in range(self.R_g):
            c = new_comp()
            for key in c:
                c[key].copy_(self.prune_out[0][key])
            self.g_pool.append(c)
        self.x_host = {}
        self.x_dev, self.xq, self.sx, self.y = {}, {}, {}, {}
        for m in ms:
            xb = WL.activation_bits(wl["cfg"], m)
            self.x_host[m] = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).pin_memory()
            self.x_dev[m] = self.x_host[m].to(device)
            self.xq[m] = torch.empty((m, self.kc), dtype=torch.uint8, device=device)
            self.sx[m] = torch.empty((1,), dtype=torch.float32, device=device)
            self.y[m] = torch.empty((m, n), dtype=torch.bfloat16, device=device)
        self.y_host = {m: torch.empty((m, n), dtype=torch.bfloat16).pin_memory() for m in ms}
        del w_dev
        torch.cuda.synchronize()

    # one call of each kind -------------------------------------------------
    def weight_op(self, w, out):
        """Weight path straight into the tile-packed layout the GEMM streams
        (one kernel: 2:4 prune/quantise/compress, or 6:8 decomposition)."""
        fn = self.sp.slide68_decompose_packed if self.is68 else self.sp.sp24_prune_compress_packed
        return fn(w, status=self.status, workspace=self.ws, out=out["packed"], scale=out["scale"])

    def act_op(self, m):
        if self.is68:
            return self.sp.slide68_lift(self.x_dev[m], status=self.status, out=self.xq[m],
                                        scale=self.sx[m], workspace=self.ws)
        return self.sp.fp8_quantize_pertensor(self.x_dev[m], status=self.status, out=self.xq[m],
                                              scale=self.sx[m], workspace=self.ws)

    def gemm_op(self, m, layer):
        c = self.g_pool[layer]
        return self.sp.sp24_gemm_packed(self.xq[m], self.sx[m], c["packed"], c["scale"], self.n,
                                        out=self.y[m], status=self.status, workspace=self.ws)

    def fused_name(self):
        return "slide68_lift_gemm_packed" if self.is68 else "sp24_quantize_gemm_packed"

    def fused_op(self, m, layer):
        c = self.g_pool[layer]
        fn = getattr(self.sp, self.fused_name())
        return fn(self.x_dev[m], c["packed"], c["scale"], self.n, out=self.y[m], xq_out=self.xq[m],
                  x_scale_out=self.sx[m], status=self.status, workspace=self.ws)

    def ops_of_step(self, s):
        """(name, callable, algorithmic bytes, flops, kernel launches) of step s."""
        n, k, kc = self.n, self.k, self.kc
        ops = []
        wi = s % self.R_w
        if self.is68:
            wname, wbytes, wl = "slide68_decompose_packed", bytes_slide68(n, k), 1
        else:
            wname, wbytes, wl = "sp24_prune_compress_packed", bytes_prune24(n, k), 1
        ops.append((wname, lambda: self.weight_op(self.w_pool[wi], self.prune_out[s % 2]), wbytes, 0, wl))
        for j, m in enumerate(self.ms):
            layer = (s * len(self.ms) + j) % self.R_g
            if self.fused[m]:
                ops.append((self.fused_name(), (lambda m=m, layer=layer: self.fused_op(m, layer)),
                            bytes_fused_gemm(m, n, k, kc), 2 * m * n * kc, 1))
                continue
            aname = "slide68_lift" if self.is68 else "fp8_quantize_pertensor"
            abytes = bytes_lift(m, k) if self.is68 else bytes_quant(m, k)
            ops.append((aname, (lambda m=m: self.act_op(m)), abytes, 0, 1))
            ops.append(("sp24_gemm_packed", (lambda m=m, layer=layer: self.gemm_op(m, layer)),
                        bytes_sparse_gemm(m, n, kc), 2 * m * n * kc, 1))
        return ops

    def step_bytes(self):
        return sum(o[2] for o in self.ops_of_step(0))

    def step_launches(self):
        return sum(o[4] for o in self.ops_of_step(0))

    def capture(self, steps, first, events):
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        evs = []
        with torch.cuda.graph(g):
            for s in range(first, first + steps):
                ops = list(self.ops_of_step(s))
                if not events:
                    for op in ops:
                        op[1]()
                    continue
                # one event pair per run of consecutive launches of one kernel,
                # so launches of the same kernel keep their programmatic
                # launch overlap (an event between them would serialise them)
                for i, j in runs_of_equal_names([op[0] for op in ops]):
                    e0 = torch.cuda.Event(enable_timing=True, external=True)
                    e1 = torch.cuda.Event(enable_timing=True, external=True)
                    e0.record()
                    for op in ops[i:j]:
                        op[1]()
                    e1.record()
                    evs.append((ops[i][0], sum(op[2] for op in ops[i:j]), sum(op[3] for op in ops[i:j]),
                                j - i, e0, e1))
        return g, evs

    # dense FP8 comparison for the GEMM shapes of this workload ------------
    def dense_compare(self, reps=50):
        """Sparse GEMM of this workload vs the dense FP8 GEMM of the same
        layer (dense W[N, K] with X quantised at K), each timed as a CUDA
        graph of `reps` launches over rotating weight copies.  The same
        sparse GEMM on the canonical (unpacked) weight layout and, for 2:4,
        with BF16 operands (values bf16 [N, K/2], X bf16) is timed alongside."""
        torch, sp = self.torch, self.sp
        n, k, kc = self.n, self.k, self.kc
        out = {}
        wq, sw = sp.fp8_quantize_pertensor(self.w_pool[0], workspace=self.ws)
        ndense = max(2, -(-3 * L2_BYTES // (n * k)))
        dpool = [wq.clone() for _ in range(ndense)]
        if self.is68:
            canon = sp.slide68_decompose(self.w_pool[0], "e4m3", workspace=self.ws)
            bf = None
        else:
            canon = sp.sp24_prune_compress(self.w_pool[0], "e4m3", workspace=self.ws)
            bf = sp.sp24_prune_compress(self.w_pool[0], "bf16", workspace=self.ws)
        ncanon = max(2, -(-3 * L2_BYTES // self.comp_bytes))
        cpool = [(canon["values"].clone(), canon["meta"].clone()) for _ in range(ncanon)]
        if bf is not None:
            nbf = max(2, -(-3 * L2_BYTES // (n * k + n * k // 8)))
            bpool = [(bf["values"].clone(), bf["meta"].clone()) for _ in range(nbf)]
        kinds = ("sparse", "dense", "canonical") + (("bf16",) if bf is not None else ())
        for m in self.ms:
            xqd, sxd = sp.fp8_quantize_pertensor(self.x_dev[m], workspace=self.ws)
            res = {}
            for kind in kinds:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    for r in range(reps):
                        if kind == "dense":
                            sp.fp8_gemm_dense(xqd, sxd, dpool[r % ndense], sw,
                                              out=self.y[m], workspace=self.ws)
                        elif kind == "canonical":
                            v, e = cpool[r % ncanon]
                            sp.sp24_gemm(self.xq[m], self.sx[m], v, e, canon["scale"],
                                         out=self.y[m], workspace=self.ws)
                        elif kind == "bf16":
                            v, e = bpool[r % nbf]
                            sp.sp24_gemm(self.x_dev[m], None, v, e, None, dtype="bf16",
                                         out=self.y[m], workspace=self.ws)
                        else:
                            c = self.g_pool[r % self.R_g]
                            sp.sp24_gemm_packed(self.xq[m], self.sx[m], c["packed"], c["scale"], n,
                                                out=self.y[m], workspace=self.ws)
                g.replay()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                g.replay()
                e1.record()
                torch.cuda.synchronize()
                res[kind] = e0.elapsed_time(e1) * 1000.0 / reps
                del g
            out[str(m)] = {"sparse_us": round(res["sparse"], 3), "dense_us": round(res["dense"], 3),
                           "speedup": round(res["dense"] / res["sparse"], 3),
                           "sparse_gbs": round(bytes_sparse_gemm(m, n, kc) / res["sparse"] / 1e3, 1),
                           "dense_gbs": round(bytes_dense_gemm(m, n, k) / res["dense"] / 1e3, 1),
                           "sparse_tflops_dense_equiv": round(2 * m * n * kc / res["sparse"] / 1e6, 2),
                           "dense_tflops": round(2 * m * n * k / res["dense"] / 1e6, 2),
                           "canonical_layout_us": round(res["canonical"], 3),
                           "canonical_layout_gbs": round(bytes_sparse_gemm(m, n, kc) / res["canonical"] / 1e3, 1)}
            if "bf16" in res:
                out[str(m)]["bf16_sparse_us"] = round(res["bf16"], 3)
                out[str(m)]["bf16_sparse_gbs"] = round(bytes_bf16_sparse_gemm(m, n, k) / res["bf16"] / 1e3, 1)
                out[str(m)]["bf16_sparse_tflops"] = round(2 * m * n * k / res["bf16"] / 1e6, 2)
        del dpool, cpool
        return out

    def _graph_us(self, fn, reps):
        """Average µs per call of `fn(r)` over a CUDA graph of `reps` calls."""
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for r in range(reps):
                fn(r)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) * 1000.0 / reps

    def finer_scales(self, reps=50):
        """Per-token activation scales and per-channel weight scales on this
        workload's shapes (2:4 only): the per-token quantiser, the per-channel
        weight path and the GEMM with both scale vectors, each timed as a
        CUDA graph over rotating inputs."""
        if self.is68:
            return None
        torch, sp = self.torch, self.sp
        n, k = self.n, self.k
        out = {}
        vals = torch.empty((n, k // 2), dtype=torch.uint8, device=self.dev)
        meta = torch.empty((n, k // 8), dtype=torch.uint8, device=self.dev)
        wsc = torch.empty((n,), dtype=torch.float32, device=self.dev)
        t = self._graph_us(lambda r: sp.sp24_prune_compress_perchannel(
            self.w_pool[r % self.R_w], out=dict(values=vals, meta=meta, scales=wsc)), max(4, reps // 5))
        out["perchannel_prune"] = {"us": round(t, 3),
                                   "gbs": round((bytes_prune24(n, k) + 4 * n) / t / 1e3, 1)}
        for m in self.ms:
            q = torch.empty((m, k), dtype=torch.uint8, device=self.dev)
            xs = torch.empty((m,), dtype=torch.float32, device=self.dev)
            tq = self._graph_us(lambda r: sp.fp8_quantize_pertoken(self.x_dev[m], out=q, scales=xs), reps)
            tg = self._graph_us(lambda r: sp.sp24_gemm_packed_scaled(
                q, xs, self.g_pool[r % self.R_g]["packed"], wsc, n, out=self.y[m], workspace=self.ws), reps)
            out[str(m)] = {"pertoken_quantize_us": round(tq, 3),
                           "pertoken_quantize_gbs": round((bytes_quant(m, k) + 4 * m) / tq / 1e3, 1),
                           "scaled_gemm_us": round(tg, 3),
                           "scaled_gemm_gbs": round((bytes_sparse_gemm(m, n, k) + 4 * m + 4 * n) / tg / 1e3, 1),
                           "scaled_gemm_tflops_dense_equiv": round(2 * m * n * k / tg / 1e6, 2)}
        return out

    def general_slide(self, reps=50):
        """The (2N-2):2N decomposition for N = 3 (4:6) and 5 (8:10) on the 6:8
        layer's shape, with K chosen so that K' = 6144 as for 6:8 (K = 4608,
        3840): the weight decomposition, the lift of each M and the sparse GEMM
        over K' from tile-packed weights, each a CUDA graph over rotating
        inputs larger than L2 (timing pools drawn on the device, N(0, 0.02))."""
        if not self.is68:
            return None
        torch, sp = self.torch, self.sp
        n, out = self.n, {}
        gen = torch.Generator(device=self.dev)
        for nn, k in ((3, 4608), (5, 3840)):
            gen.manual_seed(600 + nn)
            kp = k // (2 * nn) * 4 * (nn - 1)
            r_w = max(2, -(-3 * L2_BYTES // (2 * n * k)))
            r_g = max(2, -(-3 * L2_BYTES // (n * kp * 5 // 8)))
            wpool = [(torch.randn((n, k), generator=gen, device=self.dev) * 0.02).to(torch.bfloat16)
                     for _ in range(max(r_w, r_g))]
            vals = torch.empty((n, kp // 2), dtype=torch.uint8, device=self.dev)
            meta = torch.empty((n, kp // 8), dtype=torch.uint8, device=self.dev)
            sw = torch.empty((1,), dtype=torch.float32, device=self.dev)
            td = self._graph_us(lambda r: sp.slide_decompose(
                wpool[r % r_w], nn, workspace=self.ws, out=dict(values=vals, meta=meta, scale=sw)),
                max(4, reps // 5))
            wbytes = 2 * n * k + n * kp // 2 + n * kp // 8 + 4
            res = {"k": k, "k_prime": kp, "decompose_us": round(td, 3),
                   "decompose_gbs": round(wbytes / td / 1e3, 1)}
            layers = []
            for r in range(r_g):
                d = sp.slide_decompose(wpool[r], nn, workspace=self.ws)
                layers.append((sp.sp24_pack_weights(d["values"], d["meta"]), d["scale"]))
            del wpool
            for m in self.ms:
                x = (torch.randn((m, k), generator=gen, device=self.dev)).to(torch.bfloat16)
                xl = torch.empty((m, kp), dtype=torch.uint8, device=self.dev)
                sx = torch.empty((1,), dtype=torch.float32, device=self.dev)
                y = torch.empty((m, n), dtype=torch.bfloat16, device=self.dev)
                tl = self._graph_us(lambda r: sp.slide_lift(x, nn, workspace=self.ws, out=xl, scale=sx), reps)
                tg = self._graph_us(lambda r: sp.sp24_gemm_packed(
                    xl, sx, layers[r % r_g][0], layers[r % r_g][1], n, out=y, workspace=self.ws), reps)
                res[str(m)] = {"lift_us": round(tl, 3),
                               "lift_gbs": round((2 * m * k + m * kp + 4) / tl / 1e3, 1),
                               "gemm_us": round(tg, 3),
                               "gemm_gbs": round(bytes_sparse_gemm(m, n, kp) / tg / 1e3, 1),
                               "gemm_tflops_dense_equiv": round(2 * m * n * k / tg / 1e6, 2)}
            del layers
            out[f"{2 * nn - 2}:{2 * nn}"] = res
        return out

    def int8_compare(self, reps=50):
        """INT8 W8A8 on this workload's 2:4 shapes: the INT8 weight path
        (prune + quantise + compress, canonical layout), the per-tensor INT8
        quantiser and the INT8 sparse GEMM over tile-packed weights (rotating
        layers, larger than L2), each a CUDA graph of back-to-back calls."""
        if self.is68:
            return None
        torch, sp = self.torch, self.sp
        n, k = self.n, self.k
        outw = dict(values=torch.empty((n, k // 2), dtype=torch.int8, device=self.dev),
                    meta=torch.empty((n, k // 8), dtype=torch.uint8, device=self.dev),
                    scale=torch.empty((1,), dtype=torch.float32, device=self.dev))
        sp.sp24_prune_compress_int8(self.w_pool[0], workspace=self.ws, out=outw)
        packed = sp.sp24_pack_weights(outw["values"].view(torch.uint8), outw["meta"])
        pool = [packed.clone() for _ in range(self.R_g)]
        sw = outw["scale"].clone()
        t = self._graph_us(lambda r: sp.sp24_prune_compress_int8(self.w_pool[r % self.R_w], workspace=self.ws,
                                                                 out=outw), max(4, reps // 5))
        out = {"weight_path_us": round(t, 3), "weight_path_gbs": round(bytes_prune24(n, k) / t / 1e3, 1)}
        for m in self.ms:
            q = torch.empty((m, k), dtype=torch.int8, device=self.dev)
            sx = torch.empty((1,), dtype=torch.float32, device=self.dev)
            # one eager call of each before capture (attribute set-up, warm)
            sp.int8_quantize_pertensor(self.x_dev[m], workspace=self.ws, out=q, scale=sx)
            sp.sp24_gemm_int8_packed(q, sx, pool[0], sw, n, out=self.y[m], workspace=self.ws)
            tq = self._graph_us(lambda r: sp.int8_quantize_pertensor(self.x_dev[m], workspace=self.ws, out=q,
                                                                    scale=sx), reps)
            tg = self._graph_us(lambda r: sp.sp24_gemm_int8_packed(q, sx, pool[r % self.R_g], sw, n, out=self.y[m],
                                                                  workspace=self.ws), reps)
            out[str(m)] = {"quantize_us": round(tq, 3),
                           "quantize_gbs": round(bytes_quant(m, k) / tq / 1e3, 1),
                           "gemm_us": round(tg, 3),
                           "gemm_gbs": round(bytes_sparse_gemm(m, n, k) / tg / 1e3, 1),
                           "gemm_tops_dense_equiv": round(2 * m * n * k / tg / 1e6, 2)}
        del pool
        return out

    def fp4_compare(self, reps=50):
        """FP4 (E2M1) with 2:4 weights on this workload's shapes: the FP4
        weight path (prune + quantise + compress), the per-tensor FP4
        quantiser and the FP4 sparse GEMM (rotating layers, larger than L2),
        each a CUDA graph of back-to-back calls."""
        if self.is68:
            return None
        torch, sp = self.torch, self.sp
        n, k = self.n, self.k
        outw = dict(values=torch.empty((n, k // 4), dtype=torch.uint8, device=self.dev),
                    meta=torch.empty((n, k // 8), dtype=torch.uint8, device=self.dev),
                    scale=torch.empty((1,), dtype=torch.float32, device=self.dev))
        sp.sp24_prune_compress_fp4(self.w_pool[0], workspace=self.ws, out=outw)
        npool = max(2, -(-3 * L2_BYTES // (n * k // 4 + n * k // 8)))
        pool = [(outw["values"].clone(), outw["meta"].clone()) for _ in range(npool)]
        sw = outw["scale"].clone()
        t = self._graph_us(lambda r: sp.sp24_prune_compress_fp4(self.w_pool[r % self.R_w], workspace=self.ws,
                                                                out=outw), max(4, reps // 5))
        out = {"weight_path_us": round(t, 3), "weight_path_gbs": round(bytes_prune24_fp4(n, k) / t / 1e3, 1)}
        for m in self.ms:
            q = torch.empty((m, k // 2), dtype=torch.uint8, device=self.dev)
            sx = torch.empty((1,), dtype=torch.float32, device=self.dev)
            sp.fp4_quantize_pertensor(self.x_dev[m], workspace=self.ws, out=q, scale=sx)
            sp.sp24_gemm_fp4(q, sx, pool[0][0], pool[0][1], sw, out=self.y[m], workspace=self.ws)
            tq = self._graph_us(lambda r: sp.fp4_quantize_pertensor(self.x_dev[m], workspace=self.ws, out=q,
                                                                   scale=sx), reps)
            tg = self._graph_us(lambda r: sp.sp24_gemm_fp4(q, sx, pool[r % npool][0], pool[r % npool][1], sw,
                                                          out=self.y[m], workspace=self.ws), reps)
            out[str(m)] = {"quantize_us": round(tq, 3),
                           "quantize_gbs": round(bytes_quant_fp4(m, k) / tq / 1e3, 1),
                           "gemm_us": round(tg, 3),
                           "gemm_gbs": round(bytes_sparse_gemm_fp4(m, n, k) / tg / 1e3, 1),
                           "gemm_tflops_dense_equiv": round(2 * m * n * k / tg / 1e6, 2)}
        del pool
        return out

    def fusion_compare(self, reps=50):
        """For every M that the step runs fused: the fused launch against the
        activation kernel + GEMM pair it replaces, each as a CUDA graph of
        `reps` back-to-back repetitions over rotating weights."""
        torch = self.torch
        out = {}
        for m in self.ms:
            if m > FUSED_MAX_M:
                continue
            res = {}
            for kind in ("fused", "unfused"):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    for r in range(reps):
                        if kind == "fused":
                            self.fused_op(m, r % self.R_g)
                        else:
                            self.act_op(m)
                            self.gemm_op(m, r % self.R_g)
                g.replay()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                g.replay()
                e1.record()
                torch.cuda.synchronize()
                res[kind] = e0.elapsed_time(e1) * 1000.0 / reps
                del g
            nb = bytes_fused_gemm(m, self.n, self.k, self.kc)
            out[str(m)] = {"fused_us": round(res["fused"], 3), "unfused_us": round(res["unfused"], 3),
                           "speedup": round(res["unfused"] / res["fused"], 3),
                           "fused_gbs": round(nb / res["fused"] / 1e3, 1)}
        return out

    # e2e through the public API with host buffers ---------------------------
    def e2e(self, steps):
        torch = self.torch
        h2d = self.n * self.k * 2 + sum(m * self.k * 2 for m in self.ms)
        d2h = sum(m * self.n * 2 for m in self.ms)
        for s in range(2):
            self._e2e_step(s)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for s in range(steps):
            self._e2e_step(s)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / 1e3, h2d, d2h

    def _e2e_step(self, s):
        w = self.w_pool[s % self.R_w]
        w.copy_(self.w_host_pinned, non_blocking=True)
        for m in self.ms:
            self.x_dev[m].copy_(self.x_host[m], non_blocking=True)
        for (name, fn, nb, fl, nl) in self.ops_of_step(s):
            fn()
        for m in self.ms:
            self.y_host[m].copy_(self.y[m], non_blocking=True)


def run_gpu(args, wl, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    import __graft_entry__
    __graft_entry__.build()
    gw = GpuWorkload(wl, device, unfused=args.unfused)
    peaks = load_peaks()

    # warm-up: W eager steps (first calls set kernel attributes), then graphs
    for s in range(args.warmup):
        for op in gw.ops_of_step(s):
            op[1]()
    torch.cuda.synchronize()
    g_warm, _ = gw.capture(args.warmup, 0, events=False)
    g_timed, _ = gw.capture(args.steps, args.warmup, events=False)
    g_detail, evs = gw.capture(args.steps, args.warmup, events=True)
    g_warm.replay()
    torch.cuda.synchronize()

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        start.record()
        g_timed.replay()
        end.record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    elapsed = max_over_ranks(start.elapsed_time(end) / 1e3, device)

    # per-kernel durations (second replay of the same K steps, an event pair
    # around each run of consecutive launches of one kernel)
    g_detail.replay()
    torch.cuda.synchronize()
    per = {}
    for name, nb, fl, cnt, e0, e1 in evs:
        d = per.setdefault(name, dict(t=0.0, bytes=0, flops=0, n=0))
        d["t"] += e0.elapsed_time(e1) / 1e3
        d["bytes"] += nb
        d["flops"] += fl
        d["n"] += cnt
    assert int(gw.status.item()) == 0, "device status word set during the benchmark"

    step_bytes = gw.step_bytes()
    value = aggregate_gbs(step_bytes, args.steps, world, elapsed)
    detail_total = sum(d["t"] for d in per.values())
    dominant = max(per, key=lambda k: per[k]["t"])
    dom = per[dominant]
    traffic = load_traffic()
    tensor_bound = wl["ms"][-1] >= 1024 and dominant == "sp24_gemm_packed"
    if tensor_bound:
        achieved = dom["flops"] / dom["t"] / 1e12
        peak = peaks["bf16_tflops"] * 4.0   # 2:4 sparse FP8 = 2 x FP8 = 4 x bf16 (nominal ratio)
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "kernel": dominant, "peak_source": f"{peaks['source']} bf16 burst x4 (2:4 sparse FP8 dense-equivalent)"}
    else:
        achieved = dom["bytes"] / dom["t"] / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": round(peak, 1),
                "unit": "GB/s", "frac": round(achieved / peak, 4),
                "kernel": dominant, "peak_source": f"{peaks['source']} hbm_gbs"}
    tr = traffic.get(f"{args.workload}:{dominant}")
    roof["traffic"] = tr
    kernels = {k: {"calls": v["n"] // args.steps, "us_per_call": round(v["t"] / v["n"] * 1e6, 3),
                   "share": round(v["t"] / detail_total, 4),
                   "gbs": round(v["bytes"] / v["t"] / 1e9, 1),
                   "frac_hbm": round(v["bytes"] / v["t"] / 1e9 / peaks["hbm_gbs"], 4)}
               for k, v in per.items()}
    for k, v in per.items():
        if v["flops"]:
            kernels[k]["tflops"] = round(v["flops"] / v["t"] / 1e12, 2)

    compare = gw.dense_compare() if rank == 0 and not args.no_compare else None
    fusion = gw.fusion_compare() if rank == 0 and not args.no_compare else None
    finer = gw.finer_scales() if rank == 0 and not args.no_compare else None
    general = gw.general_slide() if rank == 0 and not args.no_compare else None
    int8 = None
    if rank == 0 and not args.no_compare:
        try:
            int8 = gw.int8_compare()
        except Exception as e:  # a failure here is recorded, never fatal to the bench line
            int8 = {"error": f"{type(e).__name__}: {e}"[:300]}
    fp4 = None
    if rank == 0 and not args.no_compare:
        try:
            fp4 = gw.fp4_compare()
        except Exception as e:  # a failure here is recorded, never fatal to the bench line
            fp4 = {"error": f"{type(e).__name__}: {e}"[:300]}
    prefill = None
    speedups = None
    if rank == 0 and args.workload == "decode" and not args.no_prefill:
        prefill = prefill_headline(device, peaks)
        try:
            speedups = speedup_headlines(device, peaks)
        except Exception as e:  # a failure here is recorded, never fatal to the bench line
            speedups = {"error": f"{type(e).__name__}: {e}"[:300]}
    e2e_t, h2d, d2h = gw.e2e(args.steps)
    e2e_t = max_over_ranks(e2e_t, device)
    del g_timed, g_detail, g_warm

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(elapsed / args.steps * 1e3, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3",
        "data": "synthetic (seeded, bf16 N(0,0.02) weights / N(0,1) activations; see workloads.py)",
        "config": {"workload": wl["name"], "n": wl["n"], "k": wl["k"], "m": list(wl["ms"]),
                   "step": ("weight 6:8 decomposition" if gw.is68 else
                            "weight 2:4 prune/quantise/compress")
                           + " into the tile-packed layout, then per M: activation quantise"
                           + (" + lift" if gw.is68 else "") + " + sparse GEMM"
                           + ("" if args.unfused else
                              f" (one fused launch for M*K <= {FUSED_ONE_LAUNCH})"),
                   "algorithmic_bytes_per_step": step_bytes,
                   "l2": f"inputs larger than L2: rotating pools of {gw.R_w} bf16 weight copies and "
                         f"{gw.R_g} compressed layers",
                   "parallelism": f"replicas x{world}"},
        "roofline": roof,
        "prefill": prefill,
        "speedups": speedups,
        "kernels": kernels,
        "sparse_vs_dense": compare,
        "fused_vs_unfused": fusion,
        "finer_scales": finer,
        "general_slide": general,
        "int8_w8a8": int8,
        "fp4_e2m1": fp4,
        "e2e": {"value": round(aggregate_gbs(step_bytes, args.steps, world, e2e_t), 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": gw.step_launches() * args.steps,
        "clocks": clocks.summary(),
        "peaks": peaks,
    }
    return line, gw


def prefill_headline(device, peaks, reps=20):
    """The tensor-bound target next to the decode headline: the prefill-shaped
    fused-QKV sparse GEMM (M4096 N12288 K4096, X with its 41 outlier columns)
    and the same-family dense FP8 GEMM on the same shapes, each timed as a
    CUDA graph of `reps` launches over rotating weight copies (pools larger
    than L2), CUDA events on the launching stream.  Roofline: 2 M N K
    dense-equivalent FLOPs per call against the sparse FP8 peak, 4 x the
    measured bf16 burst (the nominal ratios: FP8 = 2 x bf16, 2:4 = 2 x
    dense)."""
    import torch

    import structured_sparse_fp8_b200 as sp
    from structured_sparse_fp8_b200 import workloads as WL
    wl = WORKLOADS["prefill"]
    m, n, k = wl["ms"][0], wl["n"], wl["k"]
    ws = sp.Workspace(device)
    w = torch.from_numpy(WL.weight_bits(wl["cfg"]).view(np.int16)).view(torch.bfloat16).to(device)
    x = torch.from_numpy(WL.activation_bits(wl["cfg"], m).view(np.int16)).view(torch.bfloat16).to(device)
    packed, sw = sp.sp24_prune_compress_packed(w, workspace=ws)
    wq, swd = sp.fp8_quantize_pertensor(w, workspace=ws)
    xq, sx = sp.fp8_quantize_pertensor(x, workspace=ws)
    del w
    y = torch.empty((m, n), dtype=torch.bfloat16, device=device)
    ps = [packed] + [packed.clone() for _ in range(max(1, -(-3 * L2_BYTES // packed.numel())) - 1)]
    pd = [wq] + [wq.clone() for _ in range(max(1, -(-3 * L2_BYTES // wq.numel())) - 1)]
    ws.get(max(sp._lib.load().sp24_workspace_size(sp._lib.OP_GEMM_PACKED, m, n, k, 0),
               sp._lib.load().sp24_workspace_size(sp._lib.OP_GEMM_DENSE, m, n, k, 0)) + 4096)
    status = torch.zeros(1, dtype=torch.int32, device=device)

    def time_graph(fn):
        fn(0)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for r in range(reps):
                fn(r)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) * 1e3 / reps

    t_sp = time_graph(lambda r: sp.sp24_gemm_packed(xq, sx, ps[r % len(ps)], sw, n, out=y, status=status,
                                                    workspace=ws))
    t_dn = time_graph(lambda r: sp.fp8_gemm_dense(xq, sx, pd[r % len(pd)], swd, out=y, status=status,
                                                  workspace=ws))
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device status word set during the prefill timing"
    flops = 2.0 * m * n * k
    achieved = flops / t_sp / 1e6
    peak = peaks["bf16_tflops"] * 4.0
    return {"workload": wl["name"],
            "sparse_us": round(t_sp, 3), "dense_fp8_us": round(t_dn, 3), "speedup_vs_dense": round(t_dn / t_sp, 3),
            "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1),
                         "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "kernel": "sp24_gemm_packed",
                         "peak_source": f"{peaks['source']} bf16 burst x4 (2:4 sparse FP8 dense-equivalent)",
                         "traffic": load_traffic().get("prefill:sp24_gemm_packed")},
            "dense_tflops": round(flops / t_dn / 1e6, 1),
            "timing": f"CUDA graph of {reps} launches over {len(ps)} rotating packed weight copies "
                      f"({len(pd)} dense), inputs larger than L2"}


def speedup_headlines(device, peaks, reps=20):
    """The sparse-over-dense targets next to the decode headline: the MLP
    down-projection (M256 N4096 K14336, HBM-bound) against the dense FP8
    GEMM of the same family, and the 6:8 GEMM over K' = 6144 (lifted X,
    6:8 weights in the packed layout) against the dense FP8 GEMM over
    K = 4096 at M = 2048 (tensor-bound), each a CUDA graph of `reps`
    launches over rotating weight copies larger than L2, CUDA events on the
    launching stream."""
    import torch

    import structured_sparse_fp8_b200 as sp
    from structured_sparse_fp8_b200 import workloads as WL
    lib = sp._lib.load()
    ws = sp.Workspace(device)
    status = torch.zeros(1, dtype=torch.int32, device=device)

    def bf(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)

    def pool(t):
        return [t] + [t.clone() for _ in range(max(1, -(-3 * L2_BYTES // t.numel())) - 1)]

    def graph_us(fn):
        fn(0)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for r in range(reps):
                fn(r)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) * 1e3 / reps

    out = {}
    wl = WORKLOADS["downproj"]
    m, n, k = wl["ms"][0], wl["n"], wl["k"]
    w, x = bf(WL.weight_bits(wl["cfg"])), bf(WL.activation_bits(wl["cfg"], m))
    packed, sw = sp.sp24_prune_compress_packed(w, workspace=ws)
    wq, swd = sp.fp8_quantize_pertensor(w, workspace=ws)
    xq, sx = sp.fp8_quantize_pertensor(x, workspace=ws)
    del w, x
    y = torch.empty((m, n), dtype=torch.bfloat16, device=device)
    ps, pd = pool(packed), pool(wq)
    ws.get(max(lib.sp24_workspace_size(sp._lib.OP_GEMM_PACKED, m, n, k, 0),
               lib.sp24_workspace_size(sp._lib.OP_GEMM_DENSE, m, n, k, 0)) + 4096)
    t_sp = graph_us(lambda r: sp.sp24_gemm_packed(xq, sx, ps[r % len(ps)], sw, n, out=y, status=status,
                                                  workspace=ws))
    t_dn = graph_us(lambda r: sp.fp8_gemm_dense(xq, sx, pd[r % len(pd)], swd, out=y, status=status,
                                                workspace=ws))
    gbs = bytes_sparse_gemm(m, n, k) / t_sp / 1e3
    out["down_proj"] = {"workload": wl["name"], "sparse_us": round(t_sp, 3), "dense_fp8_us": round(t_dn, 3),
                        "speedup_vs_dense": round(t_dn / t_sp, 3), "sparse_gbs": round(gbs, 1),
                        "frac_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    del ps, pd, packed, wq, xq, y
    wl = WORKLOADS["slide68"]
    m, n, k = 2048, wl["n"], wl["k"]
    kp = k // 2 * 3
    w, x = bf(WL.weight_bits(wl["cfg"])), bf(WL.activation_bits(wl["cfg"], m))
    packed, sw = sp.slide68_decompose_packed(w, workspace=ws)
    xl, sxl = sp.slide68_lift(x, workspace=ws)
    wq, swd = sp.fp8_quantize_pertensor(w, workspace=ws)
    xq, sx = sp.fp8_quantize_pertensor(x, workspace=ws)
    del w, x
    y = torch.empty((m, n), dtype=torch.bfloat16, device=device)
    ps, pd = pool(packed), pool(wq)
    ws.get(max(lib.sp24_workspace_size(sp._lib.OP_GEMM_PACKED, m, n, kp, 0),
               lib.sp24_workspace_size(sp._lib.OP_GEMM_DENSE, m, n, k, 0)) + 4096)
    t_sp = graph_us(lambda r: sp.sp24_gemm_packed(xl, sxl, ps[r % len(ps)], sw, n, out=y, status=status,
                                                  workspace=ws))
    t_dn = graph_us(lambda r: sp.fp8_gemm_dense(xq, sx, pd[r % len(pd)], swd, out=y, status=status,
                                                workspace=ws))
    tf = 2.0 * m * n * kp / t_sp / 1e6
    out["slide68_m2048"] = {"workload": f"6:8 W[{n},{k}] over K'={kp} vs dense FP8 over K={k}, M={m}",
                            "sparse_us": round(t_sp, 3), "dense_fp8_us": round(t_dn, 3),
                            "speedup_vs_dense": round(t_dn / t_sp, 3),
                            "sparse_tflops_dense_equiv": round(tf, 1),
                            "frac_tensor": round(tf / (peaks["bf16_tflops"] * 4.0), 4)}
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device status word set during the speed-up timing"
    out["timing"] = f"CUDA graphs of {reps} launches over rotating weight copies, inputs larger than L2"
    return out


# ---------------------------------------------------------------- single-kernel cases
# `bench.py --kernel-case NAME` runs one library call on a fixed workload
# shape, twice as warm-up and then three times, and exits: the command the
# per-kernel ncu summaries under profiles/ are captured from (one kernel per
# case; inputs larger than L2 where the workload is).

def kernel_case(name, device):
    import torch

    import structured_sparse_fp8_b200 as sp
    from structured_sparse_fp8_b200 import workloads as WL

    def bf(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)

    ws = sp.Workspace(device)
    ws.get(256 << 20)
    w2 = None

    def w_decode():
        return bf(WL.weight_bits(2))

    if name == "quantize_small":                 # X[32, 4096] per-tensor E4M3, one thread-block cluster
        x = bf(WL.activation_bits(2, 32))
        call = lambda: sp.fp8_quantize_pertensor(x, workspace=ws)
    elif name == "quantize":                     # X[4096, 4096] per-tensor E4M3
        x = bf(WL.activation_bits(3, 4096))
        call = lambda: sp.fp8_quantize_pertensor(x, workspace=ws)
    elif name == "lift":                         # X[2048, 4096] 6:8 lift + quantise
        x = bf(WL.activation_bits(5, 2048))
        call = lambda: sp.slide68_lift(x, workspace=ws)
    elif name == "prune_packed":                 # W[11008, 4096] 2:4 prune + compress, packed
        w = w_decode()
        call = lambda: sp.sp24_prune_compress_packed(w, workspace=ws)
    elif name == "slide68_packed":               # W[4096, 4096] 6:8 decompose, packed
        w = bf(WL.weight_bits(5))
        call = lambda: sp.slide68_decompose_packed(w, workspace=ws)
    elif name in ("gemm_packed_decode", "gemm_dense_decode", "gemm_int8_decode", "fused_decode"):
        m = 1 if name == "fused_decode" else 64  # the fused call is one launch up to M*K = 8192
        w = w_decode()
        x = bf(WL.activation_bits(2, m))
        if name == "gemm_dense_decode":
            wq, swd = sp.fp8_quantize_pertensor(w, workspace=ws)
            xq, sx = sp.fp8_quantize_pertensor(x, workspace=ws)
            call = lambda: sp.fp8_gemm_dense(xq, sx, wq, swd, workspace=ws)
        elif name == "gemm_int8_decode":
            c = sp.sp24_prune_compress_int8(w, workspace=ws)
            packed = sp.sp24_pack_weights(c["values"].view(torch.uint8), c["meta"])
            xq, sx = sp.int8_quantize_pertensor(x, workspace=ws)
            call = lambda: sp.sp24_gemm_int8_packed(xq, sx, packed, c["scale"], w.shape[0], workspace=ws)
        else:
            packed, sw = sp.sp24_prune_compress_packed(w, workspace=ws)
            xq, sx = sp.fp8_quantize_pertensor(x, workspace=ws)
            if name == "fused_decode":
                call = lambda: sp.sp24_quantize_gemm_packed(x, packed, sw, w.shape[0], workspace=ws)
            else:
                call = lambda: sp.sp24_gemm_packed(xq, sx, packed, sw, w.shape[0], workspace=ws)
    elif name == "gemm_bf16_downproj":           # M256 N4096 K14336, bf16 operands
        w = bf(WL.weight_bits(4))
        x = bf(WL.activation_bits(4, 256))
        c = sp.sp24_prune_compress(w, "bf16", workspace=ws)
        call = lambda: sp.sp24_gemm(x, None, c["values"], c["meta"], None, dtype="bf16", workspace=ws)
    elif name == "gemm_scaled_prefill":          # M4096 N12288 K4096, per-token x per-channel scales
        w = bf(WL.weight_bits(3))
        x = bf(WL.activation_bits(3, 4096))
        c = sp.sp24_prune_compress_perchannel(w)
        packed = sp.sp24_pack_weights(c["values"], c["meta"])
        xq, sx = sp.fp8_quantize_pertoken(x)
        call = lambda: sp.sp24_gemm_packed_scaled(xq, sx, packed, c["scales"], w.shape[0], workspace=ws)
    elif name == "pertoken":                     # X[4096, 4096] per-token E4M3
        x = bf(WL.activation_bits(3, 4096))
        call = lambda: sp.fp8_quantize_pertoken(x)
    elif name == "perchannel":                   # W[11008, 4096] per-channel 2:4 prune
        w = w_decode()
        call = lambda: sp.sp24_prune_compress_perchannel(w)
    elif name == "int8_quantize":                # X[4096, 4096] per-tensor INT8
        x = bf(WL.activation_bits(3, 4096))
        call = lambda: sp.int8_quantize_pertensor(x, workspace=ws)
    elif name == "int8_prune":                   # W[11008, 4096] INT8 2:4 weight path
        w = w_decode()
        call = lambda: sp.sp24_prune_compress_int8(w, workspace=ws)
    elif name == "fp4_quantize":                 # X[4096, 4096] per-tensor FP4 E2M1
        x = bf(WL.activation_bits(3, 4096))
        call = lambda: sp.fp4_quantize_pertensor(x, workspace=ws)
    elif name == "fp4_prune":                    # W[11008, 4096] FP4 2:4 weight path
        w = w_decode()
        call = lambda: sp.sp24_prune_compress_fp4(w, workspace=ws)
    elif name == "gemm_fp4_decode":              # M64 N11008 K4096, FP4 A and B
        w = w_decode()
        x = bf(WL.activation_bits(2, 64))
        c = sp.sp24_prune_compress_fp4(w, workspace=ws)
        xq, sx = sp.fp4_quantize_pertensor(x, workspace=ws)
        call = lambda: sp.sp24_gemm_fp4(xq, sx, c["values"], c["meta"], c["scale"], workspace=ws)
    elif name in ("slide46_decompose", "slide46_lift"):   # 4:6 at K = 4608 (K' = 6144)
        if name == "slide46_decompose":
            w = bf(WL.random_bits((4096, 4608), 2301, scale=0.02))
            call = lambda: sp.slide_decompose(w, 3, workspace=ws)
        else:
            x = bf(WL.random_bits((2048, 4608), 2302))
            call = lambda: sp.slide_lift(x, 3, workspace=ws)
    else:
        raise SystemExit(f"unknown kernel case {name}")
    for _ in range(5):
        call()
    torch.cuda.synchronize()
    del w2
    print(json.dumps({"kernel_case": name, "ok": True}))


# ---------------------------------------------------------------- CPU oracle

def oracle_sample_step(wl, rows, rng_seed, m_cap=64):
    """One bounded oracle step: the workload's weight op on `rows` rows of W,
    then for every M (capped at `m_cap` token rows): activation quantisation
    and the float64 GEMM against those weight rows.  Returns (algorithmic
    bytes of the sample, seconds)."""
    from oracle import sp24_oracle as O
    from structured_sparse_fp8_b200 import workloads as WL
    k = wl["k"]
    w = WL.weight_bits(wl["cfg"], n=rows, k=k, layer=rng_seed + 1)
    xs = {min(m, m_cap): WL.activation_bits(wl["cfg"], m)[:min(m, m_cap)] for m in wl["ms"]}
    t0 = time.perf_counter()
    nbytes = 0
    if wl["pattern"] == "6:8":
        d = O.slide68_decompose(w, "e4m3")
        wv = O.e4m3_decode(d["expanded"])
        sw = d["scale"]
        nbytes += bytes_slide68(rows, k)
        kc = 3 * k // 2
    else:
        c = O.sp24_prune_compress(w, "e4m3")
        wv = O.e4m3_decode(O.decompress24(c["values"], c["meta"], k))
        sw = c["scale"]
        nbytes += bytes_prune24(rows, k)
        kc = k
    for m, x in xs.items():
        if wl["pattern"] == "6:8":
            xq, sx = O.slide68_lift(x)
            nbytes += bytes_lift(m, k)
        else:
            xq, sx = O.quantize_pertensor(x)
            nbytes += bytes_quant(m, k)
        O.gemm_ref(O.e4m3_decode(xq), wv, sx, sw)
        nbytes += bytes_sparse_gemm(m, rows, kc)
    return nbytes, time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def cpu_baseline(wl, budget_s=10.0, rows=128):
    total_b, total_t, n = 0, 0.0, 0
    while total_t < budget_s and n < 200:
        b, t = oracle_sample_step(wl, rows, n)
        total_b += b
        total_t += t
        n += 1
    return {"value": round(total_b / total_t / 1e9, 4), "unit": "GB/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{n} oracle steps, each on {rows} of {wl['n']} weight rows and up to 64 "
                      f"token rows per M, {total_t:.1f} s of CPU work"}


def run_reference(args, wl):
    rows = 64 if wl["ms"][-1] >= 1024 else 128
    for s in range(args.warmup):
        oracle_sample_step(wl, rows, s)
    total_b, total_t = 0, 0.0
    for s in range(args.steps):
        b, t = oracle_sample_step(wl, rows, s)
        total_b += b
        total_t += t
    value = total_b / total_t / 1e9
    cb = {"value": round(value, 4), "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
          "sample": f"each step: the oracle on {rows} of {wl['n']} weight rows and up to 64 "
                    "token rows per M of the workload"}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_t / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; see workloads.py)",
            "config": {"workload": wl["name"], "n": wl["n"], "k": wl["k"], "m": list(wl["ms"]),
                       "parallelism": "cpu oracle"},
            "cpu_baseline": cb,
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["sp24", "reference"], default="sp24")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode")
    ap.add_argument("--no-compare", action="store_true", help="skip the dense-FP8 comparison")
    ap.add_argument("--unfused", action="store_true",
                    help="quantise activations in their own launch at every M (no fused quantise + GEMM)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-case", default=None,
                    help="run one library call on a fixed shape five times and exit (for per-kernel ncu captures)")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the prefill-shaped (tensor-bound) GEMM timed next to the decode headline")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = WORKLOADS[args.workload]
    if args.kernel_case:
        import torch

        import __graft_entry__
        __graft_entry__.build()
        kernel_case(args.kernel_case, torch.device("cuda", 0))
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, wl)), flush=True)
        return

    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=__import__("torch").device("cuda", local_rank))
    line, gw = run_gpu(args, wl, rank, world, local_rank)
    if rank == 0:
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
