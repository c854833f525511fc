"""Benchmark of the FFD decode path on B200: microseconds per decode step.

A step is one pass of the whole hot path on one batch: the int4 re-quantisation
of each sequence's last key block (the append step) followed by the fused
selector + computer + split-merge kernel.  Default workload: the long-context
configuration (B1, 32 query / 8 kv heads, 131072 tokens, block 64, split 64,
delta 3, drift + 16 needles).

Contract: ``python bench.py --gpus N --steps K --warmup W`` prints one JSON line
on rank 0.  N > 1 runs one independent replica per GPU (weak scaling; the
method has no cross-GPU exchange at this size).  ``--impl reference`` times the
CPU oracle instead (rank 0 only).

Timing: K steps are replayed from CUDA graphs between two CUDA events on the
launching stream, after W warm-up steps, bracketed by a barrier and a device
synchronise; the max over ranks is reported.  Each decode launch inside the
timed region is bracketed by graph-captured timing events, which give the
dominant kernel's average duration for the roofline.  Inputs are rotated over
enough copies of the cache that each step's working set is evicted from L2
before it is reused.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import ffd_workloads as fw  # noqa: E402

DEFAULT_WORKLOAD = "long128k"
REFERENCES = {"running": 0, "sink_local": 1, "sink_local_fixed": 2}  # FFD_REFERENCE_* of include/ffd.h
METRIC = "us per decode step (128K ctx) + effective HBM TB/s of the fused decode kernel"
UNIT = "us/step"


# ------------------------------------------------------------ distributed --

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def dist_init(backend: str, world: int):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def dist_barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def dist_max(value: float, world: int, device=None) -> float:
    """Max of a float over all ranks (every rank takes part)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_sum(value: float, world: int, device=None) -> float:
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a window."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, out_path=None):
        self.gpu_index = gpu_index
        self.out_path = out_path
        self.proc = None
        self.lines = []
        self.t_start = self.t_stop = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which):
        if which == "start":
            self.t_start = time.time()
        else:
            self.t_stop = time.time()

    def stop(self):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.out_path:
            with open(self.out_path, "w") as f:
                f.write(self.FIELDS + "\n")
                for t, line in self.lines:
                    f.write(f"{t:.3f},{line}\n")

    def summary(self):
        rows = []
        for t, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((t, float(parts[1]), float(parts[2]), float(parts[3]), parts[4:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        window = [r for r in rows if self.t_start and r[0] >= self.t_start - 0.05
                  and (self.t_stop is None or r[0] <= self.t_stop + 0.05)]
        use = window if window else rows
        reasons = set()
        names = ("active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap")
        for r in use:
            for name, val in zip(names[1:], r[4][1:]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(np.median([r[1] for r in use])), "sm_max_mhz": use[0][2],
                "reasons": sorted(reasons), "samples": len(use),
                "power_w_max": max(r[3] for r in use), "in_timed_window": bool(window)}


# ------------------------------------------------------------ measurement --

def algorithmic_bytes(w, lengths, kept_tokens, dense: bool) -> dict:
    """Bytes one fused decode step must move (one launch): the last key
    block's re-quantisation (its valid K rows read, its packed rows and scales
    written), packed keys + scales of the valid blocks (skipped when dense), K
    and V of the valid tokens of the kept blocks, q, out, mask and the split
    partials (written and read once)."""
    T, S, G = w.block_size, w.split_blocks, w.group
    scan = requant = partials = 0
    for n in lengths:
        n = int(n)
        nb = -(-n // T)
        nsplit = -(-nb // S)
        if n > 0:
            requant += w.num_kv_heads * ((n - (nb - 1) * T) * 256 + T * 64 + 256)
        if not dense:
            scan += w.num_kv_heads * (n * 64 + nb * 256)
        partials += w.num_kv_heads * nsplit * G * 130 * 4 * 2
    kv = int(kept_tokens) * 2 * 128 * 2
    qo = 2 * w.batch * w.num_q_heads * 128 * 2
    mask = w.batch * w.num_kv_heads * math.ceil(w.capacity // T / 32) * 4
    return {"requant": requant, "scan": scan, "kv": kv, "q_out_mask": qo + mask,
            "partials": partials, "total": requant + scan + kv + qo + mask + partials}


def algorithmic_bytes_tr(w, lengths, kept_tokens, dense: bool) -> dict:
    """The same for the thumbnail + residual format: the re-quantisation
    writes thumbnail (32 B), residual (128 B) rows and scales; the scan reads
    thumbnails + scales of the valid blocks; the computer reads residuals and
    V of the kept tokens (their thumbnails and scales were already read by the
    scan; dense mode reads them here instead of in a scan)."""
    T, S, G = w.block_size, w.split_blocks, w.group
    scan = requant = partials = dense_extra = 0
    for n in lengths:
        n = int(n)
        nb = -(-n // T)
        nsplit = -(-nb // S)
        if n > 0:
            requant += w.num_kv_heads * ((n - (nb - 1) * T) * 256 + T * (32 + 128) + 256)
        if dense:
            dense_extra += w.num_kv_heads * (n * 32 + nb * 256)
        else:
            scan += w.num_kv_heads * (n * 32 + nb * 256)
        partials += w.num_kv_heads * nsplit * G * 130 * 4 * 2
    kv = int(kept_tokens) * (128 + 256) + dense_extra
    qo = 2 * w.batch * w.num_q_heads * 128 * 2
    mask = w.batch * w.num_kv_heads * math.ceil(w.capacity // T / 32) * 4
    return {"requant": requant, "scan": scan, "kv": kv, "q_out_mask": qo + mask,
            "partials": partials, "total": requant + scan + kv + qo + mask + partials}


def kept_tokens_from_mask(w, lengths, mask) -> tuple:
    T = w.block_size
    nblk = w.capacity // T
    kept_blocks = kept_tok = valid_blocks = 0
    for b in range(w.batch):
        n = int(lengths[b])
        nb = -(-n // T)
        valid_blocks += nb * w.num_kv_heads
        for g in range(w.num_kv_heads):
            bits = np.unpackbits(mask[b, g].astype("<u4").view(np.uint8), bitorder="little")[:nblk]
            idx = np.nonzero(bits[:nb])[0]
            kept_blocks += len(idx)
            kept_tok += int(np.minimum(T, n - idx * T).sum())
    return kept_blocks, valid_blocks, kept_tok


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy read+write)"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback 6.65 TB/s"


# the sources the decode kernel and its launch are built from
DECODE_SOURCES = ("api.cu", "decode.cu", "ffd_internal.h", "ffd_ptx.cuh", "ffd_quant.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_long_context_ffd_b200", "csrc")
    for name in DECODE_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic_per_launch(workload: str, dense: bool, fmt: str = "int4"):
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current kernel sources (else None)."""
    mode = "dense" if dense else "sparse"
    prefix = "decode_tr" if fmt == "tr" else "decode"
    path = os.path.join(ROOT, "profiles", f"{prefix}_{workload}_ncu.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m = re.search(rf"traffic_{mode}_bytes_per_launch:\s*([0-9]+)\s+source_sha:\s*([0-9a-f]+)", text)
    if not m or m.group(2) != kernel_source_hash():
        return None
    return int(m.group(1))


# ------------------------------------------------------------------ GPU arm --

class Replica:
    """One GPU's copy of the workload: R rotated layer copies of the cache,
    with the int4 scan copy ("int4") or thumbnails + residuals ("tr")."""

    def __init__(self, w, inp, device, layers, fmt="int4"):
        import torch
        from sparse_long_context_ffd_b200 import ffd
        self.torch, self.ffd = torch, ffd
        self.w, self.device, self.fmt = w, device, fmt
        self.shape = ffd.make_shape(w.batch, w.num_q_heads, w.num_kv_heads, w.capacity,
                                    w.block_size, w.split_blocks)

        def bf16(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(
                torch.bfloat16).to(device)

        q0, k0, v0 = bf16(inp["q"]), bf16(inp["k"]), bf16(inp["v"])
        self.lengths = torch.from_numpy(np.ascontiguousarray(inp["lengths"])).to(device)
        self.layers = []
        for i in range(layers):
            if fmt == "tr":
                bufs = ffd.ThumbResidBuffers(self.shape, device=device)
            else:
                bufs = ffd.DecodeBuffers(self.shape, device=device)
            layer = dict(q=q0 if i == 0 else q0.clone(), k=k0 if i == 0 else k0.clone(),
                         v=v0 if i == 0 else v0.clone(), bufs=bufs)
            if fmt == "tr":
                ffd.quantize_keys_tr(self.shape, layer["k"], self.lengths, 0, bufs.k_thumb,
                                     bufs.k_resid, bufs.k_scales)
            else:
                ffd.quantize_keys(self.shape, layer["k"], self.lengths, 0, bufs.k_packed,
                                  bufs.k_scales)
            self.layers.append(layer)
        torch.cuda.synchronize(device)

    reference = 0  # FFD_REFERENCE_RUNNING_MAX; set from --reference

    def step(self, i, delta, ev=None, fused=True):
        """One decode step: re-quantise the last key block, then the fused
        decode -- one launch (ffd_decode_step), or two (ffd_quantize_keys +
        ffd_decode) when fused is False."""
        L = self.layers[i % len(self.layers)]
        b = L["bufs"]
        tr = self.fmt == "tr"
        if not fused:
            if tr:
                self.ffd.quantize_keys_tr(self.shape, L["k"], self.lengths, self.ffd.FFD_LAST_BLOCK,
                                          b.k_thumb, b.k_resid, b.k_scales)
            else:
                self.ffd.quantize_keys(self.shape, L["k"], self.lengths, self.ffd.FFD_LAST_BLOCK,
                                       b.k_packed, b.k_scales)
        if ev is not None:
            ev[0].record()
        if tr:
            self.ffd.decode_tr(self.shape, L["q"], L["k"], L["v"], b.k_thumb, b.k_resid, b.k_scales,
                               self.lengths, delta, b.out, b.mask, b.workspace,
                               reference=self.reference, requant_last=fused)
        else:
            self.ffd.decode_ex(self.shape, L["q"], L["k"], L["v"], b.k_packed, b.k_scales,
                               self.lengths, delta, b.out, b.mask, b.workspace,
                               reference=self.reference, requant_last=fused)
        if ev is not None:
            ev[1].record()

    def check_flags(self):
        for L in self.layers:
            flags = self.ffd.check_device_status(L["bufs"].workspace)
            if flags:
                raise RuntimeError(f"device flags {flags:#x}")


NOMINAL_HBM_GBS = 8000.0  # the B200 HBM3e figure the method's target is stated against


def read_probe_gbs(device, gib=4, iters=20):
    """Streaming-read bandwidth of this GPU, measured in the run by the
    library's read probe (ffd_read_probe) over a buffer of `gib` GiB, far
    above the L2: one-pass reads, the access kind the decode step makes."""
    import torch
    from sparse_long_context_ffd_b200 import ffd
    buf = torch.empty(gib << 30, dtype=torch.uint8, device=device)
    sink = torch.zeros(1, dtype=torch.int32, device=device)
    for _ in range(3):
        ffd.read_probe(buf, sink)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    start.record()
    for _ in range(iters):
        ffd.read_probe(buf, sink)
    end.record()
    torch.cuda.synchronize(device)
    ms = start.elapsed_time(end) / iters
    del buf
    return buf_bytes_gbs(gib << 30, ms)


def buf_bytes_gbs(nbytes, ms):
    return nbytes / (ms * 1e-3) / 1e9


def error_vs_dense(rep, delta):
    """The sparse step's output against the same kernel in dense mode
    (delta = +inf) on the same inputs: max-abs, mean-abs and relative L2 over
    all output elements (what the Top-delta selection costs in accuracy)."""
    torch = rep.torch
    out = rep.layers[0]["bufs"].out
    rep.step(0, delta)
    torch.cuda.synchronize(rep.device)
    sparse = out.float().cpu().numpy().astype(np.float64)
    rep.step(0, float("inf"))
    torch.cuda.synchronize(rep.device)
    dense = out.float().cpu().numpy().astype(np.float64)
    d = sparse - dense
    return {"max_abs": float(np.abs(d).max()), "mean_abs": float(np.abs(d).mean()),
            "rel_l2": float(np.linalg.norm(d) / max(float(np.linalg.norm(dense)), 1e-30))}


def time_graph_steps(rep, delta, steps, warmup, world, device, sampler=None, spg=None, fused=True):
    """Replay K steps from CUDA graphs; returns (total_ms, per-decode ms list)."""
    torch = rep.torch
    stream = torch.cuda.Stream(device)
    spg = spg or min(steps, 200)
    spg = max(1, spg)
    graphs = {}

    def capture(n):
        ev = [(torch.cuda.Event(enable_timing=True, external=True),
               torch.cuda.Event(enable_timing=True, external=True)) for _ in range(n)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for i in range(2):  # untimed eager passes on the capture stream
                rep.step(i, delta, fused=fused)
        torch.cuda.synchronize(device)
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                rep.step(i, delta, ev[i], fused=fused)
        return g, ev

    full, rem = divmod(steps, spg)
    graphs[spg] = capture(spg)
    if rem:
        graphs[rem] = capture(rem)
    # warm-up
    wfull, wrem = divmod(warmup, spg)
    for _ in range(wfull):
        graphs[spg][0].replay()
    if wrem:
        if wrem not in graphs:
            graphs[wrem] = capture(wrem)
        graphs[wrem][0].replay()
    torch.cuda.synchronize(device)
    dist_barrier(world, device)
    torch.cuda.synchronize(device)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.mark("start")
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(full):
            graphs[spg][0].replay()
        if rem:
            graphs[rem][0].replay()
        end.record(stream)
    torch.cuda.synchronize(device)
    if sampler:
        sampler.mark("stop")
    dist_barrier(world, device)
    total_ms = start.elapsed_time(end)
    per = []
    try:
        last = graphs[rem][1] if rem else graphs[spg][1]
        per = [a.elapsed_time(b) for a, b in last]
    except RuntimeError:
        per = []
    return total_ms, per, spg


def time_gated_decodes(rep, delta, n, device):
    """Fallback per-launch timing: the stream is held by a sleep kernel while
    the host queues n steps, so each event pair brackets only the kernel."""
    torch = rep.torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    torch.cuda.synchronize(device)
    torch.cuda._sleep(int(2e8))
    for i in range(n):
        rep.step(i, delta, ev[i])
    torch.cuda.synchronize(device)
    return [a.elapsed_time(b) for a, b in ev]


def e2e_steps(w, inp, device, delta, steps):
    """End-to-end decode steps through the public API with host buffers.

    graph (the reported value): sparse_long_context_ffd_b200.step.DecodeStep,
    one call per step into the library's native step graph: the pinned H2D
    copy of the query and the new key/value rows, then the fused append +
    re-quantisation + decode launch (ffd_decode_append), which writes output
    and mask straight into pinned host memory; the call waits for the graph.
    eager: H2D, the launch and a D2H copy issued from Python each step."""
    import torch
    from sparse_long_context_ffd_b200 import ffd
    from sparse_long_context_ffd_b200.step import DecodeStep
    shape = ffd.make_shape(w.batch, w.num_q_heads, w.num_kv_heads, w.capacity, w.block_size,
                           w.split_blocks)

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    k = bf16(inp["k"]).to(device)
    v = bf16(inp["v"]).to(device)
    lengths_h = inp["lengths"]
    lengths = torch.from_numpy(np.ascontiguousarray(lengths_h)).to(device)
    B = w.batch
    last = [int(lengths_h[b]) - 1 for b in range(B)]
    # the step appends each sequence's last token again: every step does the
    # same work on the same lengths
    st = DecodeStep(shape, k, v, lengths, delta)
    st.host_q.copy_(bf16(inp["q"]))
    st.host_k_new.copy_(torch.stack([bf16(inp["k"][b, :, last[b]]) for b in range(B)]))
    st.host_v_new.copy_(torch.stack([bf16(inp["v"][b, :, last[b]]) for b in range(B)]))
    stream = torch.cuda.current_stream(device)

    def eager():
        st._body()
        stream.synchronize()

    def timed(fn):
        for _ in range(3):
            fn()
        t0 = time.perf_counter()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(steps):
            fn()
        end.record()
        torch.cuda.synchronize(device)
        return start.elapsed_time(end) / steps, (time.perf_counter() - t0) * 1e3 / steps

    graph_ms, graph_wall = timed(st.step)
    eager_ms, eager_wall = timed(eager)
    if st.check():
        raise RuntimeError("device flags raised in the end-to-end steps")
    return {"event_ms_per_step": graph_ms, "wall_ms_per_step": graph_wall,
            "eager_event_ms_per_step": eager_ms, "eager_wall_ms_per_step": eager_wall,
            "h2d": st.h2d_bytes, "d2h": st.d2h_bytes}


def layer_steps(w, inp, device, delta, steps):
    """The stand-in attention layer (random weights, hidden = Hq x 128): one
    graph per step with the pinned H2D of x, the q/k/v projections, the FFD
    append + decode, the output projection and the D2H of y."""
    import torch
    from sparse_long_context_ffd_b200 import ffd
    from sparse_long_context_ffd_b200.step import StandInAttentionLayer
    shape = ffd.make_shape(w.batch, w.num_q_heads, w.num_kv_heads, w.capacity, w.block_size,
                           w.split_blocks)

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    k = bf16(inp["k"]).to(device)
    v = bf16(inp["v"]).to(device)
    lengths = torch.from_numpy(np.ascontiguousarray(inp["lengths"])).to(device)
    hidden = w.num_q_heads * 128
    # every step re-appends at the same position, so each does the same work
    layer = StandInAttentionLayer(shape, hidden, k, v, lengths, delta, seed=w.seed, advance=False)
    layer.host_x.copy_(torch.randn((w.batch, hidden)).to(torch.bfloat16))
    for _ in range(3):
        layer.step()
    torch.cuda.synchronize(device)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        layer.step()
    end.record()
    torch.cuda.synchronize(device)
    if layer.core.check():
        raise RuntimeError("device flags raised in the layer steps")
    return {"us_per_step": start.elapsed_time(end) / steps * 1e3, "hidden": hidden,
            "how": "StandInAttentionLayer: one CUDA graph per step (H2D x, q/k/v GEMMs, "
                   "ffd_decode_append, output GEMM, D2H y), random bf16 weights"}


# ------------------------------------------------------------- CPU oracle --

_ORACLE_RATE = {}


def oracle_step_sample(w, inp, budget_s: float):
    """Time the CPU oracle, as it stands (one thread), on a bounded sample of
    one decode step: one kv-head group of sequence 0 (its last block
    re-quantised, then scan, selection and attention) over a prefix of whole
    splits sized to the time budget.  Returns (us per full step scaled by token
    count, description, seconds used)."""
    import oracle
    T, S, G = w.block_size, w.split_blocks, w.group
    n0 = int(inp["lengths"][0])
    split_tok = S * T
    key = (w.name, w.seed)
    if key not in _ORACLE_RATE:
        n = min(n0, split_tok)
        c = -(-n // T) * T  # cache rows of the sample: whole blocks
        p, s = oracle.quantize_keys(inp["k"][:1, :1, :c], np.array([n], np.int32), T)
        t0 = time.perf_counter()
        oracle.decode(inp["q"][:1, :G], inp["k"][:1, :1, :c], inp["v"][:1, :1, :c], p, s,
                      np.array([n], np.int32), T, S, w.delta)
        _ORACLE_RATE[key] = max((time.perf_counter() - t0) / n, 1e-9)
    rate = _ORACLE_RATE[key]
    n = int(budget_s / rate) // split_tok * split_tok
    n = max(min(n0, split_tok), min(n0, n))
    c = -(-n // T) * T
    k1, v1 = inp["k"][:1, :1, :c], inp["v"][:1, :1, :c]
    p1, s1 = oracle.quantize_keys(k1, np.array([n], np.int32), T)
    ln = np.array([n], np.int32)
    reps, tokens = 0, 0
    t0 = time.perf_counter()
    while True:
        oracle.quantize_keys(k1, ln, T, -1, p1, s1)
        oracle.decode(inp["q"][:1, :G], k1, v1, p1, s1, ln, T, S, w.delta)
        reps += 1
        tokens += n
        used = time.perf_counter() - t0
        if used >= 0.8 * budget_s or n < n0:
            break
    full_tokens = int(np.sum(inp["lengths"])) * w.num_kv_heads
    us = used / tokens * full_tokens * 1e6
    desc = (f"{reps} x one kv-head group (G={G}) of sequence 0 over its first {n} tokens, "
            f"scaled by token count to the full step ({full_tokens} token-heads)")
    return us, desc, used


def _oracle_unit_worker(args):
    """One host process's share of the parallel oracle sample: `reps` decode
    steps (last-block re-quantisation + the whole oracle step) of one kv-head
    group over its first n tokens.  Returns the seconds spent computing."""
    q_g, k_row, v_row, n, T, S, delta, reps = args
    import oracle
    ln = np.array([n], np.int32)
    p, s = oracle.quantize_keys(k_row, ln, T)
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.quantize_keys(k_row, ln, T, -1, p, s)
        oracle.decode(q_g, k_row, v_row, p, s, ln, T, S, delta)
    return time.perf_counter() - t0


def oracle_vs_gpu(w, inp, gpu_out, gpu_mask, pseudo_max=False) -> dict:
    """The oracle on the whole first kv-head group of sequence 0 (all its
    tokens) against the GPU's output rows and mask row of the same step."""
    import oracle
    T, S, G = w.block_size, w.split_blocks, w.group
    ln = np.ascontiguousarray(inp["lengths"][:1])
    k1, v1 = inp["k"][:1, :1], inp["v"][:1, :1]
    p1, s1 = oracle.quantize_keys(k1, ln, T)
    out, mask, _ = oracle.decode(inp["q"][:1, :G], k1, v1, p1, s1, ln, T, S, w.delta,
                                 pseudo_max=pseudo_max)
    d = np.abs(out[0] - gpu_out)
    return {"heads": f"query heads 0..{G - 1} of sequence 0 (kv-head 0), all {int(ln[0])} tokens",
            "mask_equal": bool(np.array_equal(mask[0, 0], gpu_mask)),
            "max_abs": float(d.max()), "mean_abs": float(d.mean())}


def host_cpu() -> dict:
    """The host the oracle ran on: CPU model and logical CPU count."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"model": model, "nproc": os.cpu_count()}


def oracle_parallel_sample(w, inp, budget_s: float):
    """The oracle as it stands, on every host core at once: one process per
    core, each running one decode step (last-block re-quantisation + the whole
    oracle step) of one kv-head group over a window of whole splits.  Jobs go
    round-robin over all (sequence, kv-head) units of the step, and each job's
    window starts at a different split of its sequence, so the sample covers
    the whole workload; splits are independent units of the method, so a
    window is a fair share of the step.  All start together; the slowest sets
    the time, scaled by token count to the full step.  Returns (us per full
    step, cores, description)."""
    import concurrent.futures
    import multiprocessing
    T, S, G = w.block_size, w.split_blocks, w.group
    cores = max(1, os.cpu_count() or 1)
    split_tok = S * T
    rate = _ORACLE_RATE.get((w.name, w.seed))
    if rate is None:
        oracle_step_sample(w, inp, min(budget_s, 2.0))
        rate = _ORACLE_RATE[(w.name, w.seed)]
    lengths = inp["lengths"]
    units = [(b, g) for b in range(w.batch) for g in range(w.num_kv_heads) if int(lengths[b]) > 0]
    n = max(split_tok, int(budget_s / rate) // split_tok * split_tok)
    jobs = []
    for c in range(cores):
        b, g = units[c % len(units)]
        nb_tok = int(lengths[b])
        win = min(n, nb_tok)
        nsplits = max(1, -(-nb_tok // split_tok))
        t0 = ((c // len(units)) * 7 + c) % nsplits * split_tok  # a different split per job
        t0 = min(t0, max(0, nb_tok - win)) // split_tok * split_tok
        win = min(win, nb_tok - t0)
        cap_j = -(-win // T) * T  # the window's cache rows: whole blocks
        jobs.append((np.ascontiguousarray(inp["q"][b:b + 1, g * G:(g + 1) * G]),
                     np.ascontiguousarray(inp["k"][b:b + 1, g:g + 1, t0:t0 + cap_j]),
                     np.ascontiguousarray(inp["v"][b:b + 1, g:g + 1, t0:t0 + cap_j]), win, T, S,
                     w.delta, 1))
    ctx = multiprocessing.get_context("spawn")  # the parent has a CUDA context
    with concurrent.futures.ProcessPoolExecutor(max_workers=cores, mp_context=ctx) as ex:
        list(ex.map(_oracle_unit_worker, [j[:7] + (0,) for j in jobs]))  # start and load the workers
        elapsed = list(ex.map(_oracle_unit_worker, jobs))
    wall = max(elapsed)
    tokens = sum(j[3] for j in jobs)
    full_tokens = int(np.sum(lengths)) * w.num_kv_heads
    us = wall / tokens * full_tokens * 1e6
    desc = (f"{cores} host processes at once (every core), job c = one decode step of kv-head "
            f"group (b, g) = unit c mod {len(units)} (all (sequence, kv-head) units of the step) "
            f"over a window of whole splits ({n} tokens, at most the sequence) starting at a "
            f"different split per job; {tokens} token-heads in all, scaled by token count to the "
            f"full step ({full_tokens} token-heads)")
    return us, cores, desc


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    w = fw.WORKLOADS[args.workload]
    inp = fw.make_inputs(w)
    import oracle
    oracle.build()
    budget = max(0.005, min(30.0, args.reference_budget / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_step_sample(w, inp, budget)
    samples = []
    for _ in range(args.steps):
        us1, desc1, _ = oracle_step_sample(w, inp, budget)
        samples.append(us1)
    single_us = float(np.mean(samples))
    us, cores, desc = oracle_parallel_sample(w, inp, budget)
    line = {
        "impl": "reference", "metric": METRIC, "value": us, "unit": UNIT,
        "n_gpus": args.gpus, "steps": len(samples), "warmup": args.warmup,
        "ms_per_step": us / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 select + f64 attention (CPU oracle)",
        "data": "synthetic (seeded generator; stands in for RULER/LongBench inputs)",
        "config": {"workload": w.description, "name": w.name},
        "cpu_baseline": {"value": us, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc, "host": host_cpu(), "single_thread_value": single_us,
                         "single_thread_sample": desc1},
        "e2e": {"value": us, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------- main --

def run_profile(args):
    """A few eager steps on one GPU and nothing else: the target for ncu."""
    import torch
    device = torch.device("cuda", torch.cuda.current_device())
    w = fw.WORKLOADS[args.workload]
    delta = w.delta if args.delta is None else args.delta
    inp = fw.make_inputs(w)
    rep = Replica(w, inp, device, 1, fmt=args.profile_format)
    rep.reference = REFERENCES[args.reference]
    for i in range(args.profile_steps):
        rep.step(i, delta)
    torch.cuda.synchronize(device)
    rep.check_flags()
    print(f"profile: {args.profile_steps} eager steps of {w.name} ({args.profile_format}, "
          f"delta {delta}) done")
    return 0


def run_shard_measure(args):
    """One rank's share of a W-way context-sharded decode step, on one GPU:
    the workload is the local shard (global context = W x its capacity);
    ffd_decode_partials on it, then ffd_merge_partials over W gathered
    regions (W copies of the local region: the bytes an all-gather delivers).
    The all-gather itself needs W GPUs and is not timed; its volume is
    reported."""
    import torch
    from sparse_long_context_ffd_b200 import ffd, sharded
    device = torch.device("cuda", torch.cuda.current_device())
    w = fw.WORKLOADS[args.workload]
    if args.dense:
        args.delta = float("inf")
    if args.delta is not None:
        w = fw.scaled_workload(w, delta=args.delta)
    if args.seed is not None:
        w = fw.scaled_workload(w, seed=args.seed)
    W = args.shards
    sharded.check_shard_capacity(w.capacity, w.block_size, w.split_blocks)
    inp = fw.make_inputs(w)
    rep = Replica(w, inp, device, 1)
    L = rep.layers[0]
    bufs = L["bufs"]
    off, nbytes = ffd.partials_region(rep.shape)
    gathered = torch.empty(W * nbytes, dtype=torch.uint8, device=device)
    glen = torch.from_numpy((inp["lengths"].astype(np.int64) + (W - 1) * w.capacity)
                            .astype(np.int32)).to(device)  # this shard is full in the global view
    out = torch.empty((w.batch, w.num_q_heads, 128), dtype=torch.bfloat16, device=device)
    gmask = torch.empty((w.batch, w.num_kv_heads, sharded.global_mask_words(W, w.capacity,
                         w.block_size)), dtype=torch.int32, device=device)

    def step(ev=None):
        if ev:
            ev[0].record()
        ffd.decode_partials(rep.shape, L["q"], L["k"], L["v"], bufs.k_packed, bufs.k_scales,
                            rep.lengths, w.delta, bufs.workspace, requant_last=True)
        if ev:
            ev[1].record()
        for r in range(W):  # stand-in for the all-gather (not timed below)
            gathered[r * nbytes:(r + 1) * nbytes].copy_(bufs.workspace[off:off + nbytes])
        if ev:
            ev[2].record()
        ffd.merge_partials(rep.shape, W, gathered, glen, out, gmask)
        if ev:
            ev[3].record()

    for _ in range(args.warmup):
        step()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    torch.cuda.synchronize(device)
    torch.cuda._sleep(int(1e8))
    for e in evs:
        step(e)
    torch.cuda.synchronize(device)
    part_us = float(np.mean([e[0].elapsed_time(e[1]) for e in evs])) * 1e3
    merge_us = float(np.mean([e[2].elapsed_time(e[3]) for e in evs])) * 1e3
    rep.check_flags()
    print(json.dumps({
        "metric": "us per context-sharded decode step, one rank (partials + merge; all-gather not timed)",
        "value": part_us + merge_us, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": False, "mode": "context-shard",
        "config": {"workload": w.description + f" as 1 of {W} context shards",
                   "global_context": W * w.capacity},
        "partials_us": part_us, "merge_us": merge_us,
        "exchange_bytes_per_rank": nbytes, "gathered_bytes": W * nbytes}), flush=True)
    return 0


def measure_thumb_resid(w, inp, device, args, world, l2):
    """The same decode step on the thumbnail + residual key format (2-bit
    thumbnails scanned, 8-bit residuals + V read for kept blocks): fused step,
    dense mode, and its own kept set (the thumbnail scores select differently)."""
    import torch
    probe = Replica(w, inp, device, 1, fmt="tr")
    probe.reference = REFERENCES[args.reference]
    probe.step(0, w.delta)
    torch.cuda.synchronize(device)
    mask = probe.layers[0]["bufs"].mask.cpu().numpy().view(np.uint32)
    kept_blocks, valid_blocks, kept_tok = kept_tokens_from_mask(w, inp["lengths"], mask)
    vs_dense = error_vs_dense(probe, w.delta)
    algo = algorithmic_bytes_tr(w, inp["lengths"], kept_tok, dense=False)
    valid_tok = int(np.sum(inp["lengths"])) * w.num_kv_heads
    algo_dense = algorithmic_bytes_tr(w, inp["lengths"], valid_tok, dense=True)
    layers = max(1, min(64, math.ceil(3 * l2 / min(algo["total"], algo_dense["total"]))))
    del probe
    rep = Replica(w, inp, device, layers, fmt="tr")
    rep.reference = REFERENCES[args.reference]
    steps = min(args.steps, 1000)
    total, per, _ = time_graph_steps(rep, w.delta, steps, args.warmup, world, device)
    dense_total, dense_per, _ = time_graph_steps(rep, float("inf"), min(steps, 400),
                                                 min(args.warmup, 20), world, device)
    rep.check_flags()
    peak, _ = load_peaks()
    dec = float(np.mean(per)) if per else None
    dden = float(np.mean(dense_per)) if dense_per else None
    ach = algo["total"] / (dec * 1e-3) / 1e9 if dec else None
    return {
        "ms_per_step": dist_max(total / steps, world, device),
        "decode_us": dec * 1e3 if dec else None,
        "kept_blocks": kept_blocks, "kept_fraction": kept_blocks / max(1, valid_blocks),
        "sparsity": 1.0 - kept_blocks / max(1, valid_blocks), "vs_dense": vs_dense,
        "algorithmic_bytes_per_launch": algo, "achieved_gbs": ach,
        "frac": ach / peak if ach else None,
        "traffic": ncu_traffic_per_launch(args.workload, dense=False, fmt="tr"),
        "dense_decode_us": dden * 1e3 if dden else None,
        "dense_algorithmic_bytes_per_launch": algo_dense["total"],
        "dense_achieved_gbs": algo_dense["total"] / (dden * 1e-3) / 1e9 if dden else None,
        "how": "ffd_decode_tr with requant_last (thumbnail + residual re-quantisation of the "
               "last block + thumbnail scan + residual/V computer + merge), one launch",
    }


def run_gpu(args):
    import torch
    rank, local_rank, world = dist_env()
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist_init("nccl", world)
    device = torch.device("cuda", local_rank if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(device)
    w = fw.WORKLOADS[args.workload]
    if args.dense:
        args.delta = float("inf")
    if args.delta is not None:
        w = fw.scaled_workload(w, delta=args.delta)
    if args.seed is not None:
        w = fw.scaled_workload(w, seed=args.seed)
    # each rank serves its own request: a different seed per replica
    w_rank = fw.scaled_workload(w, seed=w.seed + 1000 * rank) if rank else w
    inp = fw.make_inputs(w_rank)
    from sparse_long_context_ffd_b200 import ffd  # noqa: F401  (loads the library)

    props = torch.cuda.get_device_properties(device)
    l2 = getattr(props, "L2_cache_size", 126 * 2**20)

    # first pass: learn the kept set (same content on every layer copy)
    probe = Replica(w, inp, device, 1)
    probe.reference = REFERENCES[args.reference]
    probe.step(0, w.delta)
    torch.cuda.synchronize(device)
    mask = probe.layers[0]["bufs"].mask.cpu().numpy().view(np.uint32)
    kept_blocks, valid_blocks, kept_tok = kept_tokens_from_mask(w, inp["lengths"], mask)
    probe_out = probe.layers[0]["bufs"].out[0, :w.group].float().cpu().numpy().astype(np.float64)
    probe_mask = mask[0, 0].copy()
    vs_dense = error_vs_dense(probe, w.delta)
    algo = algorithmic_bytes(w, inp["lengths"], kept_tok, dense=False)
    valid_tok = int(np.sum(inp["lengths"])) * w.num_kv_heads
    algo_dense = algorithmic_bytes(w, inp["lengths"], valid_tok, dense=True)
    layers = max(1, min(64, math.ceil(3 * l2 / min(algo["total"], algo_dense["total"]))))
    del probe
    rep = Replica(w, inp, device, layers)
    rep.reference = REFERENCES[args.reference]

    sampler = ClockSampler(device.index, args.clocks_csv)
    sampler.start()
    time.sleep(0.8)  # let nvidia-smi start before the measured window
    torch.cuda.nvtx.range_push("ffd timed decode steps")
    total_ms, per_decode, spg = time_graph_steps(rep, w.delta, args.steps, args.warmup, world,
                                                 device, sampler)
    torch.cuda.nvtx.range_pop()
    timing_method = "graph-captured timing events around each decode launch"
    if not per_decode:
        per_decode = time_gated_decodes(rep, w.delta, min(args.steps, 64), device)
        timing_method = "gated eager loop, events around each decode launch"
    sampler.stop()
    rep.check_flags()
    ms_per_step = dist_max(total_ms / args.steps, world, device)
    decode_ms = float(np.mean(per_decode))

    # in-run flash-decoding comparison: the same kernel in dense mode
    dense_total, dense_per, _ = time_graph_steps(rep, float("inf"), min(args.steps, 400),
                                                 min(args.warmup, 20), world, device)
    dense_decode_ms = float(np.mean(dense_per)) if dense_per else None
    # the same step as two launches (ffd_quantize_keys + ffd_decode)
    two_total, two_per, _ = time_graph_steps(rep, w.delta, min(args.steps, 400),
                                             min(args.warmup, 20), world, device, fused=False)
    rep.check_flags()

    peak, peak_src = load_peaks()
    achieved = algo["total"] / (decode_ms * 1e-3) / 1e9
    traffic = ncu_traffic_per_launch(args.workload, dense=False)
    probe_gbs = read_probe_gbs(device)

    tr = None
    if not args.no_tr:
        tr = measure_thumb_resid(w, inp, device, args, world, l2)

    # the method's own regime beside the headline: the same shape with
    # concentrated attention, where few blocks are kept (timing only; the
    # oracle checks these rows in --rho-sweep and in the GPU tests), int4 and
    # the thumbnail format
    rho = None
    if not args.no_rho:
        rho = [rho_row(name, ref_name, REFERENCES[ref_name], device, min(args.steps, 200),
                       min(args.warmup, 10), world, load_peaks()[0], l2, fmt=fmt)
               for name, ref_name, fmt in (("rho1of64", "running", "int4"), ("rho0p05", "running", "int4"),
                                           ("rho1of64", "sink_local_fixed", "int4"),
                                           ("rho1of64", "running", "tr"))]

    e2e = None
    if not args.no_e2e:
        del rep
        torch.cuda.empty_cache()
        e2e = e2e_steps(w, inp, device, w.delta, args.e2e_steps)
    e2e_us = dist_max(e2e["event_ms_per_step"] * 1e3, world, device) if e2e else None
    layer = layer_steps(w, inp, device, w.delta, min(args.e2e_steps, 200)) if e2e else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        us1, desc1, used = oracle_step_sample(w, inp, args.cpu_budget)
        us, cores, desc = oracle_parallel_sample(w, inp, args.cpu_budget)
        vs_gpu = oracle_vs_gpu(w, inp, probe_out, probe_mask,
                               pseudo_max=args.reference == "sink_local")
        cpu = {"value": us, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc,
               "host": host_cpu(), "vs_gpu": vs_gpu,
               "single_thread_value": us1,
               "single_thread_sample": desc1 + f"; {used:.1f} s of CPU time"}

    clocks = sampler.summary()
    dist_barrier(world, device)
    if rank == 0:
        line = {
            "metric": METRIC, "value": ms_per_step * 1e3, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 K/V + int4xint8 scan, fp32 accumulate",
            "data": "synthetic (seeded generator; stands in for RULER/LongBench inputs)",
            "config": {"workload": w.description, "name": w.name, "delta": w.delta,
                       "reference": args.reference,
                       "kept_blocks": kept_blocks, "valid_blocks": valid_blocks,
                       "kept_fraction": kept_blocks / max(1, valid_blocks),
                       "sparsity": 1.0 - kept_blocks / max(1, valid_blocks),
                       "l2": f"inputs rotated over {layers} cache copies "
                             f"(>= 3x the {l2 >> 20} MiB L2 per cycle)",
                       "steps_per_graph": spg, "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "kernel": "ffd decode_kernel via ffd_decode_step (last-block "
                                   "re-quantisation + selector + computer + merge)",
                         "algorithmic_bytes_per_launch": algo, "launch_us": decode_ms * 1e3,
                         "launch_us_median": float(np.median(per_decode)) * 1e3,
                         "launch_us_p10": float(np.percentile(per_decode, 10)) * 1e3,
                         "launch_us_p90": float(np.percentile(per_decode, 90)) * 1e3,
                         "peak_source": peak_src, "timing": timing_method,
                         "read_probe_gbs": probe_gbs, "frac_of_read_probe": achieved / probe_gbs,
                         "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                         "read_probe": "ffd_read_probe over 4 GiB in this run (one-pass "
                                       "16-byte loads, L1 no-allocate)"},
            "vs_dense": vs_dense,
            "two_launch_step": {"ms_per_step": two_total / max(1, min(args.steps, 400)),
                                "decode_us": float(np.mean(two_per)) * 1e3 if two_per else None,
                                "how": "ffd_quantize_keys(FFD_LAST_BLOCK) + ffd_decode"},
            "dense_mode": {"decode_us": dense_decode_ms * 1e3 if dense_decode_ms else None,
                           "ms_per_step": dense_total / max(1, min(args.steps, 400)),
                           "algorithmic_bytes_per_launch": algo_dense["total"],
                           "achieved_gbs": (algo_dense["total"] / (dense_decode_ms * 1e-3) / 1e9)
                           if dense_decode_ms else None},
            "thumb_residual": tr,
            "kept_fraction_sweep": ({"workload": "long-context shape (B1 Hq32 Hkv8 N131072 T64 S64 "
                                                 "delta 3) with concentrated attention "
                                                 "(ffd_workloads.RHO_DOMINANT)",
                                     "rows": rho} if rho else None),
            "e2e": ({"value": e2e_us, "unit": UNIT, "h2d_bytes_per_step": e2e["h2d"],
                     "d2h_bytes_per_step": e2e["d2h"],
                     "wall_ms_per_step": e2e["wall_ms_per_step"],
                     "eager_value": e2e["eager_event_ms_per_step"] * 1e3,
                     "how": "public API per step (step.DecodeStep -> ffd_step_graph_run): "
                            "one native CUDA graph holding the pinned H2D of q + new K/V rows "
                            "and ffd_decode_append (cache append + last-block re-quantisation + "
                            "decode, one kernel, writing out + mask straight into pinned host "
                            "memory), then a stream sync; eager_value: H2D, launch and D2H "
                            "issued from Python each step"} if e2e else None),
            "stand_in_layer": layer,
            "cpu_baseline": cpu,
            "gpu_launches": args.steps,
            "gpu_launches_note": "one fused decode launch per timed step (the headline int4 "
                                 "path); the comparison legs run outside that window",
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


CONTEXT_SWEEP = (16384, 32768, 65536, 131072, 262144)


def run_context_sweep(args):
    """Decode time against context length: the long-context workload (B1, Hq32,
    Hkv8, T64, S64, its delta, drift and needles) at each length of
    CONTEXT_SWEEP, the fused step in sparse and in dense mode, one JSON line
    with a row per length."""
    import torch
    device = torch.device("cuda", torch.cuda.current_device())
    base = fw.WORKLOADS["long128k"]
    l2 = getattr(torch.cuda.get_device_properties(device), "L2_cache_size", 126 * 2**20)
    peak, peak_src = load_peaks()
    rows = []
    for n in CONTEXT_SWEEP:
        w = fw.scaled_workload(base, capacity=n, context=n)
        inp = fw.make_inputs(w)
        probe = Replica(w, inp, device, 1)
        probe.step(0, w.delta)
        torch.cuda.synchronize(device)
        mask = probe.layers[0]["bufs"].mask.cpu().numpy().view(np.uint32)
        kept_blocks, valid_blocks, kept_tok = kept_tokens_from_mask(w, inp["lengths"], mask)
        algo = algorithmic_bytes(w, inp["lengths"], kept_tok, dense=False)["total"]
        algo_dense = algorithmic_bytes(w, inp["lengths"], int(np.sum(inp["lengths"])) * w.num_kv_heads,
                                       dense=True)["total"]
        del probe
        layers = max(1, min(64, math.ceil(3 * l2 / min(algo, algo_dense))))
        rep = Replica(w, inp, device, layers)
        steps = min(args.steps, 400)
        _, per, _ = time_graph_steps(rep, w.delta, steps, args.warmup, 1, device)
        _, per_d, _ = time_graph_steps(rep, float("inf"), steps, args.warmup, 1, device)
        rep.check_flags()
        sp, de = float(np.mean(per)) * 1e3, float(np.mean(per_d)) * 1e3
        rows.append({"context": n, "sparse_us": sp, "dense_us": de,
                     "kept_fraction": kept_blocks / max(1, valid_blocks),
                     "sparse_frac": algo / (sp * 1e-6) / 1e9 / peak,
                     "dense_frac": algo_dense / (de * 1e-6) / 1e9 / peak})
        del rep, inp
        torch.cuda.empty_cache()
    ctx = np.array([r["context"] for r in rows], np.float64)
    fit = {m: [float(c) for c in np.polyfit(ctx / 1024.0, [r[m + "_us"] for r in rows], 1)]
           for m in ("sparse", "dense")}
    line = {"mode": "context-sweep", "metric": "us per decode launch vs context length",
            "unit": "us",
            "workload": "long-context shape (B1 Hq32 Hkv8 D128 T64 S64 delta 3, drift 0.05/token, "
                        "16 needles) at each context length",
            "peak_gbs": peak, "peak_source": peak_src,
            "rows": rows,
            "linear_fit_us_per_1k_tokens_and_intercept": fit}
    print(json.dumps(line), flush=True)
    return 0


def rho_row(name, ref_name, ref, device, steps, warmup, world, peak, l2, inp=None, dense=False,
            fmt="int4"):
    """One row of the kept-fraction sweep: the fused step on a controlled-
    sparsity workload (ffd_workloads.RHO_DOMINANT) with one reference maximum
    and key format, timed from CUDA graphs.  (The same seeded inputs are
    checked against the oracle by the GPU tests.)"""
    import torch
    w = fw.WORKLOADS[name]
    if inp is None:
        inp = fw.make_inputs(w)
    probe = Replica(w, inp, device, 1, fmt=fmt)
    probe.reference = ref
    probe.step(0, w.delta)
    torch.cuda.synchronize(device)
    mask = probe.layers[0]["bufs"].mask.cpu().numpy().view(np.uint32)
    kept_blocks, valid_blocks, kept_tok = kept_tokens_from_mask(w, inp["lengths"], mask)
    algo = (algorithmic_bytes_tr if fmt == "tr" else algorithmic_bytes)(w, inp["lengths"], kept_tok,
                                                                        dense=False)["total"]
    del probe
    row = {"workload": name, "format": fmt, "reference": ref_name,
           "kept_fraction": kept_blocks / max(1, valid_blocks), "algorithmic_bytes": algo}
    layers = max(1, min(64, math.ceil(3 * l2 / algo)))
    rep = Replica(w, inp, device, layers, fmt=fmt)
    rep.reference = ref
    _, per, _ = time_graph_steps(rep, w.delta, steps, warmup, world, device)
    us = dist_max(float(np.mean(per)) * 1e3, world, device)
    row.update({"decode_us": us, "tbs": algo / (us * 1e-6) / 1e12,
                "frac": algo / (us * 1e-6) / 1e9 / peak})
    if dense:
        _, per_d, _ = time_graph_steps(rep, float("inf"), steps, warmup, world, device)
        row["dense_us"] = dist_max(float(np.mean(per_d)) * 1e3, world, device)
    rep.check_flags()
    del rep
    torch.cuda.empty_cache()
    return row


def run_rho_sweep(args):
    """The method's own regime: decode time against the kept fraction.  The
    long-context shape with concentrated attention (ffd_workloads.RHO_DOMINANT:
    flat keys, n of every 64 blocks raised by 6 logits, so the Top-delta rule
    keeps n/64 of the blocks), the fused step timed from CUDA graphs for the
    running maximum and the pages' fixed pseudo-max threshold, beside the same
    kernel in dense mode; one JSON line.  The GPU tests check these seeded
    inputs against the oracle (tests/test_parity_gpu.py and
    tests/test_parity_tr_gpu.py: full size at 1/64 and 1/4 kept, 32K at 1/64
    and all kept)."""
    import torch
    device = torch.device("cuda", torch.cuda.current_device())
    l2 = getattr(torch.cuda.get_device_properties(device), "L2_cache_size", 126 * 2**20)
    peak, peak_src = load_peaks()
    refs = [("running", REFERENCES["running"]), ("sink_local_fixed", REFERENCES["sink_local_fixed"])]
    rows = []
    dense_us = {}
    steps = min(args.steps, 400)
    # int4 with both references, then the thumbnail format (the pages' own key
    # split) with the running maximum
    legs = [("int4", ref_name, ref) for ref_name, ref in refs] + [("tr", "running", REFERENCES["running"])]
    for name in fw.RHO_DOMINANT:
        inp = fw.make_inputs(fw.WORKLOADS[name])
        for fmt, ref_name, ref in legs:
            row = rho_row(name, ref_name, ref, device, steps, args.warmup, 1, peak, l2,
                          inp=inp, dense=fmt not in dense_us, fmt=fmt)
            dense_us[fmt] = row.get("dense_us", dense_us.get(fmt))
            row["dense_us"] = dense_us[fmt]
            row["vs_dense"] = dense_us[fmt] / row["decode_us"]
            rows.append(row)
        del inp
    line = {"mode": "rho-sweep", "metric": "us per decode launch vs kept fraction (128K), int4 and "
                                          "thumbnail + residual key formats",
            "unit": "us",
            "workload": "long-context shape (B1 Hq32 Hkv8 D128 N131072 T64 S64 delta 3) with "
                        "concentrated attention: keys 0.1 N(0,1), n of every 64 blocks raised by "
                        "6 logits (ffd_workloads.RHO_DOMINANT)",
            "peak_gbs": peak, "peak_source": peak_src,
            "parity": "checked against the oracle by the GPU tests on the same seeded inputs",
            "rows": rows}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ffd", "reference"], default="ffd")
    ap.add_argument("--workload", choices=sorted(fw.WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--delta", type=float, default=None)
    ap.add_argument("--dense", action="store_true", help="delta = +inf (flash-decoding over all blocks)")
    ap.add_argument("--seed", type=int, default=None, help="input seed (default: the workload's)")
    ap.add_argument("--clocks-csv", default=None,
                    help="also write the raw nvidia-smi clock samples of the timed window here")
    ap.add_argument("--reference", choices=sorted(REFERENCES), default="running",
                    help="Top-delta reference maximum: running max in the split, the running "
                         "max seeded with the sink/local pseudo-max, or that pseudo-max as a "
                         "fixed threshold")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rho", action="store_true",
                    help="skip the small-kept-fraction rows of the default line")
    ap.add_argument("--no-tr", action="store_true",
                    help="skip the thumbnail + residual format measurement")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--reference-budget", type=float, default=150.0)
    ap.add_argument("--context-sweep", action="store_true",
                    help="the long-context workload at 16K..256K tokens, sparse and dense (one line)")
    ap.add_argument("--rho-sweep", action="store_true",
                    help="the 128K shape with concentrated attention at kept fractions 1/64..1, "
                         "running and fixed pseudo-max references, oracle-checked (one line)")
    ap.add_argument("--shards", type=int, default=0,
                    help="time one rank's share of a context-sharded step over this many shards")
    ap.add_argument("--profile-steps", type=int, default=0,
                    help="run this many eager steps and exit (for ncu)")
    ap.add_argument("--profile-format", choices=["int4", "tr"], default="int4",
                    help="key format of the --profile-steps run")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_steps:
        return run_profile(args)
    if args.shards:
        return run_shard_measure(args)
    if args.context_sweep:
        return run_context_sweep(args)
    if args.rho_sweep:
        return run_rho_sweep(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
