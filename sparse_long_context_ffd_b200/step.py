"""Whole decode steps captured in CUDA graphs.

The pages' system part (gist.science explainer, Methodology 3, "Fused Kernel
and System Optimization": the entire decoding step is captured in a CUDA graph
to remove CPU launch overhead at small batch) applied to the FFD step:

* :class:`DecodeStep` -- one layer's FFD decode with host-side inputs and
  outputs, as the library's native step graph (``ffd_step_graph_*``): the H2D
  copy of the step's query and new K/V rows from pinned memory, optionally the
  length increment, and the fused append + re-quantisation + decode launch
  (``ffd_decode_append``), whose kernel writes the output rows and the mask
  straight into pinned host memory (or, with ``results_to_host`` off, one D2H
  copy does).  A step is one call into the library, which launches the graph
  and waits.
* :class:`StandInAttentionLayer` -- a decode-step attention layer with random
  weights (there is no checkpoint): q, k and v projections of the hidden
  state, the FFD step, the output projection, captured whole.  The
  projections are plain library GEMMs (torch.matmul); every attention step
  runs in the FFD kernel.

PyTorch provides the memory, streams and graphs; the compute of the attention
step is the CUDA library's.
"""
from __future__ import annotations

import math
from typing import Optional

from . import ffd


def _require_torch():
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("the FFD decode step needs a CUDA device")
    return torch


class DecodeStep:
    """One attention layer's decode step, captured in a CUDA graph.

    k_cache, v_cache: bf16 [B, Hkv, cap, 128] device tensors, prefilled;
    lengths: int32 [B] device tensor, the lengths BEFORE the first step when
    ``advance`` is set (each step adds one token), else the lengths including
    the new token.  fmt: "int4" (int4 scan copy + bf16 K/V) or "tr" (2-bit
    thumbnails + 8-bit residuals).  The key copies are built here from the
    cache for the current lengths.

    Per step the caller writes the query [B, Hq, 128] and the new token's K/V
    rows [B, Hkv, 128] into ``host_q``, ``host_k_new``, ``host_v_new``
    (pinned), calls :meth:`step`, and reads ``host_out`` [B, Hq, 128] and
    ``host_mask`` [B, Hkv, words].  A sequence whose length would pass the
    capacity is reported by the device flag (see :meth:`check`) and yields a
    zero row.
    """

    def __init__(self, shape: ffd.Shape, k_cache, v_cache, lengths, delta: float,
                 reference: int = ffd.FFD_REFERENCE_RUNNING_MAX, fmt: str = "int4",
                 advance: bool = False, results_to_host: bool = True):
        torch = _require_torch()
        if fmt not in ("int4", "tr"):
            raise ValueError("fmt must be 'int4' or 'tr'")
        self.torch, self.shape, self.fmt = torch, shape, fmt
        # the graph's kernel writes output and mask straight into pinned host
        # memory (no D2H copy) unless results_to_host is off
        self.results_to_host = bool(results_to_host)
        self.delta, self.reference, self.advance = float(delta), int(reference), bool(advance)
        self.k, self.v, self.lengths = k_cache, v_cache, lengths
        dev = k_cache.device
        B, Hq, Hkv, D = shape.batch, shape.num_q_heads, shape.num_kv_heads, shape.head_dim
        self.bufs = (ffd.ThumbResidBuffers(shape, device=dev) if fmt == "tr"
                     else ffd.DecodeBuffers(shape, device=dev))
        b = self.bufs
        if fmt == "tr":
            ffd.quantize_keys_tr(shape, k_cache, lengths, 0, b.k_thumb, b.k_resid, b.k_scales)
        else:
            ffd.quantize_keys(shape, k_cache, lengths, 0, b.k_packed, b.k_scales)
        nq, nk = B * Hq * D, B * Hkv * D
        self._host_in = torch.empty(nq + 2 * nk, dtype=torch.bfloat16).pin_memory()
        self._dev_in = torch.empty(nq + 2 * nk, dtype=torch.bfloat16, device=dev)
        self.host_q = self._host_in[:nq].view(B, Hq, D)
        self.host_k_new = self._host_in[nq:nq + nk].view(B, Hkv, D)
        self.host_v_new = self._host_in[nq + nk:].view(B, Hkv, D)
        self._q = self._dev_in[:nq].view(B, Hq, D)
        self._k_new = self._dev_in[nq:nq + nk].view(B, Hkv, D)
        self._v_new = self._dev_in[nq + nk:].view(B, Hkv, D)
        # output rows and mask share one device buffer, so one D2H copy returns both
        mask_shape = tuple(b.mask.shape)
        out_bytes = B * Hq * D * 2
        mask_off = (out_bytes + 15) // 16 * 16
        total = mask_off + (mask_shape[0] * mask_shape[1] * mask_shape[2]) * 4
        self._mask_off = mask_off
        self._dev_res = torch.empty(total, dtype=torch.uint8, device=dev)
        self._host_res = torch.empty(total, dtype=torch.uint8).pin_memory()
        b.out = self._dev_res[:out_bytes].view(torch.bfloat16).view(B, Hq, D)
        b.mask = self._dev_res[mask_off:].view(torch.int32).view(mask_shape)
        self.host_out = self._host_res[:out_bytes].view(torch.bfloat16).view(B, Hq, D)
        self.host_mask = self._host_res[mask_off:].view(torch.int32).view(mask_shape)
        self.h2d_bytes = self._host_in.numel() * 2
        self.d2h_bytes = total
        self._stream = torch.cuda.Stream(dev)
        self._graph: Optional[object] = None

    def _launch(self):
        b = self.bufs
        if self.advance:
            self.lengths.add_(1)
        if self.fmt == "tr":
            ffd.decode_append_tr(self.shape, self._q, self._k_new, self._v_new, self.k, self.v,
                                 b.k_thumb, b.k_resid, b.k_scales, self.lengths, self.delta, b.out,
                                 b.mask, b.workspace, reference=self.reference)
        else:
            ffd.decode_append(self.shape, self._q, self._k_new, self._v_new, self.k, self.v,
                              b.k_packed, b.k_scales, self.lengths, self.delta, b.out, b.mask,
                              b.workspace, reference=self.reference)

    def _body(self):
        self._dev_in.copy_(self._host_in, non_blocking=True)
        self._launch()
        self._host_res.copy_(self._dev_res, non_blocking=True)

    def capture(self):
        """Build the native step graph (done by the first :meth:`step`).
        Nothing runs at capture; earlier device work on the caches is ordered
        first by a device synchronisation."""
        self.torch.cuda.synchronize(self.k.device)
        b = self.bufs
        tr = self.fmt == "tr"
        self._graph = ffd.StepGraph(
            self.shape, 1 if tr else 0, self.reference, self.delta, self.advance, self._host_in,
            self._dev_in, self.k, self.v, b.k_thumb if tr else b.k_packed, b.k_resid if tr else None,
            b.k_scales, self.lengths, None if self.results_to_host else self._dev_res,
            self._host_res, self._mask_off, b.workspace)
        return self._graph

    def step(self):
        """One decode step: host inputs -> host outputs (one library call)."""
        if self._graph is None:
            self.capture()
        self._graph.run()

    def check(self) -> int:
        """Device flags (ffd.FFD_DEVICE_FLAG_*) raised since the last check."""
        return ffd.check_device_status(self.bufs.workspace)


class StandInAttentionLayer:
    """A decode-step attention layer with random weights around the FFD step.

    hidden: model width; weights drawn N(0, 1/hidden) from ``seed`` (bf16):
    w_q [hidden, Hq*128], w_k and w_v [hidden, Hkv*128], w_o [Hq*128, hidden].
    A step takes x [B, hidden] (pinned host ``host_x``), appends the new
    token's k/v to the caches, attends with FFD and writes the projected output
    [B, hidden] to ``host_y``.  lengths and ``advance`` as for DecodeStep (with
    advance off every step re-appends at position lengths - 1).  No rotary
    embedding or normalisation: this is a stand-in that exercises the step's
    data flow, not a model.
    """

    def __init__(self, shape: ffd.Shape, hidden: int, k_cache, v_cache, lengths, delta: float,
                 seed: int = 0, reference: int = ffd.FFD_REFERENCE_RUNNING_MAX, fmt: str = "int4",
                 advance: bool = True):
        torch = _require_torch()
        self.torch, self.shape = torch, shape
        dev = k_cache.device
        B, Hq, Hkv, D = shape.batch, shape.num_q_heads, shape.num_kv_heads, shape.head_dim
        gen = torch.Generator(device="cpu").manual_seed(int(seed))

        def weight(rows, cols):
            w = torch.randn((rows, cols), generator=gen, dtype=torch.float32) / math.sqrt(rows)
            return w.to(dtype=torch.bfloat16, device=dev)

        self.w_q, self.w_k = weight(hidden, Hq * D), weight(hidden, Hkv * D)
        self.w_v, self.w_o = weight(hidden, Hkv * D), weight(Hq * D, hidden)
        self.core = DecodeStep(shape, k_cache, v_cache, lengths, delta, reference=reference,
                               fmt=fmt, advance=advance)
        self.host_x = torch.empty((B, hidden), dtype=torch.bfloat16).pin_memory()
        self.host_y = torch.empty((B, hidden), dtype=torch.bfloat16).pin_memory()
        self._x = torch.empty((B, hidden), dtype=torch.bfloat16, device=dev)
        self._y = torch.empty((B, hidden), dtype=torch.bfloat16, device=dev)
        self._stream = torch.cuda.Stream(dev)
        self._graph = None

    def _body(self):
        torch, c = self.torch, self.core
        B = self.shape.batch
        self._x.copy_(self.host_x, non_blocking=True)
        torch.matmul(self._x, self.w_q, out=c._q.view(B, -1))
        torch.matmul(self._x, self.w_k, out=c._k_new.view(B, -1))
        torch.matmul(self._x, self.w_v, out=c._v_new.view(B, -1))
        c._launch()
        torch.matmul(c.bufs.out.view(B, -1), self.w_o, out=self._y)
        self.host_y.copy_(self._y, non_blocking=True)

    def capture(self):
        """As DecodeStep.capture: one eager run with the current host_x first."""
        torch = self.torch
        saved = self.core.lengths.clone()
        with torch.cuda.stream(self._stream):
            self._body()
        self._stream.synchronize()
        self.core.lengths.copy_(saved)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self._stream):
            self._body()
        self._graph = g
        torch.cuda.synchronize(self._x.device)
        return g

    def step(self):
        if self._graph is None:
            self.capture()
        self._graph.replay()
        self.torch.cuda.current_stream(self._x.device).synchronize()
