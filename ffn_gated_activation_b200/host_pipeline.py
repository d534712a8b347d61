"""Forward + backward over host-resident tensors, streamed through the GPU in
row chunks.

Rows are independent, so a [T, 2I] problem that lives in (pinned) host memory
can be cut into chunks of rows.  Each chunk's host-to-device copy, kernels
and device-to-host copy go on three CUDA streams, and consecutive chunks
overlap: while chunk k computes, chunk k + 1 is being uploaded and chunk
k - 1 downloaded, so the two copy directions run at the same time.  A ring of
device buffers (one set per chunk in flight) is reused; CUDA events order
every reuse after the download that last read the buffer.

The kernels are the library's own (``situ_glu_fwd`` / ``situ_glu_bwd``
through ``functional``); this module only moves bytes and orders streams.
Per-row and absent routing weights only: a broadcast or per-column weight's
gradient is a sum over all rows, which row chunks would have to combine.
"""
from __future__ import annotations

import torch

from . import functional


class HostPipeline:
    """Reusable streams and device buffers for ``run``.

    inter: I; dtype: gate_up's dtype (bf16 or fp32); chunk_rows: rows per
    chunk; buffers: chunks in flight (3: one uploading, one computing, one
    downloading)."""

    def __init__(self, inter: int, dtype: torch.dtype, chunk_rows: int = 4096, device=None, buffers: int = 3,
                 rw_dtype: torch.dtype = torch.float32):
        if chunk_rows <= 0 or buffers < 1:
            raise ValueError("chunk_rows and buffers must be positive")
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.inter, self.dtype, self.chunk_rows, self.rw_dtype = inter, dtype, chunk_rows, rw_dtype
        self.h2d = torch.cuda.Stream(self.device)
        self.comp = torch.cuda.Stream(self.device)
        self.d2h = torch.cuda.Stream(self.device)
        C, I, dev = chunk_rows, inter, self.device

        def ring(shape, dt):
            return [torch.empty(shape, dtype=dt, device=dev) for _ in range(buffers)]

        self.gu = ring((C, 2 * I), dtype)
        self.go = ring((C, I), dtype)
        self.rw = ring((C, 1), rw_dtype)
        self.y = ring((C, I), dtype)
        self.dgu = ring((C, 2 * I), dtype)
        self.drw = ring((C, 1), rw_dtype)
        self.uploaded = [torch.cuda.Event() for _ in range(buffers)]
        self.computed = [torch.cuda.Event() for _ in range(buffers)]
        self.released = [None] * buffers  # event recorded after the buffer's last download

    def run(self, gate_up, routing_weights, grad_out, beta: float = functional.DEFAULT_BETA,
            linear_beta: float | None = functional.DEFAULT_LINEAR_BETA, y=None, d_gate_up=None, d_rw=None):
        """Y, d_gate_up and d_routing_weights of host tensors gate_up [T, 2I],
        routing_weights [T, 1] or None, grad_out [T, I] (pinned, for the copies
        to overlap), written into host tensors (allocated pinned when None).
        Returns (y, d_gate_up, d_rw) without waiting: the caller's current
        stream is made to wait for the last download, so a synchronize of it
        (or of the device) completes the call."""
        T = gate_up.shape[0]
        I = self.inter
        if tuple(gate_up.shape) != (T, 2 * I) or tuple(grad_out.shape) != (T, I):
            raise ValueError(f"gate_up must be [T, {2 * I}] and grad_out [T, {I}]")
        if gate_up.dtype != self.dtype or grad_out.dtype != self.dtype:
            raise TypeError("gate_up and grad_out must have the pipeline's dtype")
        if gate_up.is_cuda or grad_out.is_cuda:
            raise ValueError("the inputs of a host pipeline live in host memory")
        weighted = routing_weights is not None
        if weighted and (tuple(routing_weights.shape) != (T, 1) or routing_weights.dtype != self.rw_dtype):
            raise ValueError(f"routing_weights must be [T, 1] {self.rw_dtype} (per-row weights) or None")
        pin = dict(pin_memory=True)
        if y is None:
            y = torch.empty((T, I), dtype=self.dtype, **pin)
        if d_gate_up is None:
            d_gate_up = torch.empty((T, 2 * I), dtype=self.dtype, **pin)
        if weighted and d_rw is None:
            d_rw = torch.empty((T, 1), dtype=self.rw_dtype, **pin)
        caller = torch.cuda.current_stream(self.device)
        # the host inputs may have been written by work the caller enqueued
        self.h2d.wait_stream(caller)
        nbuf = len(self.gu)
        for k, r0 in enumerate(range(0, T, self.chunk_rows)):
            r1 = min(T, r0 + self.chunk_rows)
            n = r1 - r0
            b = k % nbuf
            with torch.cuda.stream(self.h2d):
                if self.released[b] is not None:
                    self.h2d.wait_event(self.released[b])
                self.gu[b][:n].copy_(gate_up[r0:r1], non_blocking=True)
                self.go[b][:n].copy_(grad_out[r0:r1], non_blocking=True)
                if weighted:
                    self.rw[b][:n].copy_(routing_weights[r0:r1], non_blocking=True)
                self.uploaded[b].record(self.h2d)
            with torch.cuda.stream(self.comp):
                self.comp.wait_event(self.uploaded[b])
                rw = self.rw[b][:n] if weighted else None
                functional.situ_glu_fwd(self.gu[b][:n], rw, beta, linear_beta, out=self.y[b][:n], stream=self.comp)
                functional.situ_glu_bwd(self.gu[b][:n], rw, self.go[b][:n], beta, linear_beta,
                                        d_gate_up=self.dgu[b][:n], d_rw=self.drw[b][:n] if weighted else None,
                                        stream=self.comp)
                self.computed[b].record(self.comp)
            with torch.cuda.stream(self.d2h):
                self.d2h.wait_event(self.computed[b])
                y[r0:r1].copy_(self.y[b][:n], non_blocking=True)
                d_gate_up[r0:r1].copy_(self.dgu[b][:n], non_blocking=True)
                if weighted:
                    d_rw[r0:r1].copy_(self.drw[b][:n], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self.d2h)
                self.released[b] = ev
        caller.wait_stream(self.d2h)
        # the ring is used on the three streams: freeing it waits for them
        for ring in (self.gu, self.go, self.rw, self.y, self.dgu, self.drw):
            for t in ring:
                for s in (self.h2d, self.comp, self.d2h):
                    t.record_stream(s)
        return y, d_gate_up, (d_rw if weighted else None)
