"""Prefill of batches that live in host memory, with the transfers overlapped.

A caller whose inputs arrive in (pinned) host memory, and who wants y and the final state
back there, pays two PCIe transfers per call: about 0.7 GB each way for a 2.7B-shaped
16384-token batch, far longer than the prefill itself.  Done one after the other on one
stream, the copy engines carry only one direction at a time.  ``HostPrefill`` runs the
same C call (``ssd_prefill``) over two sets of device buffers and three streams -- copy in,
compute, copy out -- so that batch i's outputs go back to the host while batch i + 1's
inputs come in and batch i + 1 is computed.

Ordering, per batch i in buffer set i % 2:
  copy-in stream   waits until the outputs of batch i - 2 (same set) have left the device,
                   then copies x, dt, B, C in (one cudaMemcpyAsync per tensor)
  compute stream   waits for those copies, runs ssd_prefill into the set's y and state
  copy-out stream  waits for the prefill, copies y and the final state out
The prefills run one after another on the compute stream, so they share one workspace.
Host buffers must stay untouched until the event that ``submit`` returns has completed (for the
outputs) and until the next ``synchronize`` (for the inputs).
"""
from __future__ import annotations

import torch

from . import binding


class HostPrefill:
    def __init__(self, batch, seqlen, nheads, headdim, ngroups, dstate, chunk_len, dtype, A, D,
                 device=None):
        """``A`` and ``D`` are the layer's per-head parameters, already on the device; ``dtype``
        is the storage type of x, B, C and y (torch.bfloat16 or torch.float32)."""
        dev = torch.device(device) if device is not None else A.device
        self.dims = (batch, seqlen, nheads, headdim, ngroups, dstate)
        self.chunk_len = chunk_len
        self.A, self.D = A, D
        f32 = torch.float32

        def buffers():
            return {"x": torch.empty((batch, seqlen, nheads, headdim), device=dev, dtype=dtype),
                    "dt": torch.empty((batch, seqlen, nheads), device=dev, dtype=f32),
                    "B": torch.empty((batch, seqlen, ngroups, dstate), device=dev, dtype=dtype),
                    "C": torch.empty((batch, seqlen, ngroups, dstate), device=dev, dtype=dtype),
                    "y": torch.empty((batch, seqlen, nheads, headdim), device=dev, dtype=dtype),
                    "state": torch.empty((batch, nheads, headdim, dstate), device=dev, dtype=f32),
                    "init": torch.empty((batch, nheads, headdim, dstate), device=dev, dtype=f32)}

        self.sets = [buffers(), buffers()]
        code = binding.SSD_BF16 if dtype == torch.bfloat16 else binding.SSD_F32
        need = binding.ssd_prefill_workspace_bytes(batch, seqlen, nheads, headdim, ngroups, dstate,
                                                   chunk_len, code)
        self.workspace = torch.empty(max(need, 1), device=dev, dtype=torch.uint8)
        self.copy_in = torch.cuda.Stream(device=dev)
        self.compute = torch.cuda.Stream(device=dev)
        self.copy_out = torch.cuda.Stream(device=dev)
        self.out_done = [None, None]
        self.count = 0
        # the caller's stream may still be writing A and D
        ready = torch.cuda.current_stream(dev).record_event()
        self.compute.wait_event(ready)

    def submit(self, x, dt, B, C, y_out, state_out, init_state=None) -> torch.cuda.Event:
        """Queue one batch: host inputs x, dt, B, C (and optionally init_state), host outputs
        y_out and state_out (pinned host tensors of the layouts in include/ssd.h).  Returns
        an event that completes when y_out and state_out hold the results."""
        i = self.count % 2
        bufs = self.sets[i]
        for name, t in (("x", x), ("dt", dt), ("B", B), ("C", C), ("y", y_out), ("state", state_out)):
            if tuple(t.shape) != tuple(bufs[name].shape) or t.dtype != bufs[name].dtype:
                raise ValueError(f"{name}: expected {tuple(bufs[name].shape)} {bufs[name].dtype}, "
                                 f"got {tuple(t.shape)} {t.dtype}")
        with torch.cuda.stream(self.copy_in):
            if self.out_done[i] is not None:
                self.copy_in.wait_event(self.out_done[i])
            bufs["x"].copy_(x, non_blocking=True)
            bufs["dt"].copy_(dt, non_blocking=True)
            bufs["B"].copy_(B, non_blocking=True)
            bufs["C"].copy_(C, non_blocking=True)
            if init_state is not None:
                bufs["init"].copy_(init_state, non_blocking=True)
            arrived = self.copy_in.record_event()
        self.compute.wait_event(arrived)
        with torch.cuda.stream(self.compute):
            binding.ssd_prefill(bufs["x"], bufs["dt"], self.A, bufs["B"], bufs["C"], self.D, self.chunk_len,
                                init_state=bufs["init"] if init_state is not None else None, y=bufs["y"],
                                final_state=bufs["state"], workspace=self.workspace, stream=self.compute)
            computed = self.compute.record_event()
        self.copy_out.wait_event(computed)
        with torch.cuda.stream(self.copy_out):
            y_out.copy_(bufs["y"], non_blocking=True)
            state_out.copy_(bufs["state"], non_blocking=True)
            done = self.copy_out.record_event()
        self.out_done[i] = done
        self.count += 1
        return done

    def synchronize(self):
        for s in (self.copy_in, self.compute, self.copy_out):
            s.synchronize()
