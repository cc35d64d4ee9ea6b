"""Host-to-host layer runs with copies overlapped with compute.

`HostPipeline` feeds a sequence of host batches (router logits and token rows in pinned
host memory) through one `MoELayer` and writes each layer output back to host memory.
Three CUDA streams carry the work: host->device copies of batch i+1 and the device->host
copy of batch i-1 proceed while batch i runs the seven calls.  Two device slots per
input and output, and CUDA events between the streams, order the reuse of every slot:

    copy-in  stream:  [wait slot free] logits, x  -> slot s          [record inputs_ready]
    compute  stream:  [wait inputs_ready] route ... dispatch          [record inputs_free]
                      expert FFN, [wait out slot free] combine -> out[s] [record out_ready]
    copy-out stream:  [wait out_ready] out[s] -> host                  [record out_free]

Only PyTorch allocations, streams and events are used here; every step of the layer runs
in the library's kernels through the binding.
"""
from __future__ import annotations

import torch

from . import MoELayer, moe_combine, moe_grouped_ffn_combine


class HostPipeline:
    def __init__(self, layer: MoELayer, W1, W3, W2, slots: int = 2):
        self.L = layer
        self.W = (W1, W3, W2)
        dev = layer.idx.device
        self.dev = dev
        self.slots = slots
        T, E, d = layer.T, layer.E, layer.d
        self.logits = [torch.empty(T, E, dtype=torch.float32, device=dev) for _ in range(slots)]
        self.x = [torch.empty(T, d, dtype=torch.bfloat16, device=dev) for _ in range(slots)]
        self.out = [torch.empty(T, d, dtype=torch.bfloat16, device=dev) for _ in range(slots)]
        self.s_in = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        self.s_comp = torch.cuda.current_stream(dev)
        ev = lambda: [torch.cuda.Event() for _ in range(slots)]  # noqa: E731
        self.inputs_ready, self.inputs_free = ev(), ev()
        self.out_ready, self.out_free = ev(), ev()
        self._used = [False] * slots

    def run(self, batches, outputs):
        """batches: list of (logits_h [T,E] fp32, x_h [T,d] bf16) pinned host tensors;
        outputs: list of pinned host tensors [T,d] bf16 receiving each layer output.
        Enqueues everything and returns; synchronise (or wait on `done()`) before reading."""
        L = self.L
        W1, W3, W2 = self.W
        for i, ((lg_h, x_h), o_h) in enumerate(zip(batches, outputs)):
            s = i % self.slots
            with torch.cuda.stream(self.s_in):
                if self._used[s]:
                    self.s_in.wait_event(self.inputs_free[s])
                self.logits[s].copy_(lg_h, non_blocking=True)
                self.x[s].copy_(x_h, non_blocking=True)
                self.inputs_ready[s].record(self.s_in)
            with torch.cuda.stream(self.s_comp):
                self.s_comp.wait_event(self.inputs_ready[s])
                L.route_plan(self.logits[s])
                L.prefetch(W1, W3, W2)
                L.dispatch(self.x[s])
                if not L.fused:
                    self.inputs_free[s].record(self.s_comp)
                if L.fused_combine:
                    # GEMM 2's epilogue combines straight into this slot's output
                    if self._used[s]:
                        self.s_comp.wait_event(self.out_free[s])
                    P1, P3, P2 = L.pool
                    moe_grouped_ffn_combine(L.recv, L.plan, W1, W3, W2, P1, P3, P2, L.src, L.perm,
                                            L.gate, L.R, L.S, L.h, L.out32, self.out[s], L.err)
                else:
                    L.expert_ffn(W1, W3, W2)
                    if L.fused:  # the FFN gathered its rows from x
                        self.inputs_free[s].record(self.s_comp)
                    if self._used[s]:
                        self.s_comp.wait_event(self.out_free[s])
                    moe_combine(L.y, L.perm, L.gate, self.out[s], L.err)
                self.out_ready[s].record(self.s_comp)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.out_ready[s])
                o_h.copy_(self.out[s], non_blocking=True)
                self.out_free[s].record(self.s_out)
            self._used[s] = True

    def done(self) -> torch.cuda.Event:
        """An event recorded on the copy-out stream after the last enqueued copy."""
        e = torch.cuda.Event()
        e.record(self.s_out)
        return e
