"""Decode steps fed from host memory with the transfers hidden behind the GPU work.

A serving loop that keeps the new K/V rows, the queries and the lengths of each step in
host memory, and wants every step's attention output back on the host, pays two PCIe
transfers per step and layer. `HostStepPipeline` runs those transfers on two copy
streams with two device buffer sets, so that the host->device copy of the next layer
call and the device->host copy of the previous one overlap the append and attention
kernels of the current one. Every call still moves all of its inputs and its whole
output; only the order on the copy engines changes. The kernels are the library's,
through the session's step call (kv4.decode_step: the append and the attention in one
call, or the two baseline calls for a comparison cache).
"""
from __future__ import annotations

import torch


class HostStepPipeline:
    """Double-buffered host<->device decode steps over one or more layers.

    `layers` is a DecodeSession-like object or a list of them (one per layer, same
    shapes); each provides `step_call(batch, k, v, q, out)`, `batch(lens)` and example
    device tensors `step_k[0]`, `step_v[0]`, `q[0]`, `step_lens[0]`, `out`.
    """

    def __init__(self, layers, device=None):
        self.layers = list(layers) if isinstance(layers, (list, tuple)) else [layers]
        sess = self.layers[0]
        dev = device if device is not None else sess.out.device
        self.k = [torch.empty_like(sess.step_k[0]) for _ in range(2)]
        self.v = [torch.empty_like(sess.step_v[0]) for _ in range(2)]
        self.q = [torch.empty_like(sess.q[0]) for _ in range(2)]
        self.lens = [torch.empty_like(sess.step_lens[0]) for _ in range(2)]
        self.out = [torch.empty_like(sess.out) for _ in range(2)]
        self.h2d = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)
        self.inputs_ready = [torch.cuda.Event() for _ in range(2)]
        self.computed = [torch.cuda.Event() for _ in range(2)]
        self.copied_out = [torch.cuda.Event() for _ in range(2)]

    def bytes_per_step(self) -> tuple[int, int]:
        """(host->device, device->host) bytes moved per step, all layers."""
        n = len(self.layers)
        h2d = sum(t[0].numel() * t[0].element_size()
                  for t in (self.k, self.v, self.q, self.lens))
        d2h = self.out[0].numel() * self.out[0].element_size()
        return h2d * n, d2h * n

    def run(self, host_inputs, hout, steps, start_event=None):
        """Run decode steps `steps`. host_inputs[l] = (hk, hv, hq, hl), pinned host tensors
        of layer l indexed by step; hout[l][i] receives layer l's output of the i-th step
        run. The compute stream is the current stream; it waits for the last output copy
        before returning, so an event recorded on it afterwards closes the whole job.
        `start_event` (recorded on the compute stream) gates the first copy."""
        main = torch.cuda.current_stream()
        if start_event is not None:
            self.h2d.wait_event(start_event)
            self.d2h.wait_event(start_event)
        u = 0  # calls so far: buffer set u % 2
        for i, s in enumerate(steps):
            for li, sess in enumerate(self.layers):
                j = u % 2
                hk, hv, hq, hl = host_inputs[li]
                with torch.cuda.stream(self.h2d):
                    if u >= 2:
                        self.h2d.wait_event(self.computed[j])  # call u-2 has read set j
                    self.k[j].copy_(hk[s], non_blocking=True)
                    self.v[j].copy_(hv[s], non_blocking=True)
                    self.q[j].copy_(hq[s], non_blocking=True)
                    self.lens[j].copy_(hl[s], non_blocking=True)
                    self.inputs_ready[j].record(self.h2d)
                main.wait_event(self.inputs_ready[j])
                if u >= 2:
                    main.wait_event(self.copied_out[j])  # call u-2's output is on the host
                b = sess.batch(self.lens[j])
                sess.step_call(b, self.k[j], self.v[j], self.q[j], self.out[j])
                self.computed[j].record(main)
                with torch.cuda.stream(self.d2h):
                    self.d2h.wait_event(self.computed[j])
                    hout[li][i].copy_(self.out[j], non_blocking=True)
                    self.copied_out[j].record(self.d2h)
                u += 1
        for j in range(min(2, u)):
            main.wait_event(self.copied_out[j])
