"""Host-to-device staging of per-step inputs, overlapped with the loss.

A training step feeds the loss fresh per-step inputs (hidden states, the
teacher's top-K cache or teacher hidden states, the mask) from host memory,
while the heads stay resident.  `HostStager` keeps `depth` device copies of
those inputs and copies step i+1's batch from pinned host memory on its own
stream while step i's kernels run on the compute stream:

    stager = HostStager({"H": H_host, "topk_idx": idx_host, ...}, device)
    slot = stager.put(batch_0)                  # copy stream
    for i in range(steps):
        bufs = stager.acquire(slot, stream)     # compute waits for the copy
        if i + 1 < steps:
            nxt = stager.put(batch_{i+1})       # overlaps step i's kernels
        ... launch the loss on bufs ...
        stager.release(slot, stream)            # buffer reusable after step i
        slot = nxt

Ordering uses CUDA events only: a copy into a slot waits for the compute
stream to be done with that slot, and the compute stream waits for the copy.
The host is never blocked.  This is plumbing around the C ABI (device memory,
streams and events come from torch); no loss arithmetic happens here.
"""
from __future__ import annotations

import torch


class HostStager:
    """Ring of `depth` device buffer sets shaped like `templates` (name ->
    tensor giving shape and dtype), filled from pinned host tensors on a
    dedicated copy stream."""

    def __init__(self, templates, device, depth=2):
        if depth < 1:
            raise ValueError("depth must be >= 1")
        self.device = torch.device(device)
        self.depth = depth
        self.names = list(templates)
        self.bufs = [{k: torch.empty(t.shape, dtype=t.dtype, device=self.device)
                      for k, t in templates.items()} for _ in range(depth)]
        self.copy_stream = torch.cuda.Stream(self.device)
        self._ready = [torch.cuda.Event() for _ in range(depth)]
        self._free = [torch.cuda.Event() for _ in range(depth)]
        self._next = 0

    def put(self, host):
        """Enqueue the copy of one step's inputs (name -> pinned host tensor,
        the same names, shapes and dtypes as the templates) into the next slot;
        returns the slot.  The host tensors must stay unchanged until the copy
        has run (record `ready_event(slot)` or synchronise to know)."""
        if set(host) != set(self.names):
            raise KeyError(f"expected inputs {sorted(self.names)}, got {sorted(host)}")
        slot = self._next
        self._next = (self._next + 1) % self.depth
        bufs = self.bufs[slot]
        for k, h in host.items():
            if h.shape != bufs[k].shape or h.dtype != bufs[k].dtype:
                raise ValueError(f"{k}: {tuple(h.shape)} {h.dtype} does not match the "
                                 f"staging buffer {tuple(bufs[k].shape)} {bufs[k].dtype}")
            if h.device.type != "cpu":
                raise ValueError(f"{k} must be a host tensor")
        cs = self.copy_stream
        cs.wait_event(self._free[slot])        # no-op until the slot was released once
        with torch.cuda.stream(cs):
            for k, h in host.items():
                bufs[k].copy_(h, non_blocking=True)
        self._ready[slot].record(cs)
        return slot

    def acquire(self, slot, stream=None):
        """Make `stream` (default: the current stream) wait for the slot's copy;
        returns the slot's device buffers."""
        stream = stream if stream is not None else torch.cuda.current_stream(self.device)
        stream.wait_event(self._ready[slot])
        return self.bufs[slot]

    def release(self, slot, stream=None):
        """Mark the slot reusable once the work enqueued so far on `stream` has run."""
        stream = stream if stream is not None else torch.cuda.current_stream(self.device)
        self._free[slot].record(stream)

    def ready_event(self, slot):
        return self._ready[slot]

    @property
    def bytes_per_step(self):
        return sum(t.numel() * t.element_size() for t in self.bufs[0].values())
