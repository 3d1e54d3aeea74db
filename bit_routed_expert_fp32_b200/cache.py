"""Host-tiered experts: a layer run from a device cache of expert slots in front of its
packed buffer in page-locked host memory (moe_cache_size / moe_cache_init /
moe_cache_load in include/moe.h).

The pages' engine keeps the experts that do not fit its GPU in a pinned host-RAM arena
and moves the ones a layer needs into GPU memory a layer ahead (ossradar.top, Xolotl
README, "How it works, in one paragraph").  `ExpertCache` does the host side of that:
it decides which slot each expert goes to (free slots first, then the least recently
used expert that the current step does not need), keeps the shared expert resident,
and enqueues the loads, on the compute stream (`ensure`) or ahead of time on a copy
stream (`prefetch`, with an event the compute stream waits on).  The copies and the
table updates are the library's; the kernels read the cache like any packed buffer.
"""
from __future__ import annotations

import ctypes
from collections import OrderedDict

import numpy as np

from . import MoeError, _check, _ptr, _shape, _stream, lib


def slot_plan(resident: "OrderedDict[int, int]", n_slots: int, need, pinned=()):
    """The loads that make every expert in `need` resident: a list of (expert, slot).
    `resident` (expert -> slot, least recently used first) is updated in place: the
    needed experts become the most recently used.  Free slots go first, then the slots
    of the least recently used experts that are neither needed nor pinned.  Raises if
    the needed and pinned experts do not fit."""
    need = list(dict.fromkeys(int(e) for e in need))
    keep = set(need) | set(int(e) for e in pinned)
    if len(keep) > n_slots:
        raise ValueError(f"{len(keep)} experts needed at once but only {n_slots} slots")
    used = set(resident.values())
    free = [s for s in range(n_slots) if s not in used]
    loads = []
    for e in need:
        if e in resident:
            resident.move_to_end(e)
            continue
        if free:
            s = free.pop(0)
        else:
            victim = next(v for v in resident if v not in keep)
            s = resident.pop(victim)
        resident[e] = s
        loads.append((e, s))
    return loads


class ExpertCache:
    """A device cache of n_slots expert slots for one layer whose packed buffer
    (host_packed, numpy uint8, made page-locked here) stays in host memory."""

    def __init__(self, cfg, host_packed: np.ndarray, n_slots: int, device="cuda", stream=None):
        import torch
        self.cfg, self.n_slots, self.device = cfg, n_slots, device
        # page-locked copy of the host buffer, so that every load is an asynchronous DMA
        self.host = torch.from_numpy(np.ascontiguousarray(host_packed, np.uint8)).pin_memory()
        self._hp = ctypes.c_void_p(self.host.data_ptr())
        size = ctypes.c_size_t(0)
        _check("moe_cache_size", lib().moe_cache_size(ctypes.byref(_shape(cfg)), self._hp, n_slots,
                                                       ctypes.byref(size)))
        self.buf = torch.empty(size.value, dtype=torch.uint8, device=device)
        _check("moe_cache_init", lib().moe_cache_init(ctypes.byref(_shape(cfg)), self._hp, n_slots, _ptr(self.buf),
                                                       size.value, _stream(stream)))
        self.resident: OrderedDict[int, int] = OrderedDict()
        self.pinned = tuple(range(cfg.E, cfg.E + cfg.S))        # the shared experts stay resident
        self.loads = 0
        self.ensure(self.pinned, stream)

    def _load(self, plan, stream):
        if not plan:
            return
        ex = np.array([e for e, _ in plan], np.int32)
        sl = np.array([s for _, s in plan], np.int32)
        st = lib().moe_cache_load(ctypes.byref(_shape(self.cfg)), self._hp, self.n_slots, _ptr(self.buf),
                                  self.buf.numel(), ex.ctypes.data, sl.ctypes.data, len(plan), _stream(stream))
        if st != 0:
            raise MoeError("moe_cache_load", st)
        self.loads += len(plan)

    def ensure(self, experts, stream=None):
        """Makes the listed experts (table indices) resident, loading the missing ones on
        `stream` (the compute stream: the forward that follows sees them)."""
        self._load(slot_plan(self.resident, self.n_slots, experts, self.pinned), stream)

    def prefetch(self, experts, copy_stream, keep=()):
        """Loads the listed experts on copy_stream and returns an event recorded after
        the loads; the compute stream must wait on it (stream.wait_event) before the
        forward that reads them.  Used a layer ahead, with the next layer's routing or a
        prediction of it.  `keep`: experts a forward still in flight reads (their slots
        are not reused)."""
        import torch
        self._load(slot_plan(self.resident, self.n_slots, experts, self.pinned + tuple(keep)), copy_stream)
        ev = torch.cuda.Event()
        ev.record(copy_stream)
        return ev
