"""Per-frame KV-cache bookkeeping: pinned sink frames + sliding window.

What it computes ([LWI] "The trick: treat video like a causal stream" and
"How the cache keeps the world alive"; [WiW] second paragraph; [IW]
deployment paragraph for the dynamic window):

  * the cache holds ``sinks`` anchor slots followed by ``window`` slots for
    recent finalized frames; the current chunk is never in a slot;
  * finalized frames are appended one by one in ascending frame order;
  * the first ``sinks`` finalized frames become the anchors, slot i holding
    the i-th of them; anchors are never evicted;
  * a later frame finds the window full (``window`` non-sink frames cached)
    -> the oldest non-sink frame is evicted and the new frame takes its slot;
    otherwise it takes the lowest free window slot;
  * ``evict(keep)`` (dynamic scheduler) drops the oldest non-sink frames until
    at most ``keep`` remain; their slots become free;
  * with window == 0 and the anchors filled, an appended frame is not
    retained (reported as evicted at once, slot -1).

Readings: "which frames are anchors" = the first finalized frames (the
initial observation, [WiW]); slot reuse = the evicting frame takes the
evicted slot, else the lowest free slot (ring buffer).

Parity: pinned (worked examples of the 2+2 and 6+8 caches, closed-form ring
slot formula for a static window, set-based closed form of the visible
frames, invariants).
"""
from __future__ import annotations

from typing import Dict, List, Tuple


class CacheModel:
    """Slot table of one layer's cache (host ints only)."""

    def __init__(self, sinks: int, window: int):
        if sinks < 0 or window < 0 or sinks + window == 0:
            raise ValueError("need sinks >= 0, window >= 0, sinks + window > 0")
        self.sinks = sinks
        self.window = window
        self.slot_frame: List[int] = [-1] * (sinks + window)
        self.n_sinks_filled = 0
        self.recent: List[int] = []          # non-sink frames, oldest first
        self.frame_slot: Dict[int, int] = {}
        self.last_frame = -1

    # ------------------------------------------------------------------
    def append(self, frames) -> Tuple[List[int], List[int]]:
        """Append finalized frames; return (slot of each frame, evicted frames)."""
        slots: List[int] = []
        evicted: List[int] = []
        for f in frames:
            f = int(f)
            if f <= self.last_frame:
                raise ValueError("frame indices must be strictly increasing")
            self.last_frame = f
            if self.n_sinks_filled < self.sinks:
                s = self.n_sinks_filled
                self.n_sinks_filled += 1
            elif self.window == 0:
                slots.append(-1)
                evicted.append(f)
                continue
            elif len(self.recent) == self.window:
                old = self.recent.pop(0)
                s = self.frame_slot.pop(old)
                self.slot_frame[s] = -1
                evicted.append(old)
                self.recent.append(f)
            else:
                s = min(i for i in range(self.sinks, self.sinks + self.window)
                        if self.slot_frame[i] == -1)
                self.recent.append(f)
            self.slot_frame[s] = f
            self.frame_slot[f] = s
            slots.append(s)
        return slots, evicted

    def evict(self, keep: int) -> List[int]:
        """Drop the oldest non-sink frames until at most ``keep`` remain."""
        if keep < 0 or keep > self.window:
            raise ValueError("keep must be in [0, window]")
        out = []
        while len(self.recent) > keep:
            old = self.recent.pop(0)
            s = self.frame_slot.pop(old)
            self.slot_frame[s] = -1
            out.append(old)
        return out

    # ------------------------------------------------------------------
    def cached_frames(self) -> List[int]:
        """Cached frames in ascending frame order."""
        return sorted(f for f in self.slot_frame if f >= 0)

    def slot_map(self) -> List[int]:
        return list(self.slot_frame)

    def n_cached(self) -> int:
        return sum(1 for f in self.slot_frame if f >= 0)


def visible_frames_closed_form(first_frame: int, sinks: int, window: int) -> List[int]:
    """Frames a chunk starting at ``first_frame`` reads from the cache, stated
    as a set rather than through slots: the anchors (frames < sinks) plus the
    ``window`` most recent non-anchor frames before the chunk."""
    anchors = [f for f in range(min(sinks, first_frame))]
    lo = max(sinks, first_frame - window)
    return anchors + list(range(lo, first_frame))
