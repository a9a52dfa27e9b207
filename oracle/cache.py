"""Model of one tier of the sink + rolling-window KV cache.  (Oracle: test only.)

[orkas] section 选择三：有上限的记忆: the first chunks of the stream are kept for
good as anchors (sink); of the later chunks only a window of the most recent
ones is kept and older ones are dropped, so the cost of a new chunk does not grow
with the length of the stream. [bloom] section "Vidu S2 到底是什么" calls the
same store a rolling KV cache; [s2read] section 2.2 lists anchor chunks and a
sliding-window context.

The model is written as a list of physical slots and searches for the slot to
use, instead of computing it with modular arithmetic, so that it checks the
library's ring formula rather than restating it:

* ``sink`` slots hold chunks 0..sink-1, each in the first free sink slot;
* ``window - 1`` window slots hold the most recent history chunks (reading R1:
  the window counts the chunk being generated, which is never cached while it
  is being denoised);
* a new history chunk takes the lowest free window slot, else the slot of the
  oldest window chunk, which is evicted.
"""


class RingCacheModel:
    """Slot contents of one tier; ``append`` returns (slot, evicted chunk id)."""

    def __init__(self, sink, window):
        if sink < 0 or window < 1:
            raise ValueError("need sink >= 0 and window >= 1")
        self.sink = sink
        self.ring = window - 1
        self.slots = [None] * (sink + self.ring)
        self.count = 0  # chunks appended so far == id of the next chunk

    def append(self):
        """Store the next chunk id; return (slot or None, evicted id or None)."""
        cid = self.count
        self.count += 1
        if cid < self.sink:
            slot = self.slots.index(None)  # first free sink slot
            self.slots[slot] = cid
            return slot, None
        window_slots = range(self.sink, self.sink + self.ring)
        if not window_slots:
            return None, cid  # no window: the chunk is dropped at once
        free = [s for s in window_slots if self.slots[s] is None]
        if free:
            self.slots[free[0]] = cid
            return free[0], None
        oldest = min(window_slots, key=lambda s: self.slots[s])
        evicted = self.slots[oldest]
        self.slots[oldest] = cid
        return oldest, evicted

    def held(self):
        """Chunk ids currently cached, ascending."""
        return sorted(c for c in self.slots if c is not None)

    def attended(self):
        """Chunks the next chunk attends to: every cached chunk plus itself."""
        return self.held() + [self.count]

    def ranks(self):
        """Relocated rank of each attended chunk: its index in ``attended``."""
        return {cid: r for r, cid in enumerate(self.attended())}
