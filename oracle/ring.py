"""Per-layer rolling KV cache, oracle.

The pages: frames are generated and evicted in a sliding window, and every
layer reads and writes a rolling KV cache ("Amazon and Reactor tune Trainium
for real-time video generation", section "Three problems for generic
compilers"; "A kernel-centric path to real-time video generation on Trainium",
yomu.fyi summary, FAQ "What is the Rolling Forcing model?").

Reading taken (the pages print no data structure): a ring of W frame slots.
``head`` is the slot the next frame goes to, ``count`` the number of valid
frames.  Inserting n <= W frames writes frame i to slot (head + i) mod W, then
head <- (head + n) mod W, count <- min(W, count + n); the max(0, count + n - W)
oldest frames are evicted by being overwritten (no clearing).  Logical frame j
(0 = oldest valid) lives in slot (head - count + j) mod W.

Variant with a pinned prefix (the pages do not describe it; a common
rolling-window variant keeps the first frames of a stream, "attention sinks",
out of eviction): the first P slots take the first P frames ever inserted and
are never overwritten; later frames roll through slots P..W-1 as above.
``head`` is then the next slot of that rolling region, and logical frames are
the pinned ones (oldest first) followed by the rolling ones.
"""

import numpy as np


class RingRef:
    """Python-list ring of W slots, each holding a (K, V) frame pair or None;
    the first ``pinned`` slots hold the first frames ever inserted."""

    def __init__(self, slots, pinned=0):
        if slots <= 0:
            raise ValueError("slots must be positive")
        if pinned < 0 or pinned >= slots:
            raise ValueError("pinned must be in [0, slots)")
        self.W = int(slots)
        self.P = int(pinned)
        self.slots = [None] * self.W
        self.head = self.P          # next slot of the rolling region
        self.count = 0

    def capacity_for_insert(self):
        """Most frames one insert may carry: the free pinned slots plus the
        rolling region (a frame may not overwrite one of its own call)."""
        return max(0, self.P - self.count) + (self.W - self.P)

    def insert(self, frames):
        """Insert a list of frames (any objects); returns frames evicted."""
        n = len(frames)
        if n > self.capacity_for_insert():
            raise ValueError("cannot insert more frames than the ring can hold at once")
        R = self.W - self.P
        evicted = 0
        for f in frames:
            if self.count < self.P:
                self.slots[self.count] = f
                self.count += 1
                continue
            if self.count == self.W:
                evicted += 1
            self.slots[self.head] = f
            self.head = self.P + (self.head - self.P + 1) % R
            self.count = min(self.W, self.count + 1)
        return evicted

    def start(self):
        """Slot of the oldest valid frame of the rolling region."""
        rolling = max(0, self.count - self.P)
        return self.P + (self.head - self.P - rolling) % (self.W - self.P)

    def slot_of(self, j):
        """Slot of logical frame j (0 = oldest valid), or -1 when j is not valid."""
        if j < 0 or j >= self.count:
            return -1
        if j < self.P:
            return j
        return self.P + (self.start() - self.P + (j - self.P)) % (self.W - self.P)

    def logical_frames(self):
        """Valid frames, oldest first."""
        return [self.slots[self.slot_of(j)] for j in range(self.count)]

    def valid_slots(self):
        """Sorted physical slot indices holding valid frames."""
        return sorted(self.slot_of(j) for j in range(self.count))

    def physical_keys(self, frame_to_rows):
        """Concatenate valid frames in PHYSICAL slot order (the order attention
        reads them in); ``frame_to_rows`` maps a stored frame to its rows."""
        return np.concatenate([frame_to_rows(self.slots[s]) for s in self.valid_slots()], axis=0)
