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
"""

import numpy as np


class RingRef:
    """Python-list ring of W slots, each holding a (K, V) frame pair or None."""

    def __init__(self, slots):
        if slots <= 0:
            raise ValueError("slots must be positive")
        self.W = int(slots)
        self.slots = [None] * self.W
        self.head = 0
        self.count = 0

    def insert(self, frames):
        """Insert a list of frames (any objects); returns frames evicted."""
        n = len(frames)
        if n > self.W:
            raise ValueError("cannot insert more frames than slots")
        for i, f in enumerate(frames):
            self.slots[(self.head + i) % self.W] = f
        evicted = max(0, self.count + n - self.W)
        self.head = (self.head + n) % self.W
        self.count = min(self.W, self.count + n)
        return evicted

    def start(self):
        """Slot of the oldest valid frame."""
        return (self.head - self.count) % self.W

    def slot_of(self, j):
        """Slot of logical frame j (0 = oldest valid), or -1 when j is not valid."""
        if j < 0 or j >= self.count:
            return -1
        return (self.start() + j) % self.W

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
