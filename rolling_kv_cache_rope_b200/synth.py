"""Seeded synthetic inputs and the workload shapes of the rolling-window layer.

This module is shared by the tests, the benchmark and the oracle side of the
parity checks; it holds none of the method's arithmetic (no RoPE, no softmax,
no ring logic), only random draws and sizes.

Inputs are i.i.d. N(0, 1) draws from ``numpy.random.Generator(PCG64(seed))``
in float32, rounded to bfloat16 (nearest, ties to even) on the host, returned
as uint16 bit patterns.  The same bytes go to the GPU and to the oracle.
The pages describe the workload by shape only (23,400 query tokens, 32,760
context tokens, 12 heads; "A kernel-centric path to real-time video generation
on Trainium", ai4snews summary, second paragraph); no dataset or trained
activation is involved, so these draws stand in for real activations.
"""

from dataclasses import dataclass

import numpy as np


def _normal_bits(rng, shape):
    f = rng.standard_normal(size=shape, dtype=np.float32)
    u = f.view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_normal_bits(seed, shape):
    """uint16 bf16 patterns of N(0,1) float32 draws (PCG64(seed)), RNE-rounded."""
    return _normal_bits(np.random.Generator(np.random.PCG64(int(seed))), shape)


@dataclass(frozen=True)
class Layer:
    """Shape of one rolling-window attention layer."""
    name: str
    heads: int
    head_dim: int
    grid_h: int
    grid_w: int
    q_frames: int          # frames in the query window
    k_frames: int          # frames in the context (cached + current)
    ring_slots: int        # frame slots of the per-layer ring cache
    ring_insert: int       # frames inserted (and evicted, once full) per step
    block_frames: int      # 0 = no mask; else frame-block-causal block size
    seed: int
    pairs: tuple = (22, 21, 21)
    theta: float = 10000.0

    @property
    def frame_tokens(self):
        return self.grid_h * self.grid_w

    @property
    def Lq(self):
        return self.q_frames * self.frame_tokens

    @property
    def Lk(self):
        return self.k_frames * self.frame_tokens

    @property
    def k_t0(self):
        """Time index of the first context frame (context frames are t = 0..)."""
        return 0

    @property
    def q_t0(self):
        """Query window = the last q_frames frames of the context."""
        return self.k_frames - self.q_frames


# Tiny rolling-window layer: 4x6 grid, 2 heads, Lq 72, Lk 120, ring of 5 slots.
TINY = Layer("tiny_4x6_h2_q72_k120", 2, 128, 4, 6, 3, 5, 5, 3, 0, 1000)
# Mid-size layer: 15x26 grid, 12 heads, Lq 1,950, Lk 2,730, ring of 7 slots.
MID = Layer("mid_15x26_h12_q1950_k2730", 12, 128, 15, 26, 5, 7, 7, 5, 0, 1001)
# Paper-shaped denoise pass: 30x52 grid, 12 heads, Lq 23,400, Lk 32,760.
DENOISE = Layer("denoise_30x52_h12_q23400_k32760", 12, 128, 30, 52, 15, 21, 21, 5, 0, 1002)
# Batched two-pass launch: the denoise pass above plus a cache-update pass
# (5 query frames over the same 21-frame context), both frame-block masked.
TWO_PASS_DENOISE = Layer("twopass_denoise_q23400_k32760_b3", 12, 128, 30, 52, 15, 21, 21, 5, 3, 1003)
TWO_PASS_CACHE = Layer("twopass_cache_q7800_k32760_b3", 12, 128, 30, 52, 5, 21, 21, 5, 3, 1004)


@dataclass(frozen=True)
class Sweep:
    """Rolling sweep over many layers: per layer a 21-slot ring, 5 frames in
    per step, the ring seeded with one frame before step 0."""
    layers: int = 30
    steps: int = 8
    heads: int = 12
    head_dim: int = 128
    grid_h: int = 30
    grid_w: int = 52
    ring_slots: int = 21
    insert: int = 5
    q_frames: int = 15
    seed_frames: int = 1

    @property
    def frame_tokens(self):
        return self.grid_h * self.grid_w

    def seed(self, layer, step):
        """Seed of (layer, step); step -1 is the pre-seeded frame."""
        return 4000 + 1000 * layer + step

    def first_new_frame(self, step):
        """Absolute frame index (time t) of the first frame inserted at step."""
        return self.seed_frames + self.insert * step

    def k_frames_after(self, step):
        """Valid ring frames once ``step`` has inserted its frames."""
        return min(self.ring_slots, self.seed_frames + self.insert * (step + 1))

    def step_inputs(self, layer, step):
        """bf16 bits of (q, k_new, v_new) of (layer, step): [rows, heads, head_dim]
        arrays drawn in that order from one PCG64(seed(layer, step)) stream.
        Step -1 is the pre-seeded frame(s): q is None and k/v hold seed_frames
        frames; other steps draw q_frames query frames and insert frames."""
        rng = np.random.Generator(np.random.PCG64(self.seed(layer, step)))
        F, H, D = self.frame_tokens, self.heads, self.head_dim
        n = self.seed_frames if step < 0 else self.insert
        q = None if step < 0 else _normal_bits(rng, (self.q_frames * F, H, D))
        k = _normal_bits(rng, (n * F, H, D))
        v = _normal_bits(rng, (n * F, H, D))
        return q, k, v


SWEEP = Sweep()
