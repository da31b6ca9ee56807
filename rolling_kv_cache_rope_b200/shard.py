"""Attention of one layer split over several GPUs, one process per GPU.

Source: 12 attention heads do not divide over 8 cores, a split by heads alone
needs padding and a split of the sequence alone may cut a frame's 3D token
block, so the pages split heads over 4 cores and the sequence over 2
("Optimizing Real-Time Video Generation on Trainium Chips", item 7 "Hybrid
sharding solution"; "A kernel-centric path to real-time video generation on
Trainium", ai4snews summary, paragraph 2).

The same two cuts on GPUs, at a finer grain: the work of one sequence is
H x q_frames units, (head h, query frame f), each needing only head h's Q
rows of frame f and head h's whole K and V.  Rank r takes a contiguous run
of units in head-major order, the runs differing in length by at most one
unit, so there is no padding and no cut inside a frame; when world divides
H every rank holds whole heads.  A rank's run is a few segments (h, f0, f1)
that become single-head sequences of ONE attention launch (one view of
several heads when the rank holds whole heads): the query view
starts at frame f0, so its time index is q_t0 + f0 and its mask offset
q_frame_offset + f0 (the (h, w) position of a row depends only on the row
within its frame).  The ring of each layer shards by heads the same way: a
rank keeps the heads [h0, h1) = unit_runs(...)[rank].heads() its units touch,
in a KVRing of h1 - h0 heads fed with the head slices k_new[:, h0:h1] and
v_new[:, h0:h1] (strided views the ring insert accepts), and passes
kv_head0 = h0 when it attends over that ring.  Nothing is exchanged inside
attention; the one collective is the all-gather of the outputs for a
consumer that needs every head of every row (the output projection, outside
this library).
"""

from dataclasses import dataclass


@dataclass(frozen=True)
class UnitRun:
    """Units [u0, u1) of one sequence (unit u = head u // q_frames, query frame
    u % q_frames) held by one rank."""
    rank: int
    u0: int
    u1: int
    q_frames: int

    @property
    def units(self):
        return self.u1 - self.u0

    def segments(self):
        """(head, f0, f1) pieces of the run, in unit order."""
        out, u = [], self.u0
        while u < self.u1:
            h, f0 = divmod(u, self.q_frames)
            f1 = min(self.q_frames, f0 + (self.u1 - u))
            out.append((h, f0, f1))
            u += f1 - f0
        return out

    def heads(self):
        """The head range [h0, h1) the run touches (its K/V and ring heads)."""
        if self.units == 0:
            return (0, 0)
        return (self.u0 // self.q_frames, (self.u1 - 1) // self.q_frames + 1)


def unit_runs(H, q_frames, world):
    """Contiguous unit runs of ``world`` ranks over H * q_frames units; the
    first (H * q_frames) % world ranks take one unit more."""
    if H < 1 or q_frames < 1 or world < 1:
        raise ValueError("H, q_frames and world must be >= 1")
    n = H * q_frames
    if world > n:
        raise ValueError(f"cannot split {n} units over {world} ranks")
    base, extra = divmod(n, world)
    out, u = [], 0
    for r in range(world):
        k = base + (1 if r < extra else 0)
        out.append(UnitRun(r, u, u + k, q_frames))
        u += k
    return out


def _query_frames(seq, F):
    Lq = seq.q.shape[0]
    if Lq % F:
        raise ValueError(f"query rows ({Lq}) must be whole frames of {F} tokens")
    return Lq // F


def shard_seqs(seqs, F, rank, world, kv_head0=0):
    """The AttnSeqs of ``rank``'s units of every sequence (views of the
    callers' tensors; no copies): one view of its heads per sequence when
    every rank holds whole heads, else one single-head view per segment (one
    launch takes at most 16).  Q and O hold every head; K and V hold heads
    from ``kv_head0`` on (a rank's own ring holds only the heads its units
    touch: kv_head0 = that run's first head)."""
    from .rkv import AttnSeq
    runs = [unit_runs(seq.q.shape[1], _query_frames(seq, F), world)[rank] for seq in seqs]
    whole = [all((f0, f1) == (0, r.q_frames) for _, f0, f1 in r.segments()) for r in runs]
    if all(whole) and len({r.heads()[1] - r.heads()[0] for r in runs}) == 1:
        # whole heads everywhere (world divides H): one multi-head view per sequence
        out = []
        for seq, r in zip(seqs, runs):
            h0, h1 = r.heads()
            if h0 - kv_head0 < 0 or h1 - kv_head0 > seq.k.shape[1]:
                raise ValueError(f"heads [{h0}, {h1}) are not among the K/V heads starting at {kv_head0}")
            hs, kv = slice(h0, h1), slice(h0 - kv_head0, h1 - kv_head0)
            s = AttnSeq(seq.q[:, hs], seq.k[:, kv], seq.v[:, kv], seq.o[:, hs], q_t0=seq.q_t0, k_t0=seq.k_t0,
                        block_frames=seq.block_frames, q_frame_offset=seq.q_frame_offset)
            s.flags = seq.flags
            out.append(s)
        return out
    out = []
    for seq, run in zip(seqs, runs):
        for h, f0, f1 in run.segments():
            rows, hs, kv = slice(f0 * F, f1 * F), slice(h, h + 1), slice(h - kv_head0, h - kv_head0 + 1)
            if not 0 <= h - kv_head0 < seq.k.shape[1]:
                raise ValueError(f"head {h} is not among the K/V heads starting at {kv_head0}")
            s = AttnSeq(seq.q[rows, hs], seq.k[:, kv], seq.v[:, kv], seq.o[rows, hs], q_t0=seq.q_t0 + f0,
                        k_t0=seq.k_t0, block_frames=seq.block_frames, q_frame_offset=seq.q_frame_offset + f0)
            s.flags = seq.flags
            out.append(s)
    return out


def attn_fwd_sharded(seqs, rope, rank, world, kv_head0=0, softmax_scale=None, workspace=None, stream=None):
    """Fused attention of ``rank``'s units of every sequence in one launch;
    writes those (head, frame) blocks of each seq.o.  Returns the workspace
    (attn_fwd_varlen_workspace_size(n, 1, D) bytes for n single-head pieces)."""
    from .rkv import attn_fwd_varlen
    mine = shard_seqs(seqs, rope.grid_h * rope.grid_w, rank, world, kv_head0)
    return attn_fwd_varlen(mine, rope, softmax_scale=softmax_scale, workspace=workspace, stream=stream)


def all_gather_units(o, F, rank, world, group=None):
    """``o`` ([Lq, H, D], Lq whole frames of F tokens) holds this rank's units;
    after the call every rank holds all of them.  Each rank packs its units'
    rows into one block (padded to the largest run), one all-gather moves the
    blocks, and each is unpacked into its (head, frame) places."""
    import torch
    import torch.distributed as dist
    Lq, H, D = o.shape
    if Lq % F:
        raise ValueError(f"query rows ({Lq}) must be whole frames of {F} tokens")
    runs = unit_runs(H, Lq // F, world)
    cap = runs[0].units * F
    mine = torch.zeros((cap, D), dtype=o.dtype, device=o.device)
    at = 0
    for h, f0, f1 in runs[rank].segments():
        n = (f1 - f0) * F
        mine[at:at + n] = o[f0 * F:f1 * F, h]
        at += n
    # 16-bit data moves as int32 pairs: a plain copy, exact, in a type every
    # backend carries
    wire = (lambda t: t.view(torch.int32)) if o.element_size() == 2 and D % 2 == 0 else (lambda t: t)
    blocks = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather([wire(b) for b in blocks], wire(mine), group=group)
    for run, blk in zip(runs, blocks):
        if run.rank == rank:
            continue
        at = 0
        for h, f0, f1 in run.segments():
            n = (f1 - f0) * F
            o[f0 * F:f1 * F, h] = blk[at:at + n]
            at += n
    return o
