"""Softmax attention (SDPA) with optional 3D-RoPE and frame-block mask, float64.

The step the pages put at about 70% of compute: 23,400 query tokens attending
to 32,760 context tokens, 12 heads ("A kernel-centric path to real-time video
generation on Trainium", ai4snews summary, second paragraph; "Optimizing
Real-Time Video Generation on Trainium Chips", item 4 "Rolling Forcing
advantages").  The pages call it SDPA ("A kernel-centric path to real-time
video generation on Trainium", yomu.fyi summary, Summary), so the plain
definition applies, per head h:

    S = Q_h K_h^T * scale           (scale = 1/sqrt(D), the SDPA default)
    S[r, c] = -inf where key c is hidden from query r
    P = exp(S - rowmax(S)),  O_h = (P V_h) / rowsum(P)

A row that sees no key at all returns zeros (reading: the pages never produce
one; the plainest value for an empty average).  Layout everywhere is
token-major [L, H, D]; the pages fold the attention transposes into the kernel
("Amazon and Reactor tune Trainium for real-time video generation", section
"Results with the Neuron Kernel Interface"), so no transposed copy is part of
the definition.
"""

import numpy as np

from .rope3d import rope3d_ref
from .mask import frame_block_visible


def _one_head(qh, kh, vh, scale, visible):
    s = (qh @ kh.T) * scale
    if visible is not None:
        s = np.where(visible, s, -np.inf)
    m = np.max(s, axis=1, keepdims=True)
    empty = ~np.isfinite(m)
    m = np.where(empty, 0.0, m)
    p = np.exp(s - m)
    l = np.sum(p, axis=1, keepdims=True)
    o = p @ vh
    with np.errstate(invalid="ignore", divide="ignore"):
        o = np.where(l > 0, o / np.where(l > 0, l, 1.0), 0.0)
    return o


def attention_ref(q, k, v, scale, visible=None, row_chunk=512):
    """O float64 [Lq, H, D] from float64 q [Lq,H,D], k/v [Lk,H,D].

    ``visible`` is None (every key visible) or bool [Lq, Lk].  Rows are taken
    ``row_chunk`` at a time only to bound memory; each row's result does not
    depend on the chunking.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Lq, H, D = q.shape
    out = np.zeros((Lq, H, v.shape[2]), dtype=np.float64)
    for h in range(H):
        kh = k[:, h, :]
        vh = v[:, h, :]
        for r0 in range(0, Lq, row_chunk):
            r1 = min(Lq, r0 + row_chunk)
            vis = None if visible is None else visible[r0:r1]
            out[r0:r1, h, :] = _one_head(q[r0:r1, h, :], kh, vh, scale, vis)
    return out


def fused_attention_ref(q_raw, k_raw, v, *, scale, grid_h, grid_w,
                        rope_q, rope_k, q_t0, k_t0, pairs=(22, 21, 21), theta=10000.0,
                        block_frames=0, q_frame_offset=0, rows=None, layout="adjacent"):
    """One sequence of the batched launch: optional RoPE on Q/K, mask, attention.

    Inputs are float64 [L, H, D] (the exact values of the bf16 inputs).  The
    rotated Q and K are used unrounded.  ``rows`` (optional int array) restricts
    the output to those query rows, which is how full-size cases are sampled.
    Returns float64 [len(rows) or Lq, H, D].
    """
    q_raw = np.asarray(q_raw, dtype=np.float64)
    Lq = q_raw.shape[0]
    Lk = k_raw.shape[0]
    if rows is None:
        rows = np.arange(Lq, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    qs = q_raw[rows]
    if rope_q:
        qs = rope3d_ref(qs, q_t0, grid_h, grid_w, pairs, theta, token_index=rows, layout=layout)
    ks = k_raw
    if rope_k:
        ks = rope3d_ref(k_raw, k_t0, grid_h, grid_w, pairs, theta, layout=layout)
    visible = None
    if block_frames > 0:
        visible = frame_block_visible(Lq, Lk, grid_h * grid_w, q_frame_offset,
                                      block_frames, rows=rows)
    return attention_ref(qs, ks, v, scale, visible)


def attention_rows_ref(q_raw, k_raw, v, rows, **kw):
    """Alias of fused_attention_ref restricted to ``rows`` (sampled parity)."""
    return fused_attention_ref(q_raw, k_raw, v, rows=rows, **kw)
