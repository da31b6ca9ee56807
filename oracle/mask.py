"""Frame-block-causal visibility, integer oracle.

The pages describe two passes per sliding window -- denoising, then cache
cleanup/update -- whose attention lengths differ, batched into one run of the
shared parts ("Amazon and Reactor tune Trainium for real-time video
generation", section "Three problems for generic compilers", dynamic shapes;
"Optimizing Real-Time Video Generation on Trainium Chips", item 8 "Model
structure optimizations").  The pages print no mask.  The mask used for the
batched two-pass launch is frame-block causal: a query in frame f sees every key
whose frame lies in f's block of ``block_frames`` frames or an earlier block.

Readings taken (listed in the design notes):

* frames are counted from key frame 0 (the first key of the sequence); key
  token k lies in key frame k // F;
* query token r lies in key frame q_frame_offset + r // F; by default the query
  window is the LAST Lq/F frames of the context (bottom-right alignment), i.e.
  q_frame_offset = Lk/F - Lq/F;
* block index of a frame is floor(frame / block_frames); key visible iff
  block(key frame) <= block(query frame).
"""

import numpy as np


def default_q_frame_offset(Lq, Lk, frame_tokens):
    """Bottom-right alignment: query frame 0 is key frame Lk/F - Lq/F."""
    return Lk // frame_tokens - Lq // frame_tokens


def frame_pair_visible(n_q_frames, n_k_frames, q_frame_offset, block_frames):
    """bool [n_q_frames, n_k_frames]: may query frame a see key frame b."""
    qf = q_frame_offset + np.arange(n_q_frames, dtype=np.int64)
    kf = np.arange(n_k_frames, dtype=np.int64)
    return (kf[None, :] // block_frames) <= (qf[:, None] // block_frames)


def frame_block_visible(Lq, Lk, frame_tokens, q_frame_offset, block_frames, rows=None):
    """bool [len(rows), Lk] token-level visibility (rows default 0..Lq-1)."""
    if rows is None:
        rows = np.arange(Lq, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    qf = q_frame_offset + rows // frame_tokens
    kf = np.arange(Lk, dtype=np.int64) // frame_tokens
    return (kf[None, :] // block_frames) <= (qf[:, None] // block_frames)
