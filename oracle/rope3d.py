"""Three-axis rotary position embedding (3D-RoPE), float64 oracle.

What the pages fix: video RoPE rotates by three positions (time, height, width)
instead of the single token position used in LLMs ("Amazon and Reactor tune
Trainium for real-time video generation", section "Three problems for generic
compilers"; "Optimizing Real-Time Video Generation on Trainium Chips", item 5
"Three core bottlenecks").  It is applied to Q and K before attention.

What the pages leave open, and the reading taken here (each also listed in the
design notes):

* token order inside a frame is row-major over a grid_h x grid_w grid, frames
  follow each other: token i of a sequence whose first frame has time index t0
  sits at t = t0 + i // F, h = (i mod F) // grid_w, w = i mod grid_w with
  F = grid_h * grid_w;
* the head dimension D holds D/2 rotary pairs; pairs are adjacent elements
  (2j, 2j+1); the first ``pairs[0]`` pairs rotate with t, the next
  ``pairs[1]`` with h, the last ``pairs[2]`` with w (22/21/21 for D = 128);
* pair with local index i on an axis that owns n pairs turns by the angle
  pos * theta ** (-i / n), theta = 10000 for all three axes (the standard
  one-axis RoPE frequency law applied to an axis of 2n dimensions);
* rotation is y0 = x0 cos a - x1 sin a, y1 = x0 sin a + x1 cos a; V is not
  rotated.

Two variants the pages leave open are also computed here (the layout and the
frequency base are the two free choices of the reading above): the
"rotate-half" pair layout, where pair j holds elements (j, j + D/2) instead
of (2j, 2j+1), and a frequency base per axis, theta = (theta_t, theta_h,
theta_w).
"""

import numpy as np

AXIS_T, AXIS_H, AXIS_W = 0, 1, 2


def token_positions(token_index, t0, grid_h, grid_w):
    """(t, h, w) int64 arrays for the given token indices of one sequence."""
    i = np.asarray(token_index, dtype=np.int64)
    frame_tokens = grid_h * grid_w
    t = t0 + i // frame_tokens
    within = i % frame_tokens
    h = within // grid_w
    w = within % grid_w
    return t, h, w


def pair_axes(pairs):
    """For each rotary pair j: (axis, local index i, pairs on that axis n)."""
    axis = np.concatenate([np.full(n, a, dtype=np.int64) for a, n in enumerate(pairs)])
    local = np.concatenate([np.arange(n, dtype=np.int64) for n in pairs])
    count = np.concatenate([np.full(n, n, dtype=np.int64) for n in pairs])
    return axis, local, count


def rope_angles(token_index, t0, grid_h, grid_w, pairs, theta):
    """Rotation angle of every (token, pair): float64 [len(token_index), sum(pairs)].

    ``theta`` is one frequency base for all axes or a (t, h, w) triple."""
    t, h, w = token_positions(token_index, t0, grid_h, grid_w)
    pos = np.stack([t, h, w], axis=1).astype(np.float64)            # [L, 3]
    axis, local, count = pair_axes(pairs)
    bases = np.broadcast_to(np.asarray(theta, dtype=np.float64), (3,))
    freq = np.power(bases[axis], -local.astype(np.float64) / count.astype(np.float64))
    return pos[:, axis] * freq[None, :]                               # [L, P]


def rope3d_ref(x, t0, grid_h, grid_w, pairs=(22, 21, 21), theta=10000.0, token_index=None, layout="adjacent"):
    """Rotate x (float64 [L, H, D]) by the 3D-RoPE of its tokens.

    ``token_index`` gives each row's index within its sequence (default
    0..L-1); it lets a caller rotate a sample of rows.  ``theta``: one base or
    a (t, h, w) triple.  ``layout``: "adjacent" (pair j = elements 2j, 2j+1)
    or "half" (pair j = elements j, j + D/2).  Returns float64, same shape.
    D must equal 2 * sum(pairs).
    """
    x = np.asarray(x, dtype=np.float64)
    L, H, D = x.shape
    if D != 2 * sum(pairs):
        raise ValueError("head_dim must be twice the number of rotary pairs")
    if token_index is None:
        token_index = np.arange(L, dtype=np.int64)
    ang = rope_angles(token_index, t0, grid_h, grid_w, pairs, theta)  # [L, P]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    if layout == "adjacent":
        first, second = slice(0, D, 2), slice(1, D, 2)
    elif layout == "half":
        first, second = slice(0, D // 2), slice(D // 2, D)
    else:
        raise ValueError("layout must be 'adjacent' or 'half'")
    x0 = x[..., first]
    x1 = x[..., second]
    y = np.empty_like(x)
    y[..., first] = x0 * c - x1 * s
    y[..., second] = x0 * s + x1 * c
    return y
