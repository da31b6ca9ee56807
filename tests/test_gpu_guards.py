"""Guard regions around every output: no kernel writes a byte outside it.

A stand-in for a memory checker (which this project does not run): each
output lives inside a larger buffer filled with a sentinel bf16 pattern that
no N(0,1) draw or kernel result can produce (a quiet NaN), with guard rows
before and after it and, for row-strided and head-sliced views, guard columns
and heads around it.  After the call every byte outside the view must still
hold the sentinel, and every byte inside must have been written.  Covers the
attention output (whole tensor, head slices of a wider tensor, a row-strided
view, the tail split whose merge kernel writes the last units) and
rope3d_apply (out of place into a strided view, in place)."""

import math

import numpy as np
import pytest
import torch

from rolling_kv_cache_rope_b200.synth import bf16_normal_bits
from tests._gpu import need_gpu, to_bits, to_dev

pytestmark = pytest.mark.gpu
D = 128
SENTINEL = 0x7FC1
GUARD_ROWS = 3


def guarded(rows, heads_total, head0, heads):
    """A sentinel-filled [GUARD + rows + GUARD, heads_total, D] buffer and the
    view of its rows [GUARD, GUARD + rows) and heads [head0, head0 + heads)."""
    buf = torch.full((rows + 2 * GUARD_ROWS, heads_total, D), SENTINEL, dtype=torch.int16, device="cuda")
    view = buf.view(torch.bfloat16)[GUARD_ROWS:GUARD_ROWS + rows, head0:head0 + heads]
    return buf, view


def check_guards(buf, rows, head0, heads):
    b = to_bits(buf.view(torch.bfloat16))
    inside = np.zeros(b.shape, dtype=bool)
    inside[GUARD_ROWS:GUARD_ROWS + rows, head0:head0 + heads] = True
    assert np.all(b[~inside] == SENTINEL), "a byte outside the output view was written"
    assert not np.any(b[inside] == SENTINEL), "a byte of the output view was not written"


@pytest.mark.parametrize("Lq,Lk,H,heads_total,head0,grid", [
    (72, 120, 2, 2, 0, (4, 6)),         # whole tensor
    (300, 333, 3, 7, 2, (4, 6)),        # head slice of a wider tensor, ragged tails
    (1000, 640, 4, 9, 5, (8, 16)),      # head slice at the end of the row
    (7 * 512, 640, 12, 14, 1, (8, 16)), # 84 units on 74 pairs: tail split, merge kernel writes
])
def test_attention_output_guards(Lq, Lk, H, heads_total, head0, grid):
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    q = to_dev(bf16_normal_bits(Lq + 1, (Lq, H, D)))
    k = to_dev(bf16_normal_bits(Lk + 2, (Lk, H, D)))
    v = to_dev(bf16_normal_bits(Lk + 3, (Lk, H, D)))
    buf, o = guarded(Lq, heads_total, head0, H)
    F = grid[0] * grid[1]
    seq = rkv.AttnSeq(q, k, v, o, q_t0=1, k_t0=0, block_frames=3 if Lq % F == 0 else 0,
                      q_frame_offset=max(0, Lk // F - Lq // F))
    ws = rkv.attn_fwd_varlen([seq], rkv.make_rope(*grid), softmax_scale=1.0 / math.sqrt(D))
    rkv.rkv_attn_status(ws)
    torch.cuda.synchronize()
    check_guards(buf, Lq, head0, H)


def test_attention_two_sequences_head_slices_of_one_tensor():
    # two sequences write disjoint head slices of ONE output tensor in one launch
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    Lq, Lk, H = 300, 333, 3
    buf = torch.full((Lq + 2 * GUARD_ROWS, 2 * H + 2, D), SENTINEL, dtype=torch.int16, device="cuda")
    ob = buf.view(torch.bfloat16)
    seqs = []
    for i in range(2):
        q = to_dev(bf16_normal_bits(10 + i, (Lq, H, D)))
        k = to_dev(bf16_normal_bits(20 + i, (Lk, H, D)))
        v = to_dev(bf16_normal_bits(30 + i, (Lk, H, D)))
        seqs.append(rkv.AttnSeq(q, k, v, ob[GUARD_ROWS:GUARD_ROWS + Lq, 1 + i * H:1 + (i + 1) * H], q_t0=1))
    ws = rkv.attn_fwd_varlen(seqs, rkv.make_rope(4, 6))
    rkv.rkv_attn_status(ws)
    torch.cuda.synchronize()
    check_guards(buf, Lq, 1, 2 * H)


@pytest.mark.parametrize("L,H,heads_total,head0", [(72, 2, 2, 0), (1000, 3, 5, 1), (23400 // 10, 12, 13, 1)])
def test_rope3d_output_guards(L, H, heads_total, head0):
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    x = to_dev(bf16_normal_bits(L + 7, (L, H, D)))
    buf, y = guarded(L, heads_total, head0, H)
    rkv.rope3d_apply(x, y, t0=2, rope=rkv.make_rope(4, 6))
    torch.cuda.synchronize()
    check_guards(buf, L, head0, H)


def test_rope3d_in_place_guards():
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    L, H = 500, 3
    buf, y = guarded(L, 5, 1, H)
    y.copy_(to_dev(bf16_normal_bits(5, (L, H, D))))
    rkv.rope3d_apply(y, y, t0=0, rope=rkv.make_rope(4, 6))
    torch.cuda.synchronize()
    check_guards(buf, L, 1, H)
