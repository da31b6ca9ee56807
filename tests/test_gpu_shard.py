"""Attention split by (head, query frame) units, every rank's launch run in
turn on one GPU (the launches do not wait on one another): after all ranks of
a world have run, every output row of every head is written once and matches
the fp64 oracle on the whole sequence (RoPE on Q and K, frame-block mask)
within the attention tolerances, and matches the unsplit launch.  A rank whose
K and V hold only the heads its units touch (kv_head0) writes the same bits
as with the full K and V."""

import math

import numpy as np
import pytest
import torch

from oracle import bf16_bits_to_f64, fused_attention_ref
from rolling_kv_cache_rope_b200.synth import bf16_normal_bits
from tests._gpu import assert_attn_close, need_gpu, to_bits, to_dev, to_f64

pytestmark = pytest.mark.gpu

H, GH, GW, D = 12, 4, 6, 128
F = GH * GW
QF, KF = 5, 8
Q_T0 = KF - QF
BLOCK = 2


def inputs():
    q = bf16_normal_bits(5100, (QF * F, H, D))
    k = bf16_normal_bits(5101, (KF * F, H, D))
    v = bf16_normal_bits(5102, (KF * F, H, D))
    return q, k, v


def oracle():
    q, k, v = (bf16_bits_to_f64(x) for x in inputs())
    return fused_attention_ref(q, k, v, scale=1.0 / math.sqrt(D), grid_h=GH, grid_w=GW, rope_q=True, rope_k=True,
                               q_t0=Q_T0, k_t0=0, block_frames=BLOCK, q_frame_offset=Q_T0)


@pytest.mark.parametrize("world", [2, 3, 8])
def test_all_ranks_together_give_the_whole_output(world):
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    from rolling_kv_cache_rope_b200.shard import attn_fwd_sharded
    q, k, v = (to_dev(x) for x in inputs())
    rope = rkv.make_rope(GH, GW)
    o = torch.full((QF * F, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    seq = rkv.AttnSeq(q, k, v, o, q_t0=Q_T0, k_t0=0, block_frames=BLOCK, q_frame_offset=Q_T0)
    for rank in range(world):
        ws = attn_fwd_sharded([seq], rope, rank, world)
        rkv.rkv_attn_status(ws)
    torch.cuda.synchronize()
    got = to_f64(o)
    assert np.all(np.isfinite(got))
    assert_attn_close(got, oracle(), f"world {world}")
    whole = torch.empty_like(o)
    ws = rkv.attn_fwd_varlen([rkv.AttnSeq(q, k, v, whole, q_t0=Q_T0, k_t0=0, block_frames=BLOCK,
                                          q_frame_offset=Q_T0)], rope)
    rkv.rkv_attn_status(ws)
    assert_attn_close(got, to_f64(whole), f"world {world} vs unsplit")


def test_rank_with_only_its_own_heads_of_k_and_v():
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    from rolling_kv_cache_rope_b200.shard import attn_fwd_sharded, unit_runs
    world, rank = 8, 1
    h0, h1 = unit_runs(H, QF, world)[rank].heads()
    q, k, v = (to_dev(x) for x in inputs())
    rope = rkv.make_rope(GH, GW)
    outs = []
    for kk, vv, base in ((k, v, 0), (k[:, h0:h1].contiguous(), v[:, h0:h1].contiguous(), h0)):
        o = torch.zeros((QF * F, H, D), dtype=torch.bfloat16, device="cuda")
        seq = rkv.AttnSeq(q, kk, vv, o, q_t0=Q_T0, k_t0=0, block_frames=BLOCK, q_frame_offset=Q_T0)
        ws = attn_fwd_sharded([seq], rope, rank, world, kv_head0=base)
        rkv.rkv_attn_status(ws)
        outs.append(to_bits(o))
    assert np.array_equal(outs[0], outs[1])
    assert np.any(outs[0] != 0)
