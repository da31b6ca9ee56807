"""The tail of the persistent grid: when the last wave of work units is at
most half full, its units run as two halves over their key tiles and a second
kernel merges the halves.  These cases make that happen with small shapes
(more units than CTA pairs on a B200) and check every output against the fp64
oracle, and against the same launch with a workspace too small for the split
(no split), unmasked and frame-block masked.  The split applies when every
work unit costs the same; launches whose units differ in cost (most masked
or mixed-length launches) are scheduled longest-first instead, which the
masked and varlen cases of the other attention tests cover."""

import math

import numpy as np
import pytest
import torch

from oracle import bf16_bits_to_f64, fused_attention_ref
from rolling_kv_cache_rope_b200.synth import bf16_normal_bits
from tests._gpu import assert_attn_close, need_gpu, to_dev, to_f64

pytestmark = pytest.mark.gpu
D = 128


def run(Lq, Lk, H, grid_h, grid_w, q_t0, block_frames, q_frame_offset, seed, ws_bytes=None):
    from rolling_kv_cache_rope_b200 import rkv
    q = to_dev(bf16_normal_bits(seed, (Lq, H, D)))
    k = to_dev(bf16_normal_bits(seed + 1, (Lk, H, D)))
    v = to_dev(bf16_normal_bits(seed + 2, (Lk, H, D)))
    o = torch.full((Lq, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    seq = rkv.AttnSeq(q, k, v, o, q_t0=q_t0, k_t0=0, block_frames=block_frames, q_frame_offset=q_frame_offset)
    ws = None
    if ws_bytes is not None:
        ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    ws = rkv.attn_fwd_varlen([seq], rkv.make_rope(grid_h, grid_w), workspace=ws)
    rkv.rkv_attn_status(ws)
    torch.cuda.synchronize()
    return o


def check(Lq, Lk, H, grid_h, grid_w, block_frames, seed, q_frame_offset=None):
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    F = grid_h * grid_w
    if q_frame_offset is None:
        q_frame_offset = max(0, Lk // F - Lq // F)   # query frames are the last ones of the context
    q_t0 = q_frame_offset
    full = rkv.attn_fwd_varlen_workspace_size(1, H, D)
    assert full > 256, "workspace has no room for split partial results"
    got = run(Lq, Lk, H, grid_h, grid_w, q_t0, block_frames, q_frame_offset, seed)
    ref_nosplit = run(Lq, Lk, H, grid_h, grid_w, q_t0, block_frames, q_frame_offset, seed, ws_bytes=256)
    qf = bf16_bits_to_f64(bf16_normal_bits(seed, (Lq, H, D)))
    kf = bf16_bits_to_f64(bf16_normal_bits(seed + 1, (Lk, H, D)))
    vf = bf16_bits_to_f64(bf16_normal_bits(seed + 2, (Lk, H, D)))
    want = fused_attention_ref(qf, kf, vf, scale=1.0 / math.sqrt(D), grid_h=grid_h, grid_w=grid_w, rope_q=True,
                               rope_k=True, q_t0=q_t0, k_t0=0, block_frames=block_frames,
                               q_frame_offset=q_frame_offset)
    assert_attn_close(to_f64(got), want, "split tail")
    assert_attn_close(to_f64(ref_nosplit), want, "no split")
    assert_attn_close(to_f64(got), to_f64(ref_nosplit), "split vs no split")


def test_tail_split_unmasked():
    # 12 heads x 7 query blocks of 512 rows = 84 units: 74 in the first wave,
    # the last 10 run as halves; 5 key tiles per unit (2 + 3)
    check(Lq=7 * 512, Lk=640, H=12, grid_h=8, grid_w=16, block_frames=0, seed=700)


def test_tail_split_frame_block_masked():
    # 120-token frames, blocks of 3 frames, query frame 0 = key frame 24: the
    # first 360 query rows see 27 key frames (3,240 keys, a partial tile),
    # every later row all 3,600 keys, and every 512-row unit ends on a row
    # that sees them all, so all 84 units cost the same and the last 10 run
    # as halves
    check(Lq=7 * 512, Lk=30 * 120, H=12, grid_h=8, grid_w=15, block_frames=3, seed=701, q_frame_offset=24)
