"""The mask the attention kernel applies ON THE DEVICE, bit-exact against the
integer oracle.

attn_fwd_varlen_debug runs the attention kernel with a per-row record of what
its softmax actually saw after masking: how many scores of the row were not
-inf, the sum and the largest of their key indices, and how many 128-key
tiles the row's work unit processed.  So the record observes both device-side
parts of the mask: the tile count of each unit (tiles past it are never
loaded) and the per-element predicate on partial tiles.  With N(0,1) inputs no
visible score is -inf, so the record is exact.  For every (sequence, head,
query row) it must equal what the oracle's frame-block visibility gives for
that row: the number of visible keys, the sum of their indices, 1 + the
largest one, and the fewest tiles that hold the visible keys of every row of
the unit.  Cases: the tiny and mid layers at several block sizes and offsets,
ragged tails, three sequences in one launch, the tail split (units run as two
halves) against the same launch without it, and the full-size two-pass
launch (denoise 23,400 + cache-update 7,800 queries over 32,760 keys, blocks
of 3 frames) with and without the split.  The outputs of every debug launch
are also checked against the production entry point."""

import math

import numpy as np
import pytest
import torch

from oracle import default_q_frame_offset, frame_block_visible
from rolling_kv_cache_rope_b200.synth import MID, TINY, TWO_PASS_CACHE, TWO_PASS_DENOISE, bf16_normal_bits
from tests._gpu import assert_attn_close, need_gpu, to_dev, to_f64

pytestmark = pytest.mark.gpu
D = 128
UNIT_ROWS = 512
KEY_TILE = 128


def expected_stats(Lq, Lk, F, q_frame_offset, block_frames, chunk=512):
    """int64 [Lq, 4] from the oracle visibility: count, index sum mod 2^32,
    1 + largest visible index, key tiles of the row's 512-row unit."""
    out = np.zeros((Lq, 4), dtype=np.int64)
    keys = np.arange(Lk, dtype=np.int64)
    for r0 in range(0, Lq, chunk):
        r1 = min(Lq, r0 + chunk)
        if block_frames > 0:
            vis = frame_block_visible(Lq, Lk, F, q_frame_offset, block_frames, rows=np.arange(r0, r1))
        else:
            vis = np.ones((r1 - r0, Lk), dtype=bool)
        out[r0:r1, 0] = vis.sum(1)
        out[r0:r1, 1] = (vis @ keys) % (1 << 32)
        last = Lk - np.argmax(vis[:, ::-1], axis=1)
        out[r0:r1, 2] = np.where(vis.any(1), last, 0)
    for u0 in range(0, Lq, UNIT_ROWS):
        u1 = min(Lq, u0 + UNIT_ROWS)
        out[u0:u1, 3] = -(-out[u0:u1, 2].max() // KEY_TILE)
    return out


def run_with_stats(specs, H, grid_h, grid_w, split=True, seed0=0):
    """One debug launch of every spec; returns (row stats [sum Lq, H, 4],
    outputs of the debug launch, outputs of the production launch)."""
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    rope = rkv.make_rope(grid_h, grid_w)
    seqs_dbg, seqs_ref = [], []
    for i, sp in enumerate(specs):
        Lq, Lk = sp["Lq"], sp["Lk"]
        q = to_dev(bf16_normal_bits(seed0 + 3 * i, (Lq, H, D)))
        k = to_dev(bf16_normal_bits(seed0 + 3 * i + 1, (Lk, H, D)))
        v = to_dev(bf16_normal_bits(seed0 + 3 * i + 2, (Lk, H, D)))
        for lst in (seqs_dbg, seqs_ref):
            o = torch.full((Lq, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
            lst.append(rkv.AttnSeq(q, k, v, o, q_t0=sp.get("q_t0", 0), k_t0=0, block_frames=sp["block_frames"],
                                   q_frame_offset=sp["q_frame_offset"]))
    rows = sum(sp["Lq"] for sp in specs)
    stats = torch.full((rows, H, 4), -1, dtype=torch.int32, device="cuda")
    ws_bytes = rkv.attn_fwd_varlen_workspace_size(len(specs), H, D) if split else 256
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    rkv.attn_fwd_varlen_debug(seqs_dbg, rope, row_stats=stats, workspace=ws)
    rkv.rkv_attn_status(ws)
    rkv.attn_fwd_varlen(seqs_ref, rope, workspace=ws)
    rkv.rkv_attn_status(ws)
    torch.cuda.synchronize()
    return stats.cpu().numpy().astype(np.int64), seqs_dbg, seqs_ref


def check(specs, H, grid_h, grid_w, split=True):
    F = grid_h * grid_w
    got, seqs_dbg, seqs_ref = run_with_stats(specs, H, grid_h, grid_w, split=split)
    got[..., 1] %= 1 << 32
    row = 0
    for sp, sd, sr in zip(specs, seqs_dbg, seqs_ref):
        want = expected_stats(sp["Lq"], sp["Lk"], F, sp["q_frame_offset"], sp["block_frames"])
        g = got[row:row + sp["Lq"]]                       # [Lq, H, 4]
        for h in range(H):
            bad = np.nonzero(np.any(g[:, h] != want, axis=1))[0]
            assert bad.size == 0, (sp, h, bad[:5].tolist(), g[bad[:3], h].tolist(), want[bad[:3]].tolist())
        row += sp["Lq"]
        # the debug instantiation computes the same outputs as the production one
        assert_attn_close(to_f64(sd.o), to_f64(sr.o), what=f"debug vs production {sp}")
    return got


def S(Lq, Lk, block_frames=0, q_frame_offset=0, q_t0=0):
    return dict(Lq=Lq, Lk=Lk, block_frames=block_frames, q_frame_offset=q_frame_offset, q_t0=q_t0)


@pytest.mark.parametrize("block,offset", [(0, 0), (1, 2), (2, 2), (3, 2), (3, 0), (5, 1)])
def test_tiny_layer(block, offset):
    check([S(TINY.Lq, TINY.Lk, block, offset, TINY.q_t0)], TINY.heads, TINY.grid_h, TINY.grid_w)


@pytest.mark.parametrize("block", [0, 3])
def test_mid_layer(block):
    off = default_q_frame_offset(MID.Lq, MID.Lk, MID.frame_tokens)
    check([S(MID.Lq, MID.Lk, block, off, MID.q_t0)], MID.heads, MID.grid_h, MID.grid_w)


@pytest.mark.parametrize("block,offset", [(1, 0), (2, 1), (3, 2), (5, 0)])
def test_ragged_tails(block, offset):
    # 300 queries, 333 keys: ragged in the 128-key tile and in the 24-token frame
    check([S(300, 333, block, offset, 1)], 3, 4, 6)


def test_three_sequences_one_launch():
    check([S(7 * 24, 9 * 24 + 5, 2, 2), S(100, 333), S(13 * 24, 20 * 24, 3, 7)], 3, 4, 6)


@pytest.mark.parametrize("split", [True, False])
def test_tail_split_masked(split):
    # 12 heads x 7 blocks of 512 query rows = 84 units on 74 CTA pairs, all of
    # the same cost (each unit's last row sees all 3,600 keys; the first 360
    # rows see 3,240, a partial tile): with the split the last 10 units run as
    # two halves over their key tiles, and their records add up
    check([S(7 * 512, 30 * 120, 3, 24, q_t0=24)], 12, 8, 15, split=split)


def test_masked_longest_first_schedule():
    # units of different cost (128-token frames, query frames 0.. see 3 to 30
    # key frames): scheduled longest-first over the CTA pairs
    check([S(28 * 128, 30 * 128, 3, 0)], 12, 8, 16)


@pytest.mark.slow
@pytest.mark.parametrize("split", [True, False])
def test_two_pass_full_size(split):
    # the batched two-pass launch at full size: 31,200 query rows x 12 heads
    F = TWO_PASS_DENOISE.frame_tokens
    specs = [S(TWO_PASS_DENOISE.Lq, TWO_PASS_DENOISE.Lk, 3,
               default_q_frame_offset(TWO_PASS_DENOISE.Lq, TWO_PASS_DENOISE.Lk, F), TWO_PASS_DENOISE.q_t0),
             S(TWO_PASS_CACHE.Lq, TWO_PASS_CACHE.Lk, 3,
               default_q_frame_offset(TWO_PASS_CACHE.Lq, TWO_PASS_CACHE.Lk, F), TWO_PASS_CACHE.q_t0)]
    got = check(specs, TWO_PASS_DENOISE.heads, TWO_PASS_DENOISE.grid_h, TWO_PASS_DENOISE.grid_w, split=split)
    # the visible (query, key) pairs of the launch: 225 of 315 frame pairs for
    # the denoise pass, 99 of 105 for the cache-update pass, each F x F keys
    assert int(got[..., 0].sum()) == TWO_PASS_DENOISE.heads * F * F * (225 + 99)


@pytest.mark.slow
def test_denoise_full_size_unmasked():
    from rolling_kv_cache_rope_b200.synth import DENOISE
    check([S(DENOISE.Lq, DENOISE.Lk, 0, 0, DENOISE.q_t0)], DENOISE.heads, DENOISE.grid_h, DENOISE.grid_w)
