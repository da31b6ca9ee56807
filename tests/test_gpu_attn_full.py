"""Full-size attention, EVERY output element against the fp64 oracle.

The denoise pass (23,400 queries over 32,760 keys, 12 heads, RoPE on Q and K
in the kernel) and the batched two-pass launch (that pass plus a 7,800-query
cache-update pass, both frame-block causal) are launched exactly as the
benchmark launches them: one call, the workspace that lets the last wave of
work units run as two halves.  So every work unit, both CTAs of every pair,
both 128-row sub-tiles, every warp and both halves of every split unit are
compared element by element.  The oracle runs one head per worker process
(tests/_oracle_pool.py).  Tolerances: max |err| <= 2e-2, mean |err| <= 2e-3,
relative L2 <= 1e-2, per sequence and also per head."""

import math

import numpy as np
import pytest
import torch

from oracle import default_q_frame_offset
from rolling_kv_cache_rope_b200.synth import DENOISE, TWO_PASS_CACHE, TWO_PASS_DENOISE, bf16_normal_bits
from tests._gpu import assert_attn_close, need_gpu, to_dev, to_f64
from tests._oracle_pool import attention_by_head

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
D = 128


def run_every_row(layers, masked):
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    l0 = layers[0]
    H, F = l0.heads, l0.frame_tokens
    rope = rkv.make_rope(l0.grid_h, l0.grid_w)
    seqs, host = [], []
    for layer in layers:
        qb = bf16_normal_bits(layer.seed, (layer.Lq, H, D))
        kb = bf16_normal_bits(layer.seed + 100, (layer.Lk, H, D))
        vb = bf16_normal_bits(layer.seed + 200, (layer.Lk, H, D))
        off = default_q_frame_offset(layer.Lq, layer.Lk, F)
        o = torch.full((layer.Lq, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        seqs.append(rkv.AttnSeq(to_dev(qb), to_dev(kb), to_dev(vb), o, q_t0=layer.q_t0, k_t0=layer.k_t0,
                                block_frames=layer.block_frames if masked else 0, q_frame_offset=off))
        host.append((qb, kb, vb, off))
    ws = torch.zeros(rkv.attn_fwd_varlen_workspace_size(len(seqs), H, D), dtype=torch.uint8, device="cuda")
    rkv.attn_fwd_varlen(seqs, rope, workspace=ws)
    rkv.rkv_attn_status(ws)
    torch.cuda.synchronize()
    for layer, s, (qb, kb, vb, off) in zip(layers, seqs, host):
        want = attention_by_head(qb, kb, vb, scale=1.0 / math.sqrt(D), grid_h=layer.grid_h, grid_w=layer.grid_w,
                                 rope_q=True, rope_k=True, q_t0=layer.q_t0, k_t0=layer.k_t0,
                                 block_frames=layer.block_frames if masked else 0, q_frame_offset=off)
        got = to_f64(s.o)
        assert got.shape == want.shape
        assert_attn_close(got, want, f"{layer.name}: every row")
        for h in range(H):
            assert_attn_close(got[:, h], want[:, h], f"{layer.name}: head {h}")


def test_denoise_pass_every_row():
    run_every_row([DENOISE], masked=False)


def test_two_pass_batched_launch_every_row():
    run_every_row([TWO_PASS_DENOISE, TWO_PASS_CACHE], masked=True)
