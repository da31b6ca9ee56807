"""Fused 3D-RoPE attention on the GPU vs the fp64 oracle.

Small cases compare every output; full-size cases (23,400 x 32,760, the
two-pass launch) compare sampled query rows that include tile, unit, frame
and mask-block boundaries.  Tolerances: max |err| <= 2e-2, mean |err| <= 2e-3,
relative L2 <= 1e-2 (bf16 operands, fp32 accumulation, N(0,1) inputs)."""

import math

import numpy as np
import pytest
import torch

from oracle import bf16_bits_to_f64, default_q_frame_offset, fused_attention_ref
from rolling_kv_cache_rope_b200.synth import (DENOISE, MID, TINY, TWO_PASS_CACHE, TWO_PASS_DENOISE,
                                              bf16_normal_bits)
from tests._gpu import assert_attn_close, need_gpu, to_dev, to_f64

pytestmark = pytest.mark.gpu
D = 128


def boundary_rows(Lq, F, n_random=24, seed=0):
    cand = {0, 1, Lq - 1, Lq - 2}
    for b in (127, 128, 129, 255, 256, 257):
        cand.update({b, Lq - 1 - b})
    for f in range(1, Lq // F + 1):
        cand.update({f * F - 1, f * F})
    cand.update(np.random.default_rng(seed).integers(0, Lq, n_random).tolist())
    return np.array(sorted(r for r in cand if 0 <= r < Lq), dtype=np.int64)


def run_launch(specs, H, grid_h, grid_w, pairs=(22, 21, 21), scale=None, sample=None):
    """specs: dicts with Lq, Lk, q_t0, k_t0, rope_q, rope_k, block_frames,
    q_frame_offset, seed, [fused_qkv].  All run in ONE attn_fwd_varlen call."""
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    F = grid_h * grid_w
    host, seqs = [], []
    for sp in specs:
        Lq, Lk = sp["Lq"], sp["Lk"]
        qb = bf16_normal_bits(sp["seed"], (Lq, H, D))
        kb = bf16_normal_bits(sp["seed"] + 100, (Lk, H, D))
        vb = bf16_normal_bits(sp["seed"] + 200, (Lk, H, D))
        if sp.get("fused_qkv"):
            assert Lq == Lk
            qkv = to_dev(np.stack([qb, kb, vb], axis=1))          # [L, 3, H, D]
            q, k, v = qkv[:, 0], qkv[:, 1], qkv[:, 2]
        else:
            q, k, v = to_dev(qb), to_dev(kb), to_dev(vb)
        o = torch.full((Lq, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        seqs.append(rkv.AttnSeq(q, k, v, o, q_t0=sp["q_t0"], k_t0=sp["k_t0"], rope_q=sp["rope_q"],
                                rope_k=sp["rope_k"], block_frames=sp["block_frames"],
                                q_frame_offset=sp["q_frame_offset"]))
        host.append((qb, kb, vb))
    ws = rkv.attn_fwd_varlen(seqs, rkv.make_rope(grid_h, grid_w, pairs), softmax_scale=scale)
    rkv.rkv_attn_status(ws)
    torch.cuda.synchronize()
    results = []
    for sp, (qb, kb, vb), s in zip(specs, host, seqs):
        rows = None
        if sample is not None and sp["Lq"] > sample:
            rows = boundary_rows(sp["Lq"], F)
        ref = fused_attention_ref(bf16_bits_to_f64(qb), bf16_bits_to_f64(kb), bf16_bits_to_f64(vb),
                                  scale=scale, grid_h=grid_h, grid_w=grid_w, rope_q=sp["rope_q"],
                                  rope_k=sp["rope_k"], q_t0=sp["q_t0"], k_t0=sp["k_t0"], pairs=pairs,
                                  block_frames=sp["block_frames"], q_frame_offset=sp["q_frame_offset"], rows=rows)
        got = to_f64(s.o)
        if rows is not None:
            got = got[rows]
        results.append(assert_attn_close(got, ref, what=str(sp)))
    return results


def spec(Lq, Lk, seed, q_t0=0, k_t0=0, rope_q=True, rope_k=True, block_frames=0, q_frame_offset=0, **kw):
    d = dict(Lq=Lq, Lk=Lk, seed=seed, q_t0=q_t0, k_t0=k_t0, rope_q=rope_q, rope_k=rope_k,
             block_frames=block_frames, q_frame_offset=q_frame_offset)
    d.update(kw)
    return d


def layer_spec(layer, masked=False):
    return spec(layer.Lq, layer.Lk, layer.seed, q_t0=layer.q_t0, k_t0=layer.k_t0,
                block_frames=layer.block_frames if masked else 0,
                q_frame_offset=default_q_frame_offset(layer.Lq, layer.Lk, layer.frame_tokens))


def test_tiny_layer_all_rows():
    run_launch([layer_spec(TINY)], TINY.heads, TINY.grid_h, TINY.grid_w)


def test_tiny_layer_frame_block_mask():
    s = layer_spec(TINY)
    s.update(block_frames=3)
    run_launch([s], TINY.heads, TINY.grid_h, TINY.grid_w)


def test_mid_layer_all_rows():
    run_launch([layer_spec(MID)], MID.heads, MID.grid_h, MID.grid_w)


@pytest.mark.parametrize("Lq,Lk", [(1, 1), (1, 129), (129, 1), (128, 128), (256, 256), (257, 383), (300, 333)])
def test_ragged_shapes(Lq, Lk):
    run_launch([spec(Lq, Lk, seed=Lq * 1000 + Lk, q_t0=1)], 3, 4, 6)


@pytest.mark.parametrize("block_frames,offset", [(1, 0), (2, 1), (3, 2), (5, 0)])
def test_ragged_masked(block_frames, offset):
    run_launch([spec(300, 333, seed=70 + block_frames, q_t0=1, block_frames=block_frames, q_frame_offset=offset)],
               3, 4, 6)


@pytest.mark.parametrize("rq,rk", [(False, False), (True, False), (False, True)])
def test_rope_flags(rq, rk):
    run_launch([spec(200, 260, seed=80, q_t0=3, k_t0=1, rope_q=rq, rope_k=rk)], 2, 4, 6)


def test_custom_scale_and_axis_split():
    run_launch([spec(150, 170, seed=81, q_t0=2)], 2, 5, 7, pairs=(32, 16, 16), scale=0.05)


def test_fused_qkv_strided_views():
    run_launch([spec(520, 520, seed=82, q_t0=0, fused_qkv=True)], 4, 4, 6)


def test_varlen_three_sequences_one_launch():
    run_launch([spec(72, 120, seed=83, q_t0=2, block_frames=3, q_frame_offset=2),
                spec(500, 700, seed=84, q_t0=5),
                spec(24, 96, seed=85, q_t0=3, block_frames=1, q_frame_offset=3)], 2, 4, 6)


def test_denoise_pass_full_size_sampled():
    run_launch([layer_spec(DENOISE)], DENOISE.heads, DENOISE.grid_h, DENOISE.grid_w, sample=256)


def test_two_pass_batched_launch_sampled():
    # denoise pass (15 query frames) + cache-update pass (5 query frames), both
    # over a 21-frame context with the 3-frame block mask, in one launch
    run_launch([layer_spec(TWO_PASS_DENOISE, masked=True), layer_spec(TWO_PASS_CACHE, masked=True)],
               TWO_PASS_DENOISE.heads, TWO_PASS_DENOISE.grid_h, TWO_PASS_DENOISE.grid_w, sample=256)
