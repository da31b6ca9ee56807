"""Standalone 3D-RoPE on the GPU vs the fp64 oracle: every output within one
bf16 ulp of the oracle's correctly rounded value (nearly all identical)."""

import numpy as np
import pytest
import torch

from oracle import bf16_bits_to_f64, bf16_ulp_distance, f64_to_bf16_bits, rope3d_ref
from rolling_kv_cache_rope_b200.synth import DENOISE, MID, TINY, bf16_normal_bits
from tests._gpu import need_gpu, to_bits, to_dev

pytestmark = pytest.mark.gpu


def check_rope(L, H, grid_h, grid_w, t0, seed, in_place=False, stride_mult=1, pairs=(22, 21, 21)):
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    D = 128
    xb = bf16_normal_bits(seed, (L, H, D))
    ref = f64_to_bf16_bits(rope3d_ref(bf16_bits_to_f64(xb), t0, grid_h, grid_w, pairs))
    rope = rkv.make_rope(grid_h, grid_w, pairs)
    if stride_mult == 1:
        x = to_dev(xb)
    else:
        wide = np.zeros((L, stride_mult * H, D), dtype=np.uint16)
        wide[:, :H] = xb
        x = to_dev(wide)[:, :H, :]
    y = x if in_place else torch.empty((L, H, D), dtype=torch.bfloat16, device="cuda")
    rkv.rope3d_apply(x, y, t0=t0, rope=rope)
    torch.cuda.synchronize()
    got = to_bits(y)
    ulp = bf16_ulp_distance(got, ref)
    assert int(ulp.max()) <= 1, f"max ulp {int(ulp.max())}"
    exact = float((ulp == 0).mean())
    assert exact > 0.999, f"only {exact:.5f} of outputs identical to the oracle's rounding"
    return exact


def test_tiny_q_and_k():
    check_rope(TINY.Lq, TINY.heads, TINY.grid_h, TINY.grid_w, TINY.q_t0, TINY.seed)
    check_rope(TINY.Lk, TINY.heads, TINY.grid_h, TINY.grid_w, TINY.k_t0, TINY.seed + 1)


def test_mid_q_and_k():
    check_rope(MID.Lq, MID.heads, MID.grid_h, MID.grid_w, MID.q_t0, MID.seed)
    check_rope(MID.Lk, MID.heads, MID.grid_h, MID.grid_w, MID.k_t0, MID.seed + 1)


def test_denoise_q_full_size():
    check_rope(DENOISE.Lq, DENOISE.heads, DENOISE.grid_h, DENOISE.grid_w, DENOISE.q_t0, DENOISE.seed)


def test_denoise_k_full_size():
    check_rope(DENOISE.Lk, DENOISE.heads, DENOISE.grid_h, DENOISE.grid_w, DENOISE.k_t0, DENOISE.seed + 1)


def test_in_place_and_strided():
    check_rope(1000, 3, 4, 6, 5, 11, in_place=True)
    check_rope(1000, 3, 4, 6, 5, 12, stride_mult=3)
    check_rope(777, 2, 15, 26, 0, 13, in_place=True, stride_mult=2)


def test_ragged_and_single_row():
    check_rope(1, 1, 30, 52, 9, 14)
    check_rope(1561, 12, 30, 52, 3, 15)          # one frame plus one token
    check_rope(24 * 40 + 7, 2, 4, 6, 35, 16)     # many frames, long time axis


def test_other_axis_split():
    check_rope(300, 2, 5, 7, 1, 17, pairs=(32, 16, 16))


def test_chunk_on_three_axes():
    # splits where one 16-byte chunk (rotary pairs 4c..4c+3) holds pairs of
    # t, h and w: chunk 5 = t | h h | w; chunk 0 = t | h | w w; chunk 1 = t | h | w w
    check_rope(500, 2, 5, 7, 1, 19, pairs=(21, 2, 41))
    check_rope(500, 2, 5, 7, 1, 20, pairs=(1, 1, 62))
    check_rope(500, 2, 5, 7, 1, 21, pairs=(5, 1, 58))


def test_large_time_index():
    check_rope(200, 2, 4, 6, 1000, 18)


def _bits(t):
    return to_bits(t)


def test_batch_matches_separate_calls_and_oracle():
    # Q and K of the mid-size pass in one launch, plus a ragged third tensor
    # rotated in place: each output bit-identical to its own rope3d_apply and
    # within one ulp of the oracle
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    H, D = MID.heads, 128
    rope = rkv.make_rope(MID.grid_h, MID.grid_w)
    shapes = [(MID.Lq, MID.q_t0, 31), (MID.Lk, MID.k_t0, 32), (1000, 4, 33)]
    xs = [bf16_normal_bits(seed, (L, H, D)) for L, _, seed in shapes]
    devs = [to_dev(x) for x in xs]
    inplace = devs[2].clone()
    outs = rkv.rope3d_apply_batch([(devs[0], None, shapes[0][1]), (devs[1], None, shapes[1][1]),
                                   (inplace, inplace, shapes[2][1])], rope=rope)
    for i, (L, t0, _) in enumerate(shapes):
        alone = rkv.rope3d_apply(devs[i], t0=t0, rope=rope)
        torch.cuda.synchronize()
        assert np.array_equal(_bits(outs[i]), _bits(alone)), i
        ref = f64_to_bf16_bits(rope3d_ref(bf16_bits_to_f64(xs[i]), t0, MID.grid_h, MID.grid_w))
        assert int(bf16_ulp_distance(_bits(outs[i]), ref).max()) <= 1, i


def test_batch_full_size_q_and_k():
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    H, D = DENOISE.heads, 128
    rope = rkv.make_rope(DENOISE.grid_h, DENOISE.grid_w)
    q = to_dev(bf16_normal_bits(DENOISE.seed, (DENOISE.Lq, H, D)))
    k = to_dev(bf16_normal_bits(DENOISE.seed + 1, (DENOISE.Lk, H, D)))
    yq, yk = rkv.rope3d_apply_batch([(q, None, DENOISE.q_t0), (k, None, DENOISE.k_t0)], rope=rope)
    aq = rkv.rope3d_apply(q, t0=DENOISE.q_t0, rope=rope)
    ak = rkv.rope3d_apply(k, t0=DENOISE.k_t0, rope=rope)
    torch.cuda.synchronize()
    assert torch.equal(yq.view(torch.int16), aq.view(torch.int16))
    assert torch.equal(yk.view(torch.int16), ak.view(torch.int16))


def test_batch_strided_odd_split_and_rotate_half():
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    H, D = 2, 128
    for rope in (rkv.make_rope(5, 7, (21, 2, 41)), rkv.make_rope(5, 7, layout="half")):
        wide = to_dev(bf16_normal_bits(41, (300, 3 * H, D)))[:, :H, :]
        plain = to_dev(bf16_normal_bits(42, (77, H, D)))
        y1, y2 = rkv.rope3d_apply_batch([(wide, None, 3), (plain, None, 0)], rope=rope)
        a1 = rkv.rope3d_apply(wide, t0=3, rope=rope)
        a2 = rkv.rope3d_apply(plain, t0=0, rope=rope)
        torch.cuda.synchronize()
        assert np.array_equal(_bits(y1), _bits(a1)) and np.array_equal(_bits(y2), _bits(a2))


def test_rows_of_more_chunks_than_threads():
    # 160 heads: 2,560 chunks per row against 1,024 threads per CTA
    check_rope(40, 160, 2, 3, 1, 22)


def test_batch_of_eight():
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    H, D = 3, 128
    rope = rkv.make_rope(4, 6)
    xs = [to_dev(bf16_normal_bits(50 + i, (7 + 29 * i, H, D))) for i in range(8)]
    outs = rkv.rope3d_apply_batch([(x, None, i) for i, x in enumerate(xs)], rope=rope)
    for i, x in enumerate(xs):
        alone = rkv.rope3d_apply(x, t0=i, rope=rope)
        torch.cuda.synchronize()
        assert np.array_equal(_bits(outs[i]), _bits(alone)), i
