"""Pins of the attention oracle: closed forms, brute force, a library routine."""

import math

import numpy as np
import pytest
import torch

from oracle import attention_ref, fused_attention_ref, frame_block_visible, rope3d_ref


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_single_key_returns_its_value():
    q, k, v = rand((5, 2, 8), 0), rand((1, 2, 8), 1), rand((1, 2, 8), 2)
    o = attention_ref(q, k, v, 0.3)
    assert np.allclose(o, np.broadcast_to(v, o.shape), atol=1e-15)


def test_equal_keys_average_values():
    q, v = rand((4, 1, 8), 3), rand((6, 1, 8), 4)
    k = np.broadcast_to(rand((1, 1, 8), 5), (6, 1, 8))
    o = attention_ref(q, k, v, 1.0)
    assert np.allclose(o, np.broadcast_to(v.mean(axis=0), o.shape), atol=1e-14)


def test_two_keys_logistic_closed_form():
    # scores 1 and 0 -> weights sigma(1), sigma(-1)
    q = np.array([[[2.0, 0, 0, 0]]])
    k = np.array([[[1.0, 0, 0, 0]], [[0.0, 0, 0, 0]]])
    v = np.array([[[1.0, 0, 0, 0]], [[0.0, 1.0, 0, 0]]])
    o = attention_ref(q, k, v, 0.5)[0, 0]
    assert o[0] == pytest.approx(0.7310585786300049, abs=1e-15)
    assert o[1] == pytest.approx(0.2689414213699951, abs=1e-15)


def test_scale_enters_the_exponent():
    # with scale 1/sqrt(4) = 0.5 the score gap 2*1 becomes 1 (sigma(1) weight)
    q = np.array([[[1.0, 1.0, 1.0, 1.0]]])
    k = np.array([[[0.5, 0.5, 0.5, 0.5]], [[0.0, 0.0, 0.0, 0.0]]])
    v = np.array([[[1.0]], [[0.0]]])
    o = attention_ref(q, k, v, 1.0 / math.sqrt(4.0))
    assert o[0, 0, 0] == pytest.approx(0.7310585786300049, abs=1e-15)


def test_brute_force_loops_with_mask():
    rng = np.random.default_rng(6)
    Lq, Lk, H, D = 3, 5, 2, 4
    q, k, v = rng.standard_normal((Lq, H, D)), rng.standard_normal((Lk, H, D)), rng.standard_normal((Lk, H, D))
    vis = rng.random((Lq, Lk)) < 0.6
    vis[:, 0] = True
    o = attention_ref(q, k, v, 0.7, vis)
    for h in range(H):
        for r in range(Lq):
            w = []
            for c in range(Lk):
                if vis[r, c]:
                    w.append(math.exp(0.7 * sum(q[r, h, d] * k[c, h, d] for d in range(D))))
                else:
                    w.append(0.0)
            tot = sum(w)
            for d in range(D):
                ref = sum(w[c] * v[c, h, d] for c in range(Lk)) / tot
                assert o[r, h, d] == pytest.approx(ref, rel=1e-12, abs=1e-13)


def test_matches_torch_sdpa_float64():
    rng = np.random.default_rng(7)
    Lq, Lk, H, D = 72, 120, 2, 128
    q, k, v = rng.standard_normal((Lq, H, D)), rng.standard_normal((Lk, H, D)), rng.standard_normal((Lk, H, D))
    vis = frame_block_visible(Lq, Lk, 24, 2, 3)
    o = attention_ref(q, k, v, 1.0 / math.sqrt(D), vis)
    tq, tk, tv = (torch.from_numpy(a).permute(1, 0, 2) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(vis))
    assert np.max(np.abs(ref.permute(1, 0, 2).numpy() - o)) < 1e-12
    o2 = attention_ref(q, k, v, 1.0 / math.sqrt(D))
    ref2 = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    assert np.max(np.abs(ref2.permute(1, 0, 2).numpy() - o2)) < 1e-12


def test_fully_masked_row_is_zero():
    q, k, v = rand((2, 1, 4), 8), rand((3, 1, 4), 9), rand((3, 1, 4), 10)
    vis = np.array([[False, False, False], [True, False, True]])
    o = attention_ref(q, k, v, 1.0, vis)
    assert np.array_equal(o[0], np.zeros((1, 4)))
    assert np.all(np.isfinite(o))


def test_unmasked_is_key_permutation_invariant():
    q, k, v = rand((7, 2, 16), 11), rand((30, 2, 16), 12), rand((30, 2, 16), 13)
    perm = np.random.default_rng(14).permutation(30)
    assert np.allclose(attention_ref(q, k, v, 0.25), attention_ref(q, k[perm], v[perm], 0.25), atol=1e-14)


def test_chunking_does_not_change_rows():
    q, k, v = rand((50, 1, 8), 15), rand((9, 1, 8), 16), rand((9, 1, 8), 17)
    # equal up to BLAS summation order (its blocking depends on the row count)
    assert np.allclose(attention_ref(q, k, v, 0.5, row_chunk=7), attention_ref(q, k, v, 0.5, row_chunk=64), rtol=0, atol=1e-14)


def test_fused_is_rope_then_attention():
    rng = np.random.default_rng(18)
    q, k, v = rng.standard_normal((72, 2, 128)), rng.standard_normal((120, 2, 128)), rng.standard_normal((120, 2, 128))
    kw = dict(scale=1 / math.sqrt(128), grid_h=4, grid_w=6, rope_q=True, rope_k=True, q_t0=2, k_t0=0)
    o = fused_attention_ref(q, k, v, **kw)
    ref = attention_ref(rope3d_ref(q, 2, 4, 6), rope3d_ref(k, 0, 4, 6), v, 1 / math.sqrt(128))
    assert np.array_equal(o, ref)
    rows = np.array([3, 40, 71])
    assert np.allclose(fused_attention_ref(q, k, v, rows=rows, **kw), o[rows], atol=1e-14)


def test_fused_output_invariant_to_common_time_shift():
    # RoPE scores depend only on relative positions, so shifting both windows'
    # start frame by the same amount leaves the attention output unchanged.
    rng = np.random.default_rng(19)
    q, k, v = rng.standard_normal((48, 1, 128)), rng.standard_normal((72, 1, 128)), rng.standard_normal((72, 1, 128))
    kw = dict(scale=1 / math.sqrt(128), grid_h=4, grid_w=6, rope_q=True, rope_k=True)
    a = fused_attention_ref(q, k, v, q_t0=1, k_t0=0, **kw)
    b = fused_attention_ref(q, k, v, q_t0=9, k_t0=8, **kw)
    c = fused_attention_ref(q, k, v, q_t0=2, k_t0=0, **kw)
    assert np.max(np.abs(a - b)) < 1e-12
    assert np.max(np.abs(a - c)) > 1e-4
