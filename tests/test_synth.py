"""The seeded input recipe both sides of every parity test consume: the draws
are reproducible, their bf16 rounding is round-to-nearest-even (the same as
torch's float32 -> bfloat16 conversion), the paper-shaped workloads have the
pages' sizes (23,400 query tokens over 32,760 context tokens, 12 heads), and
the rolling sweep's schedule grows the ring 6, 11, 16, 21 frames and then
holds it full."""

import numpy as np
import torch

from rolling_kv_cache_rope_b200.synth import (DENOISE, SWEEP, TINY, TWO_PASS_CACHE, TWO_PASS_DENOISE,
                                              bf16_normal_bits)


def test_draws_are_reproducible_and_seed_dependent():
    a = bf16_normal_bits(1234, (64, 2, 128))
    assert np.array_equal(a, bf16_normal_bits(1234, (64, 2, 128)))
    assert not np.array_equal(a, bf16_normal_bits(1235, (64, 2, 128)))
    assert a.dtype == np.uint16 and a.shape == (64, 2, 128)


def test_bf16_rounding_is_nearest_even():
    rng = np.random.Generator(np.random.PCG64(77))
    f = rng.standard_normal(size=(4096,), dtype=np.float32)
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = bf16_normal_bits(77, (4096,))
    assert np.array_equal(got, want)


def test_draws_look_standard_normal():
    x = torch.from_numpy(bf16_normal_bits(5, (1 << 18,)).view(np.int16)).view(torch.bfloat16).double().numpy()
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01


def test_workload_sizes_match_the_pages():
    assert (DENOISE.Lq, DENOISE.Lk, DENOISE.heads, DENOISE.head_dim) == (23400, 32760, 12, 128)
    assert DENOISE.frame_tokens == 1560 and DENOISE.q_t0 == 6 and DENOISE.k_t0 == 0
    assert (TWO_PASS_DENOISE.Lq, TWO_PASS_CACHE.Lq, TWO_PASS_CACHE.Lk) == (23400, 7800, 32760)
    assert (TINY.Lq, TINY.Lk, TINY.heads) == (72, 120, 2)


def test_sweep_schedule():
    assert [SWEEP.k_frames_after(s) for s in range(SWEEP.steps)] == [6, 11, 16, 21, 21, 21, 21, 21]
    assert [SWEEP.first_new_frame(s) for s in range(3)] == [1, 6, 11]
    q, k, v = SWEEP.step_inputs(2, -1)
    assert q is None and k.shape == (SWEEP.frame_tokens, 12, 128) and v.shape == k.shape
    q, k, v = SWEEP.step_inputs(0, 0)
    assert q.shape == (15 * SWEEP.frame_tokens, 12, 128) and k.shape == (5 * SWEEP.frame_tokens, 12, 128)
    assert SWEEP.seed(3, 2) == 7002 and SWEEP.seed(0, -1) == 3999
