"""Rolling sweep at full size: per layer a 21-slot ring of 30x52-token frames
(12 heads), one seeded frame, then 8 steps that each insert 5 frames of raw K
(rotated on the way in) and V, and attend from a 23,400-token query window
over the ring's valid frames (Lk = 9,360 -> 32,760; K already rotated, only Q
rotated in-kernel, no mask).

Parity per step, against the oracle on the same seeded inputs:
- ring state (head, count, evicted frames, slot map) and V slots bit-exact,
  K slots within one bf16 ulp of the correctly rounded fp64 rotation;
- attention on sampled query rows (frame boundaries, first/last rows, random
  rows) against fp64 attention over the oracle's own ring contents, read in
  the same physical slot order, with the stated tolerances."""

import numpy as np
import pytest
import torch

from oracle import RingRef, bf16_bits_to_f64, bf16_ulp_distance, f64_to_bf16_bits, fused_attention_ref, rope3d_ref
from rolling_kv_cache_rope_b200.synth import SWEEP
from tests._gpu import assert_attn_close, need_gpu, to_bits, to_dev, to_f64

pytestmark = pytest.mark.gpu


def sample_rows(Lq, F, n_random, seed):
    rng = np.random.default_rng(seed)
    rows = {0, 1, Lq - 1, Lq - 2}
    for f in range(1, Lq // F):
        rows.update((f * F - 1, f * F))
    rows.update(int(r) for r in rng.integers(0, Lq, n_random))
    return np.array(sorted(rows), dtype=np.int64)


def run_layer(layer, steps):
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    sw = SWEEP
    F, H, D, W = sw.frame_tokens, sw.heads, sw.head_dim, sw.ring_slots
    rope = rkv.make_rope(sw.grid_h, sw.grid_w)
    ring = rkv.KVRing(W, F, H, D)
    ref = RingRef(W)
    ws = torch.zeros(rkv.attn_fwd_varlen_workspace_size(1, H, D), dtype=torch.uint8, device="cuda")

    def insert(k_bits, v_bits, t0):
        n = k_bits.shape[0] // F
        kr = f64_to_bf16_bits(rope3d_ref(bf16_bits_to_f64(k_bits), t0, sw.grid_h, sw.grid_w))
        frames = [(kr[i * F:(i + 1) * F], v_bits[i * F:(i + 1) * F], t0 + i) for i in range(n)]
        ev = rkv.kvcache_ring_update_rope(ring, to_dev(k_bits), to_dev(v_bits), t0, rope, n)
        assert ev == ref.insert(frames)
        assert (ring.head, ring.count) == (ref.head, ref.count)
        assert [ring.slot(j) for j in range(W)] == [ref.slot_of(j) for j in range(W)]

    _, k0, v0 = sw.step_inputs(layer, -1)
    insert(k0, v0, 0)
    lk_seen = []
    for step in range(steps):
        q_bits, k_bits, v_bits = sw.step_inputs(layer, step)
        t_new = sw.first_new_frame(step)
        insert(k_bits, v_bits, t_new)
        assert ring.count == sw.k_frames_after(step)
        # the valid slots are a prefix of the ring (filled from empty, or full)
        valid = ref.valid_slots()
        assert valid == list(range(ring.count))
        Lk = ring.count * F
        lk_seen.append(Lk)
        kview = ring.k.view(W * F, H, D)[:Lk]
        vview = ring.v.view(W * F, H, D)[:Lk]
        q = to_dev(q_bits)
        o = torch.empty_like(q)
        seq = rkv.AttnSeq(q, kview, vview, o, q_t0=t_new, rope_q=True, rope_k=False)
        rkv.attn_fwd_varlen([seq], rope, workspace=ws)
        rkv.rkv_attn_status(ws)   # raises on a device-side error
        torch.cuda.synchronize()

        # ring contents: V bit-exact, K within one ulp of the oracle rotation
        kh = to_bits(ring.k).reshape(W, F, H * D)
        vh = to_bits(ring.v).reshape(W, F, H * D)
        for s in valid:
            assert int(bf16_ulp_distance(kh[s], ref.slots[s][0].reshape(F, H * D)).max()) <= 1, (step, s)
            assert np.array_equal(vh[s], ref.slots[s][1].reshape(F, H * D)), (step, s)

        # attention over the oracle's ring, physical slot order
        k_ref = np.concatenate([bf16_bits_to_f64(ref.slots[s][0]) for s in valid]).reshape(Lk, H, D)
        v_ref = np.concatenate([bf16_bits_to_f64(ref.slots[s][1]) for s in valid]).reshape(Lk, H, D)
        rows = sample_rows(q_bits.shape[0], F, 24, seed=layer * 100 + step)
        want = fused_attention_ref(bf16_bits_to_f64(q_bits), k_ref, v_ref, scale=1.0 / np.sqrt(D),
                                   grid_h=sw.grid_h, grid_w=sw.grid_w, rope_q=True, rope_k=False,
                                   q_t0=t_new, k_t0=0, rows=rows)
        got = to_f64(o)[rows]
        assert_attn_close(got, want, f"layer {layer} step {step} Lk {Lk}")
    return lk_seen


def test_sweep_first_layer_all_steps():
    lk = run_layer(0, SWEEP.steps)
    F = SWEEP.frame_tokens
    assert lk == [f * F for f in (6, 11, 16, 21, 21, 21, 21, 21)]


def test_sweep_last_layer_all_steps():
    run_layer(SWEEP.layers - 1, SWEEP.steps)


@pytest.mark.slow
def test_sweep_all_layers():
    """All 30 layers x 8 steps.  Per step: head, count, evicted frames and the
    slot map bit-exact; the inserted K frames within one bf16 ulp of the
    correctly rounded fp64 rotation and the inserted V frames bit-exact (in
    their slots); every other valid slot unchanged since the previous step;
    attention on sampled query rows (first/last rows, both sides of every
    frame boundary, random rows) against the oracle ring.  The oracle side of
    each layer runs in a worker process (tests/_oracle_pool.py)."""
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    from tests._oracle_pool import sweep_layer, workers
    sw = SWEEP
    F, H, D, W = sw.frame_tokens, sw.heads, sw.head_dim, sw.ring_slots
    rope = rkv.make_rope(sw.grid_h, sw.grid_w)
    ws = torch.zeros(rkv.attn_fwd_varlen_workspace_size(1, H, D), dtype=torch.uint8, device="cuda")
    ahead = max(2, workers())
    futs = {layer: sweep_layer(layer, sw.steps) for layer in range(min(sw.layers, ahead))}
    for layer in range(sw.layers):
        if layer + ahead < sw.layers:
            futs[layer + ahead] = sweep_layer(layer + ahead, sw.steps)
        ring = rkv.KVRing(W, F, H, D)
        _, k0, v0 = sw.step_inputs(layer, -1)
        rkv.kvcache_ring_update_rope(ring, to_dev(k0), to_dev(v0), 0, rope, sw.seed_frames)
        expect = futs.pop(layer).result()
        for step, ex in enumerate(expect):
            q_bits, k_bits, v_bits = sw.step_inputs(layer, step)
            t_new = sw.first_new_frame(step)
            before_k, before_v = ring.k.clone(), ring.v.clone()
            kd, vd = to_dev(k_bits), to_dev(v_bits)
            ev = rkv.kvcache_ring_update_rope(ring, kd, vd, t_new, rope, sw.insert)
            rkv.rkv_ring_status()
            where = f"layer {layer} step {step}"
            assert ev == ex["evicted"], where
            assert (ring.head, ring.count) == (ex["head"], ex["count"]), where
            assert [ring.slot(j) for j in range(W)] == ex["slot_map"], where
            # the inserted frames are the newest sw.insert logical frames
            new_slots = [ring.slot(ring.count - sw.insert + i) for i in range(sw.insert)]
            for i, s in enumerate(new_slots):
                got_k = to_bits(ring.k[s]).reshape(F, H * D)
                want_k = ex["k_rot"][i * F:(i + 1) * F].reshape(F, H * D)
                assert int(bf16_ulp_distance(got_k, want_k).max()) <= 1, (where, s)
                assert torch.equal(ring.v[s], vd[i * F:(i + 1) * F]), (where, s)
            for s in ex["valid"]:
                if s not in new_slots:
                    assert torch.equal(ring.k[s], before_k[s]) and torch.equal(ring.v[s], before_v[s]), (where, s)
            Lk = ring.count * F
            q = to_dev(q_bits)
            o = torch.empty_like(q)
            seq = rkv.AttnSeq(q, ring.k.view(W * F, H, D)[:Lk], ring.v.view(W * F, H, D)[:Lk], o, q_t0=t_new,
                              rope_q=True, rope_k=False)
            rkv.attn_fwd_varlen([seq], rope, workspace=ws)
            rkv.rkv_attn_status(ws)
            torch.cuda.synchronize()
            assert_attn_close(to_f64(o)[ex["rows"]], ex["attn"], f"{where} Lk {Lk}")
            del before_k, before_v
