"""Run the fp64 oracle on all host cores for the full-size parity tests.

numpy's matrix products use every core but its elementwise steps (the
exponentials of softmax, the RoPE rotations) use one, so the full-size
oracle is split into independent pieces -- one attention head, one sweep
layer -- that run in worker processes.  The workers are started with the
"spawn" method (never forked from a process that has touched the GPU) and
each limits its BLAS library to one thread.  Every piece calls the oracle
functions unchanged; only the way the work is divided differs.
"""

import concurrent.futures
import multiprocessing
import os

import numpy as np

_POOL = None


def workers():
    return max(1, min(os.cpu_count() or 1, 32))


def pool():
    global _POOL
    if _POOL is None:
        _POOL = concurrent.futures.ProcessPoolExecutor(max_workers=workers(),
                                                       mp_context=multiprocessing.get_context("spawn"),
                                                       initializer=_init_worker)
    return _POOL


def _init_worker():
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:  # noqa: BLE001 - without threadpoolctl the workers share the cores
        pass


def _attention_head(qb, kb, vb, kw):
    from oracle import bf16_bits_to_f64, fused_attention_ref
    return fused_attention_ref(bf16_bits_to_f64(qb), bf16_bits_to_f64(kb), bf16_bits_to_f64(vb), **kw)


def attention_by_head(q_bits, k_bits, v_bits, **kw):
    """oracle.fused_attention_ref of bf16 bit arrays [L, H, D], one task per
    head; returns float64 [Lq (or len(rows)), H, D]."""
    H = q_bits.shape[1]
    futs = [pool().submit(_attention_head, np.ascontiguousarray(q_bits[:, h:h + 1]),
                          np.ascontiguousarray(k_bits[:, h:h + 1]), np.ascontiguousarray(v_bits[:, h:h + 1]), kw)
            for h in range(H)]
    return np.concatenate([f.result() for f in futs], axis=1)


def _sweep_layer(layer, steps, n_rows):
    """Expected results of one sweep layer, step by step, from the oracle:
    the ring state after each insert, the correctly rounded rotation of the
    inserted keys, and attention on sampled query rows over the oracle ring
    read in physical slot order."""
    from oracle import RingRef, bf16_bits_to_f64, f64_to_bf16_bits, fused_attention_ref, rope3d_ref
    from rolling_kv_cache_rope_b200.synth import SWEEP as sw
    F, H, D, W = sw.frame_tokens, sw.heads, sw.head_dim, sw.ring_slots
    ref = RingRef(W)
    out = []

    def insert(k_bits, v_bits, t0):
        n = k_bits.shape[0] // F
        kr = f64_to_bf16_bits(rope3d_ref(bf16_bits_to_f64(k_bits), t0, sw.grid_h, sw.grid_w))
        frames = [(kr[i * F:(i + 1) * F], v_bits[i * F:(i + 1) * F], t0 + i) for i in range(n)]
        ev = ref.insert(frames)
        return kr, ev

    _, k0, v0 = sw.step_inputs(layer, -1)
    insert(k0, v0, 0)
    for step in range(steps):
        q_bits, k_bits, v_bits = sw.step_inputs(layer, step)
        t_new = sw.first_new_frame(step)
        kr, ev = insert(k_bits, v_bits, t_new)
        valid = ref.valid_slots()
        Lk = len(valid) * F
        rows = sample_rows(q_bits.shape[0], F, n_rows, seed=layer * 100 + step)
        k_ref = np.concatenate([bf16_bits_to_f64(ref.slots[s][0]) for s in valid]).reshape(Lk, H, D)
        v_ref = np.concatenate([bf16_bits_to_f64(ref.slots[s][1]) for s in valid]).reshape(Lk, H, D)
        want = fused_attention_ref(bf16_bits_to_f64(q_bits), k_ref, v_ref, scale=1.0 / np.sqrt(D), grid_h=sw.grid_h,
                                   grid_w=sw.grid_w, rope_q=True, rope_k=False, q_t0=t_new, k_t0=0, rows=rows)
        out.append(dict(k_rot=kr, evicted=ev, head=ref.head, count=ref.count, valid=valid,
                        slot_map=[ref.slot_of(j) for j in range(W)], rows=rows, attn=want))
    return out


def sweep_layer(layer, steps, n_rows=24):
    return pool().submit(_sweep_layer, layer, steps, n_rows)


def sample_rows(Lq, F, n_random, seed):
    """First and last rows, both sides of every frame boundary, random rows."""
    rng = np.random.default_rng(seed)
    rows = {0, 1, Lq - 1, Lq - 2}
    for f in range(1, Lq // F):
        rows.update((f * F - 1, f * F))
    rows.update(int(r) for r in rng.integers(0, Lq, n_random))
    return np.array(sorted(rows), dtype=np.int64)
