"""attn_fwd_varlen_noalloc: the attention launch for callers that cannot
allocate device memory (plugin hosts that pass only inputs and outputs,
engines with a fully pre-planned memory arena, code that must not call
cudaMalloc).  Its scratch is a fixed array inside librkv.so instead of a
caller workspace.

The call goes straight through the C ABI and its output must match the
regular workspace entry point within the attention tolerances, on two calls in
a row (the second call reuses the scratch the first one left behind).  Around
those two calls torch's caching allocator must report no more allocated and
no more reserved bytes (tensors of earlier tests may be garbage-collected in
between, so the counts may only fall), and the status word the calls left in
the library's scratch
(read back with rkv_attn_noalloc_status, which allocates nothing either) must
be RKV_OK.  This file is collected last on purpose, and it passes both on its
own in a fresh process and after the rest of the suite.
"""

import ctypes
import gc
import math

import numpy as np
import pytest
import torch

from rolling_kv_cache_rope_b200.synth import TINY, bf16_normal_bits
from tests._gpu import assert_attn_close, need_gpu, to_dev, to_f64

pytestmark = pytest.mark.gpu


def _noalloc_fn(rkv):
    fn = rkv.lib().attn_fwd_varlen_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.POINTER(rkv.rkv_attn_seq), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                   ctypes.c_float, ctypes.POINTER(rkv.rkv_rope3d), ctypes.c_void_p]
    return fn


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    need_gpu()
    from rolling_kv_cache_rope_b200 import rkv
    fn = _noalloc_fn(rkv)
    H, D = TINY.heads, TINY.head_dim
    rope = rkv.make_rope(TINY.grid_h, TINY.grid_w)
    scale = 1.0 / math.sqrt(D)
    # two sequences in one launch: the tiny layer with the 3-frame block mask,
    # and a ragged unmasked one
    shapes = [(TINY.Lq, TINY.Lk, TINY.q_t0, 3, 2), (300, 333, 1, 0, 0)]
    inputs = []
    for i, (Lq, Lk, q_t0, block, off) in enumerate(shapes):
        q = to_dev(bf16_normal_bits(500 + i, (Lq, H, D)))
        k = to_dev(bf16_normal_bits(600 + i, (Lk, H, D)))
        v = to_dev(bf16_normal_bits(700 + i, (Lk, H, D)))
        inputs.append((q, k, v, q_t0, block, off))

    def seqs_with_fresh_outputs():
        seqs = []
        for q, k, v, q_t0, block, off in inputs:
            o = torch.full((q.shape[0], H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
            seqs.append(rkv.AttnSeq(q, k, v, o, q_t0=q_t0, k_t0=0, block_frames=block, q_frame_offset=off))
        return seqs

    ref = seqs_with_fresh_outputs()
    ws = rkv.attn_fwd_varlen(ref, rope, softmax_scale=scale)
    rkv.rkv_attn_status(ws)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    status = rkv.lib().rkv_attn_noalloc_status
    status.restype = ctypes.c_int
    status.argtypes = [ctypes.c_void_p]
    calls = [seqs_with_fresh_outputs() for _ in range(2)]
    arrs = [(rkv.rkv_attn_seq * len(seqs))(*[s.to_c() for s in seqs]) for seqs in calls]
    gc.collect()
    torch.cuda.synchronize()
    allocated, reserved = torch.cuda.memory_allocated(), torch.cuda.memory_reserved()
    for call, arr in enumerate(arrs):
        st = fn(arr, len(calls[call]), H, D, scale, ctypes.byref(rope), stream)
        assert st == rkv.RKV_OK, rkv.rkv_last_error_string()
        assert status(stream) == rkv.RKV_OK, rkv.rkv_last_error_string()
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() <= allocated and torch.cuda.memory_reserved() <= reserved
    for call, seqs in enumerate(calls):
        for r, s in zip(ref, seqs):
            assert_attn_close(to_f64(s.o), to_f64(r.o), what=f"no-alloc call {call}")
