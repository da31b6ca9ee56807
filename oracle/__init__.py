"""Plain, slow CPU oracle for the rolling-KV-cache / 3D-RoPE attention path.

THIS PACKAGE IS TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
it.  The product path (``rolling_kv_cache_rope_b200``) never imports it, and
this package never imports the product: the two share no code.  Only the seeded
input generator in ``rolling_kv_cache_rope_b200/synth.py`` feeds both sides,
and it holds none of the method's arithmetic.

Everything here is float64 numpy, written as the plain definition of what the
pages describe, with no blocking, fusion or reordering beyond what that
definition states:

* ``rope3d``    – token -> (t, h, w) positions and the three-axis rotary
  embedding applied to Q and K ("Amazon and Reactor tune Trainium for real-time
  video generation", section "Three problems for generic compilers": RoPE must
  handle height, width and time instead of one position).
* ``mask``      – the frame-block-causal visibility used when the denoise pass
  and the cache-update pass share one launch.
* ``attention`` – softmax attention (SDPA) from a query window to a context,
  optionally with the mask.
* ``ring``      – the per-layer rolling KV cache that inserts and evicts whole
  frames.

Every function is pinned by a ``-m "not gpu"`` test in ``tests/test_oracle_*.py``
against closed forms, invariants, library routines or brute force.
"""

from .bf16 import bf16_bits_to_f64, f64_to_bf16_bits, bf16_ulp_distance
from .rope3d import (
    AXIS_T, AXIS_H, AXIS_W,
    token_positions, pair_axes, rope_angles, rope3d_ref,
)
from .mask import frame_block_visible, frame_pair_visible, default_q_frame_offset
from .attention import attention_ref, attention_rows_ref, fused_attention_ref
from .ring import RingRef

__all__ = [
    "bf16_bits_to_f64", "f64_to_bf16_bits", "bf16_ulp_distance",
    "AXIS_T", "AXIS_H", "AXIS_W",
    "token_positions", "pair_axes", "rope_angles", "rope3d_ref",
    "frame_block_visible", "frame_pair_visible", "default_q_frame_offset",
    "attention_ref", "attention_rows_ref", "fused_attention_ref",
    "RingRef",
]
