"""ctypes binding of librkv.so (C ABI in include/rkv.h), same names as the C calls.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of librkv.so.  Tensors are torch CUDA tensors used for device memory
and streams; they are passed to the library as raw pointers and row strides.
There is no CPU fallback: importing this module raises ImportError when the
library has not been built.
"""

import ctypes
import math
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "librkv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"librkv.so not found at {LIB_PATH}; build it with "
        "`python -m rolling_kv_cache_rope_b200.build` (nvcc, sm_100a). There is no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)

RKV_OK, RKV_ERR_INVALID_ARG, RKV_ERR_UNSUPPORTED, RKV_ERR_CUDA, RKV_ERR_TIMEOUT, RKV_ERR_DEVICE_CHECK = 0, 1, 2, 3, 4, 5
RKV_ROPE_Q, RKV_ROPE_K = 1, 2
RKV_MAX_SEQS = 16
STATUS_NAMES = {0: "RKV_OK", 1: "RKV_ERR_INVALID_ARG", 2: "RKV_ERR_UNSUPPORTED", 3: "RKV_ERR_CUDA",
                4: "RKV_ERR_TIMEOUT", 5: "RKV_ERR_DEVICE_CHECK"}


class rkv_rope3d(ctypes.Structure):
    _fields_ = [("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32), ("pairs_t", ctypes.c_int32),
                ("pairs_h", ctypes.c_int32), ("pairs_w", ctypes.c_int32), ("theta", ctypes.c_float),
                ("theta_h", ctypes.c_float), ("theta_w", ctypes.c_float), ("layout", ctypes.c_int32)]


RKV_ROPE_ADJACENT, RKV_ROPE_HALF = 0, 1
RKV_ROPE_BATCH_MAX = 8


class rkv_rope_tensor(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("y", ctypes.c_void_p), ("L", ctypes.c_int64),
                ("x_row_stride", ctypes.c_int64), ("y_row_stride", ctypes.c_int64), ("t0", ctypes.c_int32)]


class rkv_attn_seq(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("o", ctypes.c_void_p),
                ("q_stride", ctypes.c_int64), ("k_stride", ctypes.c_int64), ("v_stride", ctypes.c_int64),
                ("o_stride", ctypes.c_int64), ("Lq", ctypes.c_int32), ("Lk", ctypes.c_int32),
                ("q_t0", ctypes.c_int32), ("k_t0", ctypes.c_int32), ("q_frame_offset", ctypes.c_int32),
                ("block_frames", ctypes.c_int32), ("flags", ctypes.c_uint32), ("reserved", ctypes.c_int32)]


class rkv_attn_debug(ctypes.Structure):
    _fields_ = [("row_stats", ctypes.c_void_p), ("stall", ctypes.c_uint32), ("timeout_us", ctypes.c_uint32)]


class rkv_ring_debug(ctypes.Structure):
    _fields_ = [("stall", ctypes.c_uint32), ("timeout_us", ctypes.c_uint32)]


RKV_DEBUG_STALL_NONE, RKV_DEBUG_STALL_V_READY, RKV_DEBUG_STALL_K_READY, RKV_DEBUG_STALL_P_FULL = 0, 1, 2, 3
RKV_DEBUG_STALL_BULK_LOAD = 1


class rkv_ring(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("slots", ctypes.c_int32),
                ("tokens_per_frame", ctypes.c_int32), ("H", ctypes.c_int32), ("D", ctypes.c_int32),
                ("head", ctypes.c_int32), ("count", ctypes.c_int32), ("pinned", ctypes.c_int32)]


_c = ctypes
_lib.rope3d_apply.restype = _c.c_int
_lib.rope3d_apply.argtypes = [_c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int32, _c.c_int32, _c.c_int64, _c.c_int64,
                              _c.c_int32, _c.POINTER(rkv_rope3d), _c.c_void_p]
_lib.rope3d_apply_batch.restype = _c.c_int
_lib.rope3d_apply_batch.argtypes = [_c.POINTER(rkv_rope_tensor), _c.c_int32, _c.c_int32, _c.c_int32,
                                    _c.POINTER(rkv_rope3d), _c.c_void_p]
_lib.attn_fwd_varlen_workspace_size.restype = _c.c_size_t
_lib.attn_fwd_varlen_workspace_size.argtypes = [_c.POINTER(rkv_attn_seq), _c.c_int32, _c.c_int32, _c.c_int32]
_lib.attn_fwd_varlen.restype = _c.c_int
_lib.attn_fwd_varlen.argtypes = [_c.POINTER(rkv_attn_seq), _c.c_int32, _c.c_int32, _c.c_int32, _c.c_float,
                                 _c.POINTER(rkv_rope3d), _c.c_void_p, _c.c_size_t, _c.c_void_p]
_lib.rkv_attn_status.restype = _c.c_int
_lib.rkv_attn_status.argtypes = [_c.c_void_p, _c.c_void_p]
_lib.attn_fwd_varlen_debug.restype = _c.c_int
_lib.attn_fwd_varlen_debug.argtypes = [_c.POINTER(rkv_attn_seq), _c.c_int32, _c.c_int32, _c.c_int32, _c.c_float,
                                       _c.POINTER(rkv_rope3d), _c.c_void_p, _c.c_size_t, _c.POINTER(rkv_attn_debug),
                                       _c.c_void_p]
_lib.attn_fwd_varlen_noalloc.restype = _c.c_int
_lib.attn_fwd_varlen_noalloc.argtypes = [_c.POINTER(rkv_attn_seq), _c.c_int32, _c.c_int32, _c.c_int32, _c.c_float,
                                         _c.POINTER(rkv_rope3d), _c.c_void_p]
_lib.rkv_attn_noalloc_status.restype = _c.c_int
_lib.rkv_attn_noalloc_status.argtypes = [_c.c_void_p]
_lib.rkv_attn_mask_rows.restype = _c.c_int
_lib.rkv_attn_mask_rows.argtypes = [_c.POINTER(rkv_attn_seq), _c.c_int32, _c.c_int32, _c.POINTER(rkv_rope3d),
                                    _c.POINTER(_c.c_int64), _c.POINTER(_c.c_int32), _c.POINTER(_c.c_int64)]
_lib.kvcache_ring_update.restype = _c.c_int
_lib.kvcache_ring_update.argtypes = [_c.POINTER(rkv_ring), _c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int32,
                                     _c.POINTER(_c.c_int32), _c.c_void_p]
_lib.kvcache_ring_update_rope.restype = _c.c_int
_lib.kvcache_ring_update_rope.argtypes = [_c.POINTER(rkv_ring), _c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int32,
                                          _c.c_int32, _c.POINTER(rkv_rope3d), _c.POINTER(_c.c_int32), _c.c_void_p]
_lib.kvcache_ring_update_debug.restype = _c.c_int
_lib.kvcache_ring_update_debug.argtypes = [_c.POINTER(rkv_ring), _c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int32,
                                           _c.POINTER(_c.c_int32), _c.POINTER(rkv_ring_debug), _c.c_void_p]
_lib.rkv_ring_status.restype = _c.c_int
_lib.rkv_ring_status.argtypes = [_c.c_void_p]
_lib.rkv_ring_slot.restype = _c.c_int32
_lib.rkv_ring_slot.argtypes = [_c.POINTER(rkv_ring), _c.c_int32]
_lib.rkv_last_error_string.restype = _c.c_char_p
_lib.rkv_last_error_string.argtypes = []
_lib.rkv_version.restype = _c.c_int32
_lib.rkv_version.argtypes = []


def lib():
    """The raw ctypes library (tests use it to drive the C ABI directly)."""
    return _lib


class RkvError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def rkv_last_error_string():
    return _lib.rkv_last_error_string().decode()


def rkv_version():
    return int(_lib.rkv_version())


def _check(status):
    if status != RKV_OK:
        raise RkvError(status, rkv_last_error_string())


def make_rope(grid_h, grid_w, pairs=(22, 21, 21), theta=10000.0, layout="adjacent"):
    """RoPE parameters.  ``theta``: one frequency base or a (t, h, w) triple;
    ``layout``: "adjacent" (pairs 2j, 2j+1) or "half" (pairs j, j + D/2)."""
    th = tuple(float(v) for v in theta) if isinstance(theta, (tuple, list)) else (float(theta),) * 3
    if layout not in ("adjacent", "half"):
        raise ValueError("layout must be 'adjacent' or 'half'")
    return rkv_rope3d(int(grid_h), int(grid_w), int(pairs[0]), int(pairs[1]), int(pairs[2]), th[0], th[1], th[2],
                      RKV_ROPE_HALF if layout == "half" else RKV_ROPE_ADJACENT)


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _rows(t, name):
    """Check a [L, H, D] bf16 CUDA view with contiguous rows; return its row stride."""
    import torch
    if t.dtype != torch.bfloat16 or not t.is_cuda or t.dim() != 3:
        raise ValueError(f"{name} must be a bf16 CUDA tensor of shape [L, H, D]")
    if t.stride(2) != 1 or t.stride(1) != t.shape[2]:
        raise ValueError(f"{name}: each row must hold H*D contiguous values")
    return t.stride(0)


def rope3d_apply(x, y=None, t0=0, rope=None, stream=None):
    """y = RoPE3D(x); x, y bf16 [L, H, 128] CUDA tensors (y=None -> new tensor,
    y=x -> in place).  Returns y."""
    import torch
    if y is None:
        y = torch.empty_like(x)
    xs, ys = _rows(x, "x"), _rows(y, "y")
    if tuple(x.shape) != tuple(y.shape):
        raise ValueError("x and y shapes differ")
    L, H, D = x.shape
    _check(_lib.rope3d_apply(x.data_ptr(), y.data_ptr(), L, H, D, xs, ys, int(t0), ctypes.byref(rope),
                             _stream(stream)))
    return y


def rope3d_apply_batch(items, rope=None, stream=None):
    """rope3d_apply on several tensors in one launch.  items: sequence of
    (x, y, t0) with x, y bf16 [L, H, 128] CUDA tensors of the same H (y=None ->
    new tensor, y=x -> in place).  Returns the list of y."""
    import torch
    outs = []
    arr = (rkv_rope_tensor * max(1, len(items)))()
    H = None
    for i, (x, y, t0) in enumerate(items):
        if y is None:
            y = torch.empty_like(x)
        xs, ys = _rows(x, "x"), _rows(y, "y")
        if tuple(x.shape) != tuple(y.shape):
            raise ValueError("x and y shapes differ")
        if H is None:
            H = x.shape[1]
        elif x.shape[1] != H:
            raise ValueError("all tensors of a batch must have the same number of heads")
        arr[i] = rkv_rope_tensor(x.data_ptr(), y.data_ptr(), x.shape[0], xs, ys, int(t0))
        outs.append(y)
    _check(_lib.rope3d_apply_batch(arr, len(items), H or 1, 128, ctypes.byref(rope), _stream(stream)))
    return outs


class AttnSeq:
    """One sequence of a batched attention launch (see rkv_attn_seq)."""

    def __init__(self, q, k, v, o, q_t0=0, k_t0=0, rope_q=True, rope_k=True, block_frames=0, q_frame_offset=0):
        self.q, self.k, self.v, self.o = q, k, v, o
        self.q_t0, self.k_t0 = int(q_t0), int(k_t0)
        self.flags = (RKV_ROPE_Q if rope_q else 0) | (RKV_ROPE_K if rope_k else 0)
        self.block_frames = int(block_frames)
        self.q_frame_offset = int(q_frame_offset)

    def to_c(self):
        qs, ks, vs, os_ = _rows(self.q, "q"), _rows(self.k, "k"), _rows(self.v, "v"), _rows(self.o, "o")
        if self.k.shape[0] != self.v.shape[0] or self.q.shape[0] != self.o.shape[0]:
            raise ValueError("k/v or q/o row counts differ")
        return rkv_attn_seq(self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(), self.o.data_ptr(),
                            qs, ks, vs, os_, self.q.shape[0], self.k.shape[0], self.q_t0, self.k_t0,
                            self.q_frame_offset, self.block_frames, self.flags, 0)


def attn_fwd_varlen_workspace_size(n_seqs=1, H=12, D=128):
    return int(_lib.attn_fwd_varlen_workspace_size(None, n_seqs, H, D))


def attn_fwd_varlen(seqs, rope, softmax_scale=None, workspace=None, stream=None):
    """Run every AttnSeq in ONE kernel launch; outputs are written to each seq.o.
    ``workspace`` is a uint8 CUDA tensor of attn_fwd_varlen_workspace_size()
    bytes (allocated here when None)."""
    import torch
    if not seqs:
        raise ValueError("need at least one sequence")
    H, D = seqs[0].q.shape[1], seqs[0].q.shape[2]
    arr = (rkv_attn_seq * len(seqs))(*[s.to_c() for s in seqs])
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    size = attn_fwd_varlen_workspace_size(len(seqs), H, D)
    if workspace is None:
        workspace = torch.empty(size, dtype=torch.uint8, device=seqs[0].q.device)
    _check(_lib.attn_fwd_varlen(arr, len(seqs), H, D, float(softmax_scale), ctypes.byref(rope),
                                workspace.data_ptr(), workspace.numel(), _stream(stream)))
    return workspace


def rkv_attn_status(workspace, stream=None):
    """Synchronise and raise RkvError if the last launch on ``workspace`` timed out."""
    _check(_lib.rkv_attn_status(workspace.data_ptr(), _stream(stream)))


def attn_fwd_varlen_debug(seqs, rope, row_stats=None, stall=RKV_DEBUG_STALL_NONE, timeout_us=0, softmax_scale=None,
                          workspace=None, stream=None):
    """attn_fwd_varlen with test and debug aids (see rkv.h): ``row_stats`` an
    int32 CUDA tensor of sum(Lq) * H * 4 elements that receives the per-row
    mask record; ``stall`` one of RKV_DEBUG_STALL_*; ``timeout_us`` the limit
    of every device-side wait (0 = default).  Returns the workspace."""
    import torch
    if not seqs:
        raise ValueError("need at least one sequence")
    H, D = seqs[0].q.shape[1], seqs[0].q.shape[2]
    arr = (rkv_attn_seq * len(seqs))(*[s.to_c() for s in seqs])
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    if workspace is None:
        workspace = torch.empty(attn_fwd_varlen_workspace_size(len(seqs), H, D), dtype=torch.uint8,
                                device=seqs[0].q.device)
    ptr = None
    if row_stats is not None:
        rows = sum(int(s.q.shape[0]) for s in seqs)
        if row_stats.dtype != torch.int32 or not row_stats.is_cuda or not row_stats.is_contiguous() \
                or row_stats.numel() < rows * H * 4:
            raise ValueError(f"row_stats must be a contiguous int32 CUDA tensor of >= {rows * H * 4} elements")
        ptr = row_stats.data_ptr()
    dbg = rkv_attn_debug(ptr, int(stall), int(timeout_us))
    _check(_lib.attn_fwd_varlen_debug(arr, len(seqs), H, D, float(softmax_scale), ctypes.byref(rope),
                                      workspace.data_ptr(), workspace.numel(), ctypes.byref(dbg), _stream(stream)))
    return workspace


def attn_fwd_varlen_noalloc(seqs, rope, softmax_scale=None, stream=None):
    """attn_fwd_varlen without a caller workspace (the library's fixed scratch)."""
    if not seqs:
        raise ValueError("need at least one sequence")
    H, D = seqs[0].q.shape[1], seqs[0].q.shape[2]
    arr = (rkv_attn_seq * len(seqs))(*[s.to_c() for s in seqs])
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(D)
    _check(_lib.attn_fwd_varlen_noalloc(arr, len(seqs), H, D, float(softmax_scale), ctypes.byref(rope),
                                        _stream(stream)))


def rkv_attn_noalloc_status(stream=None):
    """Synchronise and raise RkvError if the last no-alloc launch on this GPU timed out."""
    _check(_lib.rkv_attn_noalloc_status(_stream(stream)))


def attn_mask_rows(seqs, H, rope):
    """The mask and key-tile plan attn_fwd_varlen uses for ``seqs``, evaluated
    on the host by the kernel's own code (no GPU needed).  ``seqs``: AttnSeq
    objects or dicts with Lq, Lk and optional q_frame_offset, block_frames.
    Returns (limits, units): limits[i][r] = keys visible to query row r of
    sequence i (a prefix); units = int32 [n_units, 4] rows of (sequence,
    head, 512-row query block, 128-key tiles processed), in launch order."""
    import numpy as np
    descs = []
    for s in seqs:
        if isinstance(s, dict):
            descs.append(rkv_attn_seq(Lq=int(s["Lq"]), Lk=int(s["Lk"]), q_frame_offset=int(s.get("q_frame_offset", 0)),
                                      block_frames=int(s.get("block_frames", 0))))
        else:
            descs.append(rkv_attn_seq(Lq=int(s.q.shape[0]), Lk=int(s.k.shape[0]), q_frame_offset=s.q_frame_offset,
                                      block_frames=s.block_frames))
    if not descs:
        raise ValueError("need at least one sequence")
    arr = (rkv_attn_seq * len(descs))(*descs)
    lq = [d.Lq for d in descs]
    limits = np.zeros(max(1, sum(lq)), dtype=np.int64)
    n_units = sum(int(H) * ((x + 511) // 512) for x in lq)
    units = np.zeros((max(1, n_units), 4), dtype=np.int32)
    got = ctypes.c_int64(0)
    _check(_lib.rkv_attn_mask_rows(arr, len(descs), int(H), ctypes.byref(rope),
                                   limits.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                   units.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), ctypes.byref(got)))
    if got.value != n_units:
        raise RuntimeError(f"unit count {got.value} != {n_units}")
    out, at = [], 0
    for x in lq:
        out.append(limits[at:at + x].copy())
        at += x
    return out, units[:n_units]


def rkv_ring_status(stream=None):
    """Synchronise and raise RkvError if a ring insert on this GPU gave up on
    a bounded device-side wait since the last call."""
    _check(_lib.rkv_ring_status(_stream(stream)))


def _ring_buffer(t, shape, name):
    """Check a caller-supplied ring buffer: the kernels write
    slots * tokens_per_frame * H * D contiguous bf16 values from its start, so
    anything smaller, strided or on the host is refused here (the C side
    cannot see a buffer's size)."""
    import torch
    if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16:
        raise ValueError(f"ring {name} must be a bf16 tensor")
    if tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"ring {name} must be a contiguous tensor of shape {tuple(shape)} "
                         f"(got {tuple(t.shape)}, contiguous={t.is_contiguous()})")
    if not t.is_cuda:
        raise ValueError(f"ring {name} must be in CUDA device memory")
    return t


class KVRing:
    """A per-layer ring of frame slots for K and V (device bf16
    [slots][tokens_per_frame][H][D] each) plus its head/count state; the
    first ``pinned`` slots keep the first frames ever inserted."""

    def __init__(self, slots, tokens_per_frame, H, D=128, device="cuda", k=None, v=None, pinned=0):
        import torch
        if not 0 <= pinned < slots:
            raise ValueError(f"pinned ({pinned}) must be in [0, slots={slots})")
        shape = (slots, tokens_per_frame, H, D)
        self.k = torch.empty(shape, dtype=torch.bfloat16, device=device) if k is None else _ring_buffer(k, shape, "k")
        self.v = torch.empty(shape, dtype=torch.bfloat16, device=device) if v is None else _ring_buffer(v, shape, "v")
        self.c = rkv_ring(self.k.data_ptr(), self.v.data_ptr(), slots, tokens_per_frame, H, D, pinned, 0, pinned)

    @property
    def head(self):
        return self.c.head

    @property
    def count(self):
        return self.c.count

    @property
    def slots(self):
        return self.c.slots

    @property
    def pinned(self):
        return self.c.pinned

    def slot(self, j):
        return int(_lib.rkv_ring_slot(ctypes.byref(self.c), int(j)))

    def valid_rows(self):
        """Number of valid key rows when the valid slots are the prefix [0, count)
        (a ring filled from empty, or a full ring)."""
        return self.c.count * self.c.tokens_per_frame


def _ring_insert_args(ring, k_new, v_new, n_frames):
    ks, vs = _rows(k_new, "k_new"), _rows(v_new, "v_new")
    if ks != vs:
        raise ValueError("k_new and v_new must share a row stride")
    F = ring.c.tokens_per_frame
    if n_frames is None:
        n_frames = k_new.shape[0] // F
    if k_new.shape[0] < n_frames * F or v_new.shape[0] < n_frames * F:
        raise ValueError("k_new/v_new hold fewer than n_frames frames")
    return ks, int(n_frames)


def kvcache_ring_update(ring, k_new, v_new, n_frames=None, stream=None):
    """Insert n_frames frames ([n*F, H, D] bf16 CUDA tensors) into ``ring``;
    returns the number of frames evicted."""
    ks, n_frames = _ring_insert_args(ring, k_new, v_new, n_frames)
    ev = ctypes.c_int32(0)
    _check(_lib.kvcache_ring_update(ctypes.byref(ring.c), k_new.data_ptr(), v_new.data_ptr(), ks, n_frames,
                                    ctypes.byref(ev), _stream(stream)))
    return ev.value


def kvcache_ring_update_debug(ring, k_new, v_new, n_frames=None, stall=RKV_DEBUG_STALL_BULK_LOAD, timeout_us=0,
                              stream=None):
    """kvcache_ring_update with stall injection (see rkv.h); returns the
    number of frames evicted."""
    ks, n_frames = _ring_insert_args(ring, k_new, v_new, n_frames)
    ev = ctypes.c_int32(0)
    dbg = rkv_ring_debug(int(stall), int(timeout_us))
    _check(_lib.kvcache_ring_update_debug(ctypes.byref(ring.c), k_new.data_ptr(), v_new.data_ptr(), ks, n_frames,
                                          ctypes.byref(ev), ctypes.byref(dbg), _stream(stream)))
    return ev.value


def kvcache_ring_update_rope(ring, k_new, v_new, t0, rope, n_frames=None, stream=None):
    """Insert n_frames frames like kvcache_ring_update, rotating the raw keys
    k_new by RoPE3D on the way in (frame i at time t0 + i); returns the
    number of frames evicted."""
    ks, n_frames = _ring_insert_args(ring, k_new, v_new, n_frames)
    ev = ctypes.c_int32(0)
    _check(_lib.kvcache_ring_update_rope(ctypes.byref(ring.c), k_new.data_ptr(), v_new.data_ptr(), ks, n_frames,
                                         int(t0), ctypes.byref(rope), ctypes.byref(ev), _stream(stream)))
    return ev.value
