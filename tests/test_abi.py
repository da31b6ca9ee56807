"""The C ABI without a GPU: the library loads, exports every declared symbol,
and rejects invalid arguments on the host before launching anything."""

import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rkv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_]\w*\s*\*?\s+\*?([A-Za-z_]\w*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "return")))


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("rope3d_apply", "attn_fwd_varlen", "kvcache_ring_update"):
        assert n in names


def test_library_exports_every_declared_symbol(lib_path):
    lib = ctypes.CDLL(lib_path)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


@pytest.fixture(scope="module")
def rkv(lib_path):
    from rolling_kv_cache_rope_b200 import rkv as m
    return m


def fake(addr):
    return ctypes.c_void_p(addr)


def test_version(rkv):
    # the library reports the version of the header it was built from
    m = re.search(r"#define RKV_VERSION (\d+)", open(HEADER).read())
    assert m and rkv.rkv_version() == int(m.group(1)) >= 200


def ring(rkv, slots=5, F=24, H=2, D=128, head=0, count=0, k=0x10000, v=0x20000000, pinned=0):
    return rkv.rkv_ring(k, v, slots, F, H, D, head, count, pinned)


def test_ring_slot_host_logic(rkv):
    lib = rkv.lib()
    r = ring(rkv, slots=5, head=1, count=5)
    assert [lib.rkv_ring_slot(ctypes.byref(r), j) for j in range(6)] == [1, 2, 3, 4, 0, -1]
    r = ring(rkv, slots=5, head=3, count=3)
    assert [lib.rkv_ring_slot(ctypes.byref(r), j) for j in range(4)] == [0, 1, 2, -1]
    assert lib.rkv_ring_slot(ctypes.byref(r), -1) == -1
    bad = ring(rkv, slots=5, head=7, count=3)
    assert lib.rkv_ring_slot(ctypes.byref(bad), 0) == -1
    assert lib.rkv_ring_slot(None, 0) == -1


@pytest.mark.parametrize("change,n,frag", [
    (dict(), 6, "n_frames"),                 # more frames than slots
    (dict(), -1, "n_frames"),
    (dict(D=64), 1, "128"),
    (dict(head=5), 1, "head"),
    (dict(count=9), 1, "count"),
    (dict(k=0), 1, "NULL"),
    (dict(k=0x10008), 1, "aligned"),
    (dict(v=0x10000), 1, "overlap"),         # k and v buffers overlap
    (dict(pinned=5), 1, "pinned"),           # pinned must leave a rolling slot
    (dict(pinned=-1), 1, "pinned"),
    (dict(pinned=2, head=1, count=5), 1, "head"),   # head inside the pinned prefix
    (dict(pinned=2, head=3, count=1), 1, "head"),   # rolling before the prefix is full
    (dict(pinned=2, head=2, count=5), 4, "n_frames"),   # 3 rolling slots, prefix full
    (dict(pinned=2, head=2, count=1), 5, "n_frames"),   # 1 free pinned + 3 rolling
])
def test_ring_update_rejects(rkv, change, n, frag):
    lib = rkv.lib()
    r = ring(rkv, **change)
    before = (r.head, r.count)
    ev = ctypes.c_int32(-7)
    st = lib.kvcache_ring_update(ctypes.byref(r), fake(0x40000000), fake(0x50000000), 2 * 128, n,
                                 ctypes.byref(ev), None)
    assert st == rkv.RKV_ERR_INVALID_ARG
    assert frag in rkv.rkv_last_error_string()
    assert (r.head, r.count) == before and ev.value == -7


def test_ring_slot_pinned_matches_oracle(rkv):
    # slot of every logical frame, in every state a pinned ring passes through
    from oracle import RingRef
    lib = rkv.lib()
    rng = np.random.default_rng(5)
    for W, P in [(5, 1), (6, 2), (21, 3), (4, 3)]:
        ref = RingRef(W, P)
        for _ in range(40):
            n = int(rng.integers(0, ref.capacity_for_insert() + 1))
            ref.insert([None] * n)
            r = ring(rkv, slots=W, head=ref.head, count=ref.count, pinned=P)
            got = [lib.rkv_ring_slot(ctypes.byref(r), j) for j in range(-1, W + 1)]
            assert got == [ref.slot_of(j) for j in range(-1, W + 1)], (W, P, ref.head, ref.count)
    bad = ring(rkv, slots=5, head=1, count=5, pinned=2)
    assert lib.rkv_ring_slot(ctypes.byref(bad), 0) == -1


def test_ring_insert_capacity_matches_oracle(rkv):
    # over random reachable states of pinned rings, an insert is refused on
    # the host exactly when the oracle ring says it carries too many frames
    # (an accepted one then fails at the launch here: no GPU) and the state
    # is left unchanged either way
    from hypothesis import given, settings, strategies as st
    from oracle import RingRef
    lib = rkv.lib()

    @settings(max_examples=200, deadline=None)
    @given(st.integers(1, 9), st.data())
    def check(W, data):
        P = data.draw(st.integers(0, W - 1))
        ref = RingRef(W, P)
        for n in data.draw(st.lists(st.integers(0, W), max_size=6)):
            if n <= ref.capacity_for_insert():
                ref.insert([None] * n)
        n = data.draw(st.integers(0, W + 1))
        r = ring(rkv, slots=W, head=ref.head, count=ref.count, pinned=P)
        st_ = lib.kvcache_ring_update(ctypes.byref(r), fake(0x40000000), fake(0x50000000), 2 * 128, n, None, None)
        refused = st_ == rkv.RKV_ERR_INVALID_ARG and "n_frames" in rkv.rkv_last_error_string()
        assert refused == (n > ref.capacity_for_insert()), (W, P, ref.head, ref.count, n, st_)
        if n > 0:
            assert (r.head, r.count) == (ref.head, ref.count)

    check()


def test_ring_update_rejects_bad_sources(rkv):
    lib = rkv.lib()
    r = ring(rkv)
    for kn, vn, stride in [(0, 0x50000000, 256), (0x40000004, 0x50000000, 256), (0x40000000, 0x50000000, 100),
                           (0x10000, 0x50000000, 256)]:       # last: k_new overlaps the ring
        st = lib.kvcache_ring_update(ctypes.byref(r), fake(kn), fake(vn), stride, 2, None, None)
        assert st == rkv.RKV_ERR_INVALID_ARG, (kn, vn, stride)


def test_ring_update_zero_frames_is_a_host_noop(rkv):
    lib = rkv.lib()
    r = ring(rkv, head=2, count=4)
    ev = ctypes.c_int32(-1)
    assert lib.kvcache_ring_update(ctypes.byref(r), None, None, 256, 0, ctypes.byref(ev), None) == rkv.RKV_OK
    assert (r.head, r.count, ev.value) == (2, 4, 0)


def rope(rkv, **kw):
    base = dict(grid_h=4, grid_w=6, pairs=(22, 21, 21), theta=10000.0)
    base.update(kw)
    return rkv.make_rope(base["grid_h"], base["grid_w"], base["pairs"], base["theta"])


@pytest.mark.parametrize("args,frag", [
    (dict(D=64), "128"),
    (dict(x=0), "NULL"),
    (dict(x=0x1008), "aligned"),
    (dict(xs=100), "stride"),
    (dict(y=0x1100), "overlap"),
    (dict(rope_kw=dict(pairs=(20, 21, 21))), "pairs"),
    (dict(rope_kw=dict(grid_h=0)), "grid"),
    (dict(rope_kw=dict(theta=1.0)), "theta"),
])
def test_rope_rejects(rkv, args, frag):
    lib = rkv.lib()
    a = dict(x=0x1000, y=0x90000000, L=72, H=2, D=128, xs=256, ys=256)
    a.update({k: v for k, v in args.items() if k != "rope_kw"})
    r = rope(rkv, **args.get("rope_kw", {}))
    st = lib.rope3d_apply(fake(a["x"]), fake(a["y"]), a["L"], a["H"], a["D"], a["xs"], a["ys"], 0,
                          ctypes.byref(r), None)
    assert st == rkv.RKV_ERR_INVALID_ARG, rkv.rkv_last_error_string()
    assert frag in rkv.rkv_last_error_string()


def test_rope_rejects_bad_layout_and_axis_theta(rkv):
    lib = rkv.lib()
    for kw in ({"layout": 2}, {"theta_h": 0.5}, {"theta_w": float("inf")}):
        r = rope(rkv)
        for k, v in kw.items():
            setattr(r, k, v)
        st = lib.rope3d_apply(fake(0x1000), fake(0x90000000), 72, 2, 128, 256, 256, 0, ctypes.byref(r), None)
        assert st == rkv.RKV_ERR_INVALID_ARG, kw
        assert ("layout" in rkv.rkv_last_error_string()) or ("theta" in rkv.rkv_last_error_string())


def test_make_rope_variants(rkv):
    r = rkv.make_rope(4, 6, theta=(100.0, 200.0, 300.0), layout="half")
    assert (r.theta, r.theta_h, r.theta_w, r.layout) == (100.0, 200.0, 300.0, rkv.RKV_ROPE_HALF)
    d = rkv.make_rope(4, 6)
    assert (d.theta, d.theta_h, d.theta_w, d.layout) == (10000.0, 10000.0, 10000.0, rkv.RKV_ROPE_ADJACENT)
    with pytest.raises(ValueError):
        rkv.make_rope(4, 6, layout="interleaved")


def _batch(rkv, items):
    arr = (rkv.rkv_rope_tensor * max(1, len(items)))()
    for i, (x, y, L, t0) in enumerate(items):
        arr[i] = rkv.rkv_rope_tensor(x, y, L, 256, 256, t0)
    return arr


def test_rope_batch_rejects(rkv):
    lib = rkv.lib()
    r = rope(rkv)
    ok = [(0x1000, 0x90000000, 72, 0), (0x200000, 0xA0000000, 120, 1)]
    # more tensors than a launch takes
    arr = _batch(rkv, ok * 5)
    assert lib.rope3d_apply_batch(arr, 9, 2, 128, ctypes.byref(r), None) == rkv.RKV_ERR_INVALID_ARG
    assert "n must be" in rkv.rkv_last_error_string()
    assert lib.rope3d_apply_batch(None, 2, 2, 128, ctypes.byref(r), None) == rkv.RKV_ERR_INVALID_ARG
    # one tensor's output over another's input or output
    for bad in ([(0x1000, 0x90000000, 72, 0), (0x200000, 0x90000100, 120, 1)],
                [(0x1000, 0x90000000, 72, 0), (0x90000100, 0xA0000000, 120, 1)]):
        assert lib.rope3d_apply_batch(_batch(rkv, bad), 2, 2, 128, ctypes.byref(r), None) == rkv.RKV_ERR_INVALID_ARG
        assert "overlaps tensor" in rkv.rkv_last_error_string()
    # a tensor's own rules still apply
    bad = [(0x1000, 0x90000000, 72, 0), (0x0, 0xA0000000, 120, 1)]
    assert lib.rope3d_apply_batch(_batch(rkv, bad), 2, 2, 128, ctypes.byref(r), None) == rkv.RKV_ERR_INVALID_ARG
    assert "NULL" in rkv.rkv_last_error_string()
    # nothing to do: no tensors, or only empty ones
    assert lib.rope3d_apply_batch(None, 0, 2, 128, ctypes.byref(r), None) == rkv.RKV_OK
    empty = [(0x0, 0x0, 0, 0), (0x0, 0x0, 0, 3)]
    assert lib.rope3d_apply_batch(_batch(rkv, empty), 2, 2, 128, ctypes.byref(r), None) == rkv.RKV_OK


def test_rope_zero_rows_is_a_noop(rkv):
    r = rope(rkv)
    assert rkv.lib().rope3d_apply(None, None, 0, 2, 128, 256, 256, 0, ctypes.byref(r), None) == rkv.RKV_OK


@pytest.mark.parametrize("change,n,t0,rope_kw,frag", [
    ({}, 6, 0, {}, "n_frames"),
    ({}, 2, 0, {"grid_h": 5}, "tokens_per_frame"),
    ({}, 2, 0, {"pairs": (22, 21, 20)}, "pairs"),
    ({"D": 64}, 2, 0, {}, "head_dim"),
    ({"head": 9}, 2, 0, {}, "head"),
    ({}, 2, 2**31 - 1, {}, "overflows"),
])
def test_ring_update_rope_rejects(rkv, change, n, t0, rope_kw, frag):
    lib = rkv.lib()
    r = ring(rkv, **change)
    rp = rope(rkv, **rope_kw)
    before = (r.head, r.count)
    ev = ctypes.c_int32(-7)
    st = lib.kvcache_ring_update_rope(ctypes.byref(r), fake(0x40000000), fake(0x50000000), 2 * 128, n, t0,
                                      ctypes.byref(rp), ctypes.byref(ev), None)
    assert st == rkv.RKV_ERR_INVALID_ARG, rkv.rkv_last_error_string()
    assert frag in rkv.rkv_last_error_string()
    assert (r.head, r.count) == before and ev.value == -7


def test_ring_update_rope_zero_frames_is_a_host_noop(rkv):
    lib = rkv.lib()
    r = ring(rkv, head=2, count=4)
    rp = rope(rkv)
    ev = ctypes.c_int32(-1)
    assert lib.kvcache_ring_update_rope(ctypes.byref(r), None, None, 256, 0, 0, ctypes.byref(rp), ctypes.byref(ev),
                                        None) == rkv.RKV_OK
    assert (r.head, r.count, ev.value) == (2, 4, 0)


def seq(rkv, **kw):
    base = dict(q=0x100000, k=0x200000, v=0x300000, o=0x400000, q_stride=256, k_stride=256, v_stride=256,
                o_stride=256, Lq=72, Lk=120, q_t0=2, k_t0=0, q_frame_offset=2, block_frames=0, flags=3,
                reserved=0)
    base.update(kw)
    return rkv.rkv_attn_seq(**base)


@pytest.mark.parametrize("kw,frag", [
    (dict(Lq=0), "Lq"),
    (dict(k=0), "NULL"),
    (dict(v=0x300008), "aligned"),
    (dict(o_stride=128), "stride"),
    (dict(block_frames=-1), "block_frames"),
    (dict(block_frames=3, q_frame_offset=-1), "q_frame_offset"),
    (dict(flags=8), "flags"),
    (dict(reserved=1), "reserved"),
    (dict(o=0x100100), "overlaps"),
])
def test_attn_rejects(rkv, kw, frag):
    lib = rkv.lib()
    arr = (rkv.rkv_attn_seq * 1)(seq(rkv, **kw))
    r = rope(rkv)
    st = lib.attn_fwd_varlen(arr, 1, 2, 128, 0.088, ctypes.byref(r), fake(0x700000), 256, None)
    assert st == rkv.RKV_ERR_INVALID_ARG, rkv.rkv_last_error_string()
    assert frag in rkv.rkv_last_error_string()


def test_attn_outputs_may_be_head_slices_of_one_tensor(rkv):
    # four single-head sequences whose Q/O are heads 0..3 of [72, 4, 128]
    # tensors (row stride 4 heads): the strided outputs share no byte, so the
    # host checks pass (the launch itself then fails without a GPU)
    lib = rkv.lib()
    r = rope(rkv)
    q0, o0, k0 = 0x1000000, 0x2000000, 0x3000000
    def head_seq(h, o_head=None):
        return seq(rkv, q=q0 + h * 256, o=o0 + (h if o_head is None else o_head) * 256, k=k0 + h * 256,
                   v=k0 + 0x800000 + h * 256, q_stride=512, k_stride=512, v_stride=512, o_stride=512)
    arr = (rkv.rkv_attn_seq * 4)(*[head_seq(h) for h in range(4)])
    st = lib.attn_fwd_varlen(arr, 4, 1, 128, 0.088, ctypes.byref(r), fake(0x700000), 256, None)
    assert "overlaps" not in rkv.rkv_last_error_string() and st != rkv.RKV_ERR_INVALID_ARG, \
        rkv.rkv_last_error_string()
    # two sequences writing the same head, or an output on another's input
    for bad in ([head_seq(0), head_seq(1, o_head=0)],
                [head_seq(0), seq(rkv, q=o0, o=o0 + 2 * 256, k=k0, v=k0 + 0x800000, q_stride=512,
                                  k_stride=512, v_stride=512, o_stride=512)]):
        arr = (rkv.rkv_attn_seq * 2)(*bad)
        st = lib.attn_fwd_varlen(arr, 2, 1, 128, 0.088, ctypes.byref(r), fake(0x700000), 256, None)
        assert st == rkv.RKV_ERR_INVALID_ARG and "overlaps" in rkv.rkv_last_error_string()


def _views_share_a_byte(a, la, sa, b, lb, sb, width):
    return any(a + i * sa < b + j * sb + width and b + j * sb < a + i * sa + width
               for i in range(la) for j in range(lb))


def test_attn_output_overlap_check_is_exact(rkv):
    # random pairs of row-strided single-head views (row = 256 bytes): with
    # equal row strides the host check flags an output exactly when it shares
    # a byte with another sequence's output or input (brute force over the
    # rows); with different strides it flags overlapping byte spans
    from hypothesis import given, settings, strategies as st
    lib = rkv.lib()
    r = rope(rkv)
    base = 0x10000000

    @settings(max_examples=300, deadline=None)
    @given(st.integers(1, 5), st.integers(1, 5), st.sampled_from([128, 136, 256, 384, 512]),
           st.sampled_from([128, 256, 384, 512]), st.integers(0, 40), st.booleans())
    def check(la, lb, sa, sb, off16, against_output):
        a_o = base
        b_t = base + off16 * 16
        far = 0x40000000
        sa_ = sa
        sb_ = sb
        A = seq(rkv, q=far, k=far + 0x1000000, v=far + 0x2000000, o=a_o, q_stride=sa_, k_stride=128, v_stride=128,
                o_stride=sa_, Lq=la, Lk=8, q_t0=0, q_frame_offset=0, flags=0)
        if against_output:
            B = seq(rkv, q=far + 0x3000000, k=far + 0x4000000, v=far + 0x5000000, o=b_t, q_stride=sb_,
                    k_stride=128, v_stride=128, o_stride=sb_, Lq=lb, Lk=8, q_t0=0, q_frame_offset=0, flags=0)
        else:
            B = seq(rkv, q=b_t, k=far + 0x4000000, v=far + 0x5000000, o=far + 0x6000000, q_stride=sb_,
                    k_stride=128, v_stride=128, o_stride=sb_, Lq=lb, Lk=8, q_t0=0, q_frame_offset=0, flags=0)
        arr = (rkv.rkv_attn_seq * 2)(A, B)
        lib.attn_fwd_varlen(arr, 2, 1, 128, 0.088, ctypes.byref(r), fake(0x700000), 256, None)
        flagged = "overlaps" in rkv.rkv_last_error_string()
        if sa == sb:
            want = _views_share_a_byte(a_o, la, sa_ * 2, b_t, lb, sb_ * 2, 256)
        else:   # different row strides: the byte spans decide (conservative)
            want = a_o < b_t + (lb - 1) * sb_ * 2 + 256 and b_t < a_o + (la - 1) * sa_ * 2 + 256
        assert flagged == want, (la, lb, sa, sb, off16, against_output)

    check()


def test_attn_rejects_launch_level_arguments(rkv):
    lib = rkv.lib()
    arr = (rkv.rkv_attn_seq * 1)(seq(rkv))
    r = rope(rkv)
    ws = fake(0x700000)
    assert lib.attn_fwd_varlen(arr, 0, 2, 128, 0.088, ctypes.byref(r), ws, 256, None) == rkv.RKV_ERR_INVALID_ARG
    assert lib.attn_fwd_varlen(arr, 1, 2, 64, 0.088, ctypes.byref(r), ws, 256, None) == rkv.RKV_ERR_INVALID_ARG
    assert lib.attn_fwd_varlen(arr, 1, 2, 128, -1.0, ctypes.byref(r), ws, 256, None) == rkv.RKV_ERR_INVALID_ARG
    assert lib.attn_fwd_varlen(arr, 1, 2, 128, 0.088, ctypes.byref(r), None, 256, None) == rkv.RKV_ERR_INVALID_ARG
    assert lib.attn_fwd_varlen(arr, 1, 2, 128, 0.088, ctypes.byref(r), ws, 8, None) == rkv.RKV_ERR_INVALID_ARG
    many = (rkv.rkv_attn_seq * 17)(*[seq(rkv) for _ in range(17)])
    assert lib.attn_fwd_varlen(many, 17, 2, 128, 0.088, ctypes.byref(r), ws, 256, None) == rkv.RKV_ERR_UNSUPPORTED
    assert lib.attn_fwd_varlen_workspace_size(arr, 1, 2, 128) >= 4


def test_kvring_refuses_pinned_prefix_without_rolling_slot(rkv):
    with pytest.raises(ValueError):
        rkv.KVRing(3, 24, 2, pinned=3, device="cpu")
    r = rkv.KVRing(3, 24, 2, pinned=2, device="cpu")
    assert (r.head, r.count, r.pinned) == (2, 0, 2)


def test_python_binding_refuses_non_bf16(rkv):
    import torch
    x = torch.zeros(4, 2, 128, dtype=torch.float32)
    with pytest.raises(ValueError):
        rkv.rope3d_apply(x, rope=rkv.make_rope(4, 6))


def test_kvring_refuses_unfit_caller_buffers(rkv):
    # the ring kernels write slots*F*H*D contiguous bf16 values from the start
    # of each buffer, so the binding refuses anything that cannot hold them
    import torch
    shape = (3, 24, 2, 128)
    good = torch.zeros(shape, dtype=torch.bfloat16)
    bad = [torch.zeros(shape, dtype=torch.float16),                         # wrong dtype
           torch.zeros((2, 24, 2, 128), dtype=torch.bfloat16),             # too few slots
           torch.zeros((3 * 24 * 2 * 128 - 8,), dtype=torch.bfloat16),     # too few elements
           torch.zeros((3, 24, 4, 128), dtype=torch.bfloat16)[:, :, :2],   # strided view
           good]                                                           # host memory
    for b in bad:
        with pytest.raises(ValueError):
            rkv.KVRing(3, 24, 2, k=b, device="cpu")
        with pytest.raises(ValueError):
            rkv.KVRing(3, 24, 2, v=b, device="cpu")


def test_debug_entry_points_reject_bad_settings(rkv):
    lib = rkv.lib()
    arr = (rkv.rkv_attn_seq * 1)(seq(rkv))
    r = rope(rkv)
    ws = fake(0x700000)
    dbg = rkv.rkv_attn_debug(None, 99, 0)
    assert lib.attn_fwd_varlen_debug(arr, 1, 2, 128, 0.088, ctypes.byref(r), ws, 256, None, None) == \
        rkv.RKV_ERR_INVALID_ARG
    assert lib.attn_fwd_varlen_debug(arr, 1, 2, 128, 0.088, ctypes.byref(r), ws, 256, ctypes.byref(dbg), None) == \
        rkv.RKV_ERR_INVALID_ARG
    dbg = rkv.rkv_attn_debug(fake(0x800004), 0, 0)   # misaligned record
    assert lib.attn_fwd_varlen_debug(arr, 1, 2, 128, 0.088, ctypes.byref(r), ws, 256, ctypes.byref(dbg), None) == \
        rkv.RKV_ERR_INVALID_ARG
    ring = rkv.rkv_ring(fake(0x100000), fake(0x200000), 3, 24, 2, 128, 0, 0, 0)
    rd = rkv.rkv_ring_debug(7, 0)
    ev = ctypes.c_int32(0)
    assert lib.kvcache_ring_update_debug(ctypes.byref(ring), fake(0x300000), fake(0x400000), 256, 1,
                                         ctypes.byref(ev), ctypes.byref(rd), None) == rkv.RKV_ERR_INVALID_ARG
    assert lib.kvcache_ring_update_debug(ctypes.byref(ring), fake(0x300000), fake(0x400000), 256, 1,
                                         ctypes.byref(ev), None, None) == rkv.RKV_ERR_INVALID_ARG
