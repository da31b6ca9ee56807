// Rolling KV-cache update: insert whole frames of K and V into a per-layer ring
// of frame slots, evicting the oldest frames by overwriting them.
//
// Source: "Amazon and Reactor tune Trainium for real-time video generation",
// section "Three problems for generic compilers" (every layer reads and writes
// a rolling KV cache; frames are generated and evicted in a sliding window) and
// "Optimizing Real-Time Video Generation on Trainium Chips", item 6 "Neuron
// Kernel Interface" (per-layer cache copies given their own kernel).
//
// Design: a ring avoids the whole-window shift a naive sliding buffer needs;
// eviction moves no bytes.  The copy is pure HBM traffic (read n frames, write
// n frames, for K and for V), so the kernel is a coalesced grid-stride copy of
// 16-byte vectors, four independent vectors in flight per thread, one launch
// for K and V (blockIdx.y selects the tensor), grid sized to one wave of
// resident CTAs.
#include "common.cuh"

namespace rkv {

struct RingCopyArgs {
  const uint8_t* src[2];
  uint8_t* dst[2];
  int64_t src_row_stride_bytes;
  uint64_t frame_bytes;   // tokens_per_frame * H * D * 2
  uint32_t row_bytes;     // H * D * 2
  uint32_t row_vecs;      // row_bytes / 16
  uint32_t total_vecs;    // n_frames * tokens_per_frame * row_vecs
  uint32_t F;             // tokens per frame
  RingPlan plan;          // destination slot of each inserted frame
  FastDiv div_row_vecs, div_F;
};

constexpr int kRingThreads = 256;
constexpr int kRingUnroll = 4;

__global__ void __launch_bounds__(kRingThreads) ring_copy_kernel(const RingCopyArgs a) {
  const int which = blockIdx.y;  // 0 = K, 1 = V
  const uint8_t* __restrict__ src = a.src[which];
  uint8_t* __restrict__ dst = a.dst[which];
  const uint32_t stride = gridDim.x * kRingThreads;
  for (uint32_t base = blockIdx.x * kRingThreads + threadIdx.x; base < a.total_vecs;
       base += stride * kRingUnroll) {
    uint4 val[kRingUnroll];
    uint8_t* out[kRingUnroll];
#pragma unroll
    for (int u = 0; u < kRingUnroll; ++u) {
      const uint32_t v = base + u * stride;
      out[u] = nullptr;
      if (v < a.total_vecs) {
        const uint32_t row = fdiv(v, a.div_row_vecs);
        const uint32_t c = v - row * a.row_vecs;
        const uint32_t frame = fdiv(row, a.div_F);
        const uint32_t rr = row - frame * a.F;
        const int32_t slot = ring_dst_slot(a.plan, frame);
        val[u] = __ldcs(reinterpret_cast<const uint4*>(src + int64_t(row) * a.src_row_stride_bytes +
                                                        uint64_t(c) * 16u));
        out[u] = dst + uint64_t(slot) * a.frame_bytes + uint64_t(rr) * a.row_bytes + uint64_t(c) * 16u;
      }
    }
#pragma unroll
    for (int u = 0; u < kRingUnroll; ++u)
      if (out[u]) *reinterpret_cast<uint4*>(out[u]) = val[u];
  }
}

static int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

rkv_status check_ring(const rkv_ring* r) {
  if (!r) return fail(RKV_ERR_INVALID_ARG, "ring is NULL");
  if (!r->k || !r->v) return fail(RKV_ERR_INVALID_ARG, "ring k/v buffer is NULL");
  if (r->slots < 1 || r->tokens_per_frame < 1 || r->H < 1)
    return fail(RKV_ERR_INVALID_ARG, "ring slots/tokens_per_frame/H must be >= 1");
  if (r->D != 128) return fail(RKV_ERR_INVALID_ARG, "head_dim D must be 128 (got %d)", r->D);
  if (r->pinned < 0 || r->pinned >= r->slots)
    return fail(RKV_ERR_INVALID_ARG, "ring pinned %d must be in [0, slots=%d)", r->pinned, r->slots);
  if (r->head < r->pinned || r->head >= r->slots)
    return fail(RKV_ERR_INVALID_ARG, "ring head %d out of range [pinned, slots)", r->head);
  if (r->count < 0 || r->count > r->slots)
    return fail(RKV_ERR_INVALID_ARG, "ring count %d out of range", r->count);
  if (r->count < r->pinned && r->head != r->pinned)
    return fail(RKV_ERR_INVALID_ARG, "ring head must equal pinned until the pinned frames are all in");
  if (!aligned16(r->k) || !aligned16(r->v)) return fail(RKV_ERR_INVALID_ARG, "ring buffers must be 16-byte aligned");
  const uint64_t bytes = uint64_t(r->slots) * r->tokens_per_frame * r->H * r->D * 2;
  if (overlaps(r->k, bytes, r->v, bytes)) return fail(RKV_ERR_INVALID_ARG, "ring k and v buffers overlap");
  return RKV_OK;
}

rkv_status check_ring_insert(const rkv_ring* ring, const void* k_new, const void* v_new, int64_t new_row_stride,
                             int32_t n_frames) {
  const int32_t free_pinned = ring->count < ring->pinned ? ring->pinned - ring->count : 0;
  const int32_t capacity = free_pinned + (ring->slots - ring->pinned);
  if (n_frames < 0 || n_frames > capacity)
    return fail(RKV_ERR_INVALID_ARG, "n_frames %d must be in [0, %d] (free pinned slots + rolling slots)", n_frames,
                capacity);
  if (n_frames == 0) return RKV_OK;
  const int64_t row_elems = int64_t(ring->H) * ring->D;
  if (!k_new || !v_new) return fail(RKV_ERR_INVALID_ARG, "k_new/v_new is NULL");
  if (!aligned16(k_new) || !aligned16(v_new)) return fail(RKV_ERR_INVALID_ARG, "k_new/v_new must be 16-byte aligned");
  if (new_row_stride < row_elems) return fail(RKV_ERR_INVALID_ARG, "new_row_stride < H*D");
  if ((new_row_stride * 2) % 16 != 0) return fail(RKV_ERR_INVALID_ARG, "rows of k_new/v_new must be 16-byte aligned");
  const int64_t rows = int64_t(n_frames) * ring->tokens_per_frame;
  const uint64_t src_bytes = uint64_t((rows - 1) * new_row_stride + row_elems) * 2;
  const uint64_t ring_bytes = uint64_t(ring->slots) * ring->tokens_per_frame * row_elems * 2;
  if (overlaps(k_new, src_bytes, ring->k, ring_bytes) || overlaps(k_new, src_bytes, ring->v, ring_bytes) ||
      overlaps(v_new, src_bytes, ring->k, ring_bytes) || overlaps(v_new, src_bytes, ring->v, ring_bytes))
    return fail(RKV_ERR_INVALID_ARG, "new frames overlap the ring buffers");
  if (uint64_t(rows) * (row_elems * 2 / 16) >= (uint64_t(1) << 31))
    return fail(RKV_ERR_UNSUPPORTED, "insert too large for one launch");
  return RKV_OK;
}

RingPlan ring_plan(const rkv_ring* ring) {
  RingPlan p;
  p.pin_base = ring->count;
  p.n_pin = ring->count < ring->pinned ? ring->pinned - ring->count : 0;
  p.head = ring->head;
  p.end = ring->slots;
  p.len = ring->slots - ring->pinned;
  return p;
}

void ring_advance(rkv_ring* ring, int32_t n_frames, int32_t* n_evicted) {
  const RingPlan p = ring_plan(ring);
  const int32_t pinned_in = n_frames < p.n_pin ? n_frames : p.n_pin;
  const int32_t rolling = n_frames - pinned_in;
  const int32_t count = ring->count + pinned_in;
  const int32_t evicted = count + rolling > ring->slots ? count + rolling - ring->slots : 0;
  ring->head = ring->pinned + (ring->head - ring->pinned + rolling) % p.len;
  ring->count = count + rolling < ring->slots ? count + rolling : ring->slots;
  if (n_evicted) *n_evicted = evicted;
}

}  // namespace rkv

using namespace rkv;

extern "C" int32_t rkv_ring_slot(const rkv_ring* ring, int32_t j) {
  if (!ring || ring->slots < 1 || ring->pinned < 0 || ring->pinned >= ring->slots || ring->count < 0 ||
      ring->count > ring->slots || ring->head < ring->pinned || ring->head >= ring->slots)
    return -1;
  if (j < 0 || j >= ring->count) return -1;
  const int32_t P = ring->pinned;
  if (j < P) return j;
  // rolling frame j - P of count - P, the newest one in slot head - 1
  const int32_t len = ring->slots - P;
  int64_t s = (int64_t(ring->head - P) - (ring->count - P) + (j - P)) % len;
  if (s < 0) s += len;
  return int32_t(P + s);
}

extern "C" rkv_status kvcache_ring_update(rkv_ring* ring, const void* k_new, const void* v_new,
                                          int64_t new_row_stride, int32_t n_frames, int32_t* n_evicted,
                                          void* stream) {
  clear_error();
  rkv_status st = check_ring(ring);
  if (st != RKV_OK) return st;
  st = check_ring_insert(ring, k_new, v_new, new_row_stride, n_frames);
  if (st != RKV_OK) return st;
  if (n_frames > 0) {
    const int64_t row_elems = int64_t(ring->H) * ring->D;
    const uint64_t total_vecs = uint64_t(n_frames) * ring->tokens_per_frame * (row_elems * 2 / 16);
    RingCopyArgs a;
    a.src[0] = static_cast<const uint8_t*>(k_new);
    a.src[1] = static_cast<const uint8_t*>(v_new);
    a.dst[0] = static_cast<uint8_t*>(ring->k);
    a.dst[1] = static_cast<uint8_t*>(ring->v);
    a.src_row_stride_bytes = new_row_stride * 2;
    a.row_bytes = uint32_t(row_elems * 2);
    a.row_vecs = a.row_bytes / 16;
    a.frame_bytes = uint64_t(ring->tokens_per_frame) * a.row_bytes;
    a.total_vecs = uint32_t(total_vecs);
    a.F = uint32_t(ring->tokens_per_frame);
    a.plan = ring_plan(ring);
    a.div_row_vecs = make_fastdiv(a.row_vecs);
    a.div_F = make_fastdiv(a.F);
    const uint64_t per_block = uint64_t(kRingThreads) * kRingUnroll;
    uint64_t blocks = (total_vecs + per_block - 1) / per_block;
    const uint64_t wave = uint64_t(sm_count()) * (2048 / kRingThreads);  // per tensor: two resident waves in all
    if (blocks > wave) blocks = wave;
    dim3 grid(uint32_t(blocks), 2);
    ring_copy_kernel<<<grid, kRingThreads, 0, static_cast<cudaStream_t>(stream)>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "ring_copy_kernel launch");
  }
  ring_advance(ring, n_frames, n_evicted);
  return RKV_OK;
}
