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
// n frames, for K and for V).  It runs on the TMA bulk-copy engine: one CTA
// per SM, one thread issuing; each piece (up to 32 KB of whole rows of one
// frame) is loaded global -> shared memory with a bulk copy that completes on
// an mbarrier, then stored shared -> global with one bulk copy into its ring
// slot.  Six pieces are in flight per SM, about 190 KB, with no registers
// holding data; a vector copy through registers (16 B per thread, a few in
// flight) keeps far fewer bytes in flight and measured 25-35% slower.
#include <mutex>

#include "common.cuh"
#include "ring_bulk.cuh"
#include "sm100_ptx.cuh"

namespace rkv {

constexpr int kBulkThreads = 32;

// CTA b moves pieces b, b + G, b + 2G, ... of the insert (K pieces, then V).
__global__ void __launch_bounds__(kBulkThreads, 1) ring_bulk_kernel(const RingBulkArgs a) {
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ __align__(8) uint64_t full[kBulkStages];
  if (threadIdx.x != 0) return;
  bulk_copy_pieces(a, blockIdx.x, a.total, gridDim.x, ptx::smem_u32(stage_mem), full);
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

constexpr int kMaxDevices = 64;

// One timeout flag per GPU that loads the library (set by a bulk-copy wait
// that gave up; read and cleared by rkv_ring_status).  Host code must not pass
// its name to a kernel: the device address comes from cudaGetSymbolAddress.
static __device__ int32_t g_ring_timeout;
static std::mutex g_ring_mu;
static int32_t* g_ring_timeout_ptr[kMaxDevices];

rkv_status ring_timeout_flag(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(RKV_ERR_UNSUPPORTED, "device index %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_ring_mu);
  if (!g_ring_timeout_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_ring_timeout);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(ring timeout flag)");
    g_ring_timeout_ptr[dev] = static_cast<int32_t*>(ptr);
  }
  *out = g_ring_timeout_ptr[dev];
  return RKV_OK;
}

// Host side of one insert: piece geometry, grid of one CTA per SM (or fewer
// when the insert has fewer pieces), shared memory for the stages.
static rkv_status launch_ring_bulk(const rkv_ring* ring, const void* k_new, const void* v_new, int64_t new_row_stride,
                                   int32_t n_frames, const rkv_ring_debug* dbg, cudaStream_t stream) {
  RingBulkArgs a;
  rkv_status st = ring_bulk_geometry(ring, k_new, v_new, new_row_stride, n_frames, a);
  if (st != RKV_OK) return st;
  if (dbg) {
    if (dbg->timeout_us > 0) a.wait_ns = uint64_t(dbg->timeout_us) * 1000ull;
    a.stall = dbg->stall;
  }
  st = ring_timeout_flag(&a.timeout_flag);
  if (st != RKV_OK) return st;
  const int smem = int(a.stages * a.stage_bytes);
  cudaError_t e = cudaFuncSetAttribute(ring_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(ring_bulk_kernel)");
  const uint32_t grid = a.total < uint32_t(sm_count()) ? a.total : uint32_t(sm_count());
  ring_bulk_kernel<<<grid, kBulkThreads, smem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "ring_bulk_kernel launch");
  return RKV_OK;
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

static rkv_status ring_update(rkv_ring* ring, const void* k_new, const void* v_new, int64_t new_row_stride,
                              int32_t n_frames, int32_t* n_evicted, const rkv_ring_debug* dbg, void* stream) {
  rkv_status st = check_ring(ring);
  if (st != RKV_OK) return st;
  st = check_ring_insert(ring, k_new, v_new, new_row_stride, n_frames);
  if (st != RKV_OK) return st;
  if (n_frames > 0) {
    st = launch_ring_bulk(ring, k_new, v_new, new_row_stride, n_frames, dbg, static_cast<cudaStream_t>(stream));
    if (st != RKV_OK) return st;
  }
  ring_advance(ring, n_frames, n_evicted);
  return RKV_OK;
}

extern "C" rkv_status kvcache_ring_update(rkv_ring* ring, const void* k_new, const void* v_new,
                                          int64_t new_row_stride, int32_t n_frames, int32_t* n_evicted,
                                          void* stream) {
  NvtxRange nvtx_range("kvcache_ring_update");
  clear_error();
  return ring_update(ring, k_new, v_new, new_row_stride, n_frames, n_evicted, nullptr, stream);
}

extern "C" rkv_status kvcache_ring_update_debug(rkv_ring* ring, const void* k_new, const void* v_new,
                                                int64_t new_row_stride, int32_t n_frames, int32_t* n_evicted,
                                                const rkv_ring_debug* dbg, void* stream) {
  NvtxRange nvtx_range("kvcache_ring_update_debug");
  clear_error();
  if (!dbg) return fail(RKV_ERR_INVALID_ARG, "debug settings are NULL");
  if (dbg->stall > RKV_DEBUG_STALL_BULK_LOAD) return fail(RKV_ERR_INVALID_ARG, "unknown debug stall %u", dbg->stall);
  return ring_update(ring, k_new, v_new, new_row_stride, n_frames, n_evicted, dbg, stream);
}

extern "C" rkv_status rkv_ring_status(void* stream) {
  NvtxRange nvtx_range("rkv_ring_status");
  clear_error();
  int32_t* flag = nullptr;
  rkv_status st = ring_timeout_flag(&flag);
  if (st != RKV_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, flag, sizeof(host), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the ring timeout flag");
  if (host == 0) return RKV_OK;
  e = cudaMemsetAsync(flag, 0, sizeof(int32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the ring timeout flag");
  return fail(RKV_ERR_TIMEOUT, "a ring insert's bulk-copy wait gave up; the insert is incomplete");
}
