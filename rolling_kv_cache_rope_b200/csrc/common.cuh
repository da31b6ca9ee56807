// Host/device helpers shared by the librkv kernels: status plumbing, fast
// integer division by run-time constants, bf16 packing.
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include "rkv.h"

namespace rkv {

// ---- host: an NVTX range around each entry point, so a profiler's timeline
// shows which library call enqueued which kernels (a no-op when no tool is
// attached) ----
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// ---- host: per-thread last-error text ------------------------------------
void set_error(const char* fmt, ...);
void clear_error();
rkv_status fail(rkv_status code, const char* fmt, ...);
rkv_status cuda_fail(cudaError_t e, const char* what);

// ---- host: argument checks and ring bookkeeping shared by several calls ----
rkv_status check_rope(const rkv_rope3d* rope, int32_t D);          // rope3d.cu
rkv_status check_ring(const rkv_ring* ring);                       // ring_update.cu
rkv_status check_ring_insert(const rkv_ring* ring, const void* k_new, const void* v_new, int64_t new_row_stride,
                             int32_t n_frames);                     // ring_update.cu
void ring_advance(rkv_ring* ring, int32_t n_frames, int32_t* n_evicted);  // head, count, evicted

// Where the frames of one insert land.  The first n_pin frames fill the free
// slots of the pinned prefix from pin_base on; the rest roll through the
// region [end - len, end) from head on, wrapping once at most (an insert
// carries at most len rolling frames).  Without a pinned prefix n_pin = 0 and
// the region is the whole ring.
struct RingPlan {
  int32_t n_pin, pin_base, head, end, len;
};
RingPlan ring_plan(const rkv_ring* ring);  // ring_update.cu; for a checked ring
rkv_status ring_timeout_flag(int32_t** out);  // ring_update.cu: this device's ring timeout flag

__host__ __device__ __forceinline__ int32_t ring_dst_slot(const RingPlan& p, uint32_t frame) {
  const int32_t f = int32_t(frame);
  if (f < p.n_pin) return p.pin_base + f;
  const int32_t s = p.head + (f - p.n_pin);
  return s >= p.end ? s - p.len : s;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Byte ranges [a, a+na) and [b, b+nb) overlap.
inline bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return na && nb && x < y + nb && y < x + na;
}

// Do two row-strided byte ranges share a byte?  Range X holds rows
// [x + i * stride, x + i * stride + width), i < rows.  With equal strides the
// answer is exact: rows i of A and j of B meet iff, for k = i - j,
// d - width_a < k * stride < d + width_b with d = b - a; so it is enough to
// test the smallest k above (d - width_a) / stride that is a possible i - j.
// Head-sliced views of one tensor (same stride, disjoint columns) therefore
// do not overlap.  Different strides fall back to the byte spans.
inline bool rows_overlap(const void* a, int64_t rows_a, int64_t stride_a, int64_t width_a, const void* b,
                         int64_t rows_b, int64_t stride_b, int64_t width_b) {
  if (rows_a < 1 || rows_b < 1 || width_a < 1 || width_b < 1) return false;
  const uint64_t span_a = uint64_t((rows_a - 1) * stride_a + width_a);
  const uint64_t span_b = uint64_t((rows_b - 1) * stride_b + width_b);
  if (!overlaps(a, span_a, b, span_b)) return false;
  if (stride_a != stride_b || width_a > stride_a || width_b > stride_b) return true;
  const int64_t S = stride_a;
  const int64_t d = int64_t(reinterpret_cast<uintptr_t>(b)) - int64_t(reinterpret_cast<uintptr_t>(a));
  const int64_t lo = d - width_a;                           // k * S must exceed lo
  int64_t k = (lo >= 0 ? lo / S : -((-lo + S - 1) / S)) + 1;  // floor(lo / S) + 1
  if (k < -(rows_b - 1)) k = -(rows_b - 1);
  return k <= rows_a - 1 && k * S < d + width_b;
}

// ---- unsigned division by a run-time constant -----------------------------
// floor(n / d) = (umulhi(n, m) + n) >> s for every n < 2^31, with
// s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1 (Granlund and
// Montgomery, "Division by invariant integers using multiplication", 1994).
struct FastDiv {
  uint32_t d, m, s;
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  uint32_t s = 0;
  while ((uint64_t(1) << s) < d) ++s;
  f.s = s;
  f.m = uint32_t(((uint64_t(1) << 32) * ((uint64_t(1) << s) - d)) / d + 1);
  return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return (__umulhi(n, f.m) + n) >> f.s;
}

// ---- bf16 packing -----------------------------------------------------------
__device__ __forceinline__ float bf16lo_to_f32(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Two fp32 -> packed bf16x2 (lo in bits 0..15), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace rkv
