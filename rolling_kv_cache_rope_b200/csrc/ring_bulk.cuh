// Ring inserts on the TMA bulk-copy engine: how an insert of whole frames is
// cut into pieces that go global -> shared memory -> ring slot, and the
// device steps that move one piece (used by ring_bulk_kernel).
#pragma once

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace rkv {

constexpr int kBulkStages = 6;                      // most pieces in flight per CTA
constexpr uint32_t kBulkStageBytes = 32768;         // largest piece
constexpr uint64_t kBulkWaitNs = 1000000000ull;     // default limit of one wait (1 s), then give up

// Pieces of an insert: the K pieces first, then the V pieces; within a
// tensor, frame by frame, each frame as groups of rpp whole rows (or, when one
// row exceeds a stage, as cpr chunks of each row).
struct RingBulkArgs {
  const uint8_t* src[2];
  uint8_t* dst[2];
  uint64_t src_row_stride;  // bytes between source rows
  uint64_t frame_bytes;     // bytes of one ring slot
  uint32_t row_bytes;       // H * D * 2
  uint32_t F;               // rows (tokens) per frame
  uint32_t rpp;             // rows per piece
  uint32_t cpr;             // pieces across one row (1 unless a row exceeds a stage)
  uint32_t chunk;           // bytes of each row a piece covers (row_bytes when cpr = 1)
  uint32_t ppf;             // pieces per frame = ceil(F / rpp) * cpr
  uint32_t half;            // pieces of one tensor = n_frames * ppf
  uint32_t total;           // pieces of the insert = 2 * half
  uint32_t stage_bytes;     // rpp * chunk
  uint32_t stages;          // pieces in flight per CTA, 2..kBulkStages
  uint32_t contiguous;      // source rows are back to back (one load per piece)
  RingPlan plan;            // destination slot of each frame
  int32_t* timeout_flag;    // set to 1 when a wait gives up
  uint64_t wait_ns;         // limit of one wait
  uint32_t stall;           // debug: CTA 0 declares 16 bytes more for its first piece than it loads
};

struct RingPiece {
  const uint8_t* src;
  uint8_t* dst;
  uint32_t which;           // 0 = K, 1 = V
  uint32_t frame;           // frame of the insert
  uint32_t row0;            // first row of the piece within its frame
  uint32_t rows, cols;      // rows, and bytes of each row
};

__device__ __forceinline__ RingPiece ring_piece(const RingBulkArgs& a, uint32_t p) {
  RingPiece pc;
  pc.which = p >= a.half ? 1u : 0u;
  const uint32_t q = p - pc.which * a.half;
  pc.frame = q / a.ppf;
  const uint32_t k = q - pc.frame * a.ppf;
  const uint32_t rg = k / a.cpr, cc = k - rg * a.cpr;
  pc.row0 = rg * a.rpp;
  const uint32_t col0 = cc * a.chunk;
  pc.rows = min(a.rpp, a.F - pc.row0);
  pc.cols = min(a.chunk, a.row_bytes - col0);
  const int32_t slot = ring_dst_slot(a.plan, pc.frame);
  pc.src = a.src[pc.which] + (uint64_t(pc.frame) * a.F + pc.row0) * a.src_row_stride + col0;
  pc.dst = a.dst[pc.which] + uint64_t(slot) * a.frame_bytes + uint64_t(pc.row0) * a.row_bytes + col0;
  return pc;
}

// Bounded wait (at most limit_ns) for the phase of `bar` with parity
// `parity` to complete.
__device__ __forceinline__ bool bulk_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_try_wait(bar, parity))
    if (ptx::globaltimer_ns() - t0 > limit_ns) return false;
  return true;
}

// Issue the bulk load(s) of piece pc into shared memory at dst, completing on
// the mbarrier at bar.  `extra` bytes are declared on top of what is loaded
// (0 except for stall injection, which makes the barrier never complete).
__device__ __forceinline__ void bulk_load_piece(const RingBulkArgs& a, const RingPiece& pc, uint32_t dst,
                                                uint32_t bar, uint32_t extra = 0) {
  ptx::mbar_expect_tx(bar, pc.rows * pc.cols + extra);
  if (a.contiguous) {
    ptx::bulk_load(dst, pc.src, pc.rows * pc.cols, bar);
  } else {
    for (uint32_t r = 0; r < pc.rows; ++r) ptx::bulk_load(dst + r * pc.cols, pc.src + r * a.src_row_stride, pc.cols, bar);
  }
}

// Store piece pc from shared memory at src into its ring slot (one bulk group).
__device__ __forceinline__ void bulk_store_piece(const RingPiece& pc, uint32_t src) {
  ptx::bulk_store(pc.dst, src, pc.rows * pc.cols);
  ptx::bulk_commit();
}

// One thread moves pieces first, first + G, first + 2G, ... (below end) of
// the insert through the `a.stages` stages at shared address smem0, piece i
// of the list in stage i % stages, i.e. phase (i / stages) & 1 of mbarrier
// full[i % stages] (initialised here).  When a wait gives up it sets
// a.timeout_flag, lets the loads still in flight land (bounded) and stops.
__device__ __forceinline__ void bulk_copy_pieces(const RingBulkArgs& a, uint32_t first, uint32_t end, uint32_t G,
                                                 uint32_t smem0, uint64_t* full) {
  const uint32_t n = end > first ? (end - first + G - 1) / G : 0u;
  for (uint32_t s = 0; s < a.stages; ++s) ptx::mbar_init(ptx::smem_u32(&full[s]), 1);
  ptx::fence_mbar_init();
  auto piece = [&](uint32_t i) { return ring_piece(a, first + i * G); };
  auto stage = [&](uint32_t i) { return smem0 + (i % a.stages) * a.stage_bytes; };
  auto bar = [&](uint32_t i) { return ptx::smem_u32(&full[i % a.stages]); };
  uint32_t issued = 0;
  for (; issued < n && issued < a.stages; ++issued)
    bulk_load_piece(a, piece(issued), stage(issued), bar(issued),
                    (a.stall && blockIdx.x == 0 && issued == 0) ? 16u : 0u);
  uint32_t i = 0;
  for (; i < n; ++i) {
    if (!bulk_wait(bar(i), (i / a.stages) & 1u, a.wait_ns)) {
      atomicExch(a.timeout_flag, 1);
      break;
    }
    bulk_store_piece(piece(i), stage(i));
    // refill the previous piece's stage once its store has read shared memory
    // (issued == i - 1 + stages here)
    if (i >= 1 && issued < n) {
      ptx::bulk_wait_read<1>();
      bulk_load_piece(a, piece(issued), stage(issued), bar(issued));
      ++issued;
    }
  }
  // after a wait gave up on piece i: let the loads still in flight, piece i's
  // included, land (bounded) before the CTA's shared memory is released
  // (issued <= i + stages, so these pieces use distinct stages)
  for (uint32_t j = i; j < issued; ++j) bulk_wait(bar(j), (j / a.stages) & 1u, a.wait_ns);
  ptx::bulk_wait_all();
}

// Piece geometry of an insert into a checked ring (timeout_flag left null,
// default wait limit, no stall).
inline rkv_status ring_bulk_geometry(const rkv_ring* ring, const void* k_new, const void* v_new,
                                     int64_t new_row_stride, int32_t n_frames, RingBulkArgs& a) {
  a.src[0] = static_cast<const uint8_t*>(k_new);
  a.src[1] = static_cast<const uint8_t*>(v_new);
  a.dst[0] = static_cast<uint8_t*>(ring->k);
  a.dst[1] = static_cast<uint8_t*>(ring->v);
  a.row_bytes = uint32_t(int64_t(ring->H) * ring->D * 2);
  a.src_row_stride = uint64_t(new_row_stride) * 2;
  a.F = uint32_t(ring->tokens_per_frame);
  a.frame_bytes = uint64_t(a.F) * a.row_bytes;
  if (a.row_bytes <= kBulkStageBytes) {
    a.rpp = kBulkStageBytes / a.row_bytes;
    if (a.rpp > a.F) a.rpp = a.F;
    a.cpr = 1;
    a.chunk = a.row_bytes;
  } else {
    a.rpp = 1;
    a.chunk = kBulkStageBytes;
    a.cpr = (a.row_bytes + kBulkStageBytes - 1) / kBulkStageBytes;
  }
  a.stage_bytes = a.rpp * a.chunk;
  a.stages = kBulkStages;
  const uint64_t ppf = uint64_t((a.F + a.rpp - 1) / a.rpp) * a.cpr;
  const uint64_t half = uint64_t(n_frames) * ppf;
  if (2 * half >= (uint64_t(1) << 31)) return fail(RKV_ERR_UNSUPPORTED, "insert too large for one launch");
  a.ppf = uint32_t(ppf);
  a.half = uint32_t(half);
  a.total = uint32_t(2 * half);
  a.contiguous = a.src_row_stride == a.row_bytes ? 1u : 0u;
  a.plan = ring_plan(ring);
  a.timeout_flag = nullptr;
  a.wait_ns = kBulkWaitNs;
  a.stall = 0;
  return RKV_OK;
}

}  // namespace rkv
