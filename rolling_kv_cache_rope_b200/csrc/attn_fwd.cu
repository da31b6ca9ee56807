// Fused 3D-RoPE + softmax attention for sm_100a (B200), variable-length
// sequences and frame-block-causal masking, one persistent launch.
//
// What it computes (per sequence s, head h):
//   O = softmax(mask(RoPE(Q) RoPE(K)^T * scale)) V
// Source: SDPA from a 23,400-token query window to a 32,760-token context,
// 12 heads, ~70% of compute ("A kernel-centric path to real-time video
// generation on Trainium", ai4snews summary, second paragraph); attention
// transposes folded into the attention kernel and a dedicated 3D-RoPE step
// ("Amazon and Reactor tune Trainium for real-time video generation", sections
// "Three problems for generic compilers" and "Results with the Neuron Kernel
// Interface"); the denoise and cache-update passes batched into one run
// ("Optimizing Real-Time Video Generation on Trainium Chips", item 8 "Model
// structure optimizations").
//
// Design: clusters of two CTAs on two SMs share every MMA (tcgen05
// cta_group::2, M = 256 query rows), 16 warps per CTA:
//   warps 0-3   softmax for Q sub-tile 0 (one TMEM lane = one query row each)
//   warps 4-7   softmax for Q sub-tile 1
//   warps 8-11  RoPE: rotate this CTA's Q rows and its half of each K tile in
//               shared memory right after TMA lands them
//   warp 12     TMA producer for Q and K;  warp 14  TMA producer for V
//   warp 13     allocates TMEM (both CTAs); in the leader CTA one lane issues
//               every tcgen05.mma for the pair
//   warp 15     tells the leader when this CTA's V half has landed
// A work unit is (sequence, head, 512 query rows); each CTA owns 256 rows as
// two 128-row sub-tiles.  A 2-CTA MMA splits its B operand by N between the
// two CTAs, so each CTA loads and rotates only 64 keys of every 128-key K tile
// and only 64 of the 128 columns of every V tile: shared-memory traffic per SM
// (operand reads, TMA writes, RoPE) halves against a one-CTA MMA, which is
// what bounds a 128x128 tile on one SM.  Q/K/V are read straight from
// token-major [L][H][128] tensors through 3-D TMA descriptors (head is a
// coordinate), so no transpose pass exists.  S = Q K^T (128x128 fp32 per CTA)
// and the running O of both sub-tiles live in TMEM (4 x 128 columns).
// Softmax reads S with tcgen05.ld, writes P as bf16 over the first 64 columns
// of the same S region, and the PV MMA takes P straight from TMEM.  While one
// softmax warpgroup works, the tensor cores run the other sub-tile's MMAs
// (ping-pong).  The running max is only moved (and O rescaled in TMEM) when it
// grows by more than 2^8; after a unit's first tile the exponentials are taken
// against the running max while the tile max is found, and redone in the rare
// case it has to move.  Operand readiness is reported to the leader with
// cluster-scope mbarrier arrives; the leader's commits are multicast to both
// CTAs.  No TMA load uses multicast.  Waiting threads sleep in mbarrier
// try_wait (suspend-time hint).  All waits are bounded: a stuck wait makes the
// CTA stop, records RKV_ERR_TIMEOUT in the workspace and frees TMEM.
// Tail of the persistent grid: when its last wave of units is at most half
// full, those units run as two halves over their key tiles, leave
// unnormalised O, running max and row sum in the workspace, and
// attn_combine_kernel merges each pair into the output.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <functional>
#include <mutex>
#include <queue>
#include <utility>
#include <vector>

#include "common.cuh"
#include "sm100_ptx.cuh"

namespace rkv {
rkv_status check_rope(const rkv_rope3d* rope, int32_t D);

namespace attn {

constexpr int kBM = 128;             // query rows per sub-tile (one TMEM lane each)
constexpr int kSub = 2;              // sub-tiles per CTA
constexpr int kCtaRows = kBM * kSub; // 256 query rows per CTA
constexpr int kUnitRows = 2 * kCtaRows;   // 512 query rows per CTA pair
constexpr int kBN = 128;             // keys per K/V tile (per pair)
constexpr int kHD = 128;             // head dim
constexpr int kStages = 4;           // K and V pipeline depth
constexpr int kQTileBytes = kBM * kHD * 2;     // 32 KB: 128 rows x 128 cols
constexpr int kQHalfBytes = kQTileBytes / 2;   // 128 rows x 64 cols
constexpr int kKRows = kBN / 2;                // keys of a K tile held by one CTA
constexpr int kKStageBytes = kKRows * kHD * 2; // 16 KB: 64 rows x 128 cols
constexpr int kKHalfBytes = kKStageBytes / 2;  // 64 rows x 64 cols
constexpr int kVStageBytes = kBN * 64 * 2;     // 16 KB: 128 rows x 64 cols
constexpr int kThreads = 16 * 32;
constexpr int kMaxClusters = 128;    // CTA pairs a launch can have (74 on a B200)
constexpr int kMaxSched = 4096;      // work items a host-built schedule can list
constexpr int kTabEntryBytes = 32;   // cos and sin of 4 consecutive rotary pairs
constexpr int kMaxTabEntries = 768;  // 24 KB of shared memory (cos array, then sin array)
constexpr float kRescaleLog2 = 8.0f; // move the running max only past 2^8 growth
// register split (setmaxnreg): two softmax warpgroups, RoPE, producers; the
// four shares add up to the 4 x 128 registers per thread the block launches with
constexpr int kRegSoftmax = 176, kRegRope = 80, kRegProducer = 80;
static_assert(2 * kRegSoftmax + kRegRope + kRegProducer == 4 * 128, "register split must match the launch");
// setmaxnreg.inc may only raise and .dec only lower a warp's count (128 at
// launch); a .dec above the current count is an illegal instruction
static_assert(kRegSoftmax >= 128 && kRegRope <= 128 && kRegProducer <= 128, "inc/dec directions of the split");

// shared-memory map (offsets from a 1024-byte aligned base; identical in both CTAs)
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kSub * kQTileBytes;
constexpr int kOffV = kOffK + kStages * kKStageBytes;
constexpr int kOffTab = kOffV + kStages * kVStageBytes;
constexpr int kOffBar = kOffTab + kMaxTabEntries * kTabEntryBytes;
constexpr int kBarBytes = 512;
constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;   // + alignment slack

// TMEM columns: S of sub-tile b at 128*b, O of sub-tile b at 256 + 128*b
__host__ __device__ constexpr uint32_t col_s(int b) { return 128u * uint32_t(b); }
__host__ __device__ constexpr uint32_t col_o(int b) { return 256u + 128u * uint32_t(b); }
constexpr uint32_t kTmemCols = 512;

struct SeqDev {
  CUtensorMap tq, tk, tv;
  uint8_t* o;
  int64_t o_stride_bytes;
  int32_t Lq, Lk, q_t0, k_t0, q_frame_offset, block_frames;
  uint32_t flags;
  int32_t n_qblocks;
  int32_t unit_begin;
  int64_t stats_row0;   // debug launches: first row of this sequence in row_stats
};

struct Params {
  SeqDev seq[RKV_MAX_SEQS];
  int32_t n_seqs, H;
  // work items: units [0, n_whole) whole, then each of the remaining
  // n_split units as two items over the first and second half of its key
  // tiles, whose partial results go to part_o / part_ml
  int32_t total_units, n_whole, n_split;
  float* part_o;     // [2 * n_split][kUnitRows][kHD] unnormalised O
  float* part_ml;    // [2 * n_split][kUnitRows][2] running max (log2 units) and row sum
  float scale_log2;
  int32_t grid_h, grid_w;
  int32_t t_lo, n_t;
  // RoPE table: entry e holds cos (and, tab_entries entries later, sin) of 4
  // consecutive global rotary pairs.  Axis a owns entries ax_tab[a] .. as
  // [chunk k of the axis][position]; chunk k covers global pairs
  // 4*(ax_chunk0[a] + k) .. +3 (pairs outside the axis hold cos 1, sin 0).
  int32_t ax_first[3], ax_count[3], ax_chunk0[3], ax_nch[3], ax_npos[3], ax_tab[3];
  int32_t tab_entries;
  // per 16-byte chunk g of a head (pairs 4g..4g+3): entry of position 0 on the
  // axis of its first pair (lo) and of its last pair (hi); axes; and which
  // of the 4 pairs take the hi axis (0 when the chunk lies on one axis)
  int32_t ch_base_lo[16], ch_base_hi[16];
  int8_t ch_ax_lo[16], ch_ax_hi[16];
  uint32_t F;
  FastDiv div_F, div_W;
  double log2_theta[3];   // frequency base per axis (t, h, w)
  int32_t* status;
  uint64_t timeout_ns;
  // debug launches only (attn_fwd_varlen_debug): per (row, head) mask record
  // [4] int32 or null, and the handoff to skip (RKV_DEBUG_STALL_*)
  int32_t* row_stats;
  uint32_t stall;
  // work-item schedule: 0 = round-robin (cluster c takes items c, c + C, ...);
  // 1 = cluster c takes items sched[sched_off[c] .. sched_off[c + 1]) in that
  // order (a longest-first assignment built on the host when items differ in
  // cost, e.g. frame-block-masked sequences)
  int32_t use_sched;
  uint16_t sched_off[kMaxClusters + 1];
  uint16_t sched[kMaxSched];
};

// barrier indices.  The first group is used in every CTA; the second only in
// the leader (rank 0), where both CTAs arrive on it.
enum : int {
  B_QFULL = 0, B_QFREE,
  B_KFULL, B_KFREE = B_KFULL + kStages,
  B_VFULL = B_KFREE + kStages, B_VFREE = B_VFULL + kStages,
  B_SFULL = B_VFREE + kStages, B_ODONE = B_SFULL + 2, B_FINAL = B_ODONE + 2,
  B_QREADY, B_KREADY, B_VREADY = B_KREADY + kStages, B_PFULL = B_VREADY + kStages, B_OFREE = B_PFULL + 2,
  B_COUNT = B_OFREE + 2
};
static_assert(B_COUNT * 8 + 16 <= kBarBytes, "barrier area");

struct Ctx {
  uint32_t bar0;         // shared address of barrier 0
  volatile int* abort;   // CTA-wide stop flag
  const Params* p;
};

__device__ __forceinline__ uint32_t bar(const Ctx& c, int i) { return c.bar0 + 8u * uint32_t(i); }

// Bounded wait on an mbarrier phase.  Returns false when the CTA is stopping
// (this or another thread gave up); the first thread to time out records the
// status word.
__device__ __forceinline__ bool wait_phase(const Ctx& c, uint32_t b, uint32_t parity, int where) {
  if (ptx::mbar_try_wait(b, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    // sleeps in hardware until the phase completes (at most ~20 us per try)
    if (ptx::mbar_try_wait_sleep(b, parity, 20000u)) return true;
    if (*c.abort) return false;
    if (ptx::globaltimer_ns() - t0 > c.p->timeout_ns) {
      *c.abort = 1;
      atomicCAS(c.p->status, 0, int(RKV_ERR_TIMEOUT) | (where << 8));
      return false;
    }
  }
}

// The MMA issuer's wait (on barriers the peer CTA also arrives on): one
// thread, on the critical path of every key tile, so it polls without the
// suspend hint (measured a few percent faster than sleeping there).  The
// handoffs through these barriers carry TMEM or async-proxy shared-memory
// data, ordered by tcgen05 / proxy fences, so the wait keeps the default
// (CTA) scope.  Bounded like wait_phase.
__device__ __forceinline__ bool wait_phase_cluster(const Ctx& c, uint32_t b, uint32_t parity, int where) {
  if (ptx::mbar_try_wait(b, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
    if (ptx::mbar_try_wait(b, parity)) return true;
    if (*c.abort) return false;
    if (ptx::globaltimer_ns() - t0 > c.p->timeout_ns) {
      *c.abort = 1;
      atomicCAS(c.p->status, 0, int(RKV_ERR_TIMEOUT) | (where << 8));
      return false;
    }
  }
}

// Warp-uniform variant for roles whose 32 lanes continue together.
__device__ __forceinline__ bool wait_warp(const Ctx& c, uint32_t b, uint32_t parity, int where) {
  const bool ok = wait_phase(c, b, parity, where);
  return __all_sync(0xffffffffu, ok);
}

// After the CTA stopped: wait (bounded, without looking at the stop flag) for
// a TMA load this thread issued to land, so no copy still writes this CTA's
// shared memory when it exits.
__device__ __forceinline__ void drain_phase(uint32_t b, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_try_wait(b, parity))
    if (ptx::globaltimer_ns() - t0 > limit_ns) return;
}

// The last `stages` loads issued into a ring of `stages` full barriers
// starting at `bar0` (iterations [it - stages, it)), plus, when q_phases > 0,
// the last load on barrier `qbar`: wait for each (bounded).  Out of line so
// the producers' main loops keep their register allocation.
__device__ __noinline__ void drain_loads(uint32_t bar0, uint32_t it, uint32_t stages, uint32_t qbar,
                                         uint32_t q_phases, uint64_t limit_ns) {
  if (q_phases > 0) drain_phase(qbar, (q_phases - 1) & 1u, limit_ns);
  for (uint32_t i = it > stages ? it - stages : 0u; i < it; ++i)
    drain_phase(bar0 + 8u * (i % stages), (i / stages) & 1u, limit_ns);
}

// Debug launches: an index check; a failed one records RKV_ERR_DEVICE_CHECK
// (and where) in the status word and returns false so the access is skipped.
__device__ __forceinline__ bool dev_check(const Params& p, bool ok, int where) {
  if (!ok) atomicCAS(p.status, 0, int(RKV_ERR_DEVICE_CHECK) | (where << 8));
  return ok;
}

// Debug launches: one query row's record of the keys that entered its
// softmax with a finite score (count, sum of key indices, 1 + largest index)
// and of the key tiles it processed.
struct RowStats {
  uint32_t count, sum, top, tiles;
};

// Count the scores of one thread's row of a 128-key tile (first key kbase)
// that are not -inf after masking: what the softmax actually sees.
__device__ __forceinline__ void row_stats_tile(const uint32_t (&sr)[4][32], uint32_t kbase, RowStats& st) {
#pragma unroll
  for (int ch = 0; ch < 4; ++ch)
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const bool vis = sr[ch][i] != 0xFF800000u;
      const uint32_t idx = kbase + uint32_t(ch * 32 + i);
      st.count += vis ? 1u : 0u;
      st.sum += vis ? idx : 0u;
      st.top = vis ? idx + 1u : st.top;
    }
  st.tiles += 1u;
}

// Work items of CTA pair `cluster` of `n_clusters`: how many, and the k-th.
__device__ __forceinline__ int items_of(const Params& p, int cluster, int n_clusters) {
  if (p.use_sched) return int(p.sched_off[cluster + 1]) - int(p.sched_off[cluster]);
  return cluster < p.total_units ? (p.total_units - cluster + n_clusters - 1) / n_clusters : 0;
}
__device__ __forceinline__ int item_at(const Params& p, int cluster, int n_clusters, int k) {
  return p.use_sched ? int(p.sched[p.sched_off[cluster] + k]) : cluster + k * n_clusters;
}

struct Unit {
  int si, head, qb, nkt;
  int kt0, kt1;   // key tiles [kt0, kt1) of this work item
  int part;       // -1: whole unit; else index of the item's partial-result slot
};

// Keys [0, limit) of the sequence are visible to query row `row`: the whole
// context without a mask, else every key frame up to the end of the query
// frame's block.  Host and device share this code (the host evaluates it for
// the tail split and for rkv_attn_mask_rows).
__host__ __device__ __forceinline__ int64_t row_kv_limit(const SeqDev& s, const Params& p, int row) {
  if (s.block_frames <= 0) return s.Lk;
  const int64_t qf = int64_t(s.q_frame_offset) + row / int64_t(p.F);
  const int64_t blk = qf / s.block_frames;
  const int64_t lim = (blk + 1) * s.block_frames * int64_t(p.F);
  return lim < s.Lk ? lim : s.Lk;
}

// Units (512 query rows, one per CTA pair) are numbered head-major within a
// sequence (all query blocks of head 0, then head 1, ...), so the clusters in
// flight at any time share the K/V tiles of one or two heads in L2.  Masked
// sequences list their query blocks from the most to the least visible keys.
__host__ __device__ __forceinline__ Unit decode_unit(const Params& p, int item) {
  Unit r;
  int u = item;
  r.part = -1;
  if (item >= p.n_whole) {   // half of a split unit
    r.part = item - p.n_whole;
    u = p.n_whole + (r.part >> 1);
  }
  int si = 0;
  while (si + 1 < p.n_seqs && u >= p.seq[si + 1].unit_begin) ++si;
  const SeqDev& s = p.seq[si];
  const int local = u - s.unit_begin;
  r.si = si;
  r.head = local / s.n_qblocks;
  const int ord = local - r.head * s.n_qblocks;
  r.qb = s.block_frames > 0 ? (s.n_qblocks - 1 - ord) : ord;
  int last = (r.qb + 1) * kUnitRows - 1;
  if (last > s.Lq - 1) last = s.Lq - 1;
  const int64_t kv = row_kv_limit(s, p, last);
  r.nkt = int((kv + kBN - 1) / kBN);
  r.kt0 = 0;
  r.kt1 = r.nkt;
  if (r.part >= 0) {
    if (r.part & 1) r.kt0 = r.nkt / 2;
    else r.kt1 = r.nkt / 2;
  }
  return r;
}

__device__ __forceinline__ int pick3(int a, int x, int y, int z) { return a == 0 ? x : (a == 1 ? y : z); }

// Rotate 4 rotary pairs (one 16-byte chunk, bf16) by the given cos / sin.
__device__ __forceinline__ uint4 rotate_chunk(uint4 v, float4 C, float4 S) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t a = w[2 * h], b = w[2 * h + 1];
    const float2 x0 = make_float2(bf16lo_to_f32(a), bf16lo_to_f32(b));
    const float2 x1 = make_float2(bf16hi_to_f32(a), bf16hi_to_f32(b));
    const float2 nx1 = make_float2(__uint_as_float((a & 0xFFFF0000u) ^ 0x80000000u),
                                   __uint_as_float((b & 0xFFFF0000u) ^ 0x80000000u));
    const float2 c = h ? make_float2(C.z, C.w) : make_float2(C.x, C.y);
    const float2 s = h ? make_float2(S.z, S.w) : make_float2(S.x, S.y);
    const float2 y0 = __ffma2_rn(x0, c, __fmul2_rn(nx1, s));   // x0 cos - x1 sin
    const float2 y1 = __ffma2_rn(x0, s, __fmul2_rn(x1, c));    // x0 sin + x1 cos
    o[2 * h] = pack_bf16x2(y0.x, y1.x);
    o[2 * h + 1] = pack_bf16x2(y0.y, y1.y);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// RoPE of one row (chunks [kG0, kG0 + kGN) of its 16) of a 128B-swizzled
// tile in shared memory, in place.  `row_addr` is the row's address in the
// tile's first 64-column half, `half_stride` the distance to the second half.
// Chunk g lies on the same axis for every thread of a warp, so branches are
// warp-uniform, and neighbouring rows read broadcast (t, h) or adjacent (w)
// table entries.  Loads for 4 chunks are issued before their arithmetic.
//
// A chunk that straddles two axes reads both axes' entries; each axis' table
// holds cos 1 / sin 0 for pairs outside the axis, so the chunk's cos and sin
// are the elementwise product of the two cos and the sum of the two sin.
//
// kPT/kPH > 0: the axis split is known at compile time (chunk -> axis folds to
// constants and only straddling chunks load twice); kPT == 0: read it from
// the parameters.
template <int kPT, int kPH, int kG0, int kGN>
__device__ __forceinline__ void rope_row(const Params& p, uint32_t tabC, uint32_t tabS, uint32_t row_addr,
                                         uint32_t half_stride, uint32_t swz, int pt, int ph, int pw) {
#pragma unroll
  for (int g0 = kG0; g0 < kG0 + kGN; g0 += 4) {
    uint4 v[4];
    float4 C[4], S[4];
    uint32_t addr[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int g = g0 + x;
      int alo, ahi;
      if (kPT > 0) {
        alo = (4 * g) < kPT ? 0 : ((4 * g) < kPT + kPH ? 1 : 2);
        ahi = (4 * g + 3) < kPT ? 0 : ((4 * g + 3) < kPT + kPH ? 1 : 2);
      } else {
        alo = p.ch_ax_lo[g];
        ahi = p.ch_ax_hi[g];
      }
      addr[x] = row_addr + uint32_t(g >> 3) * half_stride + ((uint32_t(g & 7) ^ swz) << 4);
      v[x] = ptx::lds128(addr[x]);
      const uint32_t e_lo = uint32_t(p.ch_base_lo[g] + pick3(alo, pt, ph, pw)) * 16u;
      C[x] = ptx::lds128f(tabC + e_lo);
      S[x] = ptx::lds128f(tabS + e_lo);
      if (alo != ahi) {
        const uint32_t e_hi = uint32_t(p.ch_base_hi[g] + pick3(ahi, pt, ph, pw)) * 16u;
        const float4 C2 = ptx::lds128f(tabC + e_hi);
        const float4 S2 = ptx::lds128f(tabS + e_hi);
        C[x] = make_float4(C[x].x * C2.x, C[x].y * C2.y, C[x].z * C2.z, C[x].w * C2.w);
        S[x] = make_float4(S[x].x + S2.x, S[x].y + S2.y, S[x].z + S2.z, S[x].w + S2.w);
      }
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) ptx::sts128(addr[x], rotate_chunk(v[x], C[x], S[x]));
  }
}

// Rotate 4 rotary pairs of the rotate-half layout: element e (0..3) of the
// 8-byte word pair a (first 64 columns) with element e of b (columns + 64).
__device__ __forceinline__ void rotate_half4(uint32_t& a0, uint32_t& a1, uint32_t& b0, uint32_t& b1, float4 C,
                                             float4 S) {
  const uint32_t aw[2] = {a0, a1}, bw[2] = {b0, b1};
  uint32_t ao[2], bo[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float2 x0 = make_float2(bf16lo_to_f32(aw[h]), bf16hi_to_f32(aw[h]));
    const float2 x1 = make_float2(bf16lo_to_f32(bw[h]), bf16hi_to_f32(bw[h]));
    const float2 nx1 = make_float2(-x1.x, -x1.y);
    const float2 c = h ? make_float2(C.z, C.w) : make_float2(C.x, C.y);
    const float2 s = h ? make_float2(S.z, S.w) : make_float2(S.x, S.y);
    const float2 y0 = __ffma2_rn(x0, c, __fmul2_rn(nx1, s));   // x0 cos - x1 sin
    const float2 y1 = __ffma2_rn(x0, s, __fmul2_rn(x1, c));    // x0 sin + x1 cos
    ao[h] = pack_bf16x2(y0.x, y0.y);
    bo[h] = pack_bf16x2(y1.x, y1.y);
  }
  a0 = ao[0]; a1 = ao[1]; b0 = bo[0]; b1 = bo[1];
}

// cos / sin of table chunk tc (rotary pairs 4tc..4tc+3) for a row at (pt, ph, pw).
template <int kPT, int kPH>
__device__ __forceinline__ void tab_chunk(const Params& p, uint32_t tabC, uint32_t tabS, int tc, int pt, int ph, int pw,
                                          float4& C, float4& S) {
  int alo, ahi;
  if (kPT > 0) {
    alo = (4 * tc) < kPT ? 0 : ((4 * tc) < kPT + kPH ? 1 : 2);
    ahi = (4 * tc + 3) < kPT ? 0 : ((4 * tc + 3) < kPT + kPH ? 1 : 2);
  } else {
    alo = p.ch_ax_lo[tc];
    ahi = p.ch_ax_hi[tc];
  }
  const uint32_t e_lo = uint32_t(p.ch_base_lo[tc] + pick3(alo, pt, ph, pw)) * 16u;
  C = ptx::lds128f(tabC + e_lo);
  S = ptx::lds128f(tabS + e_lo);
  if (alo != ahi) {
    const uint32_t e_hi = uint32_t(p.ch_base_hi[tc] + pick3(ahi, pt, ph, pw)) * 16u;
    const float4 C2 = ptx::lds128f(tabC + e_hi);
    const float4 S2 = ptx::lds128f(tabS + e_hi);
    C = make_float4(C.x * C2.x, C.y * C2.y, C.z * C2.z, C.w * C2.w);
    S = make_float4(S.x + S2.x, S.y + S2.y, S.z + S2.z, S.w + S2.w);
  }
}

// rope_row for the rotate-half layout: chunk pairs g in [kG0, kG0 + kGN)
// (g < 8): chunk g of the first 64 columns holds elements 8g..8g+7, chunk g of
// the second half the elements 64 later; pair 8g + e rotates the two
// elements e.  Table chunks 2g and 2g + 1 give the cos / sin of the 8 pairs.
template <int kPT, int kPH, int kG0, int kGN>
__device__ __forceinline__ void rope_row_half(const Params& p, uint32_t tabC, uint32_t tabS, uint32_t row_addr,
                                              uint32_t half_stride, uint32_t swz, int pt, int ph, int pw) {
#pragma unroll
  for (int g0 = kG0; g0 < kG0 + kGN; g0 += 2) {
    uint4 va[2], vb[2];
    uint32_t aa[2], ab[2];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const int g = g0 + x;
      aa[x] = row_addr + ((uint32_t(g) ^ swz) << 4);
      ab[x] = aa[x] + half_stride;
      va[x] = ptx::lds128(aa[x]);
      vb[x] = ptx::lds128(ab[x]);
    }
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const int g = g0 + x;
      float4 C0, S0, C1, S1;
      tab_chunk<kPT, kPH>(p, tabC, tabS, 2 * g, pt, ph, pw, C0, S0);
      tab_chunk<kPT, kPH>(p, tabC, tabS, 2 * g + 1, pt, ph, pw, C1, S1);
      rotate_half4(va[x].x, va[x].y, vb[x].x, vb[x].y, C0, S0);
      rotate_half4(va[x].z, va[x].w, vb[x].z, vb[x].w, C1, S1);
      ptx::sts128(aa[x], va[x]);
      ptx::sts128(ab[x], vb[x]);
    }
  }
}

// (t, h, w) table positions of token `row` of a sequence whose first frame is t0.
__device__ __forceinline__ void row_positions(const Params& p, int row, int t0, int& pt, int& ph, int& pw) {
  const uint32_t f = fdiv(uint32_t(row), p.div_F);
  const uint32_t in_f = uint32_t(row) - f * p.F;
  const uint32_t hh = fdiv(in_f, p.div_W);
  pt = t0 + int(f) - p.t_lo;
  ph = int(hh);
  pw = int(in_f - hh * uint32_t(p.grid_w));
}

// Three-input max (sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// P = exp2(S * scale_log2 - m_use) for one thread's row of S (in registers),
// written as bf16 over the first 64 TMEM columns of the S region; returns the
// row sum of the fp32 P.
__device__ __forceinline__ float exp_store_tile(const uint32_t (&sr)[4][32], uint32_t tS, float scale_log2,
                                                float m_use) {
  const float2 sc2 = make_float2(scale_log2, scale_log2);
  const float2 nm2 = make_float2(-m_use, -m_use);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 x =
          __ffma2_rn(make_float2(__uint_as_float(sr[ch][2 * i]), __uint_as_float(sr[ch][2 * i + 1])), sc2, nm2);
      const float2 pp = make_float2(ptx::ex2_approx(x.x), ptx::ex2_approx(x.y));  // exp2(-inf) = 0: hidden keys
      acc[i & 3] = __fadd2_rn(acc[i & 3], pp);
      pk[i] = pack_bf16x2(pp.x, pp.y);
    }
    ptx::tmem_st16(tS + ch * 16, pk);   // P (bf16) overwrites S columns 0..63
  }
  const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
  return (a01.x + a01.y) + (a23.x + a23.y);
}

// exp_store_tile that also returns the row max of the raw scores in
// mx: the exponentials use the running max m_use and are kept unless the
// tile's own max exceeds it by more than the rescale threshold.
__device__ __forceinline__ float exp_store_tile_max(const uint32_t (&sr)[4][32], uint32_t tS, float scale_log2,
                                                    float m_use, float& mx) {
  const float2 sc2 = make_float2(scale_log2, scale_log2);
  const float2 nm2 = make_float2(-m_use, -m_use);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float s0 = __uint_as_float(sr[ch][2 * i]), s1 = __uint_as_float(sr[ch][2 * i + 1]);
      mx4[i & 3] = max3f(mx4[i & 3], s0, s1);
      const float2 x = __ffma2_rn(make_float2(s0, s1), sc2, nm2);
      const float2 pp = make_float2(ptx::ex2_approx(x.x), ptx::ex2_approx(x.y));
      acc[i & 3] = __fadd2_rn(acc[i & 3], pp);
      pk[i] = pack_bf16x2(pp.x, pp.y);
    }
    ptx::tmem_st16(tS + ch * 16, pk);   // P (bf16) overwrites S columns 0..63
  }
  mx = fmaxf(max3f(mx4[0], mx4[1], mx4[2]), mx4[3]);
  const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
  return (a01.x + a01.y) + (a23.x + a23.y);
}

// K-major operand (rows of 128 bf16 in two 64-column 128B-swizzled halves):
// 8-row groups 1024 bytes apart; k-step kk starts 32 bytes further inside a
// half, or in the second half from kk = 4.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile) { return ptx::smem_desc_sw128(tile, 16, 1024); }
__device__ __forceinline__ uint64_t kstep_off(int kk, int half_bytes) {
  return uint64_t(((kk >> 2) * half_bytes + (kk & 3) * 32) >> 4);
}
// V half (128 keys x 64 columns, 128B-swizzled) as the MN-major B operand of
// PV: keys are K, 8-key groups 1024 bytes apart; k-step kk = 16 keys = 2048 B.
__device__ __forceinline__ uint64_t desc_v(uint32_t tile) { return ptx::smem_desc_sw128(tile, kVStageBytes, 1024); }

__device__ __forceinline__ void setmaxnreg_inc_softmax() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegSoftmax));
}
__device__ __forceinline__ void setmaxnreg_dec_rope() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegRope));
}
__device__ __forceinline__ void setmaxnreg_dec_producer() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegProducer));
}

// kPT/kPH: compile-time RoPE axis split (pairs on t and h), or 0/0 for any split.
// kDebug: the instantiation behind attn_fwd_varlen_debug, which also records
// per-row mask statistics and can skip one handoff (stall injection); the
// production instantiations compile neither.
template <int kPT, int kPH, bool kHalf, bool kDebug>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t rank = ptx::cluster_ctarank();   // 0 = leader of the pair
  const int cluster = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;
  const int n_items = items_of(p, cluster, n_clusters);   // work items of this CTA pair

  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + B_COUNT * 8);
  int* abort_flag = reinterpret_cast<int*>(smem + kOffBar + B_COUNT * 8 + 4);
  uint8_t* tab = smem + kOffTab;
  Ctx c;
  c.bar0 = sbase + kOffBar;
  c.abort = abort_flag;
  c.p = &p;
  // a leader-side barrier, addressed from either CTA
  auto lbar = [&](int i) { return ptx::mapa_shared(bar(c, i), 0); };

  if (tid == 0) {
    ptx::mbar_init(bar(c, B_QFULL), 1);
    ptx::mbar_init(bar(c, B_QFREE), 1);
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(bar(c, B_KFULL + s), 1);
      ptx::mbar_init(bar(c, B_KFREE + s), 1);
      ptx::mbar_init(bar(c, B_VFULL + s), 1);
      ptx::mbar_init(bar(c, B_VFREE + s), 1);
      ptx::mbar_init(bar(c, B_KREADY + s), 2);      // one arrive per CTA
      ptx::mbar_init(bar(c, B_VREADY + s), 2);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(bar(c, B_SFULL + b), 1);
      ptx::mbar_init(bar(c, B_ODONE + b), 1);
      ptx::mbar_init(bar(c, B_PFULL + b), 8);       // one arrive per softmax warp, both CTAs
      ptx::mbar_init(bar(c, B_OFREE + b), 8);
    }
    ptx::mbar_init(bar(c, B_QREADY), 2);
    ptx::mbar_init(bar(c, B_FINAL), 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 13) {
    ptx::tmem_alloc2(ptx::smem_u32(tmem_slot), kTmemCols);
    ptx::tmem_relinquish2();
  }
  // cos/sin table (fp64 sincos rounded to fp32) for every reachable position
  for (int e = tid; e < p.tab_entries; e += kThreads) {
    const int a = e < p.ax_tab[1] ? 0 : (e < p.ax_tab[2] ? 1 : 2);
    const int rel = e - p.ax_tab[a];
    const int k = rel / p.ax_npos[a];
    const int pos_i = rel - k * p.ax_npos[a];
    const int chunk = p.ax_chunk0[a] + k;
    const int pos = a == 0 ? p.t_lo + pos_i : pos_i;
    float cs[4], sn[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int i = 4 * chunk + j - p.ax_first[a];
      double sd = 0.0, cd = 1.0;
      if (i >= 0 && i < p.ax_count[a])
        sincos(double(pos) * exp2(-(double(i) / double(p.ax_count[a])) * p.log2_theta[a]), &sd, &cd);
      cs[j] = __double2float_rn(cd);
      sn[j] = __double2float_rn(sd);
    }
    *reinterpret_cast<float4*>(tab + e * 16) = make_float4(cs[0], cs[1], cs[2], cs[3]);
    *reinterpret_cast<float4*>(tab + (p.tab_entries + e) * 16) = make_float4(sn[0], sn[1], sn[2], sn[3]);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_arrive();   // both CTAs' barriers are initialised before any remote arrive
  ptx::cluster_wait();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const uint32_t sQ = sbase + kOffQ, sK = sbase + kOffK, sV = sbase + kOffV;
  const uint32_t sTabC = sbase + kOffTab, sTabS = sTabC + uint32_t(p.tab_entries) * 16u;

  if (warp < 8) {
    // ===================== softmax (two warpgroups) =====================
    setmaxnreg_inc_softmax();
    const int wg = warp >> 2;
    const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem_base + lane_off + col_s(wg);
    const uint32_t tO = tmem_base + lane_off + col_o(wg);
    const uint32_t pfull = lbar(B_PFULL + wg), ofree = lbar(B_OFREE + wg);
    const float scale_log2 = p.scale_log2;
    uint32_t g = 0, items = 0;
    for (int k = 0; k < n_items; ++k, ++items) {
      const Unit un = decode_unit(p, item_at(p, cluster, n_clusters, k));
      const SeqDev& s = p.seq[un.si];
      const int qrow = un.qb * kUnitRows + int(rank) * kCtaRows + wg * kBM + 32 * (warp & 3) + lane;
      const int64_t my_limit = row_kv_limit(s, p, qrow < s.Lq ? qrow : s.Lq - 1);
      float m = -INFINITY, l = 0.f;
      RowStats rs = {0u, 0u, 0u, 0u};
      for (int j = un.kt0; j < un.kt1; ++j, ++g) {
        if (!wait_warp(c, bar(c, B_SFULL + wg), g & 1u, 1)) goto done;
        ptx::tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) ptx::tmem_ld32(tS + ch * 32, sr[ch]);
        ptx::tmem_wait_ld();
        const int64_t kbase = int64_t(j) * kBN;
        const int lim = kbase + kBN > my_limit ? int(my_limit - kbase) : kBN;
        // partial tile for some row of the warp: hide keys at or past each
        // row's limit (the keys of a row's mask are a prefix)
        const bool masked = __any_sync(0xffffffffu, lim < kBN);
        const float m_old = m;
        float m_new, tile_sum;
        bool need;
        if (j > un.kt0 && !masked) {
          if constexpr (kDebug) row_stats_tile(sr, uint32_t(kbase), rs);
          // speculative: exponentials against the running max while the
          // tile max is found; redone (rarely) when the max has to move
          float mx;
          tile_sum = exp_store_tile_max(sr, tS, scale_log2, m, mx);
          m_new = fmaxf(m, mx * scale_log2);
          need = m_new > m + kRescaleLog2;
          if (__any_sync(0xffffffffu, need)) {
            if (need) m = m_new;
            tile_sum = exp_store_tile(sr, tS, scale_log2, m);
          }
        } else {
          if (masked) {
#pragma unroll
            for (int ch = 0; ch < 4; ++ch)
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (ch * 32 + i >= lim) sr[ch][i] = 0xFF800000u;   // -inf
          }
          if constexpr (kDebug) row_stats_tile(sr, uint32_t(kbase), rs);
          float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int ch = 0; ch < 4; ++ch)
#pragma unroll
            for (int i = 0; i < 32; i += 2)
              mx4[(i >> 1) & 3] = max3f(mx4[(i >> 1) & 3], __uint_as_float(sr[ch][i]), __uint_as_float(sr[ch][i + 1]));
          const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
          m_new = fmaxf(m, mx * scale_log2);
          need = m_new > m + kRescaleLog2;
          if (need) m = m_new;
          const float m_use = (m == -INFINITY) ? 0.f : m;
          tile_sum = exp_store_tile(sr, tS, scale_log2, m_use);
        }
        if (j > un.kt0 && __any_sync(0xffffffffu, need)) {
          // O holds tiles 0..j-1 scaled to the old max; S(j) was committed
          // after PV(j-1), so O is complete; rescale in TMEM (PV(j) is not
          // issued before P_FULL below)
          const float f = need ? ptx::ex2_approx(m_old - m_new) : 1.0f;
#pragma unroll 1
          for (int ch = 0; ch < 8; ++ch) {
            uint32_t r[16];
            ptx::tmem_ld16(tO + ch * 16, r);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
            ptx::tmem_st16(tO + ch * 16, r);
          }
          l *= f;
        }
        l += tile_sum;
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        bool skip = false;
        if constexpr (kDebug)   // stall injection: the peer CTA's first softmax warp withholds its first P
          skip = p.stall == RKV_DEBUG_STALL_P_FULL && cluster == 0 && rank == 1 && warp == 0 && g == 0;
        if (lane == 0 && !skip) ptx::mbar_arrive_cluster(pfull);
      }
      // epilogue: O / l -> bf16 -> global (row-major [Lq][H][128])
      if (!wait_warp(c, bar(c, B_ODONE + wg), items & 1u, 3)) goto done;
      ptx::tc_fence_after();
      {
        const float inv = l > 0.f ? 1.0f / l : 0.f;
        uint8_t* orow = s.o + int64_t(qrow) * s.o_stride_bytes + int64_t(un.head) * (kHD * 2);
        uint32_t r[4][32];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) ptx::tmem_ld32(tO + ch * 32, r[ch]);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(ofree);   // O may now be overwritten
        bool store_ok = true;
        if constexpr (kDebug) {
          store_ok = dev_check(p, un.head >= 0 && un.head < p.H, 40);
          if (un.part >= 0)
            store_ok &= dev_check(p, un.part < 2 * p.n_split, 41);
          else if (qrow < s.Lq)
            store_ok &= dev_check(p, qrow >= 0 && int64_t(qrow) * s.o_stride_bytes + int64_t(un.head + 1) * (kHD * 2) <=
                                             int64_t(s.Lq - 1) * s.o_stride_bytes + int64_t(p.H) * (kHD * 2), 42);
          if (p.row_stats && qrow < s.Lq) {
            // the two halves of a split unit add up into the same record
            int32_t* rec = p.row_stats + ((s.stats_row0 + qrow) * p.H + un.head) * 4;
            atomicAdd(reinterpret_cast<unsigned*>(rec + 0), rs.count);
            atomicAdd(reinterpret_cast<unsigned*>(rec + 1), rs.sum);
            atomicMax(reinterpret_cast<unsigned*>(rec + 2), rs.top);
            atomicAdd(reinterpret_cast<unsigned*>(rec + 3), rs.tiles);
          }
        }
        if (!store_ok) {
        } else if (un.part >= 0) {
          // half of a split unit: unnormalised O, running max and row sum
          // for the combine pass
          const int64_t prow = int64_t(un.part) * kUnitRows + int(rank) * kCtaRows + wg * kBM + 32 * (warp & 3) + lane;
          uint4* dst = reinterpret_cast<uint4*>(p.part_o + prow * kHD);
#pragma unroll
          for (int ch = 0; ch < 4; ++ch)
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[ch * 8 + i] = make_uint4(r[ch][4 * i], r[ch][4 * i + 1], r[ch][4 * i + 2], r[ch][4 * i + 3]);
          reinterpret_cast<float2*>(p.part_ml)[prow] = make_float2(m, l);
        } else if (qrow < s.Lq) {
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(r[ch][2 * i]) * inv, __uint_as_float(r[ch][2 * i + 1]) * inv);
            uint4* dst = reinterpret_cast<uint4*>(orow + ch * 64);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            dst[2] = make_uint4(pk[8], pk[9], pk[10], pk[11]);
            dst[3] = make_uint4(pk[12], pk[13], pk[14], pk[15]);
          }
        }
      }
    }
  } else if (warp < 12) {
    // ===================== RoPE warpgroup =====================
    setmaxnreg_dec_rope();
    const int rt = tid - 256;
    const uint32_t qready = lbar(B_QREADY);
    uint32_t it = 0, ul = 0;
    for (int k = 0; k < n_items; ++k, ++ul) {
      const Unit un = decode_unit(p, item_at(p, cluster, n_clusters, k));
      const SeqDev& s = p.seq[un.si];
      // Every RoPE warp reaches the named barrier below, whether its own wait
      // succeeded or not, and the barrier's AND takes the stop decision for
      // all four: a warp that left alone would hold the others at it.
      const bool okq = wait_warp(c, bar(c, B_QFULL), ul & 1u, 4);
      if (okq && (s.flags & RKV_ROPE_Q)) {
        // thread rt rotates row rt of both Q sub-tiles (all 16 chunks)
        for (int b = 0; b < kSub; ++b) {
          const int row = un.qb * kUnitRows + int(rank) * kCtaRows + b * kBM + rt;
          if (row < s.Lq) {
            int pt, ph, pw;
            row_positions(p, row, s.q_t0, pt, ph, pw);
            if (kHalf)
              rope_row_half<kPT, kPH, 0, 8>(p, sTabC, sTabS, sQ + uint32_t(b * kQTileBytes + rt * 128), kQHalfBytes,
                                            uint32_t(rt & 7), pt, ph, pw);
            else
              rope_row<kPT, kPH, 0, 16>(p, sTabC, sTabS, sQ + uint32_t(b * kQTileBytes + rt * 128), kQHalfBytes,
                                        uint32_t(rt & 7), pt, ph, pw);
          }
        }
      }
      ptx::fence_proxy_async_smem();
      if (!ptx::named_sync_and(1, 128, okq)) goto done;
      if (rt == 0) ptx::mbar_arrive_cluster(qready);
      for (int j = un.kt0; j < un.kt1; ++j, ++it) {
        const uint32_t st = it % kStages, n = it / kStages;
        const bool okk = wait_warp(c, bar(c, B_KFULL + st), n & 1u, 5);
        if (okk && (s.flags & RKV_ROPE_K)) {
          // this CTA's 64 keys of the tile: two threads per key row, warps
          // 8-9 take chunks 0-7 (first 64 columns), warps 10-11 chunks 8-15
          const int r = rt & 63;
          const int row = j * kBN + int(rank) * kKRows + r;
          if (row < s.Lk) {
            int pt, ph, pw;
            row_positions(p, row, s.k_t0, pt, ph, pw);
            const uint32_t ra = sK + st * kKStageBytes + uint32_t(r * 128);
            if (kHalf) {
              // rotate-half: chunk pairs 0-3 / 4-7 (both 64-column halves)
              if (rt < 64)
                rope_row_half<kPT, kPH, 0, 4>(p, sTabC, sTabS, ra, kKHalfBytes, uint32_t(r & 7), pt, ph, pw);
              else
                rope_row_half<kPT, kPH, 4, 4>(p, sTabC, sTabS, ra, kKHalfBytes, uint32_t(r & 7), pt, ph, pw);
            } else if (rt < 64) {
              rope_row<kPT, kPH, 0, 8>(p, sTabC, sTabS, ra, kKHalfBytes, uint32_t(r & 7), pt, ph, pw);
            } else {
              rope_row<kPT, kPH, 8, 8>(p, sTabC, sTabS, ra, kKHalfBytes, uint32_t(r & 7), pt, ph, pw);
            }
          }
        }
        ptx::fence_proxy_async_smem();
        if (!ptx::named_sync_and(1, 128, okk)) goto done;
        bool skip = false;
        if constexpr (kDebug)   // stall injection: the peer CTA withholds its first rotated K tile
          skip = p.stall == RKV_DEBUG_STALL_K_READY && cluster == 0 && rank == 1 && it == 0;
        if (rt == 0 && !skip) ptx::mbar_arrive_cluster(lbar(B_KREADY + st));
      }
    }
  } else {
    setmaxnreg_dec_producer();
    if (warp == 12 && lane == 0) {
      // ===================== TMA producer: Q and this CTA's K halves =====================
      for (int i = 0; i < p.n_seqs; ++i) {
        ptx::tma_prefetch_desc(&p.seq[i].tq);
        ptx::tma_prefetch_desc(&p.seq[i].tk);
      }
      uint32_t it = 0, ul = 0;
      bool ok = true;
      for (int k = 0; k < n_items; ++k, ++ul) {
        const Unit un = decode_unit(p, item_at(p, cluster, n_clusters, k));
        const SeqDev& s = p.seq[un.si];
        if (!wait_phase(c, bar(c, B_QFREE), (ul & 1u) ^ 1u, 6)) { ok = false; break; }
        if constexpr (kDebug) {
          dev_check(p, un.head >= 0 && un.head < p.H && un.qb >= 0 && int64_t(un.qb) * kUnitRows < s.Lq, 43);
          dev_check(p, un.kt0 >= 0 && un.kt0 < un.kt1 && int64_t(un.kt1 - 1) * kBN < s.Lk, 44);
        }
        ptx::mbar_expect_tx(bar(c, B_QFULL), kSub * kQTileBytes);
        for (int b = 0; b < kSub; ++b)
          for (int h2 = 0; h2 < 2; ++h2)
            ptx::tma_load_3d(sQ + b * kQTileBytes + h2 * kQHalfBytes, &s.tq, bar(c, B_QFULL), h2 * 64, un.head,
                             un.qb * kUnitRows + int(rank) * kCtaRows + b * kBM);
        for (int j = un.kt0; j < un.kt1; ++j, ++it) {
          const uint32_t st = it % kStages, n = it / kStages;
          if (!wait_phase(c, bar(c, B_KFREE + st), (n & 1u) ^ 1u, 7)) { ok = false; break; }
          ptx::mbar_expect_tx(bar(c, B_KFULL + st), kKStageBytes);
          for (int h2 = 0; h2 < 2; ++h2)
            ptx::tma_load_3d(sK + st * kKStageBytes + h2 * kKHalfBytes, &s.tk, bar(c, B_KFULL + st), h2 * 64,
                             un.head, j * kBN + int(rank) * kKRows);
        }
        if (!ok) { ++ul; break; }
      }
      // stopped early: let this thread's last Q load and K loads land
      if (!ok) drain_loads(bar(c, B_KFULL), it, kStages, bar(c, B_QFULL), ul, p.timeout_ns);
    } else if (warp == 14 && lane == 0) {
      // ===================== TMA producer: this CTA's V column half =====================
      for (int i = 0; i < p.n_seqs; ++i) ptx::tma_prefetch_desc(&p.seq[i].tv);
      uint32_t it = 0;
      bool ok = true;
      for (int k = 0; ok && k < n_items; ++k) {
        const Unit un = decode_unit(p, item_at(p, cluster, n_clusters, k));
        const SeqDev& s = p.seq[un.si];
        for (int j = un.kt0; j < un.kt1; ++j, ++it) {
          const uint32_t st = it % kStages, n = it / kStages;
          if (!wait_phase(c, bar(c, B_VFREE + st), (n & 1u) ^ 1u, 8)) { ok = false; break; }
          ptx::mbar_expect_tx(bar(c, B_VFULL + st), kVStageBytes);
          ptx::tma_load_3d(sV + st * kVStageBytes, &s.tv, bar(c, B_VFULL + st), int(rank) * 64, un.head, j * kBN);
        }
      }
      // stopped early: let this thread's last V loads land
      if (!ok) drain_loads(bar(c, B_VFULL), it, kStages, 0u, 0u, p.timeout_ns);
    } else if (warp == 15 && lane == 0) {
      // ===================== V landed -> tell the leader =====================
      uint32_t it = 0;
      bool ok = true;
      for (int k = 0; ok && k < n_items; ++k) {
        const Unit un = decode_unit(p, item_at(p, cluster, n_clusters, k));
        for (int j = un.kt0; j < un.kt1; ++j, ++it) {
          const uint32_t st = it % kStages, n = it / kStages;
          if (!wait_phase(c, bar(c, B_VFULL + st), n & 1u, 17)) { ok = false; break; }
          bool skip = false;
          if constexpr (kDebug)   // stall injection: the peer CTA withholds its first V tile
            skip = p.stall == RKV_DEBUG_STALL_V_READY && cluster == 0 && rank == 1 && it == 0;
          if (!skip) ptx::mbar_arrive_cluster(lbar(B_VREADY + st));
        }
      }
    } else if (warp == 13 && lane == 0 && rank == 0) {
      // ===================== MMA issuer (leader CTA, for the pair) =====================
      // Waits on smem handoffs (Q/K after RoPE, V after TMA) need no tcgen05
      // fence; waits on TMEM handoffs (P written with tcgen05.st, O read by
      // the epilogue) do.  Descriptors are built once; a k-step only moves
      // the 14-bit start-address field (addresses < 256 KB, so no carry).
      const uint32_t id_s = ptx::idesc_bf16_f32(2 * kBM, kBN, false);
      const uint32_t id_pv = ptx::idesc_bf16_f32(2 * kBM, kHD, true);
      const uint64_t dq0 = desc_kmajor(sQ), dq1 = desc_kmajor(sQ + kQTileBytes);
      constexpr uint16_t kBoth = 3;
      uint32_t it = 0, g = 0, ul = 0;
      bool ok = true;
      for (int k = 0; ok && k < n_items; ++k, ++ul) {
        const Unit un = decode_unit(p, item_at(p, cluster, n_clusters, k));
        if (!wait_phase_cluster(c, bar(c, B_QREADY), ul & 1u, 9)) { ok = false; break; }
        const int nk = un.kt1 - un.kt0;   // tiles of this item; j counts them from 0
        for (int j = 0; j < nk; ++j, ++it, ++g) {
          const uint32_t st = it % kStages, n = it / kStages;
          const uint64_t dk = desc_kmajor(sK + st * kKStageBytes);
          // K(j) is waited for only where S(j) needs it: PV of tile j - 1
          // below does not, so it is not held up by K(j)'s rotation
          if (j == 0 && !wait_phase_cluster(c, bar(c, B_KREADY + st), n & 1u, 10)) { ok = false; break; }
          if (j > 0) {
            const uint32_t sp = (it - 1) % kStages, np = (it - 1) / kStages;
            if (!wait_phase_cluster(c, bar(c, B_VREADY + sp), np & 1u, 11)) { ok = false; break; }
            const uint64_t dv = desc_v(sV + sp * kVStageBytes);
            for (int b = 0; b < kSub && ok; ++b) {
              if (!wait_phase_cluster(c, bar(c, B_PFULL + b), (g - 1) & 1u, 12)) { ok = false; break; }
              if (j == 1) {
                if (!wait_phase_cluster(c, bar(c, B_OFREE + b), (ul & 1u) ^ 1u, 13)) { ok = false; break; }
              }
              ptx::tc_fence_after();
              // O_b (+)= P_b(j-1) V(j-1): P from each CTA's TMEM, V split by column halves
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                ptx::mma2_ts(tmem_base + col_o(b), tmem_base + col_s(b) + 8 * kk, dv + uint64_t(kk * (2048 >> 4)),
                             id_pv, (j > 1 || kk > 0) ? 1u : 0u);
              if (b == 0 && !wait_phase_cluster(c, bar(c, B_KREADY + st), n & 1u, 10)) { ok = false; break; }
              // S_b(j) = Q_b K(j)^T: Q rows from each CTA, keys split 64 + 64
              const uint64_t dq = b ? dq1 : dq0;
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                ptx::mma2_ss(tmem_base + col_s(b), dq + kstep_off(kk, kQHalfBytes), dk + kstep_off(kk, kKHalfBytes),
                             id_s, kk > 0 ? 1u : 0u);
              ptx::mma2_commit_mc(bar(c, B_SFULL + b), kBoth);
            }
            if (!ok) break;
            ptx::mma2_commit_mc(bar(c, B_VFREE + sp), kBoth);
          } else {
            for (int b = 0; b < kSub; ++b) {
              const uint64_t dq = b ? dq1 : dq0;
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                ptx::mma2_ss(tmem_base + col_s(b), dq + kstep_off(kk, kQHalfBytes), dk + kstep_off(kk, kKHalfBytes),
                             id_s, kk > 0 ? 1u : 0u);
              ptx::mma2_commit_mc(bar(c, B_SFULL + b), kBoth);
            }
          }
          ptx::mma2_commit_mc(bar(c, B_KFREE + st), kBoth);
          if (j == nk - 1) ptx::mma2_commit_mc(bar(c, B_QFREE), kBoth);
        }
        if (!ok) break;
        // PV of the unit's last tile
        const uint32_t sp = (it - 1) % kStages, np = (it - 1) / kStages;
        if (!wait_phase_cluster(c, bar(c, B_VREADY + sp), np & 1u, 14)) { ok = false; break; }
        const uint64_t dv = desc_v(sV + sp * kVStageBytes);
        for (int b = 0; b < kSub && ok; ++b) {
          if (!wait_phase_cluster(c, bar(c, B_PFULL + b), (g - 1) & 1u, 15)) { ok = false; break; }
          if (nk == 1) {
            if (!wait_phase_cluster(c, bar(c, B_OFREE + b), (ul & 1u) ^ 1u, 16)) { ok = false; break; }
          }
          ptx::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            ptx::mma2_ts(tmem_base + col_o(b), tmem_base + col_s(b) + 8 * kk, dv + uint64_t(kk * (2048 >> 4)), id_pv,
                         (nk > 1 || kk > 0) ? 1u : 0u);
          ptx::mma2_commit_mc(bar(c, B_ODONE + b), kBoth);
        }
        if (!ok) break;
        ptx::mma2_commit_mc(bar(c, B_VFREE + sp), kBoth);
      }
      // every MMA of the pair is complete before either CTA frees TMEM
      ptx::mma2_commit_mc(bar(c, B_FINAL), kBoth);
    }
    if (warp == 13 && lane == 0) {
      const uint64_t t0 = ptx::globaltimer_ns();
      while (!ptx::mbar_try_wait(bar(c, B_FINAL), 0)) {
        if (ptx::globaltimer_ns() - t0 > c.p->timeout_ns) {
          *c.abort = 1;
          atomicCAS(c.p->status, 0, int(RKV_ERR_TIMEOUT) | (18 << 8));
          break;
        }
      }
    }
  }
done:
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_arrive();   // neither CTA leaves while its peer may still use its barriers or TMEM
  ptx::cluster_wait();
  if (warp == 13) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc2(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// [L][H][128] bf16 view, row stride in elements; box = box_rows rows x 1 head x 64 cols.
static rkv_status make_map(CUtensorMap* m, const void* ptr, int64_t L, int H, int64_t row_stride, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(RKV_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  cuuint64_t dims[3] = {cuuint64_t(kHD), cuuint64_t(H), cuuint64_t(L)};
  cuuint64_t strides[2] = {cuuint64_t(kHD * 2), cuuint64_t(row_stride * 2)};
  cuuint32_t box[3] = {64, 1, cuuint32_t(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(RKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return RKV_OK;
}

static int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

constexpr size_t kWorkspaceBytes = 256;
constexpr int kMaxSplit = 64;   // split units per launch at most
constexpr size_t kPartBytesPerItem = size_t(kUnitRows) * (kHD * 4 + 8);

// Combine the two halves of each split unit: per query row, with M the larger
// running max, O = (O_a 2^(m_a - M) + O_b 2^(m_b - M)) / (l_a 2^(m_a - M) +
// l_b 2^(m_b - M)) -> bf16 -> the output row (the same merge the online
// softmax applies between key tiles).
struct CombineUnit {
  uint8_t* o;
  int64_t o_stride_bytes;
  int32_t Lq, head, row0, pad;
};
struct CombineArgs {
  const float* part_o;
  const float2* part_ml;
  int32_t n_split;
  CombineUnit unit[kMaxSplit];
};

constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads) attn_combine_kernel(const __grid_constant__ CombineArgs a) {
  const int64_t idx = int64_t(blockIdx.x) * kCombineThreads + threadIdx.x;   // (unit, row, 8-column group)
  if (idx >= int64_t(a.n_split) * kUnitRows * (kHD / 8)) return;
  const int u = int(idx / (kUnitRows * (kHD / 8)));
  const int rem = int(idx - int64_t(u) * kUnitRows * (kHD / 8));
  const int row = rem / (kHD / 8), cg = rem % (kHD / 8);
  const CombineUnit& cu = a.unit[u];
  const int qrow = cu.row0 + row;
  if (qrow >= cu.Lq) return;
  const int64_t ra = int64_t(2 * u) * kUnitRows + row, rb = ra + kUnitRows;
  const float2 mla = a.part_ml[ra], mlb = a.part_ml[rb];
  const float mx = fmaxf(mla.x, mlb.x);
  const float wa = mla.y > 0.f ? exp2f(mla.x - mx) : 0.f;
  const float wb = mlb.y > 0.f ? exp2f(mlb.x - mx) : 0.f;
  const float lsum = mla.y * wa + mlb.y * wb;
  const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;
  const float4* oa = reinterpret_cast<const float4*>(a.part_o + ra * kHD + cg * 8);
  const float4* ob = reinterpret_cast<const float4*>(a.part_o + rb * kHD + cg * 8);
  const float4 a0 = oa[0], a1 = oa[1], b0 = ob[0], b1 = ob[1];
  const float ca = wa * inv, cb = wb * inv;
  uint4 out;
  out.x = pack_bf16x2(a0.x * ca + b0.x * cb, a0.y * ca + b0.y * cb);
  out.y = pack_bf16x2(a0.z * ca + b0.z * cb, a0.w * ca + b0.w * cb);
  out.z = pack_bf16x2(a1.x * ca + b1.x * cb, a1.y * ca + b1.y * cb);
  out.w = pack_bf16x2(a1.z * ca + b1.z * cb, a1.w * ca + b1.w * cb);
  *reinterpret_cast<uint4*>(cu.o + int64_t(qrow) * cu.o_stride_bytes + int64_t(cu.head) * (kHD * 2) + cg * 16) = out;
}

// Launch shape of the attention kernel (attributes set, cluster of 2) and the
// number of clusters that fit on the current device at once.
// Kernel instantiation: the pages' 22/21/21 split gets a compile-time axis
// map (either pair layout); other splits read it from the parameters.  Debug
// launches (adjacent pairs only) use the kDebug instantiations.
static void (*attn_kernel_for(bool default_split, bool half, bool debug))(Params) {
  if (debug) return default_split ? attn_fwd_kernel<22, 21, false, true> : attn_fwd_kernel<0, 0, false, true>;
  if (half) return default_split ? attn_fwd_kernel<22, 21, true, false> : attn_fwd_kernel<0, 0, true, false>;
  return default_split ? attn_fwd_kernel<22, 21, false, false> : attn_fwd_kernel<0, 0, false, false>;
}

static rkv_status attn_launch_shape(bool default_split, bool half, bool debug, cudaLaunchConfig_t& cfg,
                                    cudaLaunchAttribute* attr, const void*& kern_ptr, int& max_clusters) {
  auto kern = attn_kernel_for(default_split, half, debug);
  kern_ptr = reinterpret_cast<const void*>(kern);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attn_fwd_kernel)");
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(cluster size)");
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(2 * 74);
  max_clusters = 0;
  e = cudaOccupancyMaxActiveClusters(&max_clusters, kern_ptr, &cfg);
  if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters");
  if (max_clusters < 1) return fail(RKV_ERR_UNSUPPORTED, "no 2-CTA cluster of attn_fwd_kernel fits on this device");
  return RKV_OK;
}

// Units of the last, partly filled wave of the persistent grid that are run as
// two half-units (split over their key tiles) so the wave finishes in about
// half the time; 0 when the last wave is more than half full.
// Cost of a unit in the schedule: its key tiles plus a few tiles' worth of
// per-unit work (Q load and rotation, epilogue).
constexpr int kUnitOverheadTiles = 4;

// Longest-first assignment of the units to the CTA pairs when their costs
// differ: units in decreasing cost, each to the pair with the least work so
// far (greedy LPT, within a few percent of the optimal makespan here).
// Fills p.use_sched, p.sched_off, p.sched; returns false (round-robin) when
// every unit costs the same or the launch is too large for the table.
static bool build_schedule(Params& p, int64_t units, int max_clusters) {
  p.use_sched = 0;
  if (units < 2 || units > kMaxSched) return false;
  const int C = int(std::min<int64_t>(units, max_clusters));
  if (C > kMaxClusters) return false;
  const size_t n = size_t(units);
  std::vector<int> cost(n);
  bool same = true;
  for (int u = 0; u < int(units); ++u) {
    cost[size_t(u)] = decode_unit(p, u).nkt + kUnitOverheadTiles;
    same = same && cost[size_t(u)] == cost[0];
  }
  if (same) return false;
  std::vector<int> order(n);
  for (int u = 0; u < int(units); ++u) order[size_t(u)] = u;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[size_t(a)] > cost[size_t(b)]; });
  using Load = std::pair<int64_t, int>;   // (work so far, pair)
  std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
  for (int c = 0; c < C; ++c) heap.push({0, c});
  std::vector<std::vector<int>> lists(static_cast<size_t>(C));
  for (int u : order) {
    Load l = heap.top();
    heap.pop();
    lists[size_t(l.second)].push_back(u);
    heap.push({l.first + cost[size_t(u)], l.second});
  }
  int at = 0;
  for (int c = 0; c < C; ++c) {
    p.sched_off[c] = uint16_t(at);
    for (int u : lists[size_t(c)]) p.sched[at++] = uint16_t(u);
  }
  p.sched_off[C] = uint16_t(at);
  p.use_sched = 1;
  return true;
}

static int tail_split_units(int64_t units, int clusters) {
  if (clusters < 2 || units <= clusters) return 0;
  const int64_t rest = units % clusters;
  if (rest == 0 || 2 * rest > clusters) return 0;
  return int(std::min<int64_t>(rest, kMaxSplit));
}

}  // namespace attn
}  // namespace rkv

using namespace rkv;
using namespace rkv::attn;

extern "C" size_t attn_fwd_varlen_workspace_size(const rkv_attn_seq*, int32_t, int32_t, int32_t) {
  // the status word, plus room for the partial results of the largest tail
  // split this device can take (half of its concurrent CTA pairs)
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  const void* kern = nullptr;
  int clusters = 0;
  if (attn_launch_shape(true, false, false, cfg, attr, kern, clusters) != RKV_OK) {
    clear_error();
    return kWorkspaceBytes;
  }
  const int split = std::min(clusters / 2, kMaxSplit);
  return kWorkspaceBytes + size_t(2 * split) * kPartBytesPerItem;
}

static rkv_status validate_seq(const rkv_attn_seq& s, int i, int32_t H) {
  const int64_t row = int64_t(H) * kHD;
  if (!s.q || !s.k || !s.v || !s.o) return fail(RKV_ERR_INVALID_ARG, "seq %d: NULL tensor pointer", i);
  if (!aligned16(s.q) || !aligned16(s.k) || !aligned16(s.v) || !aligned16(s.o))
    return fail(RKV_ERR_INVALID_ARG, "seq %d: tensors must be 16-byte aligned", i);
  if (s.Lq < 1 || s.Lk < 1) return fail(RKV_ERR_INVALID_ARG, "seq %d: Lq and Lk must be >= 1", i);
  const int64_t st[4] = {s.q_stride, s.k_stride, s.v_stride, s.o_stride};
  for (int j = 0; j < 4; ++j) {
    if (st[j] < row) return fail(RKV_ERR_INVALID_ARG, "seq %d: row stride < H*D", i);
    if ((st[j] * 2) % 16) return fail(RKV_ERR_INVALID_ARG, "seq %d: rows must be 16-byte aligned", i);
    if (st[j] * 2 >= (int64_t(1) << 40)) return fail(RKV_ERR_INVALID_ARG, "seq %d: row stride too large", i);
  }
  if (s.block_frames < 0) return fail(RKV_ERR_INVALID_ARG, "seq %d: block_frames < 0", i);
  if (s.block_frames > 0 && s.q_frame_offset < 0)
    return fail(RKV_ERR_INVALID_ARG, "seq %d: q_frame_offset must be >= 0 with a mask", i);
  if (s.flags & ~(RKV_ROPE_Q | RKV_ROPE_K)) return fail(RKV_ERR_INVALID_ARG, "seq %d: unknown flags", i);
  if (s.reserved != 0) return fail(RKV_ERR_INVALID_ARG, "seq %d: reserved must be 0", i);
  return RKV_OK;
}

// Launch order of the sequences (longest context first: the cheapest units
// come last, which helps the static schedule) and each one's fields that
// number and size its work units; returns the number of units.  Fills p.F,
// p.n_seqs, p.H and p.n_whole (= all units, before any tail split).
static int64_t plan_units(const rkv_attn_seq* seqs, int32_t n_seqs, int32_t H, int64_t F, Params& p,
                          int* order) {
  for (int i = 0; i < n_seqs; ++i) order[i] = i;
  for (int i = 1; i < n_seqs; ++i)
    for (int j = i; j > 0 && seqs[order[j]].Lk > seqs[order[j - 1]].Lk; --j) std::swap(order[j], order[j - 1]);
  int64_t units = 0;
  int64_t row0[RKV_MAX_SEQS];
  for (int i = 0, r = 0; i < n_seqs; r += seqs[i].Lq, ++i) row0[i] = r;
  for (int oi = 0; oi < n_seqs; ++oi) {
    const rkv_attn_seq& s = seqs[order[oi]];
    SeqDev& d = p.seq[oi];
    d.stats_row0 = row0[order[oi]];
    d.Lq = s.Lq; d.Lk = s.Lk; d.q_t0 = s.q_t0; d.k_t0 = s.k_t0;
    d.q_frame_offset = s.q_frame_offset; d.block_frames = s.block_frames; d.flags = s.flags;
    d.n_qblocks = (s.Lq + kUnitRows - 1) / kUnitRows;   // 512-row blocks, one per CTA pair
    d.unit_begin = int32_t(units);
    units += int64_t(d.n_qblocks) * H;
  }
  p.F = uint32_t(F);
  p.n_seqs = n_seqs;
  p.H = H;
  p.n_whole = int32_t(units < INT32_MAX ? units : INT32_MAX);
  return units;
}

// Checks, plans and launches one attention call (dbg = null for the
// production entry points).
static rkv_status attn_launch(const rkv_attn_seq* seqs, int32_t n_seqs, int32_t H, int32_t D, float softmax_scale,
                              const rkv_rope3d* rope, void* workspace, size_t workspace_bytes,
                              const rkv_attn_debug* dbg, void* stream) {
  if (!seqs || n_seqs < 1) return fail(RKV_ERR_INVALID_ARG, "need at least one sequence");
  if (n_seqs > RKV_MAX_SEQS) return fail(RKV_ERR_UNSUPPORTED, "at most %d sequences per launch", RKV_MAX_SEQS);
  if (H < 1) return fail(RKV_ERR_INVALID_ARG, "H must be >= 1");
  if (D != kHD) return fail(RKV_ERR_INVALID_ARG, "head_dim D must be 128 (got %d)", D);
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return fail(RKV_ERR_INVALID_ARG, "softmax_scale must be > 0");
  rkv_status st = check_rope(rope, D);
  if (st != RKV_OK) return st;
  if (!workspace || workspace_bytes < kWorkspaceBytes || !aligned16(workspace))
    return fail(RKV_ERR_INVALID_ARG, "workspace must be >= %zu bytes and 16-byte aligned", kWorkspaceBytes);
  for (int i = 0; i < n_seqs; ++i) {
    st = validate_seq(seqs[i], i, H);
    if (st != RKV_OK) return st;
  }
  // outputs may not share a byte with any input or other output; row-strided
  // views of one tensor with disjoint heads (a launch over head slices) pass
  const int64_t row_bytes = int64_t(H) * kHD * 2;
  for (int i = 0; i < n_seqs; ++i) {
    const rkv_attn_seq& s = seqs[i];
    for (int j = 0; j < n_seqs; ++j) {
      const rkv_attn_seq& t = seqs[j];
      if (rows_overlap(s.o, s.Lq, s.o_stride * 2, row_bytes, t.q, t.Lq, t.q_stride * 2, row_bytes) ||
          rows_overlap(s.o, s.Lq, s.o_stride * 2, row_bytes, t.k, t.Lk, t.k_stride * 2, row_bytes) ||
          rows_overlap(s.o, s.Lq, s.o_stride * 2, row_bytes, t.v, t.Lk, t.v_stride * 2, row_bytes) ||
          (i != j && rows_overlap(s.o, s.Lq, s.o_stride * 2, row_bytes, t.o, t.Lq, t.o_stride * 2, row_bytes)))
        return fail(RKV_ERR_INVALID_ARG, "seq %d: output overlaps an input or another output", i);
    }
  }

  Params p;
  memset(&p, 0, sizeof(p));
  const int64_t F = int64_t(rope->grid_h) * rope->grid_w;
  int order[RKV_MAX_SEQS];
  const int64_t units = plan_units(seqs, n_seqs, H, F, p, order);

  int64_t t_lo = INT64_MAX, t_hi = INT64_MIN;
  for (int oi = 0; oi < n_seqs; ++oi) {
    const rkv_attn_seq& s = seqs[order[oi]];
    SeqDev& d = p.seq[oi];
    if ((st = make_map(&d.tq, s.q, s.Lq, H, s.q_stride, kBM)) != RKV_OK) return st;
    if ((st = make_map(&d.tk, s.k, s.Lk, H, s.k_stride, kKRows)) != RKV_OK) return st;
    if ((st = make_map(&d.tv, s.v, s.Lk, H, s.v_stride, kBN)) != RKV_OK) return st;
    d.o = static_cast<uint8_t*>(s.o);
    d.o_stride_bytes = s.o_stride * 2;
    if (s.flags & RKV_ROPE_Q) {
      t_lo = std::min<int64_t>(t_lo, s.q_t0);
      t_hi = std::max<int64_t>(t_hi, int64_t(s.q_t0) + (s.Lq - 1) / F);
    }
    if (s.flags & RKV_ROPE_K) {
      t_lo = std::min<int64_t>(t_lo, s.k_t0);
      t_hi = std::max<int64_t>(t_hi, int64_t(s.k_t0) + (s.Lk - 1) / F);
    }
  }
  if (units >= (int64_t(1) << 31)) return fail(RKV_ERR_UNSUPPORTED, "too many work units");
  if (t_lo == INT64_MAX) { t_lo = 0; t_hi = -1; }
  const int64_t n_t = t_hi - t_lo + 1;
  const int32_t pairs[3] = {rope->pairs_t, rope->pairs_h, rope->pairs_w};
  for (int a = 0; a < 3; ++a)
    if (pairs[a] < 4) return fail(RKV_ERR_UNSUPPORTED, "fused RoPE needs >= 4 rotary pairs per axis");
  const int64_t npos[3] = {n_t, rope->grid_h, rope->grid_w};
  int64_t entries = 0;
  int32_t first = 0;
  for (int a = 0; a < 3; ++a) {
    p.ax_first[a] = first;
    p.ax_count[a] = pairs[a];
    p.ax_chunk0[a] = first / 4;
    p.ax_nch[a] = (first + pairs[a] - 1) / 4 - first / 4 + 1;
    p.ax_npos[a] = int32_t(std::max<int64_t>(npos[a], 1));
    p.ax_tab[a] = int32_t(std::min<int64_t>(entries, INT32_MAX));
    entries += int64_t(p.ax_npos[a]) * p.ax_nch[a];
    first += pairs[a];
  }
  if (entries > kMaxTabEntries)
    return fail(RKV_ERR_UNSUPPORTED, "RoPE positions need %lld cos/sin table entries (max %d)", (long long)entries,
                kMaxTabEntries);
  auto axis_of_pair = [&](int pr) { return pr < p.ax_first[1] ? 0 : (pr < p.ax_first[2] ? 1 : 2); };
  for (int g = 0; g < 16; ++g) {
    const int alo = axis_of_pair(4 * g), ahi = axis_of_pair(4 * g + 3);
    p.ch_ax_lo[g] = int8_t(alo);
    p.ch_ax_hi[g] = int8_t(ahi);
    p.ch_base_lo[g] = p.ax_tab[alo] + (g - p.ax_chunk0[alo]) * p.ax_npos[alo];
    p.ch_base_hi[g] = p.ax_tab[ahi] + (g - p.ax_chunk0[ahi]) * p.ax_npos[ahi];
  }
  p.n_seqs = n_seqs;
  p.H = H;
  p.scale_log2 = float(double(softmax_scale) * 1.4426950408889634);
  p.grid_h = rope->grid_h; p.grid_w = rope->grid_w;
  p.t_lo = int32_t(t_lo); p.n_t = int32_t(n_t);
  p.tab_entries = int32_t(entries);
  p.F = uint32_t(F);
  p.div_F = make_fastdiv(uint32_t(F));
  p.div_W = make_fastdiv(uint32_t(rope->grid_w));
  p.log2_theta[0] = log2(double(rope->theta));
  p.log2_theta[1] = log2(double(rope->theta_h != 0.0f ? rope->theta_h : rope->theta));
  p.log2_theta[2] = log2(double(rope->theta_w != 0.0f ? rope->theta_w : rope->theta));
  p.status = static_cast<int32_t*>(workspace);
  p.timeout_ns = 2000000000ull;
  if (dbg) {   // checked by attn_fwd_varlen_debug
    if (dbg->timeout_us > 0) p.timeout_ns = uint64_t(dbg->timeout_us) * 1000ull;
    p.row_stats = dbg->row_stats;
    p.stall = dbg->stall;
  }

  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // the 22/21/21 split of the pages' 128-dim heads gets its own instantiation
  const bool default_split = rope->pairs_t == 22 && rope->pairs_h == 21 && rope->pairs_w == 21;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  const void* kern = nullptr;
  int max_clusters = 0;
  const bool half = rope->layout == RKV_ROPE_HALF;
  if ((st = attn_launch_shape(default_split, half, dbg != nullptr, cfg, attr, kern, max_clusters)) != RKV_OK)
    return st;
  cfg.stream = cs;

  // Units of different cost (frame-block-masked sequences, or sequences of
  // different lengths in one launch) get a longest-first schedule; units of
  // one cost keep round-robin with the tail split below.
  const bool sched = build_schedule(p, units, max_clusters);
  // tail split: the last n_split units run as two half-units each when the
  // workspace can hold their partial results and every such unit has >= 2
  // key tiles
  int n_split = sched ? 0 : tail_split_units(units, max_clusters);
  if (workspace_bytes < kWorkspaceBytes + size_t(2 * n_split) * kPartBytesPerItem) n_split = 0;
  CombineArgs ca;
  memset(&ca, 0, sizeof(ca));
  for (int k = 0; k < n_split; ++k) {
    const int64_t u = units - n_split + k;
    int si = 0;
    while (si + 1 < n_seqs && u >= p.seq[si + 1].unit_begin) ++si;
    const SeqDev& d = p.seq[si];
    const int64_t local = u - d.unit_begin;
    const int head = int(local / d.n_qblocks);
    const int ord = int(local - int64_t(head) * d.n_qblocks);
    const int qb = d.block_frames > 0 ? (d.n_qblocks - 1 - ord) : ord;
    int64_t last = int64_t(qb + 1) * kUnitRows - 1;
    if (last > d.Lq - 1) last = d.Lq - 1;
    const int64_t kv = row_kv_limit(d, p, int(last));
    if ((kv + kBN - 1) / kBN < 2) { n_split = 0; break; }
    ca.unit[k].o = d.o;
    ca.unit[k].o_stride_bytes = d.o_stride_bytes;
    ca.unit[k].Lq = d.Lq;
    ca.unit[k].head = head;
    ca.unit[k].row0 = qb * kUnitRows;
  }
  ca.n_split = n_split;
  p.n_whole = int32_t(units - n_split);
  p.n_split = n_split;
  p.total_units = int32_t(units + n_split);
  p.part_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWorkspaceBytes);
  p.part_ml = p.part_o + size_t(2 * n_split) * kUnitRows * kHD;
  ca.part_o = p.part_o;
  ca.part_ml = reinterpret_cast<const float2*>(p.part_ml);

  cudaError_t e = cudaMemsetAsync(workspace, 0, kWorkspaceBytes, cs);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(workspace)");
  if (p.row_stats) {
    int64_t rows = 0;
    for (int i = 0; i < n_seqs; ++i) rows += seqs[i].Lq;
    e = cudaMemsetAsync(p.row_stats, 0, size_t(rows) * H * 4 * sizeof(int32_t), cs);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(row_stats)");
  }
  // one CTA pair per pair of SMs that can hold it (persistent)
  cfg.gridDim = dim3(uint32_t(2 * std::min<int64_t>(p.total_units, max_clusters)));
  e = cudaLaunchKernelEx(&cfg, attn_kernel_for(default_split, half, dbg != nullptr), p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attn_fwd_kernel launch");
  if (n_split > 0) {
    const int64_t threads = int64_t(n_split) * kUnitRows * (kHD / 8);
    attn_combine_kernel<<<uint32_t((threads + kCombineThreads - 1) / kCombineThreads), kCombineThreads, 0, cs>>>(ca);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "attn_combine_kernel launch");
  }
  return RKV_OK;
}

extern "C" rkv_status attn_fwd_varlen(const rkv_attn_seq* seqs, int32_t n_seqs, int32_t H, int32_t D,
                                      float softmax_scale, const rkv_rope3d* rope, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("attn_fwd_varlen");
  clear_error();
  return attn_launch(seqs, n_seqs, H, D, softmax_scale, rope, workspace, workspace_bytes, nullptr, stream);
}

extern "C" rkv_status attn_fwd_varlen_debug(const rkv_attn_seq* seqs, int32_t n_seqs, int32_t H, int32_t D,
                                            float softmax_scale, const rkv_rope3d* rope, void* workspace,
                                            size_t workspace_bytes, const rkv_attn_debug* dbg, void* stream) {
  NvtxRange nvtx_range("attn_fwd_varlen_debug");
  clear_error();
  if (!dbg) return fail(RKV_ERR_INVALID_ARG, "debug settings are NULL");
  if (dbg->stall > RKV_DEBUG_STALL_P_FULL) return fail(RKV_ERR_INVALID_ARG, "unknown debug stall %u", dbg->stall);
  if (dbg->row_stats && !aligned16(dbg->row_stats)) return fail(RKV_ERR_INVALID_ARG, "row_stats must be 16-byte aligned");
  if (rope && rope->layout != RKV_ROPE_ADJACENT)
    return fail(RKV_ERR_UNSUPPORTED, "debug launches support the adjacent RoPE pair layout only");
  return attn_launch(seqs, n_seqs, H, D, softmax_scale, rope, workspace, workspace_bytes, dbg, stream);
}

extern "C" rkv_status rkv_attn_mask_rows(const rkv_attn_seq* seqs, int32_t n_seqs, int32_t H,
                                         const rkv_rope3d* rope, int64_t* row_limit, int32_t* unit_tiles,
                                         int64_t* n_units) {
  NvtxRange nvtx_range("rkv_attn_mask_rows");
  clear_error();
  if (!seqs || n_seqs < 1) return fail(RKV_ERR_INVALID_ARG, "need at least one sequence");
  if (n_seqs > RKV_MAX_SEQS) return fail(RKV_ERR_UNSUPPORTED, "at most %d sequences per launch", RKV_MAX_SEQS);
  if (H < 1) return fail(RKV_ERR_INVALID_ARG, "H must be >= 1");
  rkv_status st = check_rope(rope, kHD);
  if (st != RKV_OK) return st;
  if (!row_limit) return fail(RKV_ERR_INVALID_ARG, "row_limit is NULL");
  for (int i = 0; i < n_seqs; ++i) {
    const rkv_attn_seq& s = seqs[i];
    if (s.Lq < 1 || s.Lk < 1) return fail(RKV_ERR_INVALID_ARG, "seq %d: Lq and Lk must be >= 1", i);
    if (s.block_frames < 0) return fail(RKV_ERR_INVALID_ARG, "seq %d: block_frames < 0", i);
    if (s.block_frames > 0 && s.q_frame_offset < 0)
      return fail(RKV_ERR_INVALID_ARG, "seq %d: q_frame_offset must be >= 0 with a mask", i);
  }
  Params p;
  memset(&p, 0, sizeof(p));
  int order[RKV_MAX_SEQS], where[RKV_MAX_SEQS];
  const int64_t units = plan_units(seqs, n_seqs, H, int64_t(rope->grid_h) * rope->grid_w, p, order);
  if (units >= (int64_t(1) << 31)) return fail(RKV_ERR_UNSUPPORTED, "too many work units");
  for (int oi = 0; oi < n_seqs; ++oi) where[order[oi]] = oi;
  int64_t off = 0;
  for (int i = 0; i < n_seqs; ++i) {
    const SeqDev& d = p.seq[where[i]];
    for (int r = 0; r < d.Lq; ++r) row_limit[off + r] = row_kv_limit(d, p, r);
    off += d.Lq;
  }
  if (unit_tiles) {
    for (int64_t u = 0; u < units; ++u) {
      const Unit un = decode_unit(p, int(u));
      unit_tiles[4 * u + 0] = order[un.si];
      unit_tiles[4 * u + 1] = un.head;
      unit_tiles[4 * u + 2] = un.qb;
      unit_tiles[4 * u + 3] = un.nkt;
    }
  }
  if (n_units) *n_units = units;
  return RKV_OK;
}

extern "C" rkv_status rkv_attn_status(void* workspace, void* stream) {
  NvtxRange nvtx_range("rkv_attn_status");
  clear_error();
  if (!workspace) return fail(RKV_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, cs);
  if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) return cuda_fail(e, "reading the attention status word");
  if (word == 0) return RKV_OK;
  e = cudaMemsetAsync(workspace, 0, sizeof(word), cs);
  if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the attention status word");
  if ((word & 0xff) == RKV_ERR_DEVICE_CHECK)
    return fail(RKV_ERR_DEVICE_CHECK, "attention debug launch: device-side index check %d failed", word >> 8);
  return fail(rkv_status(word & 0xff), "attention kernel stopped: bounded wait %d timed out", word >> 8);
}

// ---------------------------------------------------------------------------
// attn_fwd_varlen_noalloc: the same launch, with the workspace taken from a
// fixed device array inside this library instead of caller memory.  For
// callers that cannot allocate device memory themselves.
// ---------------------------------------------------------------------------
namespace rkv {
namespace attn {

constexpr size_t kNoAllocScratchBytes = 256;  // the whole fixed scratch
static_assert(kWorkspaceBytes <= kNoAllocScratchBytes, "workspace outgrew the fixed scratch");
constexpr int kMaxDevices = 64;

// Every GPU that loads librkv.so holds this array until the process exits.
// Host code must not pass its name to a kernel: on the host it is only a
// stand-in; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[kMaxDevices];

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached.
static rkv_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(RKV_ERR_UNSUPPORTED, "device index %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc attention scratch)");
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return RKV_OK;
}

}  // namespace attn
}  // namespace rkv

extern "C" rkv_status attn_fwd_varlen_noalloc(const rkv_attn_seq* seqs, int32_t n_seqs, int32_t H, int32_t D,
                                              float softmax_scale, const rkv_rope3d* rope, void* stream) {
  NvtxRange nvtx_range("attn_fwd_varlen_noalloc");
  clear_error();
  // the launch needs kWorkspaceBytes at least; with no room for partial
  // results it runs without the tail split
  const size_t need = kWorkspaceBytes;
  if (need > kNoAllocScratchBytes)
    return fail(RKV_ERR_UNSUPPORTED, "this launch needs %zu bytes of scratch; the no-alloc entry point has %zu",
                need, kNoAllocScratchBytes);
  void* ws = nullptr;
  rkv_status st = noalloc_scratch(&ws);
  if (st != RKV_OK) return st;
  return attn_launch(seqs, n_seqs, H, D, softmax_scale, rope, ws, kNoAllocScratchBytes, nullptr, stream);
}

extern "C" rkv_status rkv_attn_noalloc_status(void* stream) {
  NvtxRange nvtx_range("rkv_attn_noalloc_status");
  clear_error();
  void* ws = nullptr;
  rkv_status st = noalloc_scratch(&ws);
  if (st != RKV_OK) return st;
  return rkv_attn_status(ws, stream);
}
