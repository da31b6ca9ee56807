// Standalone 3D rotary position embedding over (t, h, w).
//
// Source: "Amazon and Reactor tune Trainium for real-time video generation",
// section "Three problems for generic compilers" (video RoPE rotates by height,
// width and time; generic compilation turns it into many tiny transfers) and
// "Optimizing Real-Time Video Generation on Trainium Chips", item 6 "Neuron
// Kernel Interface" (a dedicated 3D-RoPE kernel).  Formula: see rkv.h.
//
// Design: the op reads and writes every element once, so it is HBM-bound.
// Each CTA owns a contiguous block of rows; it first builds, in shared memory,
// the cos/sin table for the positions its rows can reach (fp64 sincos, split
// into an fp32 hi + lo pair), then streams 16-byte chunks (4 rotary pairs)
// with four chunks in flight per thread.  The rotation uses fp32 FMA; when the
// result is small against the inputs (cancellation, ~1e-4 of outputs) it is
// recomputed with error-free transforms so every output rounds to within one
// bf16 ulp of the exactly rounded value.
//
// Adjacent pairs (rope3d_adj_kernel): every thread keeps one 16-byte chunk
// position of a row (so its four pairs, their axes and table columns are
// fixed) and walks down the CTA's rows; the table is chunk-major (cos and sin
// of 4 consecutive pairs at one position, 16 bytes each), so a chunk reads 32
// bytes of table, and the exact path is out of line.  A chunk whose pairs lie
// on two or three axes reads per-row entries, so every chunk takes the same
// path.  One launch covers up to RKV_ROPE_BATCH_MAX tensors
// (rope3d_apply_batch), CTAs shared out by rows.  Rotate-half pairs
// (rope3d_half_kernel) keep the per-pair table and launch per tensor.
//
// Rotated ring insert, adjacent pairs (ring_rope_kernel): one CTA per SM; one
// thread moves V on the TMA bulk-copy engine exactly as kvcache_ring_update
// does, the other warps build the table and rotate K into the ring, so the
// table build and the rotation run under V's copy.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "ring_bulk.cuh"
#include "sm100_ptx.cuh"

namespace rkv {

struct RopeArgs {
  const uint8_t* x;        // tensor to rotate
  uint8_t* y;              // its destination (rows, or ring slots in ring mode)
  const uint8_t* x2;       // ring mode: tensor copied without rotation (V)
  uint8_t* y2;
  int64_t x_stride_bytes, y_stride_bytes;
  uint64_t slot_bytes;     // ring mode: bytes of one ring slot (one frame)
  RingPlan ring;           // ring mode: destination slot of each frame
  uint32_t L;
  uint32_t cpr;            // 16-byte chunks per row = H * 16
  uint32_t cph;            // rotate-half chunk pairs per row = H * 8
  uint32_t rows_per_cta;
  uint32_t F;              // tokens per frame
  int32_t t0;
  int32_t grid_h, grid_w;
  int32_t pt, ph, pw;      // rotary pairs per axis
  double omega[64];        // frequency of rotary pair j: theta_a^(-i/count_a), i its index on axis a
  FastDiv div_F, div_W, div_cpr, div_cph;
  // adjacent layout: axis a owns rotary pairs [ax_first[a], + ax_count[a]),
  // i.e. 16-byte chunks [ax_chunk0[a], + ax_nch[a]).  Chunk g's four pairs lie
  // on one axis, ch_axis[g], or on two or three (ch_axis[g] = -1): such a
  // chunk reads per-row table entries, region ch_multi[g] of n_multi
  int32_t ax_first[3], ax_count[3], ax_chunk0[3], ax_nch[3];
  int8_t ch_axis[16], ch_multi[16];
  int32_t n_multi;
};

// threads per CTA (rotate-half kernel): the standalone op runs one 1024-thread
// CTA per SM (each cos/sin table serves more rows); the ring insert, a short
// launch with a V copy beside it, keeps four 256-thread CTAs per SM
template <bool kRing>
constexpr int rope_threads() { return kRing ? 256 : 1024; }
constexpr int kRopeUnroll = 4;
constexpr int kRopeBatchMax = RKV_ROPE_BATCH_MAX;   // tensors of one rope3d_apply_batch launch
constexpr int kRopeMaxEntries = 4096;  // 64 KB of per-pair entries per CTA (rotate-half)
constexpr int kAdjMaxEntries = 2048;   // 128 KB of chunk entries (4 float4 arrays) per CTA (adjacent)
constexpr int kRingRopeThreads = 640;   // rotated ring insert, at most: warp 0 copies V, the rest rotate K
constexpr int kRingRopeSmem = 227 * 1024 - 256;   // its dynamic shared memory at most (V stages + table)

// One tensor of a standalone launch: source and destination rows (strides in
// bytes) and the time index of row 0's frame.
struct RopeRows {
  const uint8_t* x;
  uint8_t* y;
  int64_t xs, ys;
  int32_t t0;
};
// Tensors of a standalone launch: tensor i holds CTAs [cta0[i], cta0[i + 1]),
// rpc[i] of its L[i] rows each.
struct RopeBatch {
  int32_t n;
  uint32_t cta0[kRopeBatchMax + 1];
  uint32_t L[kRopeBatchMax], rpc[kRopeBatchMax];
  RopeRows t[kRopeBatchMax];
};

__device__ __forceinline__ int32_t pick3i(int a, int32_t x, int32_t y, int32_t z) {
  return a == 0 ? x : (a == 1 ? y : z);
}

struct TabEntry {
  float c_hi, s_hi, c_lo, s_lo;
};

// a*(ch+cl) + b*(sh+sl) with error-free products and sum (fp32).
__device__ __forceinline__ float dot2_exact(float a, float ch, float cl, float b, float sh, float sl) {
  const float p1 = a * ch;
  const float e1 = fmaf(a, ch, -p1);
  const float p2 = b * sh;
  const float e2 = fmaf(b, sh, -p2);
  const float s = p1 + p2;
  const float bb = s - p1;
  const float e3 = (p1 - (s - bb)) + (p2 - bb);
  const float lo = (e1 + e2) + (e3 + fmaf(a, cl, b * sl));
  return s + lo;
}

__device__ __forceinline__ void rotate_pair(float x0, float x1, const TabEntry& e, float& y0, float& y1) {
  y0 = fmaf(x0, e.c_hi, -x1 * e.s_hi);
  y1 = fmaf(x0, e.s_hi, x1 * e.c_hi);
  const float lim = fmaxf(fabsf(x0), fabsf(x1)) * 0x1p-12f;
  if (fabsf(y0) < lim) y0 = dot2_exact(x0, e.c_hi, e.c_lo, -x1, e.s_hi, e.s_lo);
  if (fabsf(y1) < lim) y1 = dot2_exact(x0, e.s_hi, e.s_lo, x1, e.c_hi, e.c_lo);
}

// Address of 16-byte chunk `within` of row r (frame f, row in_f of that
// frame) in the destination: a strided row, or the row's place in the ring
// slot that frame f of the insert goes to.
template <bool kRing>
__device__ __forceinline__ uint8_t* dst_chunk(const RopeArgs& a, uint8_t* base, uint32_t r, uint32_t f, uint32_t in_f,
                                              uint32_t within) {
  if (kRing) {
    const int32_t slot = ring_dst_slot(a.ring, f);
    return base + uint64_t(slot) * a.slot_bytes + (uint64_t(in_f) * a.cpr + within) * 16u;
  }
  return base + int64_t(r) * a.y_stride_bytes + uint64_t(within) * 16u;
}

// Ring mode, second tensor: copy rows [r0, r1) of x2 into the ring unrotated.
__device__ __forceinline__ void copy_rows_to_ring(const RopeArgs& a, uint32_t r0, uint32_t r1) {
  const uint32_t T = blockDim.x;
  const uint32_t c_begin = r0 * a.cpr, c_end = r1 * a.cpr;
  for (uint32_t base = c_begin + threadIdx.x; base < c_end; base += T * kRopeUnroll) {
    uint4 v[kRopeUnroll];
    uint8_t* out[kRopeUnroll];
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      const uint32_t ci = base + u * T;
      out[u] = nullptr;
      if (ci < c_end) {
        const uint32_t r = fdiv(ci, a.div_cpr);
        const uint32_t within = ci - r * a.cpr;
        const uint32_t f = fdiv(r, a.div_F);
        v[u] = __ldcs(reinterpret_cast<const uint4*>(a.x2 + int64_t(r) * a.x_stride_bytes + uint64_t(within) * 16u));
        out[u] = dst_chunk<true>(a, a.y2, r, f, r - f * a.F, within);
      }
    }
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u)
      if (out[u]) *reinterpret_cast<uint4*>(out[u]) = v[u];
  }
}

// Rotate the 8 rotary pairs (element e of chunk A, element e of chunk B),
// e = 0..7, of the rotate-half layout; pair index of element e is p0 + e.
template <typename TabIdx>
__device__ __forceinline__ void rotate_half_chunks(uint4& A, uint4& B, int32_t p0, const TabEntry* tab,
                                                   TabIdx tab_idx) {
  uint32_t a4[4] = {A.x, A.y, A.z, A.w}, b4[4] = {B.x, B.y, B.z, B.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    float y0[2], y1[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float x0 = h ? bf16hi_to_f32(a4[w]) : bf16lo_to_f32(a4[w]);
      const float x1 = h ? bf16hi_to_f32(b4[w]) : bf16lo_to_f32(b4[w]);
      rotate_pair(x0, x1, tab[tab_idx(p0 + 2 * w + h)], y0[h], y1[h]);
    }
    a4[w] = pack_bf16x2(y0[0], y0[1]);
    b4[w] = pack_bf16x2(y1[0], y1[1]);
  }
  A = make_uint4(a4[0], a4[1], a4[2], a4[3]);
  B = make_uint4(b4[0], b4[1], b4[2], b4[3]);
}

// Rotate-half layout (pair j = elements j and j + 64 of a head, i.e. element
// e of chunk c and of chunk c + 8).
// kRing = false: rotate rows of x into rows of y (rope3d_apply).
// kRing = true: blockIdx.y = 0 rotates x (K) into ring slots of y, blockIdx.y
// = 1 copies x2 (V) into ring slots of y2 (kvcache_ring_update_rope).
template <bool kRing>
__global__ void __launch_bounds__(rope_threads<kRing>()) rope3d_half_kernel(const RopeArgs a) {
  constexpr int kRopeThreads = rope_threads<kRing>();
  extern __shared__ float4 tab_raw[];
  TabEntry* tab = reinterpret_cast<TabEntry*>(tab_raw);
  const uint32_t r0 = blockIdx.x * a.rows_per_cta;
  if (r0 >= a.L) return;
  const uint32_t r1 = min(a.L, r0 + a.rows_per_cta);
  if (kRing && blockIdx.y == 1) {
    copy_rows_to_ring(a, r0, r1);
    return;
  }

  // positions this CTA can reach: frames f_lo..f_hi; rows h_lo..h_lo+nh-1;
  // columns w_lo, w_lo+1, ... (mod grid_w), nw of them (w of row r = r mod
  // grid_w because a frame holds whole grid rows)
  const uint32_t f_lo = fdiv(r0, a.div_F), f_hi = fdiv(r1 - 1, a.div_F);
  const int32_t nt = int32_t(f_hi - f_lo) + 1;
  int32_t h_lo = 0, nh = a.grid_h;
  if (f_lo == f_hi) {
    h_lo = int32_t(fdiv(r0 - f_lo * a.F, a.div_W));
    nh = int32_t(fdiv(r1 - 1 - f_lo * a.F, a.div_W)) - h_lo + 1;
  }
  int32_t w_lo = 0, nw = a.grid_w;
  if (r1 - r0 < uint32_t(a.grid_w)) {
    w_lo = int32_t(r0 - fdiv(r0, a.div_W) * uint32_t(a.grid_w));
    nw = int32_t(r1 - r0);
  }
  const int32_t base_h = nt * a.pt;
  const int32_t base_w = base_h + nh * a.ph;
  const int32_t n_entries = base_w + nw * a.pw;

  for (int32_t e = threadIdx.x; e < n_entries; e += kRopeThreads) {
    int32_t pos, i, n;
    if (e < base_h) {
      const int32_t ft = e / a.pt;
      i = e - ft * a.pt; n = a.pt; pos = a.t0 + int32_t(f_lo) + ft;
    } else if (e < base_w) {
      const int32_t hh = (e - base_h) / a.ph;
      i = (e - base_h) - hh * a.ph; n = a.ph; pos = h_lo + hh;
    } else {
      const int32_t ww = (e - base_w) / a.pw;
      i = (e - base_w) - ww * a.pw; n = a.pw;
      pos = w_lo + ww;
      if (pos >= a.grid_w) pos -= a.grid_w;
    }
    const int axis = e < base_h ? 0 : (e < base_w ? 1 : 2);
    const double ang = double(pos) * a.omega[pick3i(axis, 0, a.pt, a.pt + a.ph) + i];
    double s, c;
    sincos(ang, &s, &c);
    TabEntry t;
    t.c_hi = __double2float_rn(c);
    t.s_hi = __double2float_rn(s);
    t.c_lo = __double2float_rn(c - double(t.c_hi));
    t.s_lo = __double2float_rn(s - double(t.s_hi));
    tab[e] = t;
  }
  __syncthreads();

  {
    // units of work: chunk pairs (c, c + 8) of a head, 8 per head
    const uint32_t p_begin = r0 * a.cph, p_end = r1 * a.cph;
    for (uint32_t base = p_begin + threadIdx.x; base < p_end; base += kRopeThreads * kRopeUnroll) {
      uint4 va[kRopeUnroll], vb[kRopeUnroll];
      uint32_t row[kRopeUnroll], ca[kRopeUnroll];
#pragma unroll
      for (int u = 0; u < kRopeUnroll; ++u) {
        const uint32_t pi = base + u * kRopeThreads;
        if (pi < p_end) {
          row[u] = fdiv(pi, a.div_cph);
          const uint32_t wp = pi - row[u] * a.cph;          // head * 8 + c
          ca[u] = (wp >> 3) * 16u + (wp & 7u);               // chunk c of the head; its partner is ca + 8
          const uint8_t* src = a.x + int64_t(row[u]) * a.x_stride_bytes;
          va[u] = *reinterpret_cast<const uint4*>(src + uint64_t(ca[u]) * 16u);
          vb[u] = *reinterpret_cast<const uint4*>(src + uint64_t(ca[u] + 8u) * 16u);
        }
      }
#pragma unroll
      for (int u = 0; u < kRopeUnroll; ++u) {
        const uint32_t pi = base + u * kRopeThreads;
        if (pi >= p_end) continue;
        const uint32_t r = row[u];
        const uint32_t f = fdiv(r, a.div_F);
        const uint32_t in_f = r - f * a.F;
        const uint32_t hh = fdiv(in_f, a.div_W);
        const uint32_t ww = in_f - hh * uint32_t(a.grid_w);
        int32_t wi_off = int32_t(ww) - w_lo;
        if (wi_off < 0) wi_off += a.grid_w;
        const int32_t ti = int32_t(f - f_lo) * a.pt;
        const int32_t hi = base_h + (int32_t(hh) - h_lo) * a.ph - a.pt;
        const int32_t wi = base_w + wi_off * a.pw - a.pt - a.ph;
        const int32_t pt = a.pt, pth = a.pt + a.ph;
        rotate_half_chunks(va[u], vb[u], int32_t(ca[u] & 7u) * 8, tab, [&](int32_t p) {
          return p < pt ? ti + p : (p < pth ? hi + p : wi + p);
        });
        *reinterpret_cast<uint4*>(dst_chunk<kRing>(a, a.y, r, f, in_f, ca[u])) = va[u];
        *reinterpret_cast<uint4*>(dst_chunk<kRing>(a, a.y, r, f, in_f, ca[u] + 8u)) = vb[u];
      }
    }
  }
}

// Adjacent layout: rotate the 4 pairs of one 16-byte chunk (word k holds
// x0 in its low and x1 in its high half) with the chunk's cos C and sin S,
// in fp32 on packed f32x2 FMAs; `bad` is set when an output cancelled below
// 2^-12 of its inputs and needs the exact path.
__device__ __forceinline__ uint4 rotate4(uint4 v, float4 C, float4 S, bool& bad) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
  bool b = false;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t p = w[2 * h], q = w[2 * h + 1];
    const float2 x0 = make_float2(bf16lo_to_f32(p), bf16lo_to_f32(q));
    const float2 x1 = make_float2(bf16hi_to_f32(p), bf16hi_to_f32(q));
    const float2 nx1 = make_float2(-x1.x, -x1.y);
    const float2 c = h ? make_float2(C.z, C.w) : make_float2(C.x, C.y);
    const float2 s = h ? make_float2(S.z, S.w) : make_float2(S.x, S.y);
    const float2 y0 = __ffma2_rn(x0, c, __fmul2_rn(nx1, s));   // x0 cos - x1 sin
    const float2 y1 = __ffma2_rn(x0, s, __fmul2_rn(x1, c));    // x0 sin + x1 cos
    const float la = fmaxf(fabsf(x0.x), fabsf(x1.x)) * 0x1p-12f;
    const float lb = fmaxf(fabsf(x0.y), fabsf(x1.y)) * 0x1p-12f;
    b |= (fabsf(y0.x) < la) | (fabsf(y1.x) < la) | (fabsf(y0.y) < lb) | (fabsf(y1.y) < lb);
    o[2 * h] = pack_bf16x2(y0.x, y1.x);
    o[2 * h + 1] = pack_bf16x2(y0.y, y1.y);
  }
  bad = b;
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// The exact path of rotate4 for a chunk that cancelled: each output redone
// with its cos/sin as hi + lo and error-free products (the same result
// rotate_pair gives).  Out of line: the main loop carries none of it.
__device__ __noinline__ uint4 rotate4_exact(uint4 v, float4 C, float4 S, float4 Cl, float4 Sl) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  const float c[4] = {C.x, C.y, C.z, C.w}, s[4] = {S.x, S.y, S.z, S.w};
  const float cl[4] = {Cl.x, Cl.y, Cl.z, Cl.w}, sl[4] = {Sl.x, Sl.y, Sl.z, Sl.w};
  uint32_t o[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float y0, y1;
    rotate_pair(bf16lo_to_f32(w[k]), bf16hi_to_f32(w[k]), TabEntry{c[k], s[k], cl[k], sl[k]}, y0, y1);
    o[k] = pack_bf16x2(y0, y1);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Table entry of 16-byte chunk `chunk` (rotary pairs 4*chunk .. +3) at
// positions (p_t, p_h, p_w): cos and sin of each pair's angle rounded to
// fp32 (hi) and the fp32 rounding of the rest (lo).  Pairs on an axis outside
// the bit mask `axes` hold cos 1, sin 0.
__device__ void adj_entry(const RopeArgs& a, int32_t chunk, int axes, int32_t p_t, int32_t p_h, int32_t p_w, float4& C, float4& S,
                          float4& Cl, float4& Sl) {
  float c4[4], s4[4], cl4[4], sl4[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int32_t pr = 4 * chunk + q;
    const int ax = pr < a.ax_first[1] ? 0 : (pr < a.ax_first[2] ? 1 : 2);
    double sd = 0.0, cd = 1.0;
    if ((axes >> ax) & 1) sincos(double(pick3i(ax, p_t, p_h, p_w)) * a.omega[pr], &sd, &cd);
    c4[q] = __double2float_rn(cd);
    s4[q] = __double2float_rn(sd);
    cl4[q] = __double2float_rn(cd - double(c4[q]));
    sl4[q] = __double2float_rn(sd - double(s4[q]));
  }
  C = make_float4(c4[0], c4[1], c4[2], c4[3]);
  S = make_float4(s4[0], s4[1], s4[2], s4[3]);
  Cl = make_float4(cl4[0], cl4[1], cl4[2], cl4[3]);
  Sl = make_float4(sl4[0], sl4[1], sl4[2], sl4[3]);
}

// Adjacent layout (pairs 2j, 2j+1).  kRing: K rows go to their ring slots.  Table
// (shared memory, four float4 arrays of E entries: cos hi, sin hi, cos lo,
// sin lo).  Entry (axis a, chunk k of the axis, position index i) at
// tab_base[a] + k * npos[a] + i holds the 4 pairs of chunk ax_chunk0[a] + k
// (pairs of that chunk outside axis a hold cos 1, sin 0); a chunk whose pairs
// lie on several axes instead reads entry (region m, row r - r0) after those,
// built for each of the CTA's rows as the product of the single-axis entries
// (exact: each pair has one factor other than cos 1 / sin 0).  So every chunk
// reads one entry, and the threads of a warp take the same path whatever
// chunk positions they hold.  The first rows' loads are issued before the
// table is built, so their latency overlaps the fp64 sincos.
//
// Rows [r0, r1) by threads tid = 0 .. T-1 of the CTA (table in tab4); bar = 0
// synchronises with __syncthreads, else with named barrier `bar` over the T
// threads.
template <bool kRing>
__device__ __forceinline__ void adj_rotate(const RopeArgs& a, const RopeRows rr, uint32_t r0, uint32_t r1, uint32_t tid,
                                           uint32_t T, float4* tab4, uint32_t bar) {
  auto sync = [&]() {
    if (bar == 0)
      __syncthreads();
    else
      ptx::named_sync_and(bar, T, true);
  };
  // positions this CTA's rows reach: frames f_lo..f_hi; grid rows
  // h_lo..h_lo+nh-1; columns w_lo, w_lo+1, ... (mod grid_w), nw of them
  const uint32_t f_lo = fdiv(r0, a.div_F), f_hi = fdiv(r1 - 1, a.div_F);
  const int32_t nt = int32_t(f_hi - f_lo) + 1;
  int32_t h_lo = 0, nh = a.grid_h;
  if (f_lo == f_hi) {
    h_lo = int32_t(fdiv(r0 - f_lo * a.F, a.div_W));
    nh = int32_t(fdiv(r1 - 1 - f_lo * a.F, a.div_W)) - h_lo + 1;
  }
  int32_t w_lo = 0, nw = a.grid_w;
  if (r1 - r0 < uint32_t(a.grid_w)) {
    w_lo = int32_t(r0 - fdiv(r0, a.div_W) * uint32_t(a.grid_w));
    nw = int32_t(r1 - r0);
  }
  const int32_t npos0 = nt, npos1 = nh, npos2 = nw;
  const int32_t nrows = int32_t(r1 - r0);
  const int32_t tb0 = 0, tb1 = a.ax_nch[0] * npos0, tb2 = tb1 + a.ax_nch[1] * npos1;
  const int32_t tbm = tb2 + a.ax_nch[2] * npos2;
  const int32_t E = tbm + a.n_multi * nrows;
  float4* tC = tab4;
  float4* tS = tab4 + E;
  float4* tCl = tab4 + 2 * E;
  float4* tSl = tab4 + 3 * E;
  // thread -> (chunk position c of a row, row phase rsub): `lanes` threads per
  // row, rpp rows side by side; each thread walks rows r0 + rsub, + rpp, ...
  const uint32_t lanes = a.cpr < T ? a.cpr : T;
  const uint32_t rpp = T / lanes;
  const uint32_t rsub = tid / lanes;
  const uint32_t c0 = tid - rsub * lanes;
  const bool active = rsub < rpp;
  // the first rows' loads go out before the table is built
  uint4 v[kRopeUnroll];
  if (active) {
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      const uint32_t r = r0 + rsub + u * rpp;
      if (r < r1) v[u] = *reinterpret_cast<const uint4*>(rr.x + int64_t(r) * rr.xs + uint64_t(c0) * 16u);
    }
  }
  // single-axis entries (fp64 sincos), then the per-row entries of chunks on
  // several axes as products of those (each pair has one factor other than
  // cos 1 / sin 0, so the product and the sums are exact)
  for (int32_t e = int32_t(tid); e < tbm; e += int32_t(T)) {
    const int ax = e < tb1 ? 0 : (e < tb2 ? 1 : 2);
    const int32_t np = pick3i(ax, npos0, npos1, npos2);
    const int32_t rel = e - pick3i(ax, tb0, tb1, tb2);
    const int32_t k = rel / np, pi = rel - k * np;
    int32_t ps = ax == 0 ? rr.t0 + int32_t(f_lo) + pi : (ax == 1 ? h_lo + pi : w_lo + pi);
    if (ax == 2 && ps >= a.grid_w) ps -= a.grid_w;
    adj_entry(a, a.ax_chunk0[ax] + k, 1 << ax, ps, ps, ps, tC[e], tS[e], tCl[e], tSl[e]);
  }
  if (a.n_multi > 0) {
    sync();
    for (int32_t e = tbm + int32_t(tid); e < E; e += int32_t(T)) {
      const int32_t m = (e - tbm) / nrows;
      const uint32_t r = r0 + uint32_t(e - tbm - m * nrows);
      const uint32_t f = fdiv(r, a.div_F);
      const uint32_t in_f = r - f * a.F;
      const uint32_t hh = fdiv(in_f, a.div_W);
      int32_t wi = int32_t(in_f - hh * uint32_t(a.grid_w)) - w_lo;
      if (wi < 0) wi += a.grid_w;
      const int32_t idx[3] = {int32_t(f - f_lo), int32_t(hh) - h_lo, wi};
      int32_t g = 0;
      for (int gg = 0, seen = 0; gg < 16; ++gg)
        if (a.ch_axis[gg] < 0 && seen++ == m) g = gg;
      float4 C = make_float4(1.f, 1.f, 1.f, 1.f), S = make_float4(0.f, 0.f, 0.f, 0.f);
      float4 Cl = S, Sl = S;
#pragma unroll
      for (int ax = 0; ax < 3; ++ax) {
        const int32_t k = g - a.ax_chunk0[ax];
        if (k < 0 || k >= a.ax_nch[ax]) continue;
        const int32_t ea = pick3i(ax, tb0, tb1, tb2) + k * pick3i(ax, npos0, npos1, npos2) + idx[ax];
        const float4 c = tC[ea], s4 = tS[ea], cl = tCl[ea], sl = tSl[ea];
        C = make_float4(C.x * c.x, C.y * c.y, C.z * c.z, C.w * c.w);
        S = make_float4(S.x + s4.x, S.y + s4.y, S.z + s4.z, S.w + s4.w);
        Cl = make_float4(Cl.x + cl.x, Cl.y + cl.y, Cl.z + cl.z, Cl.w + cl.w);
        Sl = make_float4(Sl.x + sl.x, Sl.y + sl.y, Sl.z + sl.z, Sl.w + sl.w);
      }
      tC[e] = C;
      tS[e] = S;
      tCl[e] = Cl;
      tSl[e] = Sl;
    }
  }
  sync();

  if (!active) return;
  for (uint32_t c = c0; c < a.cpr; c += lanes) {
    // entry of row r: eb + ti*mt + hi*mh + wi*mw + r*mr, one term non-zero
    const int32_t g = int32_t(c & 15u);
    const int ax = a.ch_axis[g];
    int32_t eb, mt = 0, mh = 0, mw = 0, mr = 0;
    if (ax >= 0) {
      eb = pick3i(ax, tb0, tb1, tb2) + (g - a.ax_chunk0[ax]) * pick3i(ax, npos0, npos1, npos2);
      mt = ax == 0;
      mh = ax == 1;
      mw = ax == 2;
    } else {
      eb = tbm + int32_t(a.ch_multi[g]) * nrows - int32_t(r0);
      mr = 1;
    }
    for (uint32_t rb = r0 + rsub; rb < r1; rb += rpp * kRopeUnroll) {
      if (c != c0 || rb != r0 + rsub) {
#pragma unroll
        for (int u = 0; u < kRopeUnroll; ++u) {
          const uint32_t r = rb + u * rpp;
          if (r < r1) v[u] = *reinterpret_cast<const uint4*>(rr.x + int64_t(r) * rr.xs + uint64_t(c) * 16u);
        }
      }
#pragma unroll
      for (int u = 0; u < kRopeUnroll; ++u) {
        const uint32_t r = rb + u * rpp;
        if (r >= r1) continue;
        const uint32_t f = fdiv(r, a.div_F);
        const uint32_t in_f = r - f * a.F;
        const uint32_t hh = fdiv(in_f, a.div_W);
        const uint32_t ww = in_f - hh * uint32_t(a.grid_w);
        int32_t wi = int32_t(ww) - w_lo;
        if (wi < 0) wi += a.grid_w;
        const int32_t ti = int32_t(f - f_lo), hi = int32_t(hh) - h_lo;
        const int32_t e = eb + ti * mt + hi * mh + wi * mw + int32_t(r) * mr;
        const float4 C = tC[e], S = tS[e];
        bool bad;
        uint4 out = rotate4(v[u], C, S, bad);
        if (bad) out = rotate4_exact(v[u], C, S, tCl[e], tSl[e]);
        uint8_t* dst = kRing ? dst_chunk<true>(a, rr.y, r, f, in_f, c) : rr.y + int64_t(r) * rr.ys + uint64_t(c) * 16u;
        *reinterpret_cast<uint4*>(dst) = out;
      }
    }
  }
}

// Standalone op (adjacent layout): one CTA per SM over a block of rows of
// one of the launch's tensors (rope3d_apply: one tensor; rope3d_apply_batch:
// up to kRopeBatchMax, the CTAs shared out by rows).
__global__ void __launch_bounds__(1024) rope3d_adj_kernel(const RopeArgs a, const RopeBatch b) {
  extern __shared__ float4 tab4[];
  int i = 0;
  while (i + 1 < b.n && blockIdx.x >= b.cta0[i + 1]) ++i;
  const uint32_t r0 = (blockIdx.x - b.cta0[i]) * b.rpc[i];
  if (r0 >= b.L[i]) return;
  const uint32_t r1 = min(b.L[i], r0 + b.rpc[i]);
  adj_rotate<false>(a, b.t[i], r0, r1, threadIdx.x, blockDim.x, tab4, 0);
}

// Rotated ring insert (adjacent layout), one CTA per SM: one thread of warp 0
// moves the CTA's share of the V pieces on the TMA bulk-copy engine (global ->
// shared memory -> ring slot, the kvcache_ring_update path), while warps
// 1..31 build the cos/sin table and rotate the CTA's block of K rows through
// registers into the ring: the table build and the rotation run under V's
// copy.  Shared memory: V stages, then the table.  Fewer threads than the
// standalone kernel keep its registers (the V copy needs none of them).
__global__ void __launch_bounds__(kRingRopeThreads, 1) ring_rope_kernel(const RopeArgs a, const RingBulkArgs vb) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[kBulkStages];
  if (threadIdx.x < 32) {
    if (threadIdx.x == 0) bulk_copy_pieces(vb, vb.half + blockIdx.x, vb.total, gridDim.x, ptx::smem_u32(smem), full);
    return;
  }
  const uint32_t r0 = blockIdx.x * a.rows_per_cta;
  if (r0 >= a.L) return;
  const uint32_t r1 = min(a.L, r0 + a.rows_per_cta);
  adj_rotate<true>(a, RopeRows{a.x, a.y, a.x_stride_bytes, a.y_stride_bytes, a.t0}, r0, r1, threadIdx.x - 32,
                   blockDim.x - 32,
                   reinterpret_cast<float4*>(smem + vb.stages * vb.stage_bytes), 1);
}

static int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

rkv_status check_rope(const rkv_rope3d* rope, int32_t D) {
  if (!rope) return fail(RKV_ERR_INVALID_ARG, "rope parameters are NULL");
  if (rope->grid_h < 1 || rope->grid_w < 1) return fail(RKV_ERR_INVALID_ARG, "grid_h/grid_w must be >= 1");
  if (int64_t(rope->grid_h) * rope->grid_w >= (int64_t(1) << 30))
    return fail(RKV_ERR_INVALID_ARG, "frame grid too large");
  if (rope->pairs_t < 1 || rope->pairs_h < 1 || rope->pairs_w < 1)
    return fail(RKV_ERR_INVALID_ARG, "pairs per axis must be >= 1");
  if (rope->pairs_t + rope->pairs_h + rope->pairs_w != D / 2)
    return fail(RKV_ERR_INVALID_ARG, "pairs_t+pairs_h+pairs_w must equal D/2");
  if (!(rope->theta > 1.0f) || !isfinite(rope->theta)) return fail(RKV_ERR_INVALID_ARG, "theta must be finite and > 1");
  const float th[2] = {rope->theta_h, rope->theta_w};
  for (int i = 0; i < 2; ++i)
    if (th[i] != 0.0f && (!(th[i] > 1.0f) || !isfinite(th[i])))
      return fail(RKV_ERR_INVALID_ARG, "theta_h / theta_w must be 0 (= theta) or finite and > 1");
  if (rope->layout != RKV_ROPE_ADJACENT && rope->layout != RKV_ROPE_HALF)
    return fail(RKV_ERR_INVALID_ARG, "rope layout must be RKV_ROPE_ADJACENT or RKV_ROPE_HALF");
  return RKV_OK;
}

// Fill the rotation part of RopeArgs shared by both layouts.
static void fill_rope_args(RopeArgs& a, int64_t L, int32_t H, int32_t t0, const rkv_rope3d* rope) {
  a.L = uint32_t(L);
  a.cpr = uint32_t(H) * 16u;
  a.F = uint32_t(rope->grid_h) * uint32_t(rope->grid_w);
  a.t0 = t0;
  a.grid_h = rope->grid_h;
  a.grid_w = rope->grid_w;
  a.pt = rope->pairs_t;
  a.ph = rope->pairs_h;
  a.pw = rope->pairs_w;
  {
    // computed once here (fp64) instead of in every table entry on the device
    const double log2_theta[3] = {log2(double(rope->theta)),
                                  log2(double(rope->theta_h != 0.0f ? rope->theta_h : rope->theta)),
                                  log2(double(rope->theta_w != 0.0f ? rope->theta_w : rope->theta))};
    const int32_t cnt[3] = {rope->pairs_t, rope->pairs_h, rope->pairs_w};
    for (int ax = 0, j = 0; ax < 3; ++ax)
      for (int32_t i = 0; i < cnt[ax] && j < 64; ++i, ++j)
        a.omega[j] = exp2(-(double(i) / double(cnt[ax])) * log2_theta[ax]);
  }
  a.cph = uint32_t(H) * 8u;
  a.div_cph = make_fastdiv(a.cph);
  a.div_F = make_fastdiv(a.F);
  a.div_W = make_fastdiv(uint32_t(rope->grid_w));
  a.div_cpr = make_fastdiv(a.cpr);
  const int32_t pairs[3] = {rope->pairs_t, rope->pairs_h, rope->pairs_w};
  int32_t first = 0;
  for (int ax = 0; ax < 3; ++ax) {
    a.ax_first[ax] = first;
    a.ax_count[ax] = pairs[ax];
    a.ax_chunk0[ax] = first / 4;
    a.ax_nch[ax] = (first + pairs[ax] - 1) / 4 - first / 4 + 1;
    first += pairs[ax];
  }
  auto axis_of_pair = [&](int pr) { return pr < a.ax_first[1] ? 0 : (pr < a.ax_first[2] ? 1 : 2); };
  a.n_multi = 0;
  for (int g = 0; g < 16; ++g) {
    const int lo = axis_of_pair(4 * g), hi = axis_of_pair(4 * g + 3);
    a.ch_axis[g] = int8_t(lo == hi ? lo : -1);
    a.ch_multi[g] = int8_t(lo == hi ? -1 : a.n_multi++);
  }
}

// Rotate-half layout: rows per CTA under the per-pair table budget, launch
// (ring mode: two CTA rows, K rotated and V copied).
template <bool kRing>
static rkv_status launch_rope_half(RopeArgs& a, int64_t L, cudaStream_t stream) {
  const int64_t target_ctas = int64_t(sm_count()) * (kRing ? 4 : 1);
  int64_t rpc = (L + target_ctas - 1) / target_ctas;
  if (rpc < 1) rpc = 1;
  // upper bound of the table a CTA of `rows` rows builds (see the kernel)
  auto entries = [&](int64_t rows) {
    const int64_t nt = rows / a.F + 2;
    return nt * a.pt + int64_t(a.grid_h) * a.ph + std::min<int64_t>(a.grid_w, rows) * a.pw;
  };
  if (entries(1) > kRopeMaxEntries) return fail(RKV_ERR_UNSUPPORTED, "frame grid too large for the on-chip cos/sin table");
  while (rpc > 1 && entries(rpc) > kRopeMaxEntries) rpc = (rpc + 1) / 2;
  a.rows_per_cta = uint32_t(rpc);
  const int64_t grid = (L + rpc - 1) / rpc;
  const size_t smem = size_t(entries(rpc)) * sizeof(TabEntry);
  // set on every launch: the attribute belongs to the current device, and a
  // process may launch on several
  cudaError_t e = cudaFuncSetAttribute(rope3d_half_kernel<kRing>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kRopeMaxEntries * int(sizeof(TabEntry)));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(rope3d_half_kernel)");
  rope3d_half_kernel<kRing><<<dim3(uint32_t(grid), kRing ? 2u : 1u), rope_threads<kRing>(), smem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "rope3d_half_kernel launch");
  return RKV_OK;
}

// upper bound of the chunk entries a CTA of `rows` rows builds (see adj_rotate)
static int64_t adj_entries(const RopeArgs& a, int64_t rows) {
  const int64_t nt = rows / a.F + 2;
  return int64_t(a.ax_nch[0]) * nt + int64_t(a.ax_nch[1]) * a.grid_h +
         int64_t(a.ax_nch[2]) * std::min<int64_t>(a.grid_w, rows) + int64_t(a.n_multi) * rows;
}

// Adjacent layout, standalone: `lanes` threads per row (one per 16-byte
// chunk, at most 1024) times the rows side by side that fit in 1024 threads,
// one CTA per SM over all the launch's tensors (each gets CTAs in proportion
// to its rows, at least one); rows per CTA under the table budget.
static rkv_status launch_rope_adj(RopeArgs& a, const RopeRows* rows, const int64_t* L, int n, cudaStream_t stream) {
  if (adj_entries(a, 1) > kAdjMaxEntries)
    return fail(RKV_ERR_UNSUPPORTED, "frame grid too large for the on-chip cos/sin table");
  const int64_t lanes = std::min<int64_t>(a.cpr, 1024);
  const int64_t threads = lanes * std::max<int64_t>(1, 1024 / lanes);
  int64_t total = 0;
  for (int i = 0; i < n; ++i) total += L[i];
  RopeBatch b{};
  b.n = n;
  int64_t cta = 0, max_entries = 0;
  for (int i = 0; i < n; ++i) {
    int64_t c = std::max<int64_t>(1, (int64_t(sm_count()) * L[i] + total / 2) / total);
    int64_t rpc = (L[i] + c - 1) / c;
    while (rpc > 1 && adj_entries(a, rpc) > kAdjMaxEntries) rpc = (rpc + 1) / 2;
    c = (L[i] + rpc - 1) / rpc;
    b.cta0[i] = uint32_t(cta);
    b.L[i] = uint32_t(L[i]);
    b.rpc[i] = uint32_t(rpc);
    b.t[i] = rows[i];
    cta += c;
    max_entries = std::max<int64_t>(max_entries, adj_entries(a, rpc));
  }
  b.cta0[n] = uint32_t(cta);
  if (cta >= (int64_t(1) << 31)) return fail(RKV_ERR_UNSUPPORTED, "too many rows for one launch");
  const size_t smem = size_t(max_entries) * 4 * sizeof(float4);
  cudaError_t e = cudaFuncSetAttribute(rope3d_adj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kAdjMaxEntries * 4 * int(sizeof(float4)));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(rope3d_adj_kernel)");
  rope3d_adj_kernel<<<uint32_t(cta), uint32_t(threads), smem, stream>>>(a, b);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "rope3d_adj_kernel launch");
  return RKV_OK;
}

// Adjacent layout, ring insert: one CTA per SM, its K rows under the table
// budget, as many V stages as fit beside the table (the table is at most
// 64 KB, so at least 5 always do).
static rkv_status launch_ring_rope(RopeArgs& a, int64_t L, const RingBulkArgs& vb, cudaStream_t stream) {
  if (adj_entries(a, 1) > kAdjMaxEntries)
    return fail(RKV_ERR_UNSUPPORTED, "frame grid too large for the on-chip cos/sin table");
  int64_t r = (L + sm_count() - 1) / sm_count();
  if (r < 1) r = 1;
  while (r > 1 && adj_entries(a, r) > kAdjMaxEntries) r = (r + 1) / 2;
  const int64_t table = adj_entries(a, r) * 4 * int64_t(sizeof(float4));
  const int64_t stages = std::min<int64_t>(kBulkStages, (kRingRopeSmem - table) / vb.stage_bytes);
  if (stages < 2) return fail(RKV_ERR_UNSUPPORTED, "no room for the V stages beside the cos/sin table");
  RingBulkArgs v = vb;
  v.stages = uint32_t(stages);
  a.rows_per_cta = uint32_t(r);
  const int64_t grid = (L + r - 1) / r;
  const int smem = int(stages * v.stage_bytes + table);
  cudaError_t e = cudaFuncSetAttribute(ring_rope_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRingRopeSmem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(ring_rope_kernel)");
  // rotating threads: whole rows of chunks, rounded up to whole warps (the
  // named barrier counts warps; the extra threads only join it)
  const int64_t lanes = std::min<int64_t>(a.cpr, kRingRopeThreads - 32);
  const int64_t rot = lanes * std::max<int64_t>(1, (kRingRopeThreads - 32) / lanes);
  const int64_t threads = 32 + (rot + 31) / 32 * 32;
  ring_rope_kernel<<<uint32_t(grid), uint32_t(threads), smem, stream>>>(a, v);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "ring_rope_kernel launch");
  return RKV_OK;
}

// Rotated ring insert: adjacent layout on ring_rope_kernel, rotate-half on
// rope3d_half_kernel<true>.
static rkv_status launch_ring(RopeArgs& a, int64_t L, int32_t H, int32_t t0, const rkv_rope3d* rope,
                              const RingBulkArgs& vb, cudaStream_t stream) {
  fill_rope_args(a, L, H, t0, rope);
  if (rope->layout == RKV_ROPE_HALF) return launch_rope_half<true>(a, L, stream);
  return launch_ring_rope(a, L, vb, stream);
}

// Argument checks of one standalone tensor (rope3d_apply's rules).
static rkv_status check_rope_tensor(const rkv_rope_tensor& t, int32_t H, const rkv_rope3d* rope) {
  if (t.L < 0) return fail(RKV_ERR_INVALID_ARG, "L must be >= 0");
  if (t.L == 0) return RKV_OK;
  if (!t.x || !t.y) return fail(RKV_ERR_INVALID_ARG, "x/y is NULL");
  const int64_t row_elems = int64_t(H) * 128;
  if (t.x_row_stride < row_elems || t.y_row_stride < row_elems) return fail(RKV_ERR_INVALID_ARG, "row stride < H*D");
  if (!aligned16(t.x) || !aligned16(t.y) || (t.x_row_stride * 2) % 16 || (t.y_row_stride * 2) % 16)
    return fail(RKV_ERR_INVALID_ARG, "rows must be 16-byte aligned");
  const uint64_t xb = uint64_t((t.L - 1) * t.x_row_stride + row_elems) * 2;
  const uint64_t yb = uint64_t((t.L - 1) * t.y_row_stride + row_elems) * 2;
  if (t.x != t.y && overlaps(t.x, xb, t.y, yb)) return fail(RKV_ERR_INVALID_ARG, "x and y overlap without being identical");
  if (t.x == t.y && t.x_row_stride != t.y_row_stride) return fail(RKV_ERR_INVALID_ARG, "in-place call needs equal strides");
  if (t.L >= (int64_t(1) << 31) || uint64_t(t.L) * H * 16 >= (uint64_t(1) << 31))
    return fail(RKV_ERR_UNSUPPORTED, "too many rows for one launch");
  const int64_t last_t = int64_t(t.t0) + (t.L - 1) / (int64_t(rope->grid_h) * rope->grid_w);
  if (last_t > INT32_MAX) return fail(RKV_ERR_INVALID_ARG, "time index overflows int32");
  return RKV_OK;
}

// rope3d_apply / rope3d_apply_batch: check, then one launch (adjacent layout)
// or one launch per tensor (rotate-half layout).
static rkv_status rope_batch(const rkv_rope_tensor* t, int32_t n, int32_t H, int32_t D, const rkv_rope3d* rope,
                             cudaStream_t stream) {
  if (D != 128) return fail(RKV_ERR_INVALID_ARG, "head_dim D must be 128 (got %d)", D);
  rkv_status st = check_rope(rope, D);
  if (st != RKV_OK) return st;
  if (H < 1) return fail(RKV_ERR_INVALID_ARG, "H must be >= 1");
  RopeRows rows[kRopeBatchMax];
  int64_t L[kRopeBatchMax];
  int m = 0;
  for (int i = 0; i < n; ++i) {
    if ((st = check_rope_tensor(t[i], H, rope)) != RKV_OK) return st;
    if (t[i].L == 0) continue;
    const int64_t row_elems = int64_t(H) * 128;
    const uint64_t yb = uint64_t((t[i].L - 1) * t[i].y_row_stride + row_elems) * 2;
    for (int j = 0; j < n; ++j) {
      if (j == i || t[j].L == 0) continue;
      const uint64_t xb = uint64_t((t[j].L - 1) * t[j].x_row_stride + row_elems) * 2;
      const uint64_t yb2 = uint64_t((t[j].L - 1) * t[j].y_row_stride + row_elems) * 2;
      if (overlaps(t[i].y, yb, t[j].x, xb) || overlaps(t[i].y, yb, t[j].y, yb2))
        return fail(RKV_ERR_INVALID_ARG, "tensor %d's output overlaps tensor %d", i, j);
    }
    rows[m] = RopeRows{static_cast<const uint8_t*>(t[i].x), static_cast<uint8_t*>(t[i].y), t[i].x_row_stride * 2,
                       t[i].y_row_stride * 2, t[i].t0};
    L[m] = t[i].L;
    ++m;
  }
  if (m == 0) return RKV_OK;
  if (rope->layout == RKV_ROPE_HALF) {
    for (int i = 0; i < m; ++i) {
      RopeArgs a{};
      a.x = rows[i].x;
      a.y = rows[i].y;
      a.x_stride_bytes = rows[i].xs;
      a.y_stride_bytes = rows[i].ys;
      fill_rope_args(a, L[i], H, rows[i].t0, rope);
      if ((st = launch_rope_half<false>(a, L[i], stream)) != RKV_OK) return st;
    }
    return RKV_OK;
  }
  RopeArgs a{};
  fill_rope_args(a, 1, H, 0, rope);
  return launch_rope_adj(a, rows, L, m, stream);
}

}  // namespace rkv

using namespace rkv;

extern "C" rkv_status rope3d_apply(const void* x, void* y, int64_t L, int32_t H, int32_t D, int64_t x_row_stride,
                                   int64_t y_row_stride, int32_t t0, const rkv_rope3d* rope, void* stream) {
  NvtxRange nvtx_range("rope3d_apply");
  clear_error();
  const rkv_rope_tensor t = {x, y, L, x_row_stride, y_row_stride, t0};
  return rope_batch(&t, 1, H, D, rope, static_cast<cudaStream_t>(stream));
}

extern "C" rkv_status rope3d_apply_batch(const rkv_rope_tensor* tensors, int32_t n, int32_t H, int32_t D,
                                         const rkv_rope3d* rope, void* stream) {
  NvtxRange nvtx_range("rope3d_apply_batch");
  clear_error();
  if (n < 0 || n > kRopeBatchMax) return fail(RKV_ERR_INVALID_ARG, "n must be in [0, %d]", kRopeBatchMax);
  if (n > 0 && !tensors) return fail(RKV_ERR_INVALID_ARG, "tensors is NULL");
  return rope_batch(tensors, n, H, D, rope, static_cast<cudaStream_t>(stream));
}

extern "C" rkv_status kvcache_ring_update_rope(rkv_ring* ring, const void* k_new, const void* v_new,
                                               int64_t new_row_stride, int32_t n_frames, int32_t t0,
                                               const rkv_rope3d* rope, int32_t* n_evicted, void* stream) {
  NvtxRange nvtx_range("kvcache_ring_update_rope");
  clear_error();
  rkv_status st = check_ring(ring);
  if (st != RKV_OK) return st;
  st = check_rope(rope, ring->D);
  if (st != RKV_OK) return st;
  if (int64_t(rope->grid_h) * rope->grid_w != ring->tokens_per_frame)
    return fail(RKV_ERR_INVALID_ARG, "grid_h*grid_w (%d*%d) must equal tokens_per_frame (%d)", rope->grid_h,
                rope->grid_w, ring->tokens_per_frame);
  st = check_ring_insert(ring, k_new, v_new, new_row_stride, n_frames);
  if (st != RKV_OK) return st;
  if (n_frames > 0) {
    if (int64_t(t0) + n_frames - 1 > INT32_MAX) return fail(RKV_ERR_INVALID_ARG, "time index overflows int32");
    RopeArgs a{};
    a.x = static_cast<const uint8_t*>(k_new);
    a.y = static_cast<uint8_t*>(ring->k);
    a.x2 = static_cast<const uint8_t*>(v_new);
    a.y2 = static_cast<uint8_t*>(ring->v);
    a.x_stride_bytes = new_row_stride * 2;
    a.y_stride_bytes = int64_t(ring->H) * ring->D * 2;
    a.slot_bytes = uint64_t(ring->tokens_per_frame) * ring->H * ring->D * 2;
    a.ring = ring_plan(ring);
    // V goes through the bulk-copy pieces of a plain insert (the V half)
    RingBulkArgs vb;
    st = ring_bulk_geometry(ring, k_new, v_new, new_row_stride, n_frames, vb);
    if (st != RKV_OK) return st;
    st = ring_timeout_flag(&vb.timeout_flag);
    if (st != RKV_OK) return st;
    st = launch_ring(a, int64_t(n_frames) * ring->tokens_per_frame, ring->H, t0, rope, vb,
                     static_cast<cudaStream_t>(stream));
    if (st != RKV_OK) return st;
  }
  ring_advance(ring, n_frames, n_evicted);
  return RKV_OK;
}
