/*
 * rkv.h -- C ABI of librkv.so: rolling KV cache + fused 3D-RoPE attention for
 * NVIDIA B200 (sm_100a).
 *
 * Three operations make up the per-layer hot path of a streaming
 * autoregressive-diffusion video model (Rolling Forcing as the proxy):
 *
 *   rope3d_apply         3D rotary embedding over (t, h, w) of Q or K
 *   attn_fwd_varlen      softmax attention, RoPE fused into its load stage,
 *                        several sequences (e.g. the denoise pass and the
 *                        cache-update pass) in one launch, optional
 *                        frame-block-causal mask
 *   kvcache_ring_update  insert whole frames into a per-layer ring cache,
 *                        evicting the oldest frames (optionally keeping a
 *                        pinned prefix of first frames);
 *                        kvcache_ring_update_rope rotates K on the way in
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Tensors are bfloat16, token-major [L][H][D] ("row" = one token, H heads
 *    of D = 128 values).  A row stride (in ELEMENTS) lets a caller pass a view
 *    into a wider buffer (e.g. the Q part of a fused QKV projection); it must
 *    be >= H*D and make every row start 16-byte aligned.  No call transposes.
 *  - Pointers named device are CUDA device (or managed) memory; the caller owns
 *    all of it.  The library allocates no device memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls enqueue work and return without synchronising.
 *  - Every call returns an rkv_status.  Invalid arguments are rejected on the
 *    host BEFORE anything is launched; nothing traps or asserts on the device.
 *    rkv_last_error_string() describes the last failure of the calling thread.
 *  - Functions keep no state between calls (the ring state lives in the
 *    caller's rkv_ring) except two fixed device words per GPU: the status of
 *    attn_fwd_varlen_noalloc and the ring inserts' timeout flag.
 */
#ifndef RKV_H
#define RKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RKV_OK = 0,
  RKV_ERR_INVALID_ARG = 1, /* rejected on the host, nothing launched           */
  RKV_ERR_UNSUPPORTED = 2, /* well-formed but outside what the kernels handle  */
  RKV_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed                */
  RKV_ERR_TIMEOUT = 4,     /* a bounded device-side wait gave up (see below)   */
  RKV_ERR_DEVICE_CHECK = 5 /* a debug launch's device-side index check failed  */
} rkv_status;

/*
 * 3D-RoPE parameters.
 *
 * Source: "Amazon and Reactor tune Trainium for real-time video generation",
 * section "Three problems for generic compilers": in video, RoPE rotates by
 * three positions -- height, width and time -- instead of one.  The pages give
 * no formula; this library takes the plainest reading:
 *   token i of a sequence whose first frame has time index t0, on a
 *   grid_h x grid_w frame grid (F = grid_h*grid_w tokens per frame, row-major):
 *       t = t0 + i / F,  h = (i % F) / grid_w,  w = i % grid_w
 *   the D/2 rotary pairs are adjacent elements (2j, 2j+1); the first pairs_t
 *   pairs use t, the next pairs_h use h, the last pairs_w use w
 *   (pairs_t + pairs_h + pairs_w == D/2; 22/21/21 for D = 128);
 *   pair with local index k on an axis with n pairs turns by
 *       angle = pos * theta_axis^(-k/n)   (theta_axis = theta unless the
 *       per-axis bases below are set)
 *   y0 = x0 cos(angle) - x1 sin(angle);  y1 = x0 sin(angle) + x1 cos(angle).
 */
typedef struct {
  int32_t grid_h, grid_w;            /* frame grid; tokens per frame = grid_h*grid_w */
  int32_t pairs_t, pairs_h, pairs_w; /* rotary pairs per axis, sum = D/2            */
  float theta;                       /* frequency base of the t axis (and of h, w
                                        when theta_h / theta_w are 0); 10000        */
  float theta_h, theta_w;            /* frequency bases of the h and w axes; 0 =
                                        theta                                       */
  int32_t layout;                    /* RKV_ROPE_ADJACENT or RKV_ROPE_HALF          */
} rkv_rope3d;

/* rkv_rope3d.layout: which elements form rotary pair j (0 <= j < D/2) */
#define RKV_ROPE_ADJACENT 0 /* elements 2j and 2j+1 (the reading above)            */
#define RKV_ROPE_HALF 1     /* elements j and j + D/2 ("rotate-half"); the pages
                               leave the layout open, so both are offered      */

/*
 * rope3d_apply -- y = RoPE3D(x) for every row and head.
 *
 * Source: "Optimizing Real-Time Video Generation on Trainium Chips", item 6
 * "Neuron Kernel Interface" (a dedicated 3D-RoPE kernel replaced the generic
 * path) and the RoPE reading above.
 *
 *   x, y          device bf16 [L][H][D]; y may equal x (in place), otherwise
 *                 the two must not overlap.
 *   L             rows (tokens), >= 0 (0 = no-op).  H >= 1.  D == 128.
 *   x_row_stride, y_row_stride   elements between consecutive rows.
 *   t0            time index of row 0's frame.
 *   rope          frame grid and axis split.
 * Precision: rotation in fp32 with a compensated (error-free-transform) path
 * and fp64-derived cos/sin, rounded to nearest-even bf16: every output is
 * within 1 bf16 ulp of the exactly rounded result.
 * Errors: RKV_ERR_INVALID_ARG for null pointers, D != 128, bad pairs/grid,
 * misaligned rows or overlapping non-identical x/y.
 */
rkv_status rope3d_apply(const void* x, void* y, int64_t L, int32_t H, int32_t D,
                        int64_t x_row_stride, int64_t y_row_stride, int32_t t0,
                        const rkv_rope3d* rope, void* stream);

/*
 * rope3d_apply_batch -- rope3d_apply on several tensors (e.g. a layer's Q and
 * K) that share H, D and rope, in one launch.
 *
 * Source: as rope3d_apply; the pages rotate Q and K of the same window
 * ("Amazon and Reactor tune Trainium for real-time video generation", section
 * "Three problems for generic compilers").
 *
 *   tensors       host array of n descriptors (caller-owned, read during the
 *                 call): x, y, L, x_row_stride, y_row_stride, t0 exactly as
 *                 rope3d_apply's arguments of the same names.
 *   n             0 .. RKV_ROPE_BATCH_MAX (0 = no-op).
 * Each tensor's y receives what rope3d_apply on that tensor alone would write
 * (bit-identical).  With the adjacent layout all tensors share one launch
 * (CTAs shared out by rows); with the rotate-half layout they launch one after
 * another on `stream`.
 * Errors: those of rope3d_apply for any tensor, plus RKV_ERR_INVALID_ARG for
 * n out of range, a NULL array, or an output that overlaps another tensor's
 * input or output.
 */
#define RKV_ROPE_BATCH_MAX 8

typedef struct {
  const void* x;
  void* y;
  int64_t L;
  int64_t x_row_stride;
  int64_t y_row_stride;
  int32_t t0;
} rkv_rope_tensor;

rkv_status rope3d_apply_batch(const rkv_rope_tensor* tensors, int32_t n, int32_t H, int32_t D,
                              const rkv_rope3d* rope, void* stream);

/* flags of rkv_attn_seq */
#define RKV_ROPE_Q 1u /* rotate Q rows by RoPE3D (positions from q_t0) in-kernel */
#define RKV_ROPE_K 2u /* rotate K rows by RoPE3D (positions from k_t0) in-kernel */

/*
 * One sequence of a batched attention launch.
 *
 * Source: SDPA of a 23,400-token query window over a 32,760-token context,
 * 12 heads ("A kernel-centric path to real-time video generation on
 * Trainium", ai4snews summary, second paragraph); two passes per window --
 * denoise, then cache update -- with different attention lengths, batched so
 * the lighter pass does not strand hardware ("Optimizing Real-Time Video
 * Generation on Trainium Chips", item 8 "Model structure optimizations";
 * "Amazon and Reactor tune Trainium for real-time video generation", section
 * "Three problems for generic compilers").
 *
 *   q, k, v       device bf16 [Lq][H][D], [Lk][H][D], [Lk][H][D]
 *   o             device bf16 [Lq][H][D]; may share no byte with any q, k, v
 *                 or other o of the launch (row-strided views with disjoint
 *                 heads of one tensor, e.g. head slices, are fine)
 *   *_stride      elements between consecutive rows (>= H*D, 16-B aligned rows)
 *   Lq, Lk        >= 1 each
 *   q_t0, k_t0    time index of the first query / key frame (used for RoPE)
 *   block_frames  0 = every key visible.  > 0 = frame-block causal: query row r
 *                 lies in key frame qf = q_frame_offset + r / F, key c in key
 *                 frame c / F, and key c is visible iff
 *                 floor(kf / block_frames) <= floor(qf / block_frames).
 *                 (F = tokens per frame from rkv_rope3d.)
 *   q_frame_offset key-frame index of query frame 0 (>= 0); the bottom-right
 *                 alignment (query window = last frames of the context) is
 *                 Lk/F - Lq/F.
 *   flags         RKV_ROPE_Q | RKV_ROPE_K
 */
typedef struct {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  int64_t q_stride, k_stride, v_stride, o_stride;
  int32_t Lq, Lk;
  int32_t q_t0, k_t0;
  int32_t q_frame_offset;
  int32_t block_frames;
  uint32_t flags;
  int32_t reserved; /* must be 0 */
} rkv_attn_seq;

#define RKV_MAX_SEQS 16

/*
 * attn_fwd_varlen -- O = softmax(mask(RoPE(Q) RoPE(K)^T * softmax_scale)) V
 * for every sequence and head, in ONE kernel launch.
 *
 *   seqs, n_seqs   host array of 1..RKV_MAX_SEQS descriptors (read during the
 *                  call only)
 *   H >= 1, D == 128, softmax_scale > 0 (1/sqrt(128) for SDPA)
 *   rope           frame grid / axis split; required (also defines F for the
 *                  mask) even when no sequence sets a RoPE flag
 *   workspace      device memory, 16-byte aligned, not used by another call
 *                  in flight; at least 256 bytes (the device status word).
 *                  attn_fwd_varlen_workspace_size() bytes (about 20 MB on a
 *                  B200) also hold partial results for the tail of the
 *                  persistent grid: when the last wave of work units is at
 *                  most half full, those units run as two halves over their
 *                  key tiles and a second kernel merges the halves.  With a
 *                  smaller workspace the call runs without that split.
 * A query row that sees no key gets zeros.  Precision: bf16 operands, fp32
 * accumulation and softmax, bf16 output.
 * Errors: RKV_ERR_INVALID_ARG (shapes, pointers, alignment, overlap of o with
 * inputs), RKV_ERR_UNSUPPORTED (RoPE position range too large for the on-chip
 * cos/sin table, D != 128), RKV_ERR_CUDA.  A device-side wait that exceeds
 * its time limit makes the kernel stop early and record RKV_ERR_TIMEOUT in the
 * workspace; rkv_attn_status() reads it back.
 */
size_t attn_fwd_varlen_workspace_size(const rkv_attn_seq* seqs, int32_t n_seqs, int32_t H,
                                      int32_t D);
rkv_status attn_fwd_varlen(const rkv_attn_seq* seqs, int32_t n_seqs, int32_t H, int32_t D,
                           float softmax_scale, const rkv_rope3d* rope, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * rkv_attn_mask_rows -- the mask and key-tile plan attn_fwd_varlen would use,
 * evaluated on the host by the same functions the kernel compiles (a debug
 * and test aid; needs no GPU).  The frame-block-causal mask ("Amazon and
 * Reactor tune Trainium for real-time video generation", section "Three
 * problems for generic compilers", the two passes of different lengths) makes
 * every query row see a prefix of the keys, so a row's mask is one number.
 *
 *   seqs, n_seqs, H, rope   as for attn_fwd_varlen; only Lq, Lk,
 *                  q_frame_offset, block_frames and the frame grid are read
 *                  (tensor pointers and strides may be anything)
 *   row_limit      host int64 [sum of Lq]: for sequence i (in the order given)
 *                  and its query row r, entry Lq_0 + ... + Lq_{i-1} + r is the
 *                  number of leading keys row r attends to; keys at or past it
 *                  are masked
 *   unit_tiles     optional host int32 [4 * n_units]: per work unit in launch
 *                  order, (sequence index in the order given, head, 512-row
 *                  query block, key tiles of 128 keys the unit processes)
 *   n_units        optional out: number of work units, sum of H * ceil(Lq / 512)
 * Errors: RKV_ERR_INVALID_ARG (as attn_fwd_varlen for n_seqs, H, rope,
 * lengths, mask fields; row_limit NULL), RKV_ERR_UNSUPPORTED (n_seqs > 16).
 */
rkv_status rkv_attn_mask_rows(const rkv_attn_seq* seqs, int32_t n_seqs, int32_t H, const rkv_rope3d* rope,
                              int64_t* row_limit, int32_t* unit_tiles, int64_t* n_units);

/*
 * rkv_attn_status -- synchronise `stream` and return the device status word
 * an earlier attn_fwd_varlen left in `workspace` (RKV_OK or RKV_ERR_TIMEOUT),
 * then clear it.
 */
rkv_status rkv_attn_status(void* workspace, void* stream);

/*
 * attn_fwd_varlen_debug -- attn_fwd_varlen with test and debug aids: a record
 * of the mask the kernel actually applied, and stall injection for the
 * bounded device-side waits.  Same arguments as attn_fwd_varlen plus `dbg`.
 * It runs a separate instantiation of the attention kernel, compiled from the
 * same source with these aids added; results in `o` are those of
 * attn_fwd_varlen.  Adjacent RoPE pairs only (RKV_ERR_UNSUPPORTED otherwise).
 *
 * Mask record.  The frame-block-causal mask ("Amazon and Reactor tune
 * Trainium for real-time video generation", section "Three problems for
 * generic compilers": two passes per window with different attention
 * lengths) is applied on the device by the choice of key tiles a work unit
 * processes and by a per-element predicate on partial tiles.  With row_stats
 * set, every softmax thread counts, after that masking, the scores of its
 * query row that are not -inf (every other score of N(0,1)-sized inputs is
 * finite), and writes for (sequence i in the order given, query row r, head h)
 * at int32 index 4 * ((Lq_0 + ... + Lq_{i-1} + r) * H + h):
 *   [0] keys that entered the softmax, [1] the sum of their key indices
 *   (mod 2^32), [2] 1 + the largest such key index (0 if none),
 *   [3] 128-key tiles the row's work unit processed
 * (the two halves of a split tail unit add into one record).  For a row that
 * sees exactly the keys [0, n): n, n(n-1)/2, n, ceil(n/128).
 *
 * Index checks.  The debug instantiation also checks, before each global
 * store and TMA load it issues, the indices it computed against the launch's
 * shapes (head < H, query row < Lq, key tile inside [0, Lk), split-unit slot
 * inside the workspace); a failed check skips the store and records
 * RKV_ERR_DEVICE_CHECK in the workspace (rkv_attn_status reports it).  Nothing
 * traps.
 *
 * Stall injection (a test of the bounded waits that faults nothing): the
 * second CTA of the first CTA pair withholds one handoff, so the pair's MMA
 * issuer waits for it until the time limit, the kernel stops early and
 * records RKV_ERR_TIMEOUT in the workspace (rkv_attn_status reports it).
 * The outputs of that launch are then incomplete; the device stays usable.
 *
 *   dbg->row_stats   device int32 [(Lq_0 + ... + Lq_{n-1}) * H][4], 16-byte
 *                    aligned, or NULL (no record); zeroed by the call
 *   dbg->stall       RKV_DEBUG_STALL_NONE or one of the handoffs below
 *   dbg->timeout_us  limit of every device-side wait of this launch in
 *                    microseconds (0 = the default 2 s)
 * Errors: those of attn_fwd_varlen, plus RKV_ERR_INVALID_ARG for a NULL dbg,
 * an unknown stall or a misaligned row_stats.
 */
#define RKV_DEBUG_STALL_NONE 0u
#define RKV_DEBUG_STALL_V_READY 1u /* its first "V tile landed" arrive          */
#define RKV_DEBUG_STALL_K_READY 2u /* its first "K tile rotated" arrive         */
#define RKV_DEBUG_STALL_P_FULL 3u  /* its first softmax warp's first "P ready"  */

typedef struct {
  int32_t* row_stats;
  uint32_t stall;
  uint32_t timeout_us;
} rkv_attn_debug;

rkv_status attn_fwd_varlen_debug(const rkv_attn_seq* seqs, int32_t n_seqs, int32_t H, int32_t D,
                                 float softmax_scale, const rkv_rope3d* rope, void* workspace,
                                 size_t workspace_bytes, const rkv_attn_debug* dbg, void* stream);

/*
 * attn_fwd_varlen_noalloc -- attn_fwd_varlen without a caller workspace.
 *
 * The pages have no counterpart to this call; it exists for callers of this
 * library that cannot allocate device memory themselves: plugin and custom-op
 * hosts that hand a kernel only its input and output buffers, engines whose
 * device memory is fully pre-planned, and code that must not call cudaMalloc
 * (which can synchronise the device).  The caller still passes every input
 * and output; the few bytes of scratch the attention launch needs (its status
 * word, cleared at the start of every call) come from a fixed 256-byte array
 * inside librkv.so.  Every GPU that loads the library holds that array until
 * the process exits.  Nothing is allocated by this call.
 *
 *   seqs ... stream   as for attn_fwd_varlen
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and caches it; make that
 * first call before any stream capture on that device.
 * Sharing: every call on a device uses the same array, which keeps the last
 * call's contents.  Calls that overlap on the GPU (on different streams, or
 * from different host threads without ordering) race on it; serialise them.
 * Limit: the array holds only the 256 bytes a launch needs at least, so these
 * launches never split the tail of the grid (see attn_fwd_varlen's workspace)
 * and can be a few percent slower on full-size work; a launch whose minimum
 * scratch need exceeded the array would be rejected with
 * RKV_ERR_UNSUPPORTED.
 * A device-side timeout stops the kernel as in attn_fwd_varlen and is
 * recorded in the internal array; rkv_attn_noalloc_status reads it back.
 */
rkv_status attn_fwd_varlen_noalloc(const rkv_attn_seq* seqs, int32_t n_seqs, int32_t H, int32_t D,
                                   float softmax_scale, const rkv_rope3d* rope, void* stream);

/*
 * rkv_attn_noalloc_status -- rkv_attn_status for attn_fwd_varlen_noalloc:
 * synchronise `stream`, return the status word the last no-alloc launch on
 * the current device left in the library's internal array (RKV_OK or
 * RKV_ERR_TIMEOUT) and clear it.  Allocates nothing; like the launch it reads,
 * the first call on a device looks up the array's address.
 */
rkv_status rkv_attn_noalloc_status(void* stream);

/*
 * Per-layer rolling KV cache.
 *
 * Source: every layer reads and writes a rolling KV cache, and frames are
 * generated and evicted in a sliding window ("Amazon and Reactor tune Trainium
 * for real-time video generation", section "Three problems for generic
 * compilers"; a dedicated per-layer cache-copy kernel: "Optimizing Real-Time
 * Video Generation on Trainium Chips", item 6 "Neuron Kernel Interface").
 *
 * Layout: k and v are device bf16 [slots][tokens_per_frame][H][D], contiguous.
 * `count` = valid frames (0..slots).
 *
 * Pinned prefix (optional; the pages describe only the sliding window; this
 * is the common variant that keeps a stream's first frames, "attention
 * sinks", out of eviction): the first `pinned` slots (0 <= pinned < slots)
 * take the first `pinned` frames ever inserted and are never overwritten;
 * every later frame rolls through slots [pinned, slots).  pinned = 0 is the
 * plain ring.
 *
 * `head` = the slot of [pinned, slots) the next rolling frame goes to; a new
 * ring starts with head = pinned, count = 0, and head stays at pinned until
 * the pinned slots are all filled.  Logical frame j (0 = oldest valid) lives
 * in slot j when j < pinned, else in slot
 *   pinned + (head - pinned - (count - pinned) + (j - pinned)) mod (slots - pinned)
 * which for pinned = 0 is (head - count + j) mod slots.  A ring filled from
 * empty has its valid frames in the slot prefix [0, count), in any state.
 */
typedef struct {
  void* k;
  void* v;
  int32_t slots;
  int32_t tokens_per_frame;
  int32_t H;
  int32_t D;
  int32_t head;   /* updated by kvcache_ring_update (host side) */
  int32_t count;  /* updated by kvcache_ring_update (host side) */
  int32_t pinned; /* slots of the pinned prefix; fixed for the ring's life */
} rkv_ring;

/*
 * kvcache_ring_update -- insert n_frames whole frames of K and V.
 *
 *   ring           caller's ring; head/count are updated on success
 *   k_new, v_new   device bf16 [n_frames * tokens_per_frame][H][D] with row
 *                  stride new_row_stride (elements); must not overlap the ring
 *   n_frames       0..capacity (0 = no-op), capacity = the free pinned slots
 *                  max(0, pinned - count) plus the rolling slots
 *                  slots - pinned (= slots without a pinned prefix)
 *   n_evicted      optional out: frames dropped = max(0, count + n - slots)
 * The first p = min(n, max(0, pinned - count)) frames go to slots count,
 * count + 1, ...; frame i >= p goes to slot
 * pinned + (head - pinned + i - p) mod (slots - pinned).  Then
 * head = pinned + (head - pinned + n - p) mod (slots - pinned) and
 * count = min(slots, count + n).  Without a pinned prefix frame i goes to
 * slot (head + i) mod slots.  Evicted frames are overwritten, not cleared:
 * no bytes move for eviction.
 * The copy runs on the TMA bulk-copy engine; each of its waits on a bulk
 * load is bounded (1 s), after which the kernel stops, sets a per-GPU flag and
 * the insert is incomplete (its destination slots may be partly written):
 * rkv_ring_status reads that flag.
 * Errors: RKV_ERR_INVALID_ARG (n_frames above capacity or < 0, null
 * pointers, pinned/head/count out of range or inconsistent, D != 128,
 * misalignment, overlap).
 */
rkv_status kvcache_ring_update(rkv_ring* ring, const void* k_new, const void* v_new,
                               int64_t new_row_stride, int32_t n_frames, int32_t* n_evicted,
                               void* stream);

/*
 * kvcache_ring_update_rope -- kvcache_ring_update with K rotated on the way in.
 *
 * Source: the cache holds keys already rotated, so later passes read them
 * without a RoPE pass, and RoPE and the per-layer cache copy are the two
 * kernels the pages single out ("Optimizing Real-Time Video Generation on
 * Trainium Chips", item 6 "Neuron Kernel Interface"; "Amazon and Reactor tune
 * Trainium for real-time video generation", section "Three problems for
 * generic compilers").  One pass reads raw K and V once and writes the ring
 * once: HBM bytes are those of the plain copy.
 *
 *   ring, k_new, v_new, new_row_stride, n_frames, n_evicted
 *                  as for kvcache_ring_update; k_new holds UNROTATED keys
 *   t0             time index of the first inserted frame: frame i is rotated
 *                  with t = t0 + i, rows within a frame with their (h, w)
 *   rope           frame grid and axis split; grid_h*grid_w must equal the
 *                  ring's tokens_per_frame
 * The ring's K slots receive exactly what rope3d_apply(k_new) would write
 * (same arithmetic, same rounding, within 1 bf16 ulp of the exact rotation);
 * V slots receive v_new unchanged.  Slot, head, count and eviction follow
 * kvcache_ring_update.  With the adjacent layout V moves on the TMA
 * bulk-copy engine as in kvcache_ring_update (same bounded waits: a wait that
 * gives up sets the flag rkv_ring_status reports, and the insert's slots may
 * be partly written) while the other threads of each CTA rotate K.
 * Errors: those of kvcache_ring_update and rope3d_apply, plus
 * RKV_ERR_INVALID_ARG when the frame grid does not match tokens_per_frame.
 */
rkv_status kvcache_ring_update_rope(rkv_ring* ring, const void* k_new, const void* v_new,
                                    int64_t new_row_stride, int32_t n_frames, int32_t t0,
                                    const rkv_rope3d* rope, int32_t* n_evicted, void* stream);

/*
 * kvcache_ring_update_debug -- kvcache_ring_update with stall injection, a
 * test of the copy's bounded waits that faults nothing.  Same arguments plus
 * `dbg`; with dbg->stall = RKV_DEBUG_STALL_BULK_LOAD the first CTA declares
 * 16 bytes more for its first piece than it loads, so that piece's wait runs
 * out after dbg->timeout_us microseconds (0 = the default 1 s): the copy stops
 * early, sets the flag rkv_ring_status reports, and the insert is incomplete
 * (head and count still advance, as for a normal insert).  With
 * RKV_DEBUG_STALL_NONE it is kvcache_ring_update with that wait limit.
 * Errors: those of kvcache_ring_update, plus RKV_ERR_INVALID_ARG for a NULL
 * dbg or an unknown stall.
 */
#define RKV_DEBUG_STALL_BULK_LOAD 1u

typedef struct {
  uint32_t stall;
  uint32_t timeout_us;
} rkv_ring_debug;

rkv_status kvcache_ring_update_debug(rkv_ring* ring, const void* k_new, const void* v_new,
                                     int64_t new_row_stride, int32_t n_frames, int32_t* n_evicted,
                                     const rkv_ring_debug* dbg, void* stream);

/*
 * rkv_ring_status -- synchronise `stream` and report whether a ring insert on
 * the current GPU gave up on a bounded device-side wait since the last call:
 * RKV_ERR_TIMEOUT (the flag is then cleared) or RKV_OK.  Errors:
 * RKV_ERR_CUDA when the flag cannot be read.
 */
rkv_status rkv_ring_status(void* stream);

/* Slot of logical frame j (0 = oldest valid), or -1 when j is not a valid
 * frame or the ring is malformed. */
int32_t rkv_ring_slot(const rkv_ring* ring, int32_t logical_frame);

/* Text of the last error returned on the calling thread ("" if none). */
const char* rkv_last_error_string(void);

/* Library version, major*10000 + minor*100 + patch.  A caller compiled
 * against this header can compare it with RKV_VERSION: the structs above
 * changed layout between minor versions (rkv_ring gained `pinned`,
 * rkv_rope3d its per-axis bases and layout in 0.2). */
#define RKV_VERSION 200
int32_t rkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RKV_H */
