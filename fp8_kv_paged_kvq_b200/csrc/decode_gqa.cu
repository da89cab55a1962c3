// Split-KV paged decode attention for query-head groups of up to 16 heads per
// KV head (FP8 E4M3 or BF16 cache), plus the log-sum-exp combine.
//
// What it computes: one new query token per sequence attends over the
// sequence's cached tokens through its page table; FP8 codes are converted
// on read ("Công thức của Cloudflare để phục vụ Kimi và GLM ..." (manulx.blog),
// section "Bộ nhớ đệm KV FP8 tăng gấp đôi dung lượng ngữ cảnh"; "Cloudflare:
// Kleinere Modellbereitstellung senkt Speicherbedarf, doch Sicherheit wird zum
// Prüfstein" (remio.ai), section "Warum kleinere Cloudflare-Caches reine
// Geschwindigkeit schlagen").  Decode is bound by memory bandwidth, so the
// design goal is to keep HBM busy:
//
//  * Work split.  The work units are 16-token tiles of one (sequence, KV
//    head) segment, flattened in (b, h, tile) order after aborted and empty
//    sequences are dropped.  Persistent CTA c takes one contiguous range of
//    units: [c*U/N, (c+1)*U/N) when all sequences have the same length (with
//    N a multiple of the segments when there are CTAs enough, so that ranges
//    start on segment edges), and for ragged batches equal shares of
//    weighted units, each segment counting kPieceCost more, so that a CTA
//    crossing many short segments gets fewer tiles.  A CTA's range covers a
//    few segments ("pieces").  Each piece leaves one partial (o, lse) in the
//    workspace at slot c + segment, which is unique because both c and the
//    segment index grow along the unit order.  A combine launch merges the
//    partials of each segment.
//  * Pipeline.  Every warp streams its own tiles (n = warp + NW*k of the
//    CTA's range) through S private ring slots: lane 0 issues the TMA loads
//    of a tile (16 rows of K and of V for one page and head, 128-byte
//    swizzle) completed on the slot's mbarrier, and re-issues the slot as soon
//    as the warp holds that tile's fragments in registers.  Each warp keeps
//    its own online-softmax state; the warps' states are merged per piece.
//  * Math.  QK^T and PV run on tensor cores (mma.m16n8k16, FP32
//    accumulate) with the token axis as M and the 8 query heads of a group
//    as N, so no MMA row is padding.  E4M3 codes become f16 with the hardware
//    conversion (exact: every E4M3 value is an f16 value); per-tensor and
//    per-head scales are folded into the score scale and the output.  The
//    probability tile is moved from the score layout into the PV operand
//    layout with movmatrix.  The BF16 cache uses bf16 MMAs and splits P
//    into a bf16 high and low part so that P keeps 16 significant bits.
//    V's d axis (and K's, consistently with Q) is permuted per thread so
//    that each thread reads whole 16-byte swizzled chunks with
//    conflict-free shared loads.
#include <mutex>

#include "kvq_device.cuh"
#include "kvq_internal.h"
#include "kvq_decode.h"

namespace kvq {

// Largest batch the decode kernels accept (three per-sequence arrays live in shared memory).
constexpr int32_t kGqaMaxBatch = 8000;   // three [B+1] arrays in shared memory

// ---------------------------------------------------------------------------
// Shared memory layout traits
// ---------------------------------------------------------------------------
template <bool FP8, int D>
struct Layout {
  static constexpr int kElem = FP8 ? 1 : 2;
  static constexpr int kRowBytes = D * kElem;          // one token row of one head
  static constexpr int kTileBytes = 16 * kRowBytes;    // 16 tokens
  static constexpr bool kSw64 = (kRowBytes == 64);     // fp8, D = 64
  static constexpr int kBoxBytes = kSw64 ? 64 : 128;   // inner extent of one TMA box
  static constexpr int kBoxes = kRowBytes / kBoxBytes; // boxes per tile
  static constexpr int kBoxElems = kBoxBytes / kElem;
  static constexpr int kKSteps = D / 16;               // MMA k-steps over the head dim
  static constexpr int kMTiles = D / 16;               // V^T row tiles
  static constexpr int kKChunks = kRowBytes / 64;      // 16-byte K chunks per thread and row
  static constexpr int kKStepsPerChunk = 16 / (4 * kElem);

  // Byte offset of 16-byte chunk c of row r inside a swizzled tile.
  static __device__ __forceinline__ uint32_t chunk_off(int r, int c) {
    if (kSw64) return r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
    return (c >> 3) * 2048 + r * 128 + (((c & 7) ^ (r & 7)) << 4);
  }
  // K chunk loaded by thread-in-group tig in its i-th load of a row.
  static __device__ __forceinline__ int k_chunk(int i, int tig) {
    if (kKChunks == 4) return 4 * tig + ((i + 2 * (tig >> 1)) & 3);
    return kKChunks * tig + i;
  }
  // First of the four head dims that k-step j covers for thread tig.
  static __device__ __forceinline__ int k_dbase(int j, int tig) {
    return k_chunk(j / kKStepsPerChunk, tig) * (16 / kElem) + 4 * (j % kKStepsPerChunk);
  }
  // Head dim of output row r (0: row g, 1: row g+8) of V^T m-tile i for group g.
  static __device__ __forceinline__ int v_dim(int i, int r, int g) {
    if (!FP8 && D == 128) return (i < 4 ? 8 * g + 2 * i : 64 + 8 * g + 2 * (i - 4)) + r;
    return (D / 8) * g + 2 * i + r;
  }
};

// ---------------------------------------------------------------------------
// Kernel parameters
// ---------------------------------------------------------------------------
struct GqaParams {
  CacheView c;
  const uint16_t* q;
  int32_t Hq, G;
  const int32_t* block_table;
  int32_t max_pages;
  const int32_t* seq_lens;
  int32_t B;
  const uint8_t* abort_mask;
  float sm_scale;
  float* out;
  float* lse;
  int32_t* ws_pre;   // [B+2] unit prefix, then the count of working CTAs (written by CTA 0)
  int32_t* ws_bounds;  // [num_ctas+1] first unit of each working CTA, then U
  float* ws_lse;     // [slots][G]
  float* ws_o;       // [slots][G][Dv]
  int32_t num_ctas;
};

// Tokens of sequence b that decode reads (0 if aborted; the abort mask is
// consulted only when use_abort is set).
__device__ __forceinline__ int32_t seq_tokens(const GqaParams& p, int b, bool use_abort) {
  if (use_abort && p.abort_mask != nullptr && p.abort_mask[b]) return 0;
  int64_t n = p.seq_lens[b];
  n = n < 0 ? 0 : n;
  const int64_t cap = static_cast<int64_t>(p.max_pages) * p.c.ps;
  return static_cast<int32_t>(n > cap ? cap : n);
}

// Each (sequence, KV head) segment with tiles also carries kPieceCost
// virtual units in the split: a piece ends with the warps' merge and the
// partial's write, and the next one starts with its query and scale loads,
// about as long as this many tiles take to stream.  Without them a CTA whose
// range crosses many short segments ends well after the others.
constexpr int32_t kPieceCost = 48;

// Exclusive prefixes over b of Hkv * tiles_b (pre[0..B], the units) and of
// Hkv * (tiles_b + kPieceCost if tiles_b > 0) (wpre[0..B], the weighted units
// the split divides), tiles_b = ceil(tokens_b / 16): each thread sums a run of
// sequences, a warp scan and the warps' totals give each run its start.
// Also keeps each sequence's token count in ntok[b].  Called by all threads
// of the block; scratch holds two ints per warp.
__device__ void block_prefix_units(const GqaParams& p, int32_t* pre, int32_t* wpre,
                                   int32_t* ntok, int32_t* scratch, bool use_abort) {
  const int nthr = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = nthr >> 5;
  const int per = (p.B + nthr - 1) / nthr;
  const int lo = min(p.B, tid * per), hi = min(p.B, lo + per);
  auto units = [&](int b) { return p.c.Hkv * ((seq_tokens(p, b, use_abort) + 15) >> 4); };
  int32_t sum = 0, wsum = 0;
  for (int b = lo; b < hi; ++b) {
    const int32_t x = units(b);
    sum += x;
    wsum += x > 0 ? x + p.c.Hkv * kPieceCost : 0;
  }
  int32_t incl = sum, wincl = wsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    const int32_t wv = __shfl_up_sync(0xffffffffu, wincl, o);
    if (lane >= o) {
      incl += v;
      wincl += wv;
    }
  }
  if (lane == 31) {
    scratch[warp] = incl;
    scratch[nw + warp] = wincl;
  }
  __syncthreads();
  int32_t run = incl - sum, wrun = wincl - wsum;
  for (int w = 0; w < warp; ++w) {
    run += scratch[w];
    wrun += scratch[nw + w];
  }
  for (int b = lo; b < hi; ++b) {
    pre[b] = run;
    wpre[b] = wrun;
    ntok[b] = seq_tokens(p, b, use_abort);
    const int32_t x = units(b);
    run += x;
    wrun += x > 0 ? x + p.c.Hkv * kPieceCost : 0;
  }
  if (tid == nthr - 1) {                    // the last run ends at B
    pre[p.B] = run;
    wpre[p.B] = wrun;
  }
  __syncthreads();
}

// First real unit at or after weighted position w (0 <= w <= wpre[B]): in
// sequence b each of its Hkv segments spans tiles_b + kPieceCost weighted
// units, the virtual ones first.
__device__ __forceinline__ int32_t real_unit(const GqaParams& p, const int32_t* pre,
                                             const int32_t* wpre, int64_t w) {
  if (w >= wpre[p.B]) return pre[p.B];
  int lo = 0, hi = p.B;                     // largest b with wpre[b] <= w (a sequence with tiles)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (wpre[mid] <= w) lo = mid; else hi = mid;
  }
  const int32_t tiles = (pre[lo + 1] - pre[lo]) / p.c.Hkv;
  const int32_t len = tiles + kPieceCost;
  const int32_t off = static_cast<int32_t>(w - wpre[lo]);
  const int32_t h = off / len, r = off - h * len;
  return pre[lo] + h * tiles + max(0, r - kPieceCost);
}

// CTAs (or CTA pairs) that get units: at most num_ctas, at least min_units
// units each when there are enough (the 8-head kernel asks for
// kMinTilesPerCta: fewer, longer ranges for small batches, so fewer pieces to
// merge and more tiles in flight per warp), and never more than U, so that
// every working CTA owns at least one unit.  The decode kernels write the
// count they used next to the unit prefix, where the combine reads it.
constexpr int32_t kMinTilesPerCta = 32;
__device__ __forceinline__ int64_t working_ctas(int64_t num_ctas, int64_t U, int64_t min_units) {
  const int64_t n = U / min_units;
  return min(num_ctas, n > 1 ? n : (U > 0 ? int64_t{1} : int64_t{0}));
}

// Segment containing unit u: largest b with pre[b] <= u (pre has B+1 entries).
__device__ __forceinline__ int find_seq(const int32_t* pre, int B, int32_t u) {
  int lo = 0, hi = B;            // invariant: pre[lo] <= u < pre[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (pre[mid] <= u) lo = mid; else hi = mid;
  }
  return lo;
}

struct Piece {
  int32_t b, h, seg;    // sequence, kv head, segment index b*Hkv + h
  int32_t t0, nt;       // first tile in the segment, tiles in this piece
  int32_t n0;           // first CTA-local tile number of the piece
  int32_t ntok;         // tokens of the sequence
};

// Next piece starting at unit u (< u1).  pre is followed in shared memory
// by the weighted prefix and the sequences' token counts (B+1 each).
__device__ __forceinline__ Piece make_piece(const GqaParams& p, const int32_t* pre, int32_t u,
                                            int32_t u1, int32_t n0) {
  Piece pc;
  pc.b = find_seq(pre, p.B, u);
  const int32_t tiles_b = (pre[pc.b + 1] - pre[pc.b]) / p.c.Hkv;
  const int32_t r = u - pre[pc.b];
  pc.h = r / tiles_b;
  pc.t0 = r - pc.h * tiles_b;
  pc.nt = min(tiles_b - pc.t0, u1 - u);
  pc.seg = pc.b * p.c.Hkv + pc.h;
  pc.n0 = n0;
  pc.ntok = pre[2 * (p.B + 1) + pc.b];
  return pc;
}

// ---------------------------------------------------------------------------
// The decode kernel
// ---------------------------------------------------------------------------
template <bool FP8, int D, int NT, int NW, int S>
struct GqaKernel {
  using L = Layout<FP8, D>;
  static constexpr int kThreads = NW * 32;
  static constexpr int kHeads = NT * 8;
  static constexpr int kStageBytes = 2 * L::kTileBytes;     // K tile then V tile
  static constexpr int kSlots = NW * S;                      // S ring slots per warp
  // shared memory carve-up (bytes)
  static constexpr int kOffStages = 0;
  static constexpr int kOffBars = kOffStages + kSlots * kStageBytes;
  static constexpr int kOffPage = kOffBars + kSlots * 8;
  static constexpr int kOffRedM = kOffPage + kSlots * 4;
  static constexpr int kOffRedL = kOffRedM + NW * kHeads * 4;
  static constexpr int kOffRedO = kOffRedL + NW * kHeads * 4;
  static constexpr int kOffMisc = kOffRedO + NW * kHeads * D * 4;   // flag, scratch
  static constexpr int kMiscInts = 4 + kThreads;
  // per-tensor or per-head scales of K and V, for up to kScaleHeads KV heads
  static constexpr int kScaleHeads = 64;
  static constexpr int kOffScales = kOffMisc + kMiscInts * 4;
  static constexpr int kOffPre = kOffScales + 2 * kScaleHeads * 4;
  // pre[B+1], wpre[B+1], ntok[B+1]
  static size_t smem_bytes(int B) { return 1024 + kOffPre + static_cast<size_t>(B + 1) * 12; }
};

// Registers: two CTAs per SM for one n-tile (128 per thread), and for the FP8
// kernel 120, so that the tag check launched before it (128 threads of 32
// registers per SM) fits beside its two CTAs and they start while it runs.
template <bool FP8, int D, int NT, int NW, int S>
__global__ void __maxnreg__(NT == 1 ? (FP8 ? 120 : 128) : 255)
    gqa_decode_kernel(const __grid_constant__ CUtensorMap k_map,
                      const __grid_constant__ CUtensorMap v_map, const GqaParams p) {
  using K = GqaKernel<FP8, D, NT, NW, S>;
  using L = typename K::L;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + K::kOffBars);
  int32_t* slot_page = reinterpret_cast<int32_t*>(smem + K::kOffPage);
  float* red_m = reinterpret_cast<float*>(smem + K::kOffRedM);
  float* red_l = reinterpret_cast<float*>(smem + K::kOffRedL);
  float* red_o = reinterpret_cast<float*>(smem + K::kOffRedO);
  volatile int32_t* abort_flag = reinterpret_cast<int32_t*>(smem + K::kOffMisc);
  int32_t* scratch = reinterpret_cast<int32_t*>(smem + K::kOffMisc) + 4;
  int32_t* pre = reinterpret_cast<int32_t*>(smem + K::kOffPre);
  int32_t* wpre = pre + p.B + 1;
  int32_t* ntok = wpre + p.B + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();                                 // the combine may launch (it waits for us)
  if (threadIdx.x == 0) {
    for (int i = 0; i < K::kSlots; ++i) mbar_init(&full[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (lane == 0) { tma_prefetch_desc(&k_map); tma_prefetch_desc(&v_map); }

  // The work plan.  Before the dependency wait the kernel reads only what the
  // kernel launched just before it does not write (sequence lengths,
  // block-table entries, per-tensor or per-head scales) and writes nothing to
  // global memory: it lays out the units as if no request were aborted and
  // looks up its first pages.  After the wait it
  // reads the abort mask and redoes the plan only if some request aborted.
  // The units go to the first N CTAs, every one of which owns at least one
  // unit (the combine relies on it).
  const int cw = warp;
  int64_t U = 0, N = 0;
  int32_t u0 = 0, u1 = 0, kw = 0;
  bool plain_split = false;                    // the plain c*U/N ranges
  auto plan = [&](bool use_abort) {
    block_prefix_units(p, pre, wpre, ntok, scratch, use_abort);  // includes __syncthreads
    U = pre[p.B];
    // Every sequence as long as the others (in tiles) and at least two CTAs
    // per segment: each segment gets the same number k >= 1 of CTAs, so CTA
    // boundaries fall on segment boundaries and no CTA holds two pieces.
    // Equal lengths with fewer CTAs (where idle CTAs would cost more than the
    // extra pieces): the stream-K split of the units, every CTA then holding
    // one or two pieces.  Ragged batches: the stream-K split of the weighted
    // units, each segment counting kPieceCost extra, so that a CTA whose
    // range crosses many short segments gets fewer tiles.
    const int32_t t0 = p.B > 0 ? pre[1] - pre[0] : 0;
    int uneven = 0;
    for (int b = threadIdx.x; b < p.B; b += blockDim.x) uneven |= (pre[b + 1] - pre[b]) != t0;
    uneven = __syncthreads_or(uneven);
    const int64_t segs = static_cast<int64_t>(p.B) * p.c.Hkv;
    const bool aligned = !uneven && t0 > 0 && 2 * segs <= p.num_ctas;
    if (aligned) {
      const int64_t tseg = U / segs;               // tiles of one segment
      int64_t k = p.num_ctas / segs;
      const int64_t kmax = tseg / kMinTilesPerCta;
      k = min(k, kmax > 1 ? kmax : int64_t{1});
      N = segs * k;
    } else {
      N = working_ctas(p.num_ctas, U, kMinTilesPerCta);
    }
    const bool works = static_cast<int64_t>(blockIdx.x) < N;
    plain_split = !uneven;                    // c*U/N, no weights
    if (!uneven) {
      u0 = works ? static_cast<int32_t>(U * blockIdx.x / N) : 0;
      u1 = works ? static_cast<int32_t>(U * (blockIdx.x + 1) / N) : 0;
    } else {                                    // equal shares of the weighted units
      const int64_t W = wpre[p.B];
      u0 = works ? real_unit(p, pre, wpre, W * blockIdx.x / N) : 0;
      u1 = works ? real_unit(p, pre, wpre, W * (blockIdx.x + 1) / N) : 0;
    }
    // warp cw takes the CTA's tiles n = cw + NW*k, k = 0 .. kw-1
    const int32_t n_cta = u1 - u0;
    kw = n_cta > cw ? (n_cta - cw + NW - 1) / NW : 0;
  };
  // TMA coordinates of warp-local tile k0 + lane (page id; kv head << 16 | row offset).
  auto lookup = [&](int32_t k0, int32_t& page, int32_t& hy) {
    page = 0;
    hy = 0;
    const int32_t k = k0 + lane;
    if (k < kw) {
      const int32_t u = u0 + cw + NW * k;
      const int b = find_seq(pre, p.B, u);
      const int32_t tiles_b = (pre[b + 1] - pre[b]) / p.c.Hkv;
      const int32_t r = u - pre[b];
      const int32_t h = r / tiles_b;
      const int32_t t = r - h * tiles_b;
      page = p.block_table[static_cast<int64_t>(b) * p.max_pages + (t * 16) / p.c.ps];
      hy = (h << 16) | ((t * 16) % p.c.ps);
    }
  };
  int32_t cur_page, cur_hy, nxt_page, nxt_hy, batch0 = 0;
  // Per-tensor or per-head scales into shared memory (made visible by the
  // plan's barriers).  They are read before the dependency wait too: only
  // kvq_scale_from_amax writes them, and it lets no kernel start before it
  // ends.
  if (FP8 && p.c.scale_mode <= 1 && p.c.Hkv <= K::kScaleHeads) {
    float* sk = reinterpret_cast<float*>(smem + K::kOffScales);
    const float* vs = p.c.v_pages ? p.c.v_scale : p.c.k_scale;
    const int nh = p.c.scale_mode == 0 ? 1 : p.c.Hkv;
    for (int i = threadIdx.x; i < nh; i += blockDim.x) {
      sk[i] = p.c.k_scale[i];
      sk[K::kScaleHeads + i] = vs[i];
    }
  }
  plan(false);
  lookup(0, cur_page, cur_hy);
  lookup(32, nxt_page, nxt_hy);

  pdl_wait();                                    // the previous kernel (validate) has finished
  if (p.abort_mask != nullptr) {
    int any = 0;
    for (int b = threadIdx.x; b < p.B; b += blockDim.x) any |= p.abort_mask[b];
    if (__syncthreads_or(any)) {
      plan(true);
      lookup(0, cur_page, cur_hy);
      lookup(32, nxt_page, nxt_hy);
    }
  }
  if (blockIdx.x == 0) {
    for (int b = threadIdx.x; b <= p.B; b += blockDim.x) p.ws_pre[b] = pre[b];
    // N, negated when the split is the weighted one (the combine then looks
    // the pieces up in the CTAs' starts rather than in c*U/N)
    if (threadIdx.x == 0) {
      p.ws_pre[p.B + 1] = plain_split ? static_cast<int32_t>(N) : -static_cast<int32_t>(N);
      p.ws_bounds[N] = static_cast<int32_t>(U);
    }
  }
  // where this CTA's units start, for the combine's piece lookup
  if (threadIdx.x == 0 && static_cast<int64_t>(blockIdx.x) < N) p.ws_bounds[blockIdx.x] = u0;
  if (u0 >= u1) return;                          // no units: nothing issued, nothing to wait on

  // ---------------- this warp's pipeline ----------------
  // The warp keeps its tiles in its own S slots (slot k % S).  When it has
  // pulled tile k's fragments into registers it issues the TMA loads of tile
  // k + S into the same slot.  The loads are marked evict-first in L2: the
  // cache is streamed once per call.
  uint64_t* my_full = full + cw * S;
  uint8_t* my_stage = smem + K::kOffStages + cw * S * K::kStageBytes;
  int32_t* my_page = slot_page + cw * S;
  const uint64_t l2_stream = l2_policy_evict_first();
  int32_t issued = 0;                            // tiles of this warp issued so far
  // Issue warp-local tile `issued` (all lanes call; tiles go out in order).
  auto issue_next = [&]() {
    const int32_t k = issued++;
    if (k >= batch0 + 32) {                      // warp-uniform
      cur_page = nxt_page;
      cur_hy = nxt_hy;
      batch0 += 32;
      lookup(batch0 + 32, nxt_page, nxt_hy);
    }
    const int32_t page = __shfl_sync(0xffffffffu, cur_page, k - batch0);
    const int32_t hy = __shfl_sync(0xffffffffu, cur_hy, k - batch0);
    if (lane == 0) {
      const int sl = k % S;
      my_page[sl] = page;
      uint8_t* st = my_stage + sl * K::kStageBytes;
      fence_proxy_async_smem();                  // earlier reads of this slot before the TMA writes
      mbar_arrive_expect_tx(&my_full[sl], K::kStageBytes);
#pragma unroll
      for (int x = 0; x < L::kBoxes; ++x) {
        tma_load_4d_hint(st + x * 2048, &k_map, &my_full[sl], x * L::kBoxElems, hy & 0xFFFF,
                         hy >> 16, page, l2_stream);
        tma_load_4d_hint(st + L::kTileBytes + x * 2048, &v_map, &my_full[sl], x * L::kBoxElems,
                         hy & 0xFFFF, hy >> 16, page, l2_stream);
      }
    }
  };
  while (issued < S && issued < kw) issue_next();

  const int g = lane >> 2, tig = lane & 3;
  const float kNegInf = -__int_as_float(0x7f800000);
  // Scores are exponentiated against a per-head reference max that only moves
  // when a score exceeds it by more than kSlack (base-2 units): probabilities
  // then stay <= 2^kSlack, exact in f16 and fp32, and the cross-lane max and
  // the accumulator rescale run only on the rare tiles that move it.
  constexpr float kSlack = 8.0f;
  const bool tok_mode = FP8 && p.c.scale_mode == 2;

  int32_t n_begin = 0;
  for (int32_t u = u0; u < u1;) {
    const Piece pc = make_piece(p, pre, u, u1, n_begin);
    // per-segment constants
    const int hk = pc.h;
    float alpha = p.sm_scale * kLog2e, vscale = 1.0f;
    if (FP8 && p.c.scale_mode <= 1) {
      const int i = p.c.scale_mode == 0 ? 0 : hk;
      if (p.c.Hkv <= K::kScaleHeads) {
        const float* sk = reinterpret_cast<const float*>(smem + K::kOffScales);
        alpha *= sk[i];
        vscale = sk[K::kScaleHeads + i];
      } else {
        alpha *= p.c.k_scale[i];
        vscale = (p.c.v_pages ? p.c.v_scale : p.c.k_scale)[i];
      }
    }
    // Q fragments (B operand of QK^T): head nt*8+g, dims k_dbase(j)..+3
    uint32_t qb[NT][L::kKSteps][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int hq = nt * 8 + g;
      const bool valid = hq < p.G;
      const uint16_t* qrow =
          p.q + (static_cast<int64_t>(pc.b) * p.Hq + hk * p.G + (valid ? hq : 0)) * D;
#pragma unroll
      for (int j = 0; j < L::kKSteps; ++j) {
        uint2 w = make_uint2(0u, 0u);
        if (valid) w = *reinterpret_cast<const uint2*>(qrow + L::k_dbase(j, tig));
        if (FP8) {
          qb[nt][j][0] = pack_f16x2(bf16lo_to_f32(w.x), bf16hi_to_f32(w.x));
          qb[nt][j][1] = pack_f16x2(bf16lo_to_f32(w.y), bf16hi_to_f32(w.y));
        } else {
          qb[nt][j][0] = w.x;
          qb[nt][j][1] = w.y;
        }
      }
    }
    float o_acc[NT][L::kMTiles][4];
    float m_ref[NT][2], l_run[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m_ref[nt][0] = m_ref[nt][1] = kNegInf;
      l_run[nt][0] = l_run[nt][1] = 0.0f;
#pragma unroll
      for (int i = 0; i < L::kMTiles; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) o_acc[nt][i][e] = 0.0f;
    }

    // first CTA-local tile of this warp in the piece
    int32_t n = pc.n0 + ((cw - pc.n0 % NW) + NW) % NW;
    for (; n < pc.n0 + pc.nt; n += NW) {
      const int32_t k = (n - cw) / NW;           // warp-local tile index
      const int sl = k % S;
      const uint32_t ph = static_cast<uint32_t>(k / S) & 1u;
      if (*abort_flag) continue;
      if (!mbar_wait(&my_full[sl], ph)) { *abort_flag = 1; continue; }
      const uint32_t kbase = smem_u32(my_stage + sl * K::kStageBytes);
      const uint32_t vbase = kbase + L::kTileBytes;
      const int32_t tok0 = (pc.t0 + (n - pc.n0)) * 16;   // first token of the tile
      const bool tail = tok0 + 16 > pc.ntok;

      // ---- fragments: K rows g, g+8; V rows 2tig, 2tig+1, 2tig+8, 2tig+9 ----
      uint4 kr[2][L::kKChunks];
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int i = 0; i < L::kKChunks; ++i)
          kr[r][i] = lds128(kbase + L::chunk_off(g + 8 * r, L::k_chunk(i, tig)));
      constexpr int kVWords = (FP8 && D == 64) ? 2 : ((!FP8 && D == 128) ? 8 : 4);
      uint32_t vr[4][kVWords];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = 2 * tig + (r & 1) + 8 * (r >> 1);
        if (FP8 && D == 64) {
          const uint2 w = lds64(vbase + L::chunk_off(row, g >> 1) + 8 * (g & 1));
          vr[r][0] = w.x; vr[r][1] = w.y;
        } else if (!FP8 && D == 128) {
          const uint4 a = lds128(vbase + L::chunk_off(row, g));
          const uint4 b = lds128(vbase + L::chunk_off(row, 8 + g));
          vr[r][0] = a.x; vr[r][1] = a.y; vr[r][2] = a.z; vr[r][3] = a.w;
          vr[r][4] = b.x; vr[r][5] = b.y; vr[r][6] = b.z; vr[r][7] = b.w;
        } else {
          const uint4 a = lds128(vbase + L::chunk_off(row, g));
          vr[r][0] = a.x; vr[r][1] = a.y; vr[r][2] = a.z; vr[r][3] = a.w;
        }
      }
      const int32_t page = tok_mode ? my_page[sl] : 0;
      __syncwarp();
      if (issued < kw) issue_next();             // refill this slot with tile k + S

      // ---- S^T = K Q^T : rows = tokens g, g+8; cols = heads (two chains) ----
      float sa[NT][4], sb[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sa[nt][e] = sb[nt][e] = 0.0f;
#pragma unroll
      for (int ci = 0; ci < L::kKChunks; ++ci) {
        const uint32_t w0[4] = {kr[0][ci].x, kr[0][ci].y, kr[0][ci].z, kr[0][ci].w};
        const uint32_t w1[4] = {kr[1][ci].x, kr[1][ci].y, kr[1][ci].z, kr[1][ci].w};
#pragma unroll
        for (int jj = 0; jj < L::kKStepsPerChunk; ++jj) {
          const int j = ci * L::kKStepsPerChunk + jj;
          uint32_t a0, a1, a2, a3;
          if (FP8) {
            e4m3x4_to_f16x2x2(w0[jj], a0, a2);   // row g:   dims d,d+1 | d+2,d+3
            e4m3x4_to_f16x2x2(w1[jj], a1, a3);   // row g+8
          } else {
            a0 = w0[2 * jj];
            a2 = w0[2 * jj + 1];
            a1 = w1[2 * jj];
            a3 = w1[2 * jj + 1];
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            float (&acc)[4] = (j & 1) ? sb[nt] : sa[nt];
            if (FP8) mma_f16_16816(acc, a0, a1, a2, a3, qb[nt][j][0], qb[nt][j][1]);
            else mma_bf16_16816(acc, a0, a1, a2, a3, qb[nt][j][0], qb[nt][j][1]);
          }
        }
      }

      if (tail) {
        // zero V rows past the end so stale bytes (possibly NaN codes) cannot
        // reach the accumulator through a zero probability
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int row = 2 * tig + (r & 1) + 8 * (r >> 1);
          if (tok0 + row >= pc.ntok)
#pragma unroll
            for (int w = 0; w < kVWords; ++w) vr[r][w] = 0u;
        }
      }
      // per-token scales (TOKEN mode): K and V of rows g, g+8
      float ks_row[2] = {1.0f, 1.0f}, vs_row[2] = {1.0f, 1.0f};
      if (tok_mode) {
        const bool in = page >= 0 && page < p.c.P;
        const int64_t base = (static_cast<int64_t>(in ? page : 0) * p.c.Hkv + hk) * p.c.ps +
                             (tok0 % p.c.ps);
        const float* vsp = p.c.v_pages ? p.c.v_scale : p.c.k_scale;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          ks_row[r] = in ? p.c.k_scale[base + g + 8 * r] : 0.0f;
          vs_row[r] = in ? vsp[base + g + 8 * r] : 0.0f;
        }
      }

      // ---- scores (base 2) and the lazily moved reference max ----
      float x[NT][4];
      bool grow = false;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v = (sa[nt][e] + sb[nt][e]) * alpha;
          if (tok_mode) v *= ks_row[e >> 1];
          if (tail && tok0 + g + 8 * (e >> 1) >= pc.ntok) v = kNegInf;
          x[nt][e] = v;
          grow |= v > m_ref[nt][e & 1] + kSlack;
        }
      if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float mb[2] = {fmaxf(x[nt][0], x[nt][2]), fmaxf(x[nt][1], x[nt][3])};
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            mb[c] = fmaxf(mb[c], __shfl_xor_sync(0xffffffffu, mb[c], 4));
            mb[c] = fmaxf(mb[c], __shfl_xor_sync(0xffffffffu, mb[c], 8));
            mb[c] = fmaxf(mb[c], __shfl_xor_sync(0xffffffffu, mb[c], 16));
            if (mb[c] > m_ref[nt][c]) {
              const float r = ex2(m_ref[nt][c] - mb[c]);     // 0 on the first tile
              l_run[nt][c] *= r;
#pragma unroll
              for (int i = 0; i < L::kMTiles; ++i) {
                o_acc[nt][i][c] *= r;
                o_acc[nt][i][c + 2] *= r;
              }
              m_ref[nt][c] = mb[c];
            }
          }
        }
      }

      // ---- probabilities, moved into the PV operand layout ----
      uint32_t pb[NT][2][2];   // [nt][hi/lo part][b0b1, b2b3]
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float pr[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) pr[e] = ex2(x[nt][e] - m_ref[nt][e & 1]);
        l_run[nt][0] += pr[0] + pr[2];
        l_run[nt][1] += pr[1] + pr[3];
        if (tok_mode) {
#pragma unroll
          for (int e = 0; e < 4; ++e) pr[e] *= vs_row[e >> 1];
        }
        if (FP8) {
          pb[nt][0][0] = movmatrix_trans(pack_f16x2(pr[0], pr[1]));
          pb[nt][0][1] = movmatrix_trans(pack_f16x2(pr[2], pr[3]));
        } else {
          const uint32_t h0 = pack_bf16x2(pr[0], pr[1]);
          const uint32_t h1 = pack_bf16x2(pr[2], pr[3]);
          const uint32_t l0 = pack_bf16x2(pr[0] - bf16lo_to_f32(h0), pr[1] - bf16hi_to_f32(h0));
          const uint32_t l1 = pack_bf16x2(pr[2] - bf16lo_to_f32(h1), pr[3] - bf16hi_to_f32(h1));
          pb[nt][0][0] = movmatrix_trans(h0);
          pb[nt][0][1] = movmatrix_trans(h1);
          pb[nt][1][0] = movmatrix_trans(l0);
          pb[nt][1][1] = movmatrix_trans(l1);
        }
      }

      // ---- O^T += V^T P^T : rows = head dims, cols = heads ----
#pragma unroll
      for (int i = 0; i < L::kMTiles; ++i) {
        uint32_t a0, a1, a2, a3;
        if (FP8) {
          const int wi = i >> 1;                          // word holding the dim pair
          const uint32_t sel = (i & 1) ? 0x7362u : 0x5140u;
          const uint32_t t01 = prmt(vr[0][wi], vr[1][wi], sel);   // tokens 2tig, 2tig+1
          const uint32_t t89 = prmt(vr[2][wi], vr[3][wi], sel);   // tokens 2tig+8, 2tig+9
          e4m3x4_to_f16x2x2(t01, a0, a1);                 // dims v_dim(i,0) | v_dim(i,1)
          e4m3x4_to_f16x2x2(t89, a2, a3);
        } else {
          a0 = prmt(vr[0][i], vr[1][i], 0x5410u);
          a1 = prmt(vr[0][i], vr[1][i], 0x7632u);
          a2 = prmt(vr[2][i], vr[3][i], 0x5410u);
          a3 = prmt(vr[2][i], vr[3][i], 0x7632u);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (FP8) {
            mma_f16_16816(o_acc[nt][i], a0, a1, a2, a3, pb[nt][0][0], pb[nt][0][1]);
          } else {
            mma_bf16_16816(o_acc[nt][i], a0, a1, a2, a3, pb[nt][0][0], pb[nt][0][1]);
            mma_bf16_16816(o_acc[nt][i], a0, a1, a2, a3, pb[nt][1][0], pb[nt][1][1]);
          }
        }
      }
    }

    // ---- merge the warps' states for this piece ----
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float l = l_run[nt][c];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        const int head = nt * 8 + 2 * tig + c;
        if (g == 0) {
          red_m[cw * K::kHeads + head] = m_ref[nt][c];
          red_l[cw * K::kHeads + head] = l;
        }
#pragma unroll
        for (int i = 0; i < L::kMTiles; ++i)
#pragma unroll
          for (int r = 0; r < 2; ++r)
            red_o[(cw * K::kHeads + head) * D + L::v_dim(i, r, g)] = o_acc[nt][i][c + 2 * r];
      }
    __syncthreads();
    if (!*abort_flag) {
      const int32_t slot = blockIdx.x + pc.seg;
      const int ctid = threadIdx.x;
      for (int idx = ctid; idx < p.G * D; idx += NW * 32) {
        const int head = idx / D, d = idx - head * D;
        float M = kNegInf;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, red_m[w * K::kHeads + head]);
        const float muse = (M == kNegInf) ? 0.0f : M;
        float Lsum = 0.0f, O = 0.0f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          const float f = ex2(red_m[w * K::kHeads + head] - muse);
          Lsum += f * red_l[w * K::kHeads + head];
          O += f * red_o[(w * K::kHeads + head) * D + d];
        }
        p.ws_o[(static_cast<int64_t>(slot) * p.G + head) * D + d] = O * (vscale / Lsum);
        if (d == 0) p.ws_lse[static_cast<int64_t>(slot) * p.G + head] = (M + __log2f(Lsum)) * kLn2;
      }
    }
    __syncthreads();
    u += pc.nt;
    n_begin += pc.nt;
  }
  // After a timed-out wait the loops above stop consuming: wait (bounded) for
  // this warp's loads still in flight before the CTA's shared memory is freed.
  if (*abort_flag && lane == 0)
    for (int32_t k = issued > S ? issued - S : 0; k < issued; ++k)
      mbar_wait(&my_full[k % S], static_cast<uint32_t>(k / S) & 1u);
}

// ---------------------------------------------------------------------------
// Log-sum-exp combine.  Grid (segment = (sequence, KV head), head chunk): a
// block merges the partials of up to kCombHeads query heads of one segment.
// The decode launch gave its units to N CTAs (the count it wrote after the
// unit prefix), CTA c taking
// [c*U/N, (c+1)*U/N), so unit u belongs to CTA ((u+1)*N - 1) / U and the
// pieces of a segment with units [S, E) are exactly the CTAs cs..ce that own
// S and E - 1, every one of them non-empty.  out = sum_k exp(lse_k - M) / L *
// o_k with M the largest lse_k and L the sum of exp(lse_k - M).  Each group
// of four outputs has 2^lanes_log2 consecutive threads (sub-lanes): sub-lane
// j takes pieces j, j + 2^lanes_log2, ... in rounds of kCombGroup loads with
// a running maximum and sum, any number of them, and the sub-lanes' states
// are then merged pairwise through shuffles.  Several sub-lanes serve
// segments split into many pieces (small batches), where one thread's rounds
// of loads would follow one another.
// ---------------------------------------------------------------------------
struct CombineParams {
  const int32_t* ws_pre;
  const int32_t* ws_bounds;   // first unit of each working CTA (then U), or null: c*U/N
  const float* ws_lse;
  const float* ws_o;
  int32_t B, Hkv, G, Hq, Dv, heads_per_block, lanes_log2;
  float* out;
  float* lse;
};

constexpr int kCombHeads = 32;        // heads per block at most
constexpr int kCombOutputs = 2048;    // outputs per block (heads_per_block * Dv) at most
constexpr int kCombMaxThreads = kCombOutputs / 4;   // threads per block at most
constexpr int kCombGroup = 4;         // pieces per round of loads
constexpr int kCombMaxLanesLog2 = 3;  // at most 8 sub-lanes per group of four outputs
constexpr int kCombMaxBounds = 2048;  // CTA starts staged in shared memory at most

// CTA of a launch with N working CTAs over U units that owns unit u.
__device__ __forceinline__ int64_t owner_cta(int64_t u, int64_t N, int64_t U) {
  return ((u + 1) * N - 1) / U;
}

// blockDim = heads_per_block * Dv / 4 * 2^lanes_log2 (in whole warps, at
// most kCombMaxThreads), so the blocks are small.  No minimum of resident
// blocks is asked for: under 64 registers the double-buffered loads spill.
__global__ void __launch_bounds__(kCombMaxThreads, 1) lse_combine_kernel(const CombineParams p) {
  pdl_wait();                                    // the decode kernel has finished
  // Only now may a kernel launched after this one start (its work before its
  // own wait then overlaps the merge): a tag check writes its clean result
  // before its wait, and the decode kernel reads the abort mask until it ends.
  pdl_trigger();
  const int32_t seg = blockIdx.x;
  const int32_t b = seg / p.Hkv, h = seg - b * p.Hkv;
  const int32_t h0 = blockIdx.y * p.heads_per_block;            // first head of this block
  const int32_t nh = min(p.heads_per_block, p.G - h0);
  const int64_t U = p.ws_pre[p.B];
  const int32_t tiles_b = (p.ws_pre[b + 1] - p.ws_pre[b]) / p.Hkv;
  float* out = p.out + (static_cast<int64_t>(b) * p.Hq + h * p.G + h0) * p.Dv;
  float* lse = p.lse ? p.lse + static_cast<int64_t>(b) * p.Hq + h * p.G + h0 : nullptr;
  const int dq = p.Dv >> 2;                     // outputs in groups of four dims
  const int n4 = nh * dq;
  const int lg = p.lanes_log2, nl = 1 << lg;
  const int i4 = threadIdx.x >> lg;             // this thread's group
  const int sub = threadIdx.x & (nl - 1);       // and its sub-lane in the group
  const bool mine = i4 < n4;
  const int hh = mine ? i4 / dq : 0, d = mine ? (i4 - hh * dq) * 4 : 0;
  const bool vec_out = (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
  auto store = [&](const float4& acc) {
    float* dst = out + hh * p.Dv + d;
    if (vec_out) {
      *reinterpret_cast<float4*>(dst) = acc;
    } else {
      dst[0] = acc.x;
      dst[1] = acc.y;
      dst[2] = acc.z;
      dst[3] = acc.w;
    }
  };
  if (tiles_b == 0) {                           // the same for the whole block
    if (mine && sub == 0) store(make_float4(0.f, 0.f, 0.f, 0.f));
    if (lse && mine && sub == 0 && d == 0) lse[hh] = -__int_as_float(0x7f800000);
    return;
  }
  // U >= tiles_b > 0 here
  const int64_t S = p.ws_pre[b] + static_cast<int64_t>(h) * tiles_b, E = S + tiles_b;
  // the decode launch's working CTAs, negated after a weighted split
  const int32_t nflag = p.ws_pre[p.B + 1];
  const int64_t N = nflag < 0 ? -static_cast<int64_t>(nflag) : nflag;
  const bool weighted = nflag < 0 && p.ws_bounds != nullptr;
  // After a weighted split the CTAs' starts come into shared memory in one
  // round of loads (when they fit) for the searches below.
  __shared__ int32_t s_bounds[kCombMaxBounds];
  const bool staged = weighted && N + 1 <= kCombMaxBounds;
  if (staged) {
    for (int i = threadIdx.x; i <= N; i += blockDim.x) s_bounds[i] = p.ws_bounds[i];
    __syncthreads();
  }
  const int32_t* bounds = staged ? s_bounds : p.ws_bounds;
  // CTA holding unit u: c*U/N's owner, or after a weighted split the last CTA
  // whose range starts at or before u (a CTA with an empty range shares its
  // start with the next one)
  auto owner = [&](int64_t u) -> int64_t {
    if (!weighted) return owner_cta(u, N, U);
    int64_t lo = 0, hi = N;
    while (hi - lo > 1) {
      const int64_t mid = (lo + hi) >> 1;
      if (bounds[mid] <= u) lo = mid; else hi = mid;
    }
    return lo;
  };
  const int64_t cs = owner(S);
  const int np = static_cast<int>(owner(E - 1) - cs + 1);
  const int64_t slot0 = cs + seg;               // slot of piece k: slot0 + k
  // This sub-lane's pieces sub, sub + nl, ... (none for threads past the
  // block's outputs, which still take part in the shuffles), in groups of
  // kCombGroup with a running maximum m, sum l and output acc (rescaled by
  // exp(m_old - m_new) when m moves); the loads of the next group are issued
  // before the current group is merged.  A single piece comes out bit for
  // bit (weight exp(0) = 1, l = 1, and the empty sub-lanes weigh 0).
  const int my_np = mine && sub < np ? (np - 1 - sub) / nl + 1 : 0;
  const int64_t row0 = (slot0 + sub) * p.G + h0 + hh;   // my piece k at row0 + k * rstep
  const int64_t rstep = static_cast<int64_t>(nl) * p.G;
  float4 o[2][kCombGroup];
  float a[2][kCombGroup];
  auto load_group = [&](int x, int base) {
#pragma unroll
    for (int k = 0; k < kCombGroup; ++k) {
      if (base + k < my_np) {
        const int64_t row = row0 + static_cast<int64_t>(base + k) * rstep;
        o[x][k] = *reinterpret_cast<const float4*>(p.ws_o + row * p.Dv + d);
        a[x][k] = p.ws_lse[row];
      }
    }
  };
  const float kNegInf = -__int_as_float(0x7f800000);
  float m = kNegInf, l = 0.0f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  auto merge = [&](int x, int base) {
    float mg = m;
#pragma unroll
    for (int k = 0; k < kCombGroup; ++k)
      if (base + k < my_np) mg = fmaxf(mg, a[x][k]);
    const float r = __expf(m - mg);                // 0 on the first group
    l *= r;
    acc.x *= r;
    acc.y *= r;
    acc.z *= r;
    acc.w *= r;
#pragma unroll
    for (int k = 0; k < kCombGroup; ++k) {
      if (base + k < my_np) {
        const float w = __expf(a[x][k] - mg);
        l += w;
        acc.x += w * o[x][k].x;
        acc.y += w * o[x][k].y;
        acc.z += w * o[x][k].z;
        acc.w += w * o[x][k].w;
      }
    }
    m = mg;
  };
  // two buffers used alternately with constant indices (registers)
  load_group(0, 0);
  for (int base = 0; base < my_np; base += 2 * kCombGroup) {
    if (base + kCombGroup < my_np) load_group(1, base + kCombGroup);
    merge(0, base);
    if (base + kCombGroup >= my_np) break;
    if (base + 2 * kCombGroup < my_np) load_group(0, base + 2 * kCombGroup);
    merge(1, base + kCombGroup);
  }
  // merge the sub-lanes' states pairwise (an empty state has m = -inf, l = 0)
  for (int x = 1; x < nl; x <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, x);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, x);
    float4 a2;
    a2.x = __shfl_xor_sync(0xffffffffu, acc.x, x);
    a2.y = __shfl_xor_sync(0xffffffffu, acc.y, x);
    a2.z = __shfl_xor_sync(0xffffffffu, acc.z, x);
    a2.w = __shfl_xor_sync(0xffffffffu, acc.w, x);
    const float mg = fmaxf(m, m2);
    const float ref = mg == -__int_as_float(0x7f800000) ? 0.0f : mg;
    const float f1 = __expf(m - ref), f2 = __expf(m2 - ref);
    l = l * f1 + l2 * f2;
    acc.x = acc.x * f1 + a2.x * f2;
    acc.y = acc.y * f1 + a2.y * f2;
    acc.z = acc.z * f1 + a2.z * f2;
    acc.w = acc.w * f1 + a2.w * f2;
    m = mg;
  }
  if (!mine || sub != 0) return;
  if (np > 1) {
    const float inv = 1.0f / l;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
  }
  if (lse && d == 0) lse[hh] = np == 1 ? m : m + __logf(l);
  store(acc);
}

// ---------------------------------------------------------------------------
// Host side: tensor maps, occupancy, dispatch
// ---------------------------------------------------------------------------
cudaError_t launch_lse_combine(const int32_t* ws_pre, const int32_t* ws_bounds,
                               const float* ws_lse, const float* ws_o, int32_t B, int32_t Hkv,
                               int32_t G, int32_t Hq, int32_t Dv, int32_t num_ctas, float* out,
                               float* lse, cudaStream_t stream) {
  CombineParams cp;
  cp.ws_pre = ws_pre;
  cp.ws_bounds = ws_bounds;
  cp.ws_lse = ws_lse;
  cp.ws_o = ws_o;
  cp.B = B;
  cp.Hkv = Hkv;
  cp.G = G;
  cp.Hq = Hq;
  cp.Dv = Dv;
  cp.out = out;
  cp.lse = lse;
  if (Dv % 4 != 0 || Dv > kCombOutputs) return cudaErrorInvalidValue;
  // Sub-lanes: a segment has about num_ctas / segments + 1 pieces.  Up to
  // two rounds of loads stay on one thread; beyond that each sub-lane gets
  // up to kCombGroup pieces (one round), with at most 2^kCombMaxLanesLog2
  // sub-lanes and one head's groups within a block.
  const int64_t segs = static_cast<int64_t>(B) * Hkv;
  const int64_t pieces = (segs > 0 ? num_ctas / segs : 0) + 1;
  int lg = 0;
  if (pieces > 2 * kCombGroup)
    while (lg < kCombMaxLanesLog2 && (static_cast<int64_t>(kCombGroup) << lg) < pieces) ++lg;
  while (lg > 0 && ((Dv / 4) << lg) > kCombMaxThreads) --lg;
  cp.lanes_log2 = lg;
  int hpb = (kCombOutputs >> lg) / Dv;
  hpb = hpb < 1 ? 1 : (hpb > kCombHeads ? kCombHeads : hpb);
  hpb = hpb > G ? G : hpb;
  cp.heads_per_block = hpb;
  // 2^lg threads per four outputs of the block, in whole warps
  const int threads = (((hpb * (Dv / 4)) << lg) + 31) / 32 * 32;
  const dim3 grid(static_cast<unsigned>(B * Hkv), static_cast<unsigned>((G + hpb - 1) / hpb));
  if (B * Hkv == 0) return cudaSuccess;
  return launch_pdl(lse_combine_kernel, grid, dim3(threads), 0, stream, cp);
}

// Opt the kernel into the largest dynamic shared memory it can ask for, once
// per device (the attribute is per function and device).
template <bool FP8, int D, int NT, int NW, int NS>
static cudaError_t prepare_gqa(int dev) {
  using K = GqaKernel<FP8, D, NT, NW, NS>;
  static std::mutex mu;
  static bool done[64] = {};
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(gqa_decode_kernel<FP8, D, NT, NW, NS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(K::smem_bytes(kGqaMaxBatch)));
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

template <bool FP8, int D, int NT, int NW, int NS>
static cudaError_t run_gqa(const DecodeArgs& a, const CUtensorMap& km, const CUtensorMap& vm) {
  using K = GqaKernel<FP8, D, NT, NW, NS>;
  auto kern = gqa_decode_kernel<FP8, D, NT, NW, NS>;
  const size_t smem = K::smem_bytes(a.B);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = prepare_gqa<FP8, D, NT, NW, NS>(dev);
  if (e != cudaSuccess) return e;
  GqaParams p;
  p.c = a.c;
  p.q = a.q;
  p.Hq = a.Hq;
  p.G = a.Hq / a.c.Hkv;
  p.block_table = a.block_table;
  p.max_pages = a.max_pages;
  p.seq_lens = a.seq_lens;
  p.B = a.B;
  p.abort_mask = a.abort_mask;
  p.sm_scale = a.sm_scale;
  p.out = a.out;
  p.lse = a.lse;
  p.num_ctas = a.num_ctas;
  WorkspaceLayout wl = workspace_layout(a.B, a.c.Hkv, p.G, a.c.Dv, a.num_ctas);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  p.ws_pre = reinterpret_cast<int32_t*>(ws + wl.off_pre);
  p.ws_bounds = reinterpret_cast<int32_t*>(ws + wl.off_bounds);
  p.ws_lse = reinterpret_cast<float*>(ws + wl.off_lse);
  p.ws_o = reinterpret_cast<float*>(ws + wl.off_o);
  e = launch_pdl(kern, dim3(a.num_ctas), dim3(K::kThreads), smem, a.stream, km, vm, p);
  if (e != cudaSuccess) return e;
  return launch_lse_combine(p.ws_pre, p.ws_bounds, p.ws_lse, p.ws_o, a.B, a.c.Hkv, p.G, a.Hq,
                            a.c.Dv, a.num_ctas, a.out, a.lse, a.stream);
}

// Consumer warps and pipeline depth per configuration.
// Warps per CTA and ring slots per warp: 8 warps, about 8 KB of slots per
// warp (two CTAs per SM for 8-head groups, 16 warps streaming per SM).
template <bool FP8, int D, int NT>
struct GqaConfig {
  static constexpr int kNW = 8;
  static constexpr int kStage = 2 * 16 * D * (FP8 ? 1 : 2);
  static constexpr int kNS = 8192 / kStage > 1 ? 8192 / kStage : 1;
};

template <bool FP8, int D, int NT>
static int gqa_blocks_per_sm(int dev, int B) {
  using C = GqaConfig<FP8, D, NT>;
  using K = GqaKernel<FP8, D, NT, C::kNW, C::kNS>;
  // cache the last query per device: the answer depends only on B here
  static std::mutex mu;
  static int last_b[64], last_n[64];
  static bool have[64] = {};
  if (dev < 0 || dev >= 64) return 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (have[dev] && last_b[dev] == B) return last_n[dev];
  }
  if (prepare_gqa<FP8, D, NT, C::kNW, C::kNS>(dev) != cudaSuccess) return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gqa_decode_kernel<FP8, D, NT, C::kNW, C::kNS>,
                                                    K::kThreads, K::smem_bytes(B)) != cudaSuccess)
    return 0;
  std::lock_guard<std::mutex> lock(mu);
  last_b[dev] = B;
  last_n[dev] = n;
  have[dev] = true;
  return n;
}

int gqa_default_ctas(bool fp8, int D, int G, int B) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  int per = 0;
  const bool two = G > 8;
#define KVQ_OCC(F, DD, NTT) per = gqa_blocks_per_sm<F, DD, NTT>(dev, B)
  if (fp8) {
    if (D == 64) { if (two) KVQ_OCC(true, 64, 2); else KVQ_OCC(true, 64, 1); }
    else { if (two) KVQ_OCC(true, 128, 2); else KVQ_OCC(true, 128, 1); }
  } else {
    if (D == 64) { if (two) KVQ_OCC(false, 64, 2); else KVQ_OCC(false, 64, 1); }
    else { if (two) KVQ_OCC(false, 128, 2); else KVQ_OCC(false, 128, 1); }
  }
#undef KVQ_OCC
  if (per <= 0) return 0;
  return sms * per;
}

cudaError_t launch_gqa_decode(const DecodeArgs& a, const CUtensorMap& km, const CUtensorMap& vm) {
  const int G = a.Hq / a.c.Hkv;
  const bool two = G > 8;
  const int D = a.c.Dk;
#define KVQ_RUN(F, DD, NTT)                                                                  \
  return run_gqa<F, DD, NTT, GqaConfig<F, DD, NTT>::kNW, GqaConfig<F, DD, NTT>::kNS>(a, km, vm)
  if (a.c.fp8) {
    if (D == 64) { if (two) KVQ_RUN(true, 64, 2); else KVQ_RUN(true, 64, 1); }
    else { if (two) KVQ_RUN(true, 128, 2); else KVQ_RUN(true, 128, 1); }
  } else {
    if (D == 64) { if (two) KVQ_RUN(false, 64, 2); else KVQ_RUN(false, 64, 1); }
    else { if (two) KVQ_RUN(false, 128, 2); else KVQ_RUN(false, 128, 1); }
  }
#undef KVQ_RUN
}

// Box geometry of the TMA tile loads for a (dtype, head dim) pair.
void gqa_tma_box(bool fp8, int D, int* box_elems, int* swizzle_bytes) {
  const int row = D * (fp8 ? 1 : 2);
  if (row == 64) { *box_elems = 64; *swizzle_bytes = 64; }
  else { *box_elems = 128 / (fp8 ? 1 : 2); *swizzle_bytes = 128; }
}

}  // namespace kvq
