// Wide-group FP8 decode on tcgen05 tensor cores: 128 query heads attend to
// one KV head whose keys have 576 dims and whose values are the first 512
// dims of the keys, one FP32 scale per token, pages of a multiple of 64
// tokens.  Here QK^T and PV are real dense contractions (128 rows), so they
// run on the tensor cores with accumulators in tensor memory.
//
// What it computes is the same decode attention as the 8-head kernel (an
// FP8 cache read through its page table, converted on read: "Công thức của
// Cloudflare để phục vụ Kimi và GLM ..." (manulx.blog), section "Bộ nhớ đệm KV
// FP8 tăng gấp đôi dung lượng ngữ cảnh").
//
// Layout of the work
//  * A thread-block cluster of two CTAs on two SMs works on one stretch of
//    one sequence; its MMAs use cta_group::2 with M = 128 query heads (64
//    per SM), so each SM keeps S and O for its own 64 heads.  O (64 heads x
//    512 dims, FP32) takes 256 TMEM columns per SM.
//  * Blocks of 64 tokens.  QK^T: kind::f8f6f4 straight on the stored E4M3
//    key codes (no conversion of K).  Each BF16 query row is split into two
//    E4M3 terms: hi = E4M3(q*2^e), lo = E4M3(q*2^e - hi), with a per-row
//    power of two 2^e that puts max|q*2^e| in [128, 256).  A BF16 value has
//    8 significant bits and hi keeps 4, so the residual fits in lo exactly
//    for every element with |q*2^e| >= 2^-2; smaller ones are rounded at the
//    E4M3 subnormal step 2^-9 (at most 2^-10 away, against a row maximum of
//    at least 128).  A pre-pass writes both terms of every (sequence, 64-head
//    half) as the shared-memory image the MMAs read.
//  * MMA issue: one warp issues every QK^T (18 K-steps of 32 dims, both
//    query terms, into one of three S accumulators, so it runs up to three
//    blocks ahead of the softmax) and another every PV (both value-dim
//    halves, N = 256 each), each in block order.  Each runs its loop as a
//    whole warp with warp-uniform operands (descriptors from the
//    shared-memory base, the constant tensor-memory base, the block
//    counters) and one lane chosen by elect.sync issues: a lane issuing
//    from divergent code takes about a hundred cycles per MMA, a warp with
//    uniform operands a few tens, close to the pipe's own rate for these
//    shapes.
//  * PV: kind::f8f6f4 as well, on the stored value codes.  P, with the
//    token's scale folded in and a per-head power of two 2^f, is split into
//    three E4M3 terms (t0 = E4M3(v), t1 = E4M3(v - t0), t2 = E4M3(v - t0 -
//    t1): about 12 significant bits, against the 8 of two terms, which
//    peaky score rows showed to be too few); the power of two moves only
//    when a block would exceed the E4M3 range (O is then rescaled in TMEM
//    with the reference max), and the epilogue multiplies by 2^-f.
//  * The B operand of QK^T is split by tokens between the two SMs (the
//    leader holds tokens 0-31 of the block, the other SM tokens 32-63), and
//    both SMs' key loads complete on the leader's barrier.  The B operand of
//    PV is split by value dims, and a pair MMA reads both SMs' halves at the
//    same shared-memory offset, so PV cannot read the key stage in place:
//    each SM copies the raw code atoms of its 32 tokens (4 KB each, 128-byte
//    swizzle kept) into its own value buffer and into the other SM's, with
//    bulk shared-memory copies (16 KB per block per SM, no conversion).
//  * Softmax: eight warps per SM; each thread holds one head and 16 of the
//    block's 64 tokens (TMEM lane quarter and column half), and the four
//    warps holding the same 32 heads exchange partial maxima and sums
//    through shared memory.  Scores are scaled to base 2 and exponentiated
//    against a reference max that moves only when a score exceeds it by 2^8
//    (then O is rescaled in TMEM).  A block's token scales are read before
//    its S is waited for, and a rescale of O waits for the previous block's
//    PV only after this block's P is stored, so that wait overlaps the P
//    terms.
//  * Warp roles per CTA: 0 TMA producer (five key stages, page ids read 32
//    blocks ahead); 1 QK^T and 2 PV issue (leader CTA only; warp 1 also owns
//    the tensor memory); 3-10 softmax, P and O read-out; 11 token scales for
//    the softmax and the value copies.  S has three buffers; V and P two
//    each, freed by the completion of the PV that read them.
//  * Work split as in the 8-head kernel: the pre-pass also writes the prefix
//    of 64-token blocks over the sequences, the blocks of all sequences are
//    split evenly over the CTA pairs (split-KV), each pair writes one
//    partial (o, lse) per sequence piece at slot pair + sequence, and the
//    log-sum-exp combine merges them.
#include <mutex>

#include "kvq_decode.h"
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace wide {

constexpr int kHq = 128;   // query heads
constexpr int kH = 64;     // heads per CTA
constexpr int kDk = 576;
constexpr int kDv = 512;
constexpr int kBlk = 64;   // tokens per block
constexpr int kWarpMma = 1;                           // warp 1 QK^T, warp 2 PV
constexpr int kWarpSoftmax = kWarpMma + 2;            // 8 softmax warps
constexpr int kWarpV = kWarpSoftmax + 8;              // scales and value copies
constexpr int kThreads = 32 * (kWarpV + 1);

constexpr int kNK = 5;                                // key stages
constexpr int kQkAtom = 32 * 128;                     // 32 token rows x 128 dims
constexpr int kStage = 4 * kQkAtom + 32 * 64;         // + 64-dim tail: 18,432 B
constexpr int kQAtom = 64 * 128;                      // 64 head rows x 128 dims
constexpr int kQPart = 4 * kQAtom + 64 * 64;          // one E4M3 term: 36,864 B
constexpr int kQImage = 2 * kQPart + kH * 4;          // hi, lo, 2^-e per head
constexpr int kVHalf = kBlk * 128;                    // 64 tokens x 128 value dims, E4M3
constexpr int kVBuf = 2 * kVHalf;                     // one CTA's 256 value dims
constexpr int kPTerms = 3;                            // E4M3 terms of P
constexpr int kPTerm = kH * kBlk;                     // one term: 64 heads x 64 tokens
constexpr int kPBuf = kPTerms * kPTerm;
constexpr int kNSc = 4;                               // scale ring entries
constexpr int kNP = 2;                                // P buffers (freed with V: kPvDone)
constexpr int kNS = 3;                                // S buffers

constexpr int kOffQ = 0;
constexpr int kOffK = 74752;                          // kQImage rounded up to 1 KB
constexpr int kOffV = kOffK + kNK * kStage;           // 2 buffers
constexpr int kOffP = kOffV + 2 * kVBuf;              // kNP buffers
constexpr int kOffKSc = kOffP + kNP * kPBuf;          // token scales per key stage
constexpr int kOffScR = kOffKSc + kNK * kBlk * 4;     // scale ring read by the softmax
constexpr int kOffScMax = kOffScR + kNSc * kBlk * 4;  // largest scale of each ring entry
constexpr int kOffXm = kOffScMax + kNSc * 4;
constexpr int kOffXl = kOffXm + 2 * 256 * 4;         // xm: two blocks' partial maxima
constexpr int kOffFlag = kOffXl + 256 * 4;            // per key stage: page in range
constexpr int kOffBars = kOffFlag + 32;
enum {
  // completed in the leader CTA
  kKFull = 0,
  kSFree = kKFull + kNK,
  kQReady = kSFree + kNS,
  kPReady = kQReady + 1,
  kVReady = kPReady + 2,
  kOFree = kVReady + 2,
  // arrive in both CTAs (multicast commits)
  kSFull = kOFree + 1,
  kKFree = kSFull + kNS,
  kPvDone = kKFree + kNK,
  // local
  kKPeerFull = kPvDone + 2,
  kScL = kKPeerFull + kNK,
  kScR = kScL + kNK,
  kQFull = kScR + kNSc,
  kVFull = kQFull + 1,
  kDrain = kVFull + 2,
  kNumBars = kDrain + 2
};
constexpr int kOffTmem = kOffBars + kNumBars * 8;
constexpr int kSmemBytes = 1024 + kOffTmem + 16;
static_assert(kQImage <= kOffK, "query image overlaps the key stages");
static_assert(kNK <= 8, "stage flags");
static_assert(kSmemBytes <= 232448, "shared memory");

// TMEM columns: O at [0, 256) (value-dim half h of the pair at 128*h), S
// buffer s at 256 + 32*s.
static_assert(256 + 32 * kNS <= 512, "tensor memory");
constexpr uint32_t kTmemCols = 512;
// The kernel allocates all 512 columns, so the allocation starts at lane 0,
// column 0: the MMA warps address tensor memory from this constant (a
// uniform operand), and a pair whose allocation reports another address
// records kErrTmemBase and does no work.
constexpr uint32_t kTmemBase = 0;
constexpr uint32_t kColS = 256;

// Instruction descriptors (kind::f8f6f4, E4M3 x E4M3): FP32 accumulate
// (bit 4), M = 128 (m_dim = 8 at bit 24), N >> 3 at bit 17; QK^T both
// K-major (N = 64 tokens); PV with B (the values) MN-major (bit 16), N = 256
// value dims.
constexpr uint32_t kIdescQK = (1u << 4) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 16) | ((256u >> 3) << 17) | ((128u >> 4) << 24);

// 2^f as a float, f in [-126, 127]
__device__ __forceinline__ float pow2f(int f) { return __int_as_float((f + 127) << 23); }
// f with v * 2^f in [128, 256) for a positive normal v, held to [-120, 120]
// (subnormal v count as 2^-127)
__device__ __forceinline__ int pow2_exponent(float v) {
  const int e = static_cast<int>((__float_as_uint(v) >> 23) & 255u) - 127;
  const int f = 7 - e;
  return f > 120 ? 120 : (f < -120 ? -120 : f);
}

// byte offset of 16-byte chunk c of row r in a 128-byte-swizzled atom
__host__ __device__ __forceinline__ uint32_t sw128(int r, int c) {
  return r * 128 + ((c ^ (r & 7)) << 4);
}
// ... in a 64-byte-swizzled atom
__host__ __device__ __forceinline__ uint32_t sw64(int r, int c) {
  return r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
}
// byte offset of 16-dim chunk cg (0..35) of head row h in one E4M3 term of the query image
__host__ __device__ __forceinline__ uint32_t q_chunk_off(int h, int cg) {
  return cg < 32 ? (cg >> 3) * kQAtom + sw128(h, cg & 7) : 4 * kQAtom + sw64(h, cg - 32);
}

struct Params {
  CacheView c;
  const uint16_t* q;        // bf16 [B][128][576]
  const int32_t* block_table;
  int32_t max_pages;
  const int32_t* seq_lens;
  int32_t B;
  const uint8_t* abort_mask;
  float sm_scale;
  int32_t* ws_pre;          // [B+2] prefix of 64-token blocks, then the working pairs (pre-pass)
  float* ws_lse;            // [slots][128]
  float* ws_o;              // [slots][128][512]
  uint8_t* ws_q;            // [B][2][kQImage] query images (written by the pre-pass)
  int32_t num_pairs;
};

__device__ __forceinline__ int32_t seq_tokens(const Params& p, int b) {
  if (p.abort_mask != nullptr && p.abort_mask[b]) return 0;
  int64_t n = p.seq_lens[b];
  n = n < 0 ? 0 : n;
  const int64_t cap = static_cast<int64_t>(p.max_pages) * p.c.ps;
  return static_cast<int32_t>(n > cap ? cap : n);
}

// Pre-pass, one launch of 2B + 1 CTAs.  CTA 2b + r writes the query image
// of sequence b, heads 64r..64r+63 (skipped when the sequence has no
// tokens); the last CTA writes the exclusive prefix over b of
// ceil(tokens_b / 64) into ws_pre[0..B].
constexpr int kPrepThreads = 256;
__global__ void __launch_bounds__(kPrepThreads) wide_prep_kernel(const Params p) {
  pdl_trigger();                                 // the decode kernel may launch and set up
  pdl_wait();                                    // the previous kernel (validate) has finished
  const int tid = threadIdx.x;
  if (blockIdx.x == 2 * p.B) {
    // each thread sums a run of sequences; a warp scan and the warps' totals
    // give each run its start
    __shared__ int32_t warp_tot[kPrepThreads / 32];
    const int lane = tid & 31, warp = tid >> 5;
    const int per = (p.B + kPrepThreads - 1) / kPrepThreads;
    const int lo = min(p.B, tid * per), hi = min(p.B, lo + per);
    int32_t sum = 0;
    for (int b = lo; b < hi; ++b) sum += (seq_tokens(p, b) + kBlk - 1) / kBlk;
    int32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int32_t run = incl - sum;
    for (int w = 0; w < warp; ++w) run += warp_tot[w];
    for (int b = lo; b < hi; ++b) {
      p.ws_pre[b] = run;
      run += (seq_tokens(p, b) + kBlk - 1) / kBlk;
    }
    if (tid == kPrepThreads - 1) {
      p.ws_pre[p.B] = run;                               // the last run ends at B
      p.ws_pre[p.B + 1] = min(p.num_pairs, run);         // working pairs, as the decode kernel
    }
    return;
  }
  const int b = blockIdx.x >> 1, r = blockIdx.x & 1;
  if (seq_tokens(p, b) == 0) return;
  const int h = tid >> 2, qd = tid & 3;                  // head, quarter of 144 dims
  const uint16_t* qrow = p.q + (static_cast<int64_t>(b) * kHq + 64 * r + h) * kDk + qd * 144;
  uint8_t* img = p.ws_q + (static_cast<int64_t>(b) * 2 + r) * kQImage;
  uint4 w[18];
#pragma unroll
  for (int k = 0; k < 18; ++k) w[k] = *reinterpret_cast<const uint4*>(qrow + 8 * k);
  float amax = 0.0f;
#pragma unroll
  for (int k = 0; k < 18; ++k) {
    const uint32_t ws[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
#pragma unroll
    for (int t = 0; t < 4; ++t)
      amax = fmaxf(amax, fmaxf(fabsf(bf16lo_to_f32(ws[t])), fabsf(bf16hi_to_f32(ws[t]))));
  }
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  int e = 0;
  if (amax > 0.0f) {
    const int E = static_cast<int>((__float_as_uint(amax) >> 23) & 255) - 127;
    e = 7 - E;                                           // max|q| * 2^e in [128, 256)
    e = e > 100 ? 100 : (e < -100 ? -100 : e);
  }
  const float sc = ldexpf(1.0f, e);
  if (qd == 0) reinterpret_cast<float*>(img + 2 * kQPart)[h] = ldexpf(1.0f, -e);
#pragma unroll
  for (int c = 0; c < 9; ++c) {                          // 16-dim chunks of this quarter
    const uint32_t ws[8] = {w[2 * c].x, w[2 * c].y, w[2 * c].z, w[2 * c].w,
                            w[2 * c + 1].x, w[2 * c + 1].y, w[2 * c + 1].z, w[2 * c + 1].w};
    uint32_t hi[4] = {0, 0, 0, 0}, lo[4] = {0, 0, 0, 0};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float x0 = bf16lo_to_f32(ws[k]) * sc, x1 = bf16hi_to_f32(ws[k]) * sc;
      const uint32_t h01 = f32x2_to_e4m3x2(x0, x1);
      const uint32_t hf16 = e4m3x2_to_f16x2(h01);
      const float r0 = x0 - __half2float(__ushort_as_half(static_cast<uint16_t>(hf16 & 0xFFFFu)));
      const float r1 = x1 - __half2float(__ushort_as_half(static_cast<uint16_t>(hf16 >> 16)));
      const uint32_t l01 = f32x2_to_e4m3x2(r0, r1);
      hi[k >> 1] |= h01 << (16 * (k & 1));
      lo[k >> 1] |= l01 << (16 * (k & 1));
    }
    const uint32_t off = q_chunk_off(h, 9 * qd + c);
    *reinterpret_cast<uint4*>(img + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(img + kQPart + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
}

__device__ __forceinline__ int find_seq(const int32_t* pre, int B, int32_t u) {
  int lo = 0, hi = B;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(pre + mid) <= u) lo = mid; else hi = mid;
  }
  return lo;
}

// Waits give up after about a second, or at once when any wait of the
// launch has already given up (the word is global, so both CTAs see it).
// CTA-scope acquire: what a waiter then reads is in its own CTA's shared
// memory or tensor memory, or (the V conversion) in the other CTA's key
// stage, which TMA wrote before the load's completion reached the barrier.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*reinterpret_cast<volatile uint32_t*>(&g_error_flags) & kErrWaitTimeout) return false;
      if (globaltimer_ns() - t0 > 1000000000ull) {
        atomicOr(&g_error_flags, kErrWaitTimeout);
        return false;
      }
    }
  }
}

// Arrive on barrier `bar` (an offset in this CTA's shared memory) of the leader CTA.
__device__ __forceinline__ void arrive_leader(uint64_t* bar, uint32_t rank) {
  if (rank == 0) mbar_arrive(bar);
  else mbar_arrive_remote(mapa_shared(smem_u32(bar), 0));
}

__device__ __forceinline__ void named_bar(uint32_t id, uint32_t n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Iterate this pair's pieces: calls f(b, t0, nt) for every (sequence, first
// block, block count) in order.  All roles walk the same pieces.
template <class F>
__device__ __forceinline__ void for_pieces(const Params& p, int32_t u0, int32_t u1, F&& f) {
  for (int32_t u = u0; u < u1;) {
    const int b = find_seq(p.ws_pre, p.B, u);
    const int32_t t0 = u - __ldg(p.ws_pre + b);
    const int32_t nt = min(__ldg(p.ws_pre + b + 1) - u, u1 - u);
    f(b, t0, nt);
    u += nt;
  }
}

// A bounded wait whose result is the same for every lane of the warp.
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, wait_bar(bar, parity));
}

// Two MMA warps of the leader CTA: one issues QK^T of every block (18
// K-steps x 2 query terms into one S accumulator), the other PV of every
// block for both value-dim halves, each in block order.  Each runs its loop
// as a whole warp with warp-uniform operands (descriptors from the
// shared-memory base, the constant tensor-memory base, the block counters)
// and one elected lane issues each tcgen05 instruction.
__device__ __forceinline__ void qk_warp(const Params& p, uint8_t* smem, uint64_t* bars,
                                        int32_t u0, int32_t u1) {
  const uint32_t sq = smem_u32(smem + kOffQ), sk = smem_u32(smem + kOffK);
  constexpr uint64_t kLo = kQPart >> 4;                // the lo term, as a descriptor offset
  int32_t j = 0, item = 0;
  bool ok = true;
  for_pieces(p, u0, u1, [&](int, int32_t, int32_t nt) {
    ok = ok && wait_bar_warp(&bars[kQReady], item & 1);
    for (int32_t i = 0; i < nt && ok; ++i, ++j) {
      const int s = j % kNK, s3 = j % kNS;
      ok = wait_bar_warp(&bars[kKFull + s], static_cast<uint32_t>(j / kNK) & 1u);
      if (ok && j >= kNS)
        ok = wait_bar_warp(&bars[kSFree + s3], static_cast<uint32_t>((j / kNS) & 1) ^ 1u);
      if (!ok) break;
      tc_fence_after();
      const uint32_t d = kTmemBase + kColS + 32 * s3;
      const uint32_t sks = sk + s * kStage;
      const uint64_t qa = smem_desc(sq, 16, 1024, 2), ka = smem_desc(sks, 16, 1024, 2);
      const uint64_t qt = smem_desc(sq + 4 * kQAtom, 16, 512, 4);
      const uint64_t kt = smem_desc(sks + 4 * kQkAtom, 16, 512, 4);
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {          // dims 0..511: 128-byte-swizzled atoms
        const uint64_t qo = qa + (((ks >> 2) * kQAtom + (ks & 3) * 32) >> 4);
        const uint64_t ko = ka + (((ks >> 2) * kQkAtom + (ks & 3) * 32) >> 4);
        umma_pair_f8_warp(d, qo, ko, kIdescQK, ks > 0 ? 1u : 0u);
        umma_pair_f8_warp(d, qo + kLo, ko, kIdescQK, 1u);
      }
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {           // dims 512..575: the 64-byte-swizzled tail
        umma_pair_f8_warp(d, qt + ((ks * 32) >> 4), kt + ((ks * 32) >> 4), kIdescQK, 1u);
        umma_pair_f8_warp(d, qt + ((ks * 32) >> 4) + kLo, kt + ((ks * 32) >> 4), kIdescQK, 1u);
      }
      umma_commit_pair_warp(&bars[kSFull + s3]);
      umma_commit_pair_warp(&bars[kKFree + s]);
    }
    ++item;
  });
  umma_commit_pair_local_warp(&bars[kDrain]);
  mbar_wait_cluster(&bars[kDrain], 0);
}

__device__ __forceinline__ void pv_warp(const Params& p, uint8_t* smem, uint64_t* bars,
                                        int32_t u0, int32_t u1) {
  const uint32_t sv = smem_u32(smem + kOffV), sp = smem_u32(smem + kOffP);
  int32_t j = 0, item = 0;
  bool ok = true;
  for_pieces(p, u0, u1, [&](int, int32_t, int32_t nt) {
    for (int32_t i = 0; i < nt && ok; ++i, ++j) {
      const int x = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      ok = wait_bar_warp(&bars[kPReady + x], ph) && wait_bar_warp(&bars[kVReady + x], ph);
      // O must be free of the previous piece's epilogue
      if (ok && i == 0 && item > 0) ok = wait_bar_warp(&bars[kOFree], (item - 1) & 1);
      if (!ok) break;
      tc_fence_after();
      // A: P, one K-major tile per term (rows of 64 token codes, 64-byte
      // swizzle); B: the value codes, MN-major, 8-token groups of 1 KB;
      // value half h into O columns [128h, 128h + 128)
      const uint64_t pa = smem_desc(sp + (j % kNP) * kPBuf, 16, 512, 4);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint64_t va = smem_desc(sv + x * kVBuf + h * kVHalf, kVHalf, 1024, 2);
#pragma unroll
        for (int ks = 0; ks < kBlk / 32; ++ks)
#pragma unroll
          for (int t = 0; t < kPTerms; ++t)
            umma_pair_f8_warp(kTmemBase + 128 * h, pa + ((t * kPTerm + 32 * ks) >> 4),
                              va + ((ks * 4096) >> 4), kIdescPV,
                              (i == 0 && ks == 0 && t == 0) ? 0u : 1u);
      }
      umma_commit_pair_warp(&bars[kPvDone + x]);   // frees V buffer x and P buffer j % 2
    }
    ++item;
  });
  umma_commit_pair_local_warp(&bars[kDrain + 1]);
  mbar_wait_cluster(&bars[kDrain + 1], 0);
}

__global__ void __launch_bounds__(kThreads, 1)
    wide_decode_kernel(const __grid_constant__ CUtensorMap kmap_qk,
                       const __grid_constant__ CUtensorMap kmap_tail, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t rank = cluster_ctarank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmem);
  volatile int32_t* flag = reinterpret_cast<volatile int32_t*>(smem + kOffFlag);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNK; ++s) {
      mbar_init(&bars[kKFull + s], 1);
      mbar_init(&bars[kKFree + s], 3);   // the QK^T warp's commit + both CTAs' V warps
      mbar_init(&bars[kKPeerFull + s], 1);
      mbar_init(&bars[kScL + s], 1);
    }
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&bars[kSFree + s], 16);       // per softmax warp, both CTAs
      mbar_init(&bars[kSFull + s], 1);   // the QK^T warp's commit
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[kPReady + s], 16);
      mbar_init(&bars[kVReady + s], 2);         // one V warp per CTA
      mbar_init(&bars[kPvDone + s], 1);  // the PV warp's commit
      mbar_init(&bars[kVFull + s], 1);          // plus 16 KB of copies
    }
    for (int s = 0; s < kNSc; ++s) mbar_init(&bars[kScR + s], 1);
    mbar_init(&bars[kQReady], 2);
    mbar_init(&bars[kOFree], 16);
    mbar_init(&bars[kQFull], 1);
    for (int s = 0; s < 2; ++s) mbar_init(&bars[kDrain + s], 1);
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int pair = blockIdx.x >> 1;
  cluster_sync_all();                            // both CTAs' barriers and TMEM ready
  pdl_trigger();                                 // the combine may launch (it waits for us)
  pdl_wait();                                    // the pre-pass has finished

  // The blocks go to the first N = min(num_pairs, U) pairs, so that every
  // working pair has at least one (the combine relies on it); the others
  // get an empty range and only set up and tear down.
  const int64_t U = __ldg(p.ws_pre + p.B);
  const int64_t N = working_ctas(p.num_pairs, U, 1);     // min(pairs, U)
  if (tbase != kTmemBase && threadIdx.x == 0) atomicOr(&g_error_flags, kErrTmemBase);
  const bool works = pair < N && tbase == kTmemBase;
  const int32_t u0 = works ? static_cast<int32_t>(U * pair / N) : 0;
  const int32_t u1 = works ? static_cast<int32_t>(U * (pair + 1) / N) : 0;
  const int32_t nblk = u1 - u0;

  if (warp == 0) {
    // ---------------- TMA producer (whole warp: page ids 32 blocks ahead) ----------------
    auto lookup = [&](int32_t jj, int32_t& page, int32_t& y) {
      page = -1;
      y = 0;
      if (jj < nblk) {
        const int32_t u = u0 + jj;
        const int b = find_seq(p.ws_pre, p.B, u);
        const int32_t tok = (u - __ldg(p.ws_pre + b)) * kBlk;
        page = __ldg(p.block_table + static_cast<int64_t>(b) * p.max_pages + tok / p.c.ps);
        y = tok % p.c.ps;
      }
    };
    if (lane == 0) {
      tma_prefetch_desc(&kmap_qk);
      tma_prefetch_desc(&kmap_tail);
    }
    int32_t cur_page, cur_y, nxt_page, nxt_y;
    lookup(lane, cur_page, cur_y);
    bool ok = true;
    int32_t issued = 0;
    for (int32_t jb = 0; jb < nblk; jb += 32) {
      lookup(jb + 32 + lane, nxt_page, nxt_y);     // in flight while this batch issues
      const int nb = min(32, nblk - jb);
      for (int k = 0; k < nb; ++k) {
        const int32_t page = __shfl_sync(0xffffffffu, cur_page, k);
        const int32_t y = __shfl_sync(0xffffffffu, cur_y, k);
        if (lane == 0 && ok) {
          const int32_t j = jb + k;
          const int s = j % kNK;
          const uint32_t n = static_cast<uint32_t>(j / kNK);
          ok = wait_bar(&bars[kKFree + s], (n & 1u) ^ 1u);
          if (ok) {
            const bool in = page >= 0 && page < p.c.P;
            flag[s] = in ? 1 : 0;
            const uint32_t kfull = mapa_shared(smem_u32(&bars[kKFull + s]), 0);
            if (rank == 0) mbar_arrive_expect_tx(&bars[kKFull + s], 2 * kStage);
            uint8_t* st = smem + kOffK + s * kStage;
            const int yq = y + 32 * static_cast<int>(rank);    // this SM's token half
#pragma unroll
            for (int a = 0; a < 4; ++a)
              tma_load_4d_pair(st + a * kQkAtom, &kmap_qk, kfull, a * 128, yq, 0, page);
            tma_load_4d_pair(st + 4 * kQkAtom, &kmap_tail, kfull, 512, yq, 0, page);
            mbar_arrive_expect_tx(&bars[kScL + s], in ? kBlk * 4 : 0);
            if (in)
              bulk_load(smem + kOffKSc + s * kBlk * 4,
                        p.c.k_scale + static_cast<int64_t>(page) * p.c.ps + y, kBlk * 4,
                        &bars[kScL + s]);
            ++issued;
          }
        }
      }
      cur_page = nxt_page;
      cur_y = nxt_y;
    }
    if (lane == 0) {
      // Loads still in flight after a failed wait land before the CTA exits
      // (each earlier load of a stage completed before its reuse).
      for (int32_t j = issued > kNK ? issued - kNK : 0; j < issued; ++j) {
        const uint32_t ph = static_cast<uint32_t>(j / kNK) & 1u;
        if (rank == 0) mbar_wait_cluster(&bars[kKFull + j % kNK], ph);
        mbar_wait_cluster(&bars[kScL + j % kNK], ph);
      }
    }
  } else if (warp < kWarpSoftmax) {
    // ---------------- MMA issue (leader CTA): QK^T warp, PV warp ----------------
    if (rank == 0) {
      if (warp == kWarpMma) qk_warp(p, smem, bars, u0, u1);
      else pv_warp(p, smem, bars, u0, u1);
    }
  } else if (warp == kWarpV) {
    // ---------------- token scales and value copies ----------------
    // Per block: the token scales for the softmax (0 past the end of the
    // sequence or off the cache) and their maximum, first, so the softmax
    // never waits for the copies.  Then, once the block's key stages have
    // landed in both CTAs and value buffer x is free in both, lane 0 copies
    // the raw code atoms of this CTA's 32 tokens into both CTAs' buffers:
    // PV half k covers value dims 256k + [0, 256), of which CTA r holds
    // 256k + 128r + [0, 128), key-stage atom 2k + r of either CTA; this CTA's
    // tokens are rows 32*rank + [0, 32) of every buffer.
    const float* kscl = reinterpret_cast<const float*>(smem + kOffKSc);
    float* ring = reinterpret_cast<float*>(smem + kOffScR);
    float* ring_max = reinterpret_cast<float*>(smem + kOffScMax);
    int32_t j = 0, pending = -1;   // a block whose copies into this CTA were not waited for
    bool ok = true;
    for_pieces(p, u0, u1, [&](int b, int32_t t0, int32_t nt) {
      const int32_t ntok = seq_tokens(p, b);
      for (int32_t i = 0; i < nt; ++i, ++j) {
        const int s = j % kNK, x = j & 1, e = j & (kNSc - 1);
        const uint32_t n = static_cast<uint32_t>(j / kNK);
        const int32_t nvalid = min(kBlk, ntok - (t0 + i) * kBlk);
        ok = ok && wait_bar(&bars[kScL + s], n & 1u);
        if (ok) {
          const bool in = flag[s] != 0;
          const float2 sv = reinterpret_cast<const float2*>(kscl + s * kBlk)[lane];
          const float s0 = in && 2 * lane < nvalid ? sv.x : 0.0f;
          const float s1 = in && 2 * lane + 1 < nvalid ? sv.y : 0.0f;
          reinterpret_cast<float2*>(ring + e * kBlk)[lane] = make_float2(s0, s1);
          float mx = fmaxf(s0, s1);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          if (lane == 0) ring_max[e] = mx;
        }
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&bars[kScR + e]);
        // both CTAs' stages have landed: the leader's barrier counts both
        // loads, and the leader forwards its completion
        ok = ok && wait_bar(&bars[rank == 0 ? kKFull + s : kKPeerFull + s], n & 1u);
        if (rank == 0 && lane == 0 && ok)
          mbar_arrive_remote(mapa_shared(smem_u32(&bars[kKPeerFull + s]), 1));
        // buffer x is free in both CTAs once PV(j - 2) has completed
        if (j >= 2) ok = ok && wait_bar(&bars[kPvDone + x], ((j >> 1) & 1) ^ 1);
        if (lane == 0 && ok) {
          mbar_arrive_expect_tx(&bars[kVFull + x], kVBuf);   // own two atoms + the peer's two
          const uint8_t* st = smem + kOffK + s * kStage;
          const uint32_t dst = smem_u32(smem + kOffV + x * kVBuf) + rank * kQkAtom;
#pragma unroll
          for (int k = 0; k < 2; ++k)
#pragma unroll
            for (uint32_t r = 0; r < 2; ++r)
              bulk_copy_to_cluster(mapa_shared(dst + k * kVHalf, r), st + (2 * k + r) * kQkAtom,
                                   kQkAtom, mapa_shared(smem_u32(&bars[kVFull + x]), r));
          pending = j;
        }
        ok = ok && wait_bar(&bars[kVFull + x], (j >> 1) & 1);
        if (ok) pending = -1;
        // rows past the end of the sequence may hold any codes, NaN patterns
        // among them, which a zero probability would not cancel
        if (ok && nvalid < kBlk) {
          uint8_t* vb = smem + kOffV + x * kVBuf;
          const int nrow = kBlk - nvalid;
          for (int idx = lane; idx < 2 * nrow * 8; idx += 32) {
            const int k = idx / (nrow * 8), rr = idx - k * nrow * 8;
            *reinterpret_cast<uint4*>(vb + k * kVHalf + (nvalid + (rr >> 3)) * 128 + (rr & 7) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0 && ok) {
          arrive_leader(&bars[kVReady + x], rank);
          // the copies out of this CTA's stage have landed in both CTAs
          mbar_arrive(&bars[kKFree + s]);
          mbar_arrive_remote(mapa_shared(smem_u32(&bars[kKFree + s]), rank ^ 1u));
        }
      }
    });
    // copies into this CTA after a wait that gave up land before the CTA exits
    if (lane == 0 && pending >= 0)
      mbar_wait_cluster(&bars[kVFull + (pending & 1)], (pending >> 1) & 1);
  } else {
    // ---------------- softmax warps: scores, P, epilogue ----------------
    // Eight warps.  Warp w reads TMEM lane quarter q = w % 4 (lane L = 32q +
    // lane: head L % 64, token half L / 64) and column half ch of the block's
    // 32 columns per lane, i.e. tokens 32*(L/64) + 16*ch + [0, 16).  The four
    // warps holding the same 32 heads (quarters q and q^2, both column
    // halves) exchange partial maxima and sums through shared memory.
    const int mt = threadIdx.x - 32 * kWarpSoftmax;       // 0..255
    const int q4 = warp & 3, ch = (warp - kWarpSoftmax) >> 2;
    const int L = 32 * q4 + lane;                         // this thread's TMEM lane
    const int hl = L & 63, half = L >> 6;                 // head (in this CTA), token half
    const int part = 2 * half + ch;                       // which 16 of the head's 64 tokens
    const uint32_t tl = tbase + (static_cast<uint32_t>(32 * q4) << 16);
    const float* qexp = reinterpret_cast<const float*>(smem + kOffQ + 2 * kQPart);
    const float* ring = reinterpret_cast<const float*>(smem + kOffScR);
    const float* ring_max = reinterpret_cast<const float*>(smem + kOffScMax);
    float* xm = reinterpret_cast<float*>(smem + kOffXm);
    float* xl = reinterpret_cast<float*>(smem + kOffXl);
    const float kNegInf = -__int_as_float(0x7f800000);
    const uint32_t group_bar = 3 + (warp & 1);            // the four warps of these heads
    int32_t j = 0, item = 0, q_loads = 0;
    bool ok = true;
    // Every softmax thread runs the same loop trips and barriers; after a
    // failed wait (ok == false) the work is skipped but the barriers kept.
    // Each warp reports to the MMA issuers on its own (counts of 16: eight
    // warps in each CTA).
    for_pieces(p, u0, u1, [&](int b, int32_t t0, int32_t nt) {
      const int32_t ntok = seq_tokens(p, b);
      // ---- this CTA's half of the query image (the previous piece's QK^T
      // has finished: its last S was read before its epilogue) ----
      if (mt == 0 && ok) {
        const uint8_t* img = p.ws_q + (static_cast<int64_t>(b) * 2 + rank) * kQImage;
        mbar_arrive_expect_tx(&bars[kQFull], kQImage);
#pragma unroll 1
        for (int c = 0; c < kQImage; c += 8192)
          bulk_load(smem + kOffQ + c, img + c, min(8192, kQImage - c), &bars[kQFull]);
        ++q_loads;
      }
      ok = ok && wait_bar(&bars[kQFull], item & 1);
      if (mt == 0 && ok) arrive_leader(&bars[kQReady], rank);
      // read once: the next piece's image load (by thread 0 after its last
      // PV, which needs every warp's last P) may overwrite it
      const float alpha = p.sm_scale * kLog2e * qexp[hl];

      float m_ref = kNegInf, l_part = 0.0f;
      int f_p = 0;              // P is stored as E4M3 terms of p * s * 2^f_p
      bool f_set = false;       // f_p chosen (some block had p * s > 0)
      for (int32_t i = 0; i < nt; ++i, ++j) {
        const int s2 = j & 1, s3 = j % kNS;
        const int32_t nvalid = min(kBlk, ntok - (t0 + i) * kBlk);
        ok = ok && wait_bar(&bars[kScR + (j & (kNSc - 1))], (j >> 2) & 1);
        float sc[16];
        const float smax = ring_max[j & (kNSc - 1)];
        {
          const float4* s4 = reinterpret_cast<const float4*>(ring + (j & (kNSc - 1)) * kBlk + 16 * part);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float4 v = s4[k];
            sc[4 * k] = v.x;
            sc[4 * k + 1] = v.y;
            sc[4 * k + 2] = v.z;
            sc[4 * k + 3] = v.w;
          }
        }
        ok = ok && wait_bar(&bars[kSFull + s3], static_cast<uint32_t>(j / kNS) & 1u);
        ok = __all_sync(0xffffffffu, ok);                   // tcgen05.ld is warp-collective
        tc_fence_after();
        // the block's scores
        float sacc[16];
        if (ok) {
          uint32_t r0[16];
          tmem_ld16(tl + kColS + 32 * s3 + 16 * ch, r0);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) sacc[c] = __uint_as_float(r0[c]);
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) sacc[c] = 0.0f;
        }
        tc_fence_before();
        // this thread's 16 token scales (0 past the end of the sequence or off
        // the cache) and the block's largest scale
        float x[16];
        float bm = kNegInf;
#pragma unroll
        for (int c = 0; c < 16; ++c)
          x[c] = sacc[c] * (alpha * sc[c]);
        if (nvalid < kBlk) {
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (16 * part + c >= nvalid) x[c] = kNegInf;
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) bm = fmaxf(bm, x[c]);
        // partial maxima, double-buffered by block parity: the next write to
        // this buffer comes after the next block's barrier, which the other
        // three warps pass only after this block's reads
        float* xmj = xm + s2 * 256;
        xmj[part * 64 + hl] = bm;
        named_bar(group_bar, 128);                        // this warp's S loads are done too
        if (lane == 0 && ok) arrive_leader(&bars[kSFree + s3], rank);
#pragma unroll
        for (int o = 1; o < 4; ++o) bm = fmaxf(bm, xmj[((part + o) & 3) * 64 + hl]);
        // Move the reference max when a score exceeds it by 2^8, and the
        // power of two of P when this block's bound on p * s (its largest
        // p, against the new reference, times its largest scale) would pass
        // the E4M3 range at the current one; the new power puts the bound in
        // [128, 256).  Either move rescales O.  The vote keeps the TMEM
        // accesses warp-uniform; the other three warps of these 32 heads see
        // the same head maxima and scales and decide alike.
        const float m_new = bm > m_ref + 8.0f ? fmaxf(m_ref, bm) : m_ref;
        const float vb = ex2(bm - m_new) * smax;
        int f_new = f_p;
        if (vb > 0.0f && (!f_set || vb * pow2f(f_p) > 448.0f)) f_new = pow2_exponent(vb);
        const bool rescale = __any_sync(0xffffffffu, m_new != m_ref || f_new != f_p);
        float r = 1.0f;
        if (rescale) {
          const float rm = ex2(m_ref - m_new);            // 0 on the first block, 1 if unmoved
          // before f is first set every P was 0, so O needs no power-of-two factor
          r = f_set ? rm * pow2f(f_new) * pow2f(-f_p) : rm;
          l_part *= rm;
        }
        m_ref = m_new;
        f_p = f_new;
        f_set = f_set || vb > 0.0f;
        // ---- P (token scale and 2^f folded in) as E4M3 terms: the A operand of PV ----
        const float g = pow2f(f_p);
        uint32_t pt[kPTerms][4] = {};
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
          const float p0 = ex2(x[c] - m_ref), p1 = ex2(x[c + 1] - m_ref);
          l_part += p0 + p1;
          float a0 = p0 * sc[c] * g, a1 = p1 * sc[c + 1] * g;
#pragma unroll
          for (int t = 0; t < kPTerms; ++t) {
            const uint32_t code = f32x2_to_e4m3x2(a0, a1);
            pt[t][c >> 2] |= code << (16 * ((c >> 1) & 1));
            if (t + 1 < kPTerms) {                        // the residual for the next term
              const uint32_t hf = e4m3x2_to_f16x2(code);
              a0 -= __half2float(__ushort_as_half(static_cast<uint16_t>(hf & 0xFFFFu)));
              a1 -= __half2float(__ushort_as_half(static_cast<uint16_t>(hf >> 16)));
            }
          }
        }
        const int pb = j % kNP;
        if (j >= kNP)                                     // P buffer free: PV(j - 2) done
          ok = ok && wait_bar(&bars[kPvDone + pb], static_cast<uint32_t>((j >> 1) & 1) ^ 1u);
        if (ok) {
          // term t, row hl: the codes of tokens 0-63, 16 per chunk
          uint8_t* pbuf = smem + kOffP + pb * kPBuf;
#pragma unroll
          for (int t = 0; t < kPTerms; ++t)
            *reinterpret_cast<uint4*>(pbuf + t * kPTerm + sw64(hl, part)) =
                make_uint4(pt[t][0], pt[t][1], pt[t][2], pt[t][3]);
        }
        if (rescale && i > 0) {
          // O rescale, after P(j) is stored: O must not be in use by PV(j-1)
          ok = ok && wait_bar(&bars[kPvDone + ((j - 1) & 1)], ((j - 1) >> 1) & 1);
          ok = __all_sync(0xffffffffu, ok);
          tc_fence_after();
          if (ok) {                                       // this warp's half of O's columns
#pragma unroll 1
            for (int cc = 4 * ch; cc < 4 * ch + 4; ++cc) {
              uint32_t o[32];
              tmem_ld32(tl + 32 * cc, o);
              tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * r);
              tmem_st32(tl + 32 * cc, o);
            }
            tmem_wait_st();
          }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && ok) arrive_leader(&bars[kPReady + s2], rank);
      }

      // ---- epilogue: O / l and lse for this piece ----
      {
        const int32_t jl = j - 1;
        ok = ok && wait_bar(&bars[kPvDone + (jl & 1)], (jl >> 1) & 1);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        xl[part * 64 + hl] = l_part;
        named_bar(group_bar, 128);
        float l_tot = l_part;
#pragma unroll
        for (int o = 1; o < 4; ++o) l_tot += xl[((part + o) & 3) * 64 + hl];
        const float inv = pow2f(-f_p) / l_tot;            // P was stored times 2^f_p
        const int hg = 64 * static_cast<int>(rank) + hl;
        const int64_t slot = pair + b;
        float* orow = p.ws_o + (slot * kHq + hg) * kDv;
#pragma unroll 1
        for (int cc = 4 * ch; cc < 4 * ch + 4 && ok; ++cc) {
          uint32_t o[32];
          tmem_ld32(tl + 32 * cc, o);
          tmem_wait_ld();
          // column 32*cc: value-dim half cc/4, this lane half's 128 dims
          const int dv0 = 256 * (cc >> 2) + 128 * half + 32 * (cc & 3);
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            *reinterpret_cast<float4*>(orow + dv0 + k) =
                make_float4(__uint_as_float(o[k]) * inv, __uint_as_float(o[k + 1]) * inv,
                            __uint_as_float(o[k + 2]) * inv, __uint_as_float(o[k + 3]) * inv);
        }
        if (part == 0 && ok) p.ws_lse[slot * kHq + hg] = (m_ref + __log2f(l_tot)) * kLn2;
        tc_fence_before();
        // xl is rewritten at the next piece's epilogue, after many group barriers
        __syncwarp();
        if (lane == 0 && ok) arrive_leader(&bars[kOFree], rank);
      }
      ++item;
    });
    // a query-image load whose wait gave up lands before the CTA exits
    if (mt == 0 && q_loads > 0) mbar_wait_cluster(&bars[kQFull], (q_loads - 1) & 1);
  }

  __syncthreads();
  cluster_sync_all();            // the leader's MMAs no longer read this CTA's memory
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, kTmemCols);
  }
}

}  // namespace wide

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static cudaError_t prepare_wide(int dev) {
  static std::mutex mu;
  static bool done[64] = {};
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(wide::wide_decode_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       wide::kSmemBytes);
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

int wide_default_pairs(int B) {
  (void)B;   // the wide kernel's shared memory does not depend on the batch size
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  static std::mutex mu;
  static int last_n[64];
  static bool have[64] = {};
  if (dev < 0 || dev >= 64) return 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (have[dev]) return last_n[dev];
  }
  if (prepare_wide(dev) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(wide::kThreads);
  cfg.dynamicSmemBytes = wide::kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, wide::wide_decode_kernel, &cfg) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  last_n[dev] = n;
  have[dev] = true;
  return n;
}

size_t wide_q_image_bytes() { return static_cast<size_t>(2) * wide::kQImage; }

cudaError_t launch_wide_decode(const DecodeArgs& a, const CUtensorMap& kqk,
                               const CUtensorMap& ktail) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = prepare_wide(dev);
  if (e != cudaSuccess) return e;
  wide::Params p;
  p.c = a.c;
  p.q = a.q;
  p.block_table = a.block_table;
  p.max_pages = a.max_pages;
  p.seq_lens = a.seq_lens;
  p.B = a.B;
  p.abort_mask = a.abort_mask;
  p.sm_scale = a.sm_scale;
  p.num_pairs = a.num_ctas;
  WorkspaceLayout wl =
      workspace_layout(a.B, 1, wide::kHq, wide::kDv, a.num_ctas, wide_q_image_bytes());
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  p.ws_pre = reinterpret_cast<int32_t*>(ws + wl.off_pre);
  p.ws_lse = reinterpret_cast<float*>(ws + wl.off_lse);
  p.ws_o = reinterpret_cast<float*>(ws + wl.off_o);
  p.ws_q = ws + wl.off_extra;
  e = prefer_max_shared(wide::wide_prep_kernel);
  if (e != cudaSuccess) return e;
  e = launch_pdl(wide::wide_prep_kernel, dim3(2 * a.B + 1), dim3(wide::kPrepThreads), 0,
                 a.stream, p);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.num_ctas);
  cfg.blockDim = dim3(wide::kThreads);
  cfg.dynamicSmemBytes = wide::kSmemBytes;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, wide::wide_decode_kernel, kqk, ktail, p);
  if (e != cudaSuccess) return e;
  return launch_lse_combine(p.ws_pre, nullptr, p.ws_lse, p.ws_o, a.B, 1, wide::kHq, wide::kHq,
                            wide::kDv, a.num_ctas, a.out, a.lse, a.stream);
}

}  // namespace kvq
