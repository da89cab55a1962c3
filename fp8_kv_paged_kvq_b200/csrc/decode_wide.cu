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
//  * One thread issues a tcgen05.mma about every 55 cycles, while an
//    M=128, N=64, K=32 E4M3 MMA takes the tensor core about 16.  So the
//    hi and lo chains of QK^T accumulate into two separate S buffers, each
//    issued by its own warp, and a third warp issues PV: the three streams
//    together keep the tensor core fed.  The softmax adds the two S terms.
//  * PV: kind::f16.  P goes to f16 with the token's scale folded in; V is
//    converted from E4M3 to f16 (exact).  Each SM converts only the half
//    of the 512 value dims that its half of the MMA's B operand holds.
//  * The B operand of QK^T is split by tokens between the two SMs (the
//    leader holds tokens 0-31 of the block, the other SM tokens 32-63), and
//    both SMs' key loads complete on the leader's barrier.  The B operand of
//    PV is split by value dims, so the V conversion reads the 32 tokens it
//    lacks from the other SM's stage through distributed shared memory
//    instead of loading them again.
//  * Softmax: each SM's TMEM lane holds one head and 32 of the block's 64
//    tokens (the two halves of the N range sit in lanes 0-63 and 64-127), so
//    a head's two lanes exchange one float per block.  Scores are scaled to
//    base 2 and exponentiated against a reference max that moves only when a
//    score exceeds it by 2^8 (then O is rescaled in TMEM).
//  * Warp roles per CTA: 0 TMA producer (three key stages, page ids read 32
//    blocks ahead); 1 TMEM owner and QK-hi issuer; 10 QK-lo issuer; 11 PV
//    issuer (issuers run in the leader CTA only); 2-5 softmax, P and O
//    read-out; 6-9 V conversion.  S and converted V are double-buffered,
//    P triple-buffered.
//  * Work split as in the 8-head kernel: the pre-pass also writes the prefix
//    of 64-token blocks over the sequences, the blocks of all sequences are
//    split evenly over the CTA pairs (split-KV), each pair writes one
//    partial (o, lse) per sequence piece at slot pair + sequence, and the
//    log-sum-exp combine merges them.
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
constexpr int kThreads = 384;
constexpr int kWarpQkHi = 1, kWarpQkLo = 10, kWarpPv = 11;

constexpr int kNK = 3;                                // key stages
constexpr int kQkAtom = 32 * 128;                     // 32 token rows x 128 dims
constexpr int kStage = 4 * kQkAtom + 32 * 64;         // + 64-dim tail: 18,432 B
constexpr int kQAtom = 64 * 128;                      // 64 head rows x 128 dims
constexpr int kQPart = 4 * kQAtom + 64 * 64;          // one E4M3 term: 36,864 B
constexpr int kQImage = 2 * kQPart + kH * 4;          // hi, lo, 2^-e per head
constexpr int kVHalf = kBlk * 128 * 2;                // 64 tokens x 128 dims f16
constexpr int kVBuf = 2 * kVHalf;
constexpr int kPBuf = kH * kBlk * 2;
constexpr int kNSc = 4;                               // scale ring entries
constexpr int kNP = 3;                                // P buffers

constexpr int kOffQ = 0;
constexpr int kOffK = 74752;                          // kQImage rounded up to 1 KB
constexpr int kOffV = kOffK + kNK * kStage;           // 2 buffers
constexpr int kOffP = kOffV + 2 * kVBuf;              // kNP buffers
constexpr int kOffKSc = kOffP + kNP * kPBuf;          // token scales per key stage
constexpr int kOffScR = kOffKSc + kNK * kBlk * 4;     // scale ring read by the softmax
constexpr int kOffXm = kOffScR + kNSc * kBlk * 4;
constexpr int kOffXl = kOffXm + 2 * 128 * 4;         // xm: two blocks' head maxima
constexpr int kOffFlag = kOffXl + 128 * 4;            // per key stage: page in range
constexpr int kOffBars = kOffFlag + 16;
enum {
  // completed in the leader CTA
  kKFull = 0, kSFree = 3, kQReady = 5, kPReady = 6, kVReady = 8, kOFree = 10,
  // arrive in both CTAs (multicast commits)
  kSHi = 11, kSLo = 13, kKFree = 15, kPvDone = 18, kPFree = 20,
  // local
  kKPeerFull = 23, kScL = 26, kScR = 29, kQFull = 33, kDrain = 34, kNumBars = 37
};
constexpr int kOffTmem = kOffBars + kNumBars * 8;
constexpr int kSmemBytes = 1024 + kOffTmem + 16;
static_assert(kQImage <= kOffK, "query image overlaps the key stages");
static_assert(kSmemBytes <= 232448, "shared memory");

// TMEM columns: O at [0, 256) (PV instruction i at 128*i), S_hi buffers at
// 256 + 32*s, S_lo buffers at 320 + 32*s.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColSHi = 256, kColSLo = 320;

// Instruction descriptors: FP32 accumulate (bit 4), M = 128 (m_dim = 8 at
// bit 24), N >> 3 at bit 17; QK^T E4M3 x E4M3 both K-major; PV f16 x f16
// with B (the values) MN-major (bit 16).
constexpr uint32_t kIdescQK = (1u << 4) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 16) | ((256u >> 3) << 17) | ((128u >> 4) << 24);

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
  int32_t* ws_pre;          // [B+1] prefix of 64-token blocks (written by the pre-pass)
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
  const int tid = threadIdx.x;
  if (blockIdx.x == 2 * p.B) {
    __shared__ int32_t scratch[kPrepThreads];
    const int per = (p.B + kPrepThreads - 1) / kPrepThreads;
    const int lo = tid * per, hi = min(p.B, lo + per);
    int32_t sum = 0;
    for (int b = lo; b < hi; ++b) sum += (seq_tokens(p, b) + kBlk - 1) / kBlk;
    scratch[tid] = sum;
    __syncthreads();
    if (tid == 0) {
      int32_t run = 0;
      for (int t = 0; t < kPrepThreads; ++t) {
        const int32_t v = scratch[t];
        scratch[t] = run;
        run += v;
      }
      p.ws_pre[p.B] = run;
    }
    __syncthreads();
    int32_t run = scratch[tid];
    for (int b = lo; b < hi; ++b) {
      p.ws_pre[b] = run;
      run += (seq_tokens(p, b) + kBlk - 1) / kBlk;
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

// One QK^T chain (18 MMAs of K = 32) of the query term at `sq` against key stage `sk`.
__device__ __forceinline__ void issue_qk(uint32_t d, uint32_t sq, uint32_t sk) {
#pragma unroll
  for (int ks = 0; ks < kDk / 32; ++ks) {
    uint64_t ad, bd;
    if (ks < 16) {
      ad = smem_desc(sq + (ks >> 2) * kQAtom + (ks & 3) * 32, 16, 1024, 2);
      bd = smem_desc(sk + (ks >> 2) * kQkAtom + (ks & 3) * 32, 16, 1024, 2);
    } else {
      ad = smem_desc(sq + 4 * kQAtom + (ks - 16) * 32, 16, 512, 4);
      bd = smem_desc(sk + 4 * kQkAtom + (ks - 16) * 32, 16, 512, 4);
    }
    umma_pair_f8(d, ad, bd, kIdescQK, ks > 0 ? 1u : 0u);
  }
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
      mbar_init(&bars[kKFree + s], 4);        // two QK chains + both CTAs' V conversion
      mbar_init(&bars[kKPeerFull + s], 1);
      mbar_init(&bars[kScL + s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[kSFree + s], 2);
      mbar_init(&bars[kPReady + s], 2);
      mbar_init(&bars[kVReady + s], 2);
      mbar_init(&bars[kSHi + s], 1);
      mbar_init(&bars[kSLo + s], 1);
      mbar_init(&bars[kPvDone + s], 1);
    }
    for (int s = 0; s < kNP; ++s) mbar_init(&bars[kPFree + s], 1);
    for (int s = 0; s < kNSc; ++s) mbar_init(&bars[kScR + s], 1);
    mbar_init(&bars[kQReady], 2);
    mbar_init(&bars[kOFree], 2);
    mbar_init(&bars[kQFull], 1);
    for (int s = 0; s < 3; ++s) mbar_init(&bars[kDrain + s], 1);
    fence_barrier_init();
  }
  if (warp == kWarpQkHi) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int pair = blockIdx.x >> 1;
  cluster_sync_all();                            // both CTAs' barriers and TMEM ready

  const int64_t U = __ldg(p.ws_pre + p.B);
  const int32_t u0 = static_cast<int32_t>(U * pair / p.num_pairs);
  const int32_t u1 = static_cast<int32_t>(U * (pair + 1) / p.num_pairs);
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
  } else if (warp == kWarpQkHi || warp == kWarpQkLo) {
    // ---------------- QK^T issue, one E4M3 term per warp (leader CTA) ----------------
    if (rank == 0 && lane == 0) {
      const int part = warp == kWarpQkLo ? 1 : 0;
      const uint32_t sq = smem_u32(smem + kOffQ) + part * kQPart;
      const uint32_t sk = smem_u32(smem + kOffK);
      const uint32_t dcol = tbase + (part ? kColSLo : kColSHi);
      uint64_t* s_full = &bars[part ? kSLo : kSHi];
      int32_t j = 0, item = 0;
      bool ok = true;
      for_pieces(p, u0, u1, [&](int, int32_t, int32_t nt) {
        ok = ok && wait_bar(&bars[kQReady], item & 1);
        for (int32_t i = 0; i < nt && ok; ++i, ++j) {
          const int s = j % kNK, s2 = j & 1;
          ok = wait_bar(&bars[kKFull + s], static_cast<uint32_t>(j / kNK) & 1u);
          if (ok && part == 0)     // the other CTA's V conversion learns that both stages landed
            mbar_arrive_remote(mapa_shared(smem_u32(&bars[kKPeerFull + s]), 1));
          if (ok && j >= 2) ok = wait_bar(&bars[kSFree + s2], ((j >> 1) & 1) ^ 1);
          if (!ok) break;
          tc_fence_after();
          issue_qk(dcol + 32 * s2, sq, sk + s * kStage);
          umma_commit_pair(&s_full[s2]);
          umma_commit_pair(&bars[kKFree + s]);
        }
        ++item;
      });
      // every MMA issued has finished before either CTA leaves
      umma_commit_pair_local(&bars[kDrain + part]);
      mbar_wait_cluster(&bars[kDrain + part], 0);
    }
  } else if (warp == kWarpPv) {
    // ---------------- PV issue (leader CTA) ----------------
    if (rank == 0 && lane == 0) {
      const uint32_t sv = smem_u32(smem + kOffV), sp = smem_u32(smem + kOffP);
      int32_t j = 0, item = 0;
      bool ok = true;
      for_pieces(p, u0, u1, [&](int, int32_t, int32_t nt) {
        for (int32_t i = 0; i < nt && ok; ++i, ++j) {
          const int x = j & 1;
          const uint32_t ph = (j >> 1) & 1;
          ok = wait_bar(&bars[kPReady + x], ph) && wait_bar(&bars[kVReady + x], ph);
          if (ok && i == 0 && item > 0) ok = wait_bar(&bars[kOFree], (item - 1) & 1);
          if (!ok) break;
          tc_fence_after();
          const uint32_t spj = sp + (j % kNP) * kPBuf;
#pragma unroll
          for (int ks = 0; ks < kBlk / 16; ++ks)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const uint64_t a = smem_desc(spj + ks * 32, 16, 1024, 2);
              const uint64_t bd =
                  smem_desc(sv + x * kVBuf + hf * kVHalf + ks * 4096, 1024, 2048, 2);
              umma_pair_f16(tbase + 128 * hf, a, bd, kIdescPV, (i == 0 && ks == 0) ? 0u : 1u);
            }
          umma_commit_pair(&bars[kPvDone + x]);
          umma_commit_pair(&bars[kPFree + j % kNP]);
        }
        ++item;
      });
      umma_commit_pair_local(&bars[kDrain + 2]);
      mbar_wait_cluster(&bars[kDrain + 2], 0);
    }
  } else if (warp >= 6) {
    // ---------------- V conversion: E4M3 codes -> f16 B operand of PV ----------------
    const int vt = threadIdx.x - 192;                     // 0..127
    const int tt = vt & 63, vh = vt >> 6;                 // token, PV instruction half
    const int row = tt & 31;
    // token tt sits in the key stage of CTA tt / 32; this CTA's value dims
    // 256*vh + 128*rank + [0, 128) are atom 2*vh + rank of that stage
    const uint32_t src = mapa_shared(smem_u32(smem + kOffK), static_cast<uint32_t>(tt >> 5)) +
                         (2 * vh + rank) * kQkAtom;
    const float* kscl = reinterpret_cast<const float*>(smem + kOffKSc);
    float* ring = reinterpret_cast<float*>(smem + kOffScR);
    int32_t j = 0;
    bool ok = true;
    for_pieces(p, u0, u1, [&](int b, int32_t t0, int32_t nt) {
      const int32_t ntok = seq_tokens(p, b);
      for (int32_t i = 0; i < nt; ++i, ++j) {
        const int s = j % kNK, x = j & 1;
        const uint32_t n = static_cast<uint32_t>(j / kNK);
        // both CTAs' stages have landed: the leader's barrier counts both
        // loads, and the leader's QK-hi issuer forwards its completion
        ok = ok && wait_bar(&bars[rank == 0 ? kKFull + s : kKPeerFull + s], n & 1u);
        ok = ok && wait_bar(&bars[kScL + s], n & 1u);
        if (j >= 2) ok = ok && wait_bar(&bars[kPvDone + x], ((j >> 1) & 1) ^ 1);
        if (ok) {
          const int32_t nvalid = min(kBlk, ntok - (t0 + i) * kBlk);
          const bool valid = tt < nvalid;
          const uint32_t sa = src + s * kStage;
          uint8_t* dst = smem + kOffV + x * kVBuf + vh * kVHalf;
          uint4 wv[8];                                    // all eight loads in flight at once
#pragma unroll
          for (int c = 0; c < 8; ++c)
            wv[c] = valid ? ld_cluster128(sa + sw128(row, c)) : make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int c = 0; c < 8; ++c) {                   // 16 codes = dims 16c..16c+15
            const uint4 w = wv[c];
            uint32_t f[8];
            e4m3x4_to_f16x2x2(w.x, f[0], f[1]);
            e4m3x4_to_f16x2x2(w.y, f[2], f[3]);
            e4m3x4_to_f16x2x2(w.z, f[4], f[5]);
            e4m3x4_to_f16x2x2(w.w, f[6], f[7]);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {              // 8 dims per 16-byte V chunk
              const int cc = 2 * c + hh;
              const uint32_t off = (cc >> 3) * 1024 + (tt >> 3) * 2048 + (tt & 7) * 128 +
                                   (((cc & 7) ^ (tt & 7)) << 4);
              *reinterpret_cast<uint4*>(dst + off) =
                  make_uint4(f[4 * hh], f[4 * hh + 1], f[4 * hh + 2], f[4 * hh + 3]);
            }
          }
          if (vt < kBlk)      // token scales for the softmax (0 past the end or off the cache)
            ring[(j & (kNSc - 1)) * kBlk + vt] = (flag[s] != 0 && vt < nvalid) ? kscl[s * kBlk + vt] : 0.0f;
        }
        fence_proxy_async_smem();
        named_bar(2, 128);
        if (vt == 0 && ok) {      // the softmax and the PV issuer first, then the stage
          mbar_arrive(&bars[kScR + (j & (kNSc - 1))]);
          arrive_leader(&bars[kVReady + x], rank);
          mbar_arrive(&bars[kKFree + s]);
          mbar_arrive_remote(mapa_shared(smem_u32(&bars[kKFree + s]), rank ^ 1u));
        }
      }
    });
  } else {
    // ---------------- softmax warps: scores, P, epilogue ----------------
    const int mt = threadIdx.x - 64;                      // 0..127
    const int L = 32 * (warp & 3) + lane;                 // this thread's TMEM lane
    const int hl = L & 63, half = L >> 6;                 // head (in this CTA), token half
    const uint32_t tl = tbase + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    const float* qexp = reinterpret_cast<const float*>(smem + kOffQ + 2 * kQPart);
    const float* ring = reinterpret_cast<const float*>(smem + kOffScR);
    float* xm = reinterpret_cast<float*>(smem + kOffXm);
    float* xl = reinterpret_cast<float*>(smem + kOffXl);
    const float kNegInf = -__int_as_float(0x7f800000);
    int32_t j = 0, item = 0, q_loads = 0;
    bool ok = true;
    // Every softmax thread runs the same loop trips and named barriers; after
    // a failed wait (ok == false) the work is skipped but the barriers kept.
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

      float m_ref = kNegInf, l_part = 0.0f;
      for (int32_t i = 0; i < nt; ++i, ++j) {
        const int s2 = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const int32_t nvalid = min(kBlk, ntok - (t0 + i) * kBlk);
        ok = ok && wait_bar(&bars[kSHi + s2], ph) && wait_bar(&bars[kSLo + s2], ph);
        ok = ok && wait_bar(&bars[kScR + (j & (kNSc - 1))], (j >> 2) & 1);
        ok = __all_sync(0xffffffffu, ok);                   // tcgen05.ld is warp-collective
        tc_fence_after();
        uint32_t rh[32], rl[32];
        if (ok) {
          tmem_ld32(tl + kColSHi + 32 * s2, rh);
          tmem_ld32(tl + kColSLo + 32 * s2, rl);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) rh[c] = rl[c] = 0u;
        }
        tc_fence_before();
        // this thread's 32 token scales (0 past the end of the sequence or off the cache)
        float sc[32];
        {
          const float4* s4 =
              reinterpret_cast<const float4*>(ring + (j & (kNSc - 1)) * kBlk + 32 * half);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float4 v = s4[k];
            sc[4 * k] = v.x;
            sc[4 * k + 1] = v.y;
            sc[4 * k + 2] = v.z;
            sc[4 * k + 3] = v.w;
          }
        }
        const float alpha = p.sm_scale * kLog2e * qexp[hl];
        float x[32];
        float bm = kNegInf;
#pragma unroll
        for (int c = 0; c < 32; ++c) x[c] = (__uint_as_float(rh[c]) + __uint_as_float(rl[c])) * (alpha * sc[c]);
        if (nvalid < kBlk) {
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (32 * half + c >= nvalid) x[c] = kNegInf;
        }
#pragma unroll
        for (int c = 0; c < 32; ++c) bm = fmaxf(bm, x[c]);
        // head maxima, double-buffered by block parity: the next write to this
        // half comes after the next block's barrier, which the partner passes
        // only after this read
        float* xmj = xm + s2 * 128;
        xmj[L] = bm;
        named_bar(1, 128);                                // every S load of this block done
        if (mt == 0 && ok) arrive_leader(&bars[kSFree + s2], rank);
        bm = fmaxf(bm, xmj[L ^ 64]);
        // Move the reference max when a score exceeds it by 2^8.  The vote keeps
        // the TMEM accesses warp-uniform; the warp holding the other token half
        // of the same 32 heads sees the same head maxima and votes alike.
        if (__any_sync(0xffffffffu, bm > m_ref + 8.0f)) {
          const float m_new = fmaxf(m_ref, bm);
          const float r = ex2(m_ref - m_new);             // 0 on the first block, 1 if unmoved
          l_part *= r;
          if (i > 0) {
            // O must not be in use by the previous block's PV
            ok = ok && wait_bar(&bars[kPvDone + ((j - 1) & 1)], ((j - 1) >> 1) & 1);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if (ok) {
#pragma unroll 1
              for (int cc = 0; cc < 8; ++cc) {
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
          m_ref = m_new;
        }
        // ---- P (f16, token scale folded in) into the A operand of PV ----
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float p0 = ex2(x[c] - m_ref), p1 = ex2(x[c + 1] - m_ref);
          l_part += p0 + p1;
          pk[c >> 1] = pack_f16x2(p0 * sc[c], p1 * sc[c + 1]);
        }
        const int pb = j % kNP;
        if (j >= kNP)                                     // P buffer free: PV(j - kNP) done
          ok = ok && wait_bar(&bars[kPFree + pb], static_cast<uint32_t>((j / kNP) & 1) ^ 1u);
        if (ok) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            *reinterpret_cast<uint4*>(smem + kOffP + pb * kPBuf + sw128(hl, 4 * half + k)) =
                make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
        tc_fence_before();
        fence_proxy_async_smem();
        named_bar(1, 128);
        if (mt == 0 && ok) arrive_leader(&bars[kPReady + s2], rank);
      }

      // ---- epilogue: O / l and lse for this piece ----
      {
        const int32_t jl = j - 1;
        ok = ok && wait_bar(&bars[kPvDone + (jl & 1)], (jl >> 1) & 1);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        xl[L] = l_part;
        named_bar(1, 128);
        const float l_tot = l_part + xl[L ^ 64];
        const float inv = 1.0f / l_tot;
        const int hg = 64 * static_cast<int>(rank) + hl;
        const int64_t slot = pair + b;
        float* orow = p.ws_o + (slot * kHq + hg) * kDv;
#pragma unroll 1
        for (int cc = 0; cc < 8 && ok; ++cc) {
          uint32_t o[32];
          tmem_ld32(tl + 32 * cc, o);
          tmem_wait_ld();
          const int dv0 = 256 * (cc >> 2) + 128 * half + 32 * (cc & 3);
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            *reinterpret_cast<float4*>(orow + dv0 + k) =
                make_float4(__uint_as_float(o[k]) * inv, __uint_as_float(o[k + 1]) * inv,
                            __uint_as_float(o[k + 2]) * inv, __uint_as_float(o[k + 3]) * inv);
        }
        if (half == 0 && ok) p.ws_lse[slot * kHq + hg] = (m_ref + __log2f(l_tot)) * kLn2;
        tc_fence_before();
        named_bar(1, 128);
        if (mt == 0 && ok) arrive_leader(&bars[kOFree], rank);
      }
      ++item;
    });
    // a query-image load whose wait gave up lands before the CTA exits
    if (mt == 0 && q_loads > 0) mbar_wait_cluster(&bars[kQFull], (q_loads - 1) & 1);
  }

  __syncthreads();
  cluster_sync_all();            // the leader's MMAs no longer read this CTA's memory
  if (warp == kWarpQkHi) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, kTmemCols);
  }
}

}  // namespace wide

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static cudaError_t prepare_wide(int dev) {
  static bool done[64] = {};
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
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
  static int last_n[64];
  static bool have[64] = {};
  if (dev < 0 || dev >= 64) return 0;
  if (have[dev]) return last_n[dev];
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
  wide::wide_prep_kernel<<<2 * a.B + 1, wide::kPrepThreads, 0, a.stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.num_ctas);
  cfg.blockDim = dim3(wide::kThreads);
  cfg.dynamicSmemBytes = wide::kSmemBytes;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, wide::wide_decode_kernel, kqk, ktail, p);
  if (e != cudaSuccess) return e;
  return launch_lse_combine(p.ws_pre, p.ws_lse, p.ws_o, a.B, 1, wide::kHq, wide::kHq, wide::kDv,
                            a.num_ctas, a.out, a.lse, a.stream);
}

}  // namespace kvq
