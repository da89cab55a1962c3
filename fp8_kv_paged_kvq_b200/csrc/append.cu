// Write path of the FP8 cache: amax / scale, tag bump on reallocation, and
// quantize-on-append with 16-byte vector stores.
//
// Sources: the decode pool stores keys and values as E4M3 instead of BF16
// ("Công thức của Cloudflare để phục vụ Kimi và GLM ..." (manulx.blog),
// section "Bộ nhớ đệm KV FP8 tăng gấp đôi dung lượng ngữ cảnh"); each physical
// page's tag changes on reallocation ("Cloudflare: Kleinere
// Modellbereitstellung senkt Speicherbedarf, doch Sicherheit wird zum
// Prüfstein" (remio.ai), section "Sicherheit gemeinsamer KV-Caches wird zum
// Produktionsthema").
#include <mutex>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

template <typename K>
cudaError_t prefer_max_shared(K* kernel) {
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev]) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

// ---------------------------------------------------------------------------
// amax: one block per (row chunk, head or all heads); 16-byte loads.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* __restrict__ x, int64_t T,
                                                   int32_t H, int32_t D, int32_t per_head,
                                                   float* __restrict__ amax_io) {
  const int32_t vec_per_row = D / 8;                    // uint4 = 8 bf16
  const int32_t rows_h = per_head ? 1 : H;              // heads this block covers
  const int32_t h0 = per_head ? blockIdx.y : 0;
  const int64_t n_vec = T * rows_h * vec_per_row;
  float m = 0.0f;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n_vec;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / vec_per_row;                // (t, h-in-block)
    const int32_t v = static_cast<int32_t>(i % vec_per_row);
    const int64_t t = row / rows_h;
    const int32_t h = h0 + static_cast<int32_t>(row % rows_h);
    const uint4 w = *reinterpret_cast<const uint4*>(x + ((t * H + h) * D) + v * 8);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      m = fmaxf(m, fabsf(bf16lo_to_f32(ws[k])));        // fmaxf drops NaN operands
      m = fmaxf(m, fabsf(bf16hi_to_f32(ws[k])));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 1; k < (int)(blockDim.x >> 5); ++k) m = fmaxf(m, red[k]);
    // Non-negative floats order like their bit patterns.
    atomicMax(reinterpret_cast<unsigned int*>(amax_io + h0), __float_as_uint(m));
  }
}

__global__ void scale_from_amax_kernel(const float* __restrict__ amax, float* __restrict__ scale,
                                       int32_t n) {
  const int32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float a = amax[i];
    scale[i] = (a > 0.0f) ? __fdiv_rn(a, 448.0f) : 1.0f;
  }
}

// ---------------------------------------------------------------------------
// Append: the token blocks quantize and write the new rows (a warp per
// head and 8 tokens, or per row; see append_rows_batched and the per-row
// path in append_kernel), lanes holding 16-value groups written with one
// 16-byte store each; the last block bumps the tags of reallocated pages.
// ---------------------------------------------------------------------------
// The quotient v / s that the E4M3 encode rounds, RN(v / s), without a
// hardware division per value.  r = RN(1/s) is worked out once per scale.
//  * s a power of two: r = 1/s exactly and q0 = RN(v r) = RN(v / s).
//  * otherwise Markstein's correction: q0 = RN(v r), rem = RN(v - q0 s) (one
//    FMA), q1 = RN(q0 + rem r) (one FMA) equals RN(v / s) for every bf16 v
//    and every float s whose values and intermediates stay normal; checked
//    over all 128 bf16 significands x all 2^23 float significands (powers of
//    two only shift every step).  That holds for |s| in [2^-40, 2^40] and
//    2^-100 <= |v| < 2^88.  Below 2^-100 the quotient is under 2^-59 and
//    encodes to a signed zero, whatever its magnitude; the sign is taken
//    from q0, the sign of v r (zeros included).  From 2^88 up (infinities
//    and NaNs too) the caller divides.
struct QuantScale {
  float s, r;
  int kind;          // 0: divide; 1: product (s a power of two); 2: corrected product
};

__device__ __forceinline__ QuantScale quant_scale(float s) {
  const float as = fabsf(s);
  const bool in = as >= 0x1p-40f && as <= 0x1p40f;               // NaN: out
  const bool pow2 = (__float_as_uint(s) & 0x7FFFFFu) == 0u;
  return QuantScale{s, __frcp_rn(s), in ? (pow2 ? 1 : 2) : 0};
}

template <bool kPow2>
__device__ __forceinline__ float quant_quotient(float v, float s, float r) {
  const float q0 = v * r;
  if (kPow2) return q0;
  const float rem = fmaf(-q0, s, v);
  const float q1 = fmaf(rem, r, q0);
  return __uint_as_float((__float_as_uint(q1) & 0x7FFFFFFFu) | (__float_as_uint(q0) & 0x80000000u));
}

// Eight bf16 values to eight E4M3 codes by the quotient above.  Without
// kPow2, big collects the bf16 exponent fields plus 41: bit 15 or 31 set
// means a value of magnitude 2^88 or more (infinities, NaNs), which the
// caller sends to the division.
template <bool kPow2>
__device__ __forceinline__ uint2 quantize8_mul(const uint4 a, float s, float r, uint32_t& big) {
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
  uint32_t pairs[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (!kPow2) big |= (w[k] & 0x7F807F80u) + 0x14801480u;
    pairs[k] = f32x2_to_e4m3x2(quant_quotient<kPow2>(bf16lo_to_f32(w[k]), s, r),
                               quant_quotient<kPow2>(bf16hi_to_f32(w[k]), s, r));   // lo | hi << 8
  }
  return make_uint2(pairs[0] | (pairs[1] << 16), pairs[2] | (pairs[3] << 16));
}

// The same codes through the IEEE division (a call of its own, so it costs
// nothing where it is skipped).
__device__ __noinline__ uint2 quantize8_div(const uint4 a, float s) {
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
  uint32_t pairs[4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    pairs[k] = f32x2_to_e4m3x2(__fdiv_rn(bf16lo_to_f32(w[k]), s),
                               __fdiv_rn(bf16hi_to_f32(w[k]), s));
  return make_uint2(pairs[0] | (pairs[1] << 16), pairs[2] | (pairs[3] << 16));
}

// Eight bf16 values to eight E4M3 codes of v / s: E(RN(v / s)), rounding to
// nearest even with saturation in the conversion.
__device__ __forceinline__ uint2 quantize8(const uint4 a, const QuantScale& d) {
  uint32_t big = 0u;
  if (d.kind == 1) return quantize8_mul<true>(a, d.s, d.r, big);
  const uint2 c = quantize8_mul<false>(a, d.s, d.r, big);
  return d.kind == 2 && (big & 0x80008000u) == 0u ? c : quantize8_div(a, d.s);
}

// One float value, the same way (the exhaustive check of the quotient):
// the corrected product where its argument holds, else the division.
__device__ __forceinline__ uint32_t quantize1(float v, const QuantScale& d) {
  const uint32_t ev = (__float_as_uint(v) >> 23) & 0xFFu;
  float q;
  if (d.kind == 1) q = quant_quotient<true>(v, d.s, d.r);
  else if (d.kind == 2 && ev < 215u) q = quant_quotient<false>(v, d.s, d.r);
  else q = __fdiv_rn(v, d.s);
  return f32x2_to_e4m3x2(q, 0.0f) & 0xFFu;
}

__device__ __forceinline__ float amax8(const uint4 a) {
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
  float m = 0.0f;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    m = fmaxf(m, fmaxf(fabsf(bf16lo_to_f32(w[k])), fabsf(bf16hi_to_f32(w[k]))));
  return m;                                   // fmaxf drops NaN operands
}

constexpr int kAppendWarps = 8;
constexpr int kRowsPerWarp = 8;      // (token, head) rows per warp in the batched case

struct AppendArgs {
  CacheView c;
  const uint16_t* k_new;
  const uint16_t* v_new;
  const int32_t* slot_mapping;
  int32_t T;
  const int32_t* realloc_pages;
  int32_t n_realloc;
  int32_t token_blocks;  // blocks that handle tokens; the next block bumps tags
  int32_t batched;       // rows per warp: kRowsPerWarp (batched case) or 1
};

// The common case: K and V head dims that are multiples of 16, whose
// 16-value groups per token (gt = Dk/16 + Dv/16) divide the warp into tp =
// 32 / gt tokens (2 for d 128, 4 for d 64), and a per-tensor or per-head
// scale.  A warp takes kRowsPerWarp tokens of one KV head in kRowsPerWarp /
// tp passes; lane l holds group l % gt (the K row's groups, then the V
// row's) of token l / gt of each pass: two 16-byte loads of bf16, one
// 16-byte store of 16 codes.  All loads are issued before any conversion
// (eight 16-byte loads per lane in flight).  Warp w takes head w % Hkv of
// tokens kRowsPerWarp * (w / Hkv) + [0, kRowsPerWarp): it writes consecutive
// slots of one head (contiguous bytes when the tokens' slots are
// consecutive), and the warps of a block, consecutive heads of the same
// tokens, read one contiguous span of the new K and V rows.
constexpr int kMaxPass = 4;          // kRowsPerWarp / tp for tp >= 2

template <bool FP8>
__device__ __forceinline__ void append_rows_batched(const AppendArgs& a, int32_t w, int lane) {
  const CacheView& c = a.c;
  const int32_t h = w % c.Hkv;
  const int32_t tb = (w / c.Hkv) * kRowsPerWarp;
  const int32_t gk = c.Dk / 16, gt = gk + c.Dv / 16;
  const int32_t tp = 32 / gt, passes = kRowsPerWarp / tp;
  const int32_t sub = lane / gt, g = lane - sub * gt;
  const bool isk = g < gk;
  const int32_t e = 16 * (isk ? g : g - gk);
  uint4 x[kMaxPass][2];
#pragma unroll
  for (int p = 0; p < kMaxPass; ++p) {
    x[p][0] = x[p][1] = make_uint4(0, 0, 0, 0);
    const int64_t t = tb + p * tp + sub;
    if (p < passes && t < a.T) {
      const uint16_t* src =
          (isk ? a.k_new + (t * c.Hkv + h) * c.Dk : a.v_new + (t * c.Hkv + h) * c.Dv) + e;
      x[p][0] = __ldg(reinterpret_cast<const uint4*>(src));
      x[p][1] = __ldg(reinterpret_cast<const uint4*>(src + 8));
    }
  }
  // Lane i works out token tb + i's cache row (-1: none) in 32-bit
  // arithmetic; the warp reads it by shuffle.
  int64_t my_row = -1;
  if (lane < kRowsPerWarp && tb + lane < a.T) {
    const int32_t slot = __ldg(a.slot_mapping + tb + lane);
    if (slot >= 0 && static_cast<int64_t>(slot) < static_cast<int64_t>(c.P) * c.ps) {
      const uint32_t pg = static_cast<uint32_t>(slot) / static_cast<uint32_t>(c.ps);
      const uint32_t o = static_cast<uint32_t>(slot) - pg * static_cast<uint32_t>(c.ps);
      my_row = (static_cast<int64_t>(pg) * c.Hkv + h) * c.ps + o;
    }
  }
  // FP8: the product quotient for every value, or the division for all of
  // this lane's values when one of them is 2^88 or more, an infinity or a
  // NaN (bf16 exponent field plus 41 carries into bit 15 or 31), or the
  // scale is out of the product's range
  QuantScale qs{1.0f, 1.0f, 1};
  bool slow = false;
  if (FP8) {
    qs = quant_scale((isk ? c.k_scale : c.v_scale)[c.scale_mode == 0 ? 0 : h]);
    uint32_t big = 0u;
#pragma unroll
    for (int p = 0; p < kMaxPass; ++p)
#pragma unroll
      for (int j = 0; j < 2; ++j)
        big |= ((x[p][j].x & 0x7F807F80u) + 0x14801480u) | ((x[p][j].y & 0x7F807F80u) + 0x14801480u) |
               ((x[p][j].z & 0x7F807F80u) + 0x14801480u) | ((x[p][j].w & 0x7F807F80u) + 0x14801480u);
    slow = qs.kind == 0 || (qs.kind == 2 && (big & 0x80008000u) != 0u);
  }
#pragma unroll
  for (int p = 0; p < kMaxPass; ++p) {
    const int64_t prow = __shfl_sync(0xffffffffu, my_row, (p * tp + sub) & 31);
    if (p >= passes || prow < 0) continue;
    if (FP8) {
      uint2 lo, hi;
      uint32_t unused = 0u;
      if (slow) {
        lo = quantize8_div(x[p][0], qs.s);
        hi = quantize8_div(x[p][1], qs.s);
      } else if (qs.kind == 1) {
        lo = quantize8_mul<true>(x[p][0], qs.s, qs.r, unused);
        hi = quantize8_mul<true>(x[p][1], qs.s, qs.r, unused);
      } else {
        lo = quantize8_mul<false>(x[p][0], qs.s, qs.r, unused);
        hi = quantize8_mul<false>(x[p][1], qs.s, qs.r, unused);
      }
      uint8_t* dst = static_cast<uint8_t*>(isk ? c.k_pages : c.v_pages) +
                     prow * (isk ? c.Dk : c.Dv) + e;
      *reinterpret_cast<uint4*>(dst) = make_uint4(lo.x, lo.y, hi.x, hi.y);
    } else {
      uint16_t* dst = static_cast<uint16_t*>(isk ? c.k_pages : c.v_pages) +
                      prow * (isk ? c.Dk : c.Dv) + e;
      reinterpret_cast<uint4*>(dst)[0] = x[p][0];
      reinterpret_cast<uint4*>(dst)[1] = x[p][1];
    }
  }
}

__global__ void __launch_bounds__(kAppendWarps * 32, 4) append_kernel(AppendArgs a) {
  pdl_trigger();            // the tag check may start loading its block-table entries
  const CacheView& c = a.c;
  if (static_cast<int32_t>(blockIdx.x) >= a.token_blocks) {
    for (int32_t i = threadIdx.x; i < a.n_realloc; i += blockDim.x) {
      const int32_t p = a.realloc_pages[i];
      if (p >= 0 && p < c.P) atomicAdd(c.tags + p, 1u);
    }
    return;
  }
  const int lane = threadIdx.x & 31;
  if (a.batched > 1) {
    const int32_t w = static_cast<int32_t>(blockIdx.x) * kAppendWarps + (threadIdx.x >> 5);
    if (c.fp8) append_rows_batched<true>(a, w, lane);
    else append_rows_batched<false>(a, w, lane);
    return;
  }
  const uint32_t row = blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
  if (static_cast<int64_t>(row) >= static_cast<int64_t>(a.T) * c.Hkv) return;
  const int32_t t = static_cast<int32_t>(row / static_cast<uint32_t>(c.Hkv));
  const int32_t h = static_cast<int32_t>(row) - t * c.Hkv;
  const int32_t slot = a.slot_mapping[t];
  if (slot < 0 || static_cast<int64_t>(slot) >= static_cast<int64_t>(c.P) * c.ps) return;
  const uint32_t pg = static_cast<uint32_t>(slot) / static_cast<uint32_t>(c.ps);
  const uint32_t o = static_cast<uint32_t>(slot) - pg * static_cast<uint32_t>(c.ps);
  const int64_t prow = (static_cast<int64_t>(pg) * c.Hkv + h) * c.ps + o;   // [P][Hkv][ps] row
  // 16-value groups (two 16-byte loads, one 16-byte store of codes) when
  // both head dims allow, else 8-value groups
  const bool g16 = c.Dk % 16 == 0 && (c.v_pages == nullptr || c.Dv % 16 == 0);
  const int32_t gw = g16 ? 16 : 8;
  const int32_t nk = c.Dk / gw, nv = c.v_pages == nullptr ? 0 : c.Dv / gw;
  const uint16_t* ksrc = a.k_new + (static_cast<int64_t>(t) * c.Hkv + h) * c.Dk;
  const uint16_t* vsrc = a.v_new + (static_cast<int64_t>(t) * c.Hkv + h) * c.Dv;
  if (!c.fp8) {
    uint16_t* kdst = static_cast<uint16_t*>(c.k_pages) + prow * c.Dk;
    uint16_t* vdst = static_cast<uint16_t*>(c.v_pages) + prow * c.Dv;
    for (int32_t g = lane; g < nk + nv; g += 32) {
      const bool isk = g < nk;
      const int32_t e = gw * (isk ? g : g - nk);
      const uint4* src = reinterpret_cast<const uint4*>((isk ? ksrc : vsrc) + e);
      uint4* dst = reinterpret_cast<uint4*>((isk ? kdst : vdst) + e);
      dst[0] = src[0];
      if (g16) dst[1] = src[1];
    }
    return;
  }
  float sk, sv = 1.0f;
  if (c.scale_mode == 0) {
    sk = c.k_scale[0];
    if (nv) sv = c.v_scale[0];
  } else if (c.scale_mode == 1) {
    sk = c.k_scale[h];
    if (nv) sv = c.v_scale[h];
  } else {
    // per-token scale: amax over each row, reduced across the warp
    float ak = 0.0f, av = 0.0f;
    for (int32_t g = lane; g < nk + nv; g += 32) {
      const bool isk = g < nk;
      const uint4* src = reinterpret_cast<const uint4*>((isk ? ksrc : vsrc) + gw * (isk ? g : g - nk));
      float m = amax8(src[0]);
      if (g16) m = fmaxf(m, amax8(src[1]));
      if (isk) ak = fmaxf(ak, m);
      else av = fmaxf(av, m);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      ak = fmaxf(ak, __shfl_xor_sync(0xffffffffu, ak, off));
      av = fmaxf(av, __shfl_xor_sync(0xffffffffu, av, off));
    }
    sk = (ak > 0.0f) ? __fdiv_rn(ak, 448.0f) : 1.0f;
    sv = (av > 0.0f) ? __fdiv_rn(av, 448.0f) : 1.0f;
    if (lane == 0) {
      c.k_scale[prow] = sk;
      if (nv) c.v_scale[prow] = sv;
    }
  }
  uint8_t* kdst = static_cast<uint8_t*>(c.k_pages) + prow * c.Dk;
  uint8_t* vdst = nv ? static_cast<uint8_t*>(c.v_pages) + prow * c.Dv : nullptr;
  const QuantScale qk = quant_scale(sk), qv = quant_scale(sv);
  for (int32_t g = lane; g < nk + nv; g += 32) {
    const bool isk = g < nk;
    const int32_t e = gw * (isk ? g : g - nk);
    const uint4* src = reinterpret_cast<const uint4*>((isk ? ksrc : vsrc) + e);
    uint8_t* dst = (isk ? kdst : vdst) + e;
    const uint2 lo = quantize8(src[0], isk ? qk : qv);
    if (g16) {
      const uint2 hi = quantize8(src[1], isk ? qk : qv);
      *reinterpret_cast<uint4*>(dst) = make_uint4(lo.x, lo.y, hi.x, hi.y);
    } else {
      *reinterpret_cast<uint2*>(dst) = lo;
    }
  }
}

// ---------------------------------------------------------------------------
// Exhaustive codec check: encode the floats with bit patterns start + i.
// ---------------------------------------------------------------------------
__global__ void encode_bits_kernel(uint32_t start, uint32_t count, uint8_t* __restrict__ out) {
  const uint64_t i4 = (static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4u;
  if (i4 >= count) return;
  const uint32_t b = start + static_cast<uint32_t>(i4);     // bit patterns wrap mod 2^32
  if (i4 + 4u <= count) {
    const uint32_t lo = f32x2_to_e4m3x2(__uint_as_float(b), __uint_as_float(b + 1u));
    const uint32_t hi = f32x2_to_e4m3x2(__uint_as_float(b + 2u), __uint_as_float(b + 3u));
    *reinterpret_cast<uint32_t*>(out + i4) = lo | (hi << 16);   // out is 4-byte aligned
  } else {
    for (uint64_t k = i4; k < count; ++k)
      out[k] = static_cast<uint8_t>(
          f32x2_to_e4m3x2(__uint_as_float(start + static_cast<uint32_t>(k)), 0.0f) & 0xFFu);
  }
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
cudaError_t launch_amax(const uint16_t* x, int64_t T, int32_t H, int32_t D, int32_t per_head,
                        float* amax_io, cudaStream_t stream) {
  const int64_t rows = T * (per_head ? 1 : H);
  const int64_t n_vec = rows * (D / 8);
  if (n_vec == 0) return cudaSuccess;
  const int64_t want = (n_vec + 255) / 256;
  const unsigned gx = static_cast<unsigned>(want < 4096 ? want : 4096);
  dim3 grid(gx, per_head ? H : 1);
  amax_kernel<<<grid, 256, 0, stream>>>(x, T, H, D, per_head, amax_io);
  return cudaGetLastError();
}

cudaError_t launch_scale_from_amax(const float* amax, float* scale, int32_t n,
                                   cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  scale_from_amax_kernel<<<(n + 255) / 256, 256, 0, stream>>>(amax, scale, n);
  return cudaGetLastError();
}

cudaError_t launch_append(const CacheView& c, const uint16_t* k_new, const uint16_t* v_new,
                          const int32_t* slot_mapping, int32_t T, const int32_t* realloc_pages,
                          int32_t n_realloc, cudaStream_t stream) {
  AppendArgs a;
  a.c = c;
  a.k_new = k_new;
  a.v_new = v_new;
  a.slot_mapping = slot_mapping;
  a.T = T;
  a.realloc_pages = realloc_pages;
  a.n_realloc = n_realloc;
  const int64_t rows = static_cast<int64_t>(T) * c.Hkv;
  const int32_t gt = c.Dk / 16 + c.Dv / 16;   // 16-value groups per token (batched case)
  const bool batched = c.v_pages != nullptr && c.Dk % 16 == 0 && c.Dv % 16 == 0 && gt >= 4 &&
                       gt <= 16 && 32 % gt == 0 &&
                       (!c.fp8 || c.scale_mode != 2);
  a.batched = batched ? kRowsPerWarp : 1;
  // batched: one warp per (head, group of kRowsPerWarp tokens); else one per row
  const int64_t warps =
      batched ? (static_cast<int64_t>(T) + kRowsPerWarp - 1) / kRowsPerWarp * c.Hkv : rows;
  a.token_blocks = static_cast<int32_t>((warps + kAppendWarps - 1) / kAppendWarps);
  const int32_t blocks = a.token_blocks + (n_realloc > 0 ? 1 : 0);
  if (blocks == 0) return cudaSuccess;
  append_kernel<<<blocks, kAppendWarps * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

// Exhaustive check of the append path's quantize step:
// out[i] = E(bits(start + i) / scale) with the same division and conversion.
__global__ void quantize_bits_kernel(uint32_t start, uint32_t count, float scale,
                                     uint8_t* __restrict__ out) {
  const uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= count) return;
  out[i] = static_cast<uint8_t>(
      quantize1(__uint_as_float(start + static_cast<uint32_t>(i)), quant_scale(scale)));
}

cudaError_t launch_quantize_bits(uint32_t start, uint32_t count, float scale, uint8_t* out,
                                 cudaStream_t stream) {
  if (count == 0) return cudaSuccess;
  quantize_bits_kernel<<<static_cast<unsigned>((static_cast<uint64_t>(count) + 255) / 256), 256,
                         0, stream>>>(start, count, scale, out);
  return cudaGetLastError();
}

cudaError_t launch_encode_bits(uint32_t start, uint32_t count, uint8_t* out,
                               cudaStream_t stream) {
  if (count == 0) return cudaSuccess;
  const uint64_t threads = (static_cast<uint64_t>(count) + 3u) / 4u;
  encode_bits_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(start, count,
                                                                                        out);
  return cudaGetLastError();
}

}  // namespace kvq
