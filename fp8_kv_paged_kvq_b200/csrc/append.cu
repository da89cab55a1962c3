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
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

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
// Append: one warp per (token, kv head); the last block also bumps tags.
// ---------------------------------------------------------------------------
// Quantize one row of D bf16 values (D % 16 == 0) into E4M3 codes at dst
// with 16-byte stores; s is the row's scale.
__device__ __forceinline__ void quantize_row(const uint16_t* __restrict__ src,
                                             uint8_t* __restrict__ dst, int32_t D, float s,
                                             int lane) {
  for (int32_t g = lane; g < D / 16; g += 32) {
    const uint4 a = *reinterpret_cast<const uint4*>(src + g * 16);
    const uint4 b = *reinterpret_cast<const uint4*>(src + g * 16 + 8);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t pairs[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float lo = __fdiv_rn(bf16lo_to_f32(w[k]), s);
      const float hi = __fdiv_rn(bf16hi_to_f32(w[k]), s);
      pairs[k] = f32x2_to_e4m3x2(lo, hi);               // 16 bits: lo code | hi code << 8
    }
    uint4 out;
    out.x = pairs[0] | (pairs[1] << 16);
    out.y = pairs[2] | (pairs[3] << 16);
    out.z = pairs[4] | (pairs[5] << 16);
    out.w = pairs[6] | (pairs[7] << 16);
    *reinterpret_cast<uint4*>(dst + g * 16) = out;
  }
}

__device__ __forceinline__ float row_amax(const uint16_t* __restrict__ src, int32_t D, int lane) {
  float m = 0.0f;
  for (int32_t g = lane; g < D / 8; g += 32) {
    const uint4 a = *reinterpret_cast<const uint4*>(src + g * 8);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      m = fmaxf(m, fabsf(bf16lo_to_f32(w[k])));
      m = fmaxf(m, fabsf(bf16hi_to_f32(w[k])));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

__device__ __forceinline__ void copy_row_bf16(const uint16_t* __restrict__ src,
                                              uint16_t* __restrict__ dst, int32_t D, int lane) {
  for (int32_t g = lane; g < D / 8; g += 32)
    *reinterpret_cast<uint4*>(dst + g * 8) = *reinterpret_cast<const uint4*>(src + g * 8);
}

struct AppendArgs {
  CacheView c;
  const uint16_t* k_new;
  const uint16_t* v_new;
  const int32_t* slot_mapping;
  int32_t T;
  const int32_t* realloc_pages;
  int32_t n_realloc;
  int32_t token_blocks;  // blocks that handle tokens; the next block bumps tags
};

constexpr int kAppendWarps = 8;

__global__ void __launch_bounds__(kAppendWarps * 32) append_kernel(AppendArgs a) {
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
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kAppendWarps + (threadIdx.x >> 5);
  if (row >= static_cast<int64_t>(a.T) * c.Hkv) return;
  const int32_t t = static_cast<int32_t>(row / c.Hkv);
  const int32_t h = static_cast<int32_t>(row % c.Hkv);
  const int64_t slot = a.slot_mapping[t];
  if (slot < 0 || slot >= static_cast<int64_t>(c.P) * c.ps) return;
  const int64_t p = slot / c.ps, o = slot % c.ps;
  const int64_t prow = (p * c.Hkv + h) * c.ps + o;   // [P][Hkv][ps] row index
  for (int part = 0; part < 2; ++part) {
    if (part == 1 && c.v_pages == nullptr) break;
    const int32_t D = part ? c.Dv : c.Dk;
    const uint16_t* src = (part ? a.v_new : a.k_new) + (static_cast<int64_t>(t) * c.Hkv + h) * D;
    if (!c.fp8) {
      uint16_t* dst = static_cast<uint16_t*>(part ? c.v_pages : c.k_pages) + prow * D;
      copy_row_bf16(src, dst, D, lane);
      continue;
    }
    float* sc = part ? c.v_scale : c.k_scale;
    float s;
    if (c.scale_mode == 0) {
      s = sc[0];
    } else if (c.scale_mode == 1) {
      s = sc[h];
    } else {
      const float amax = row_amax(src, D, lane);
      s = (amax > 0.0f) ? __fdiv_rn(amax, 448.0f) : 1.0f;
      if (lane == 0) sc[prow] = s;
    }
    uint8_t* dst = static_cast<uint8_t*>(part ? c.v_pages : c.k_pages) + prow * D;
    quantize_row(src, dst, D, s, lane);
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
  a.token_blocks = static_cast<int32_t>((rows + kAppendWarps - 1) / kAppendWarps);
  const int32_t blocks = a.token_blocks + (n_realloc > 0 ? 1 : 0);
  if (blocks == 0) return cudaSuccess;
  append_kernel<<<blocks, kAppendWarps * 32, 0, stream>>>(a);
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
