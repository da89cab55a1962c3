// Batched page-tag validation, run as its own launch before decode reads the
// cache (not fused into attention, where thread groups could race on it):
// "Cloudflare: Kleinere Modellbereitstellung senkt Speicherbedarf, doch
// Sicherheit wird zum Prüfstein" (remio.ai), section "Sicherheit gemeinsamer
// KV-Caches wird zum Produktionsthema"; "Cloudflare zrýchľuje inferenciu
// modelov Kimi a GLM kompresiou cache a váh" (aifeed.sk), section "Kvalita
// odpovedí a integrita spoločnej cache".
//
// Grid: (chunks of kChunk entries, B).  The mask is cleared by a memset on
// the same stream first; a block that finds a bad entry writes 1.  The cost
// is launch latency plus two dependent loads per entry (the block table /
// expected tag, then the live-tag gather), so each thread keeps kPerThread
// independent entries in flight.
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

constexpr int kValThreads = 256;
constexpr int kPerThread = 8;
constexpr int kChunk = kValThreads * kPerThread;

__global__ void __launch_bounds__(kValThreads)
    validate_kernel(const uint32_t* __restrict__ tags, int32_t P,
                    const int32_t* __restrict__ block_table,
                    const uint32_t* __restrict__ expected, const int32_t* __restrict__ seq_lens,
                    int32_t ps, int32_t max_pages, uint8_t* __restrict__ abort_mask) {
  const int32_t b = blockIdx.y;
  int64_t n = seq_lens[b];
  n = n < 0 ? 0 : n;
  const int64_t cap = static_cast<int64_t>(max_pages) * ps;
  n = n > cap ? cap : n;
  const int32_t npages = static_cast<int32_t>((n + ps - 1) / ps);
  const int32_t base = blockIdx.x * kChunk;
  if (base >= npages) return;                          // block-uniform
  const int32_t* bt = block_table + static_cast<int64_t>(b) * max_pages;
  const uint32_t* ex = expected + static_cast<int64_t>(b) * max_pages;
  int32_t page[kPerThread];
  uint32_t want[kPerThread];
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int32_t i = base + k * kValThreads + threadIdx.x;   // coalesced
    page[k] = 0;
    want[k] = 0;
    if (i < npages) {
      page[k] = bt[i];
      want[k] = ex[i];
    }
  }
  int bad = 0;
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int32_t i = base + k * kValThreads + threadIdx.x;
    if (i < npages) {
      const int32_t p = page[k];
      if (p < 0 || p >= P) bad = 1;
      else if (tags[p] != want[k]) bad = 1;
    }
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) abort_mask[b] = 1;
}

cudaError_t launch_validate(const uint32_t* tags, int32_t P, const int32_t* block_table,
                            const uint32_t* expected, const int32_t* seq_lens, int32_t ps,
                            int32_t B, int32_t max_pages, uint8_t* abort_mask,
                            cudaStream_t stream) {
  if (B == 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(abort_mask, 0, static_cast<size_t>(B), stream);
  if (e != cudaSuccess) return e;
  dim3 grid((max_pages + kChunk - 1) / kChunk, B);
  validate_kernel<<<grid, kValThreads, 0, stream>>>(tags, P, block_table, expected, seq_lens, ps,
                                                    max_pages, abort_mask);
  return cudaGetLastError();
}

cudaError_t read_and_clear_error_flags(uint32_t* flags) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(flags, g_error_flags, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_error_flags, &zero, sizeof(uint32_t));
}

}  // namespace kvq
