// Batched page-tag validation, run as its own launch before decode reads the
// cache (not fused into attention, where thread groups could race on it):
// "Cloudflare: Kleinere Modellbereitstellung senkt Speicherbedarf, doch
// Sicherheit wird zum Prüfstein" (remio.ai), section "Sicherheit gemeinsamer
// KV-Caches wird zum Produktionsthema"; "Cloudflare zrýchľuje inferenciu
// modelov Kimi a GLM kompresiou cache a váh" (aifeed.sk), section "Kvalita
// odpovedí a integrita spoločnej cache".
//
// Each request gets a thread-block cluster of C <= 8 CTAs, enough that one
// round of loads covers its block-table row: CTA r checks entries
// r*kPerCta + k*kValThreads + tid (+ C*kPerCta per further round).  The CTAs
// combine their flags through distributed shared memory and rank 0 writes the
// request's mask byte, so no separate clear is needed.  The cost is launch
// latency plus, after the sequence length, two dependent loads per entry:
// the block-table entry with its expected tag, then the live tag.
#include <cooperative_groups.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace cg = cooperative_groups;

constexpr int kValThreads = 512;
constexpr int kPerThread = 8;
constexpr int kPerCta = kValThreads * kPerThread;
constexpr int kMaxCluster = 8;

__global__ void __launch_bounds__(kValThreads)
    validate_kernel(const uint32_t* __restrict__ tags, int32_t P,
                    const int32_t* __restrict__ block_table,
                    const uint32_t* __restrict__ expected, const int32_t* __restrict__ seq_lens,
                    int32_t ps, int32_t max_pages, uint8_t* __restrict__ abort_mask,
                    int32_t* __restrict__ n_aborted, int32_t* __restrict__ first_bad) {
  // Launched as a programmatic dependent of the previous kernel (kvq_append
  // in a decode step), whose launch it overlaps.  The sequence lengths, the
  // block table and the expected tags are read before the wait: a kernel
  // that lets this one start early (kvq_append, which triggers at its start)
  // never writes them, and whatever wrote them earlier in the stream finished
  // before that kernel began.  The live tags, which kvq_append bumps, are
  // read only after the wait.
  pdl_trigger();
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int32_t b = blockIdx.x / C;
  __shared__ int32_t flag;          // this CTA's first failing entry, or INT32_MAX
  __shared__ int32_t warp_min[kValThreads / 32];
  int64_t n = seq_lens[b];
  n = n < 0 ? 0 : n;
  const int64_t cap = static_cast<int64_t>(max_pages) * ps;
  n = n > cap ? cap : n;
  const int32_t npages = static_cast<int32_t>((n + ps - 1) / ps);
  const int32_t* bt = block_table + static_cast<int64_t>(b) * max_pages;
  const uint32_t* ex = expected + static_cast<int64_t>(b) * max_pages;
  int32_t page[kPerThread];
  uint32_t want[kPerThread];
  auto load_round = [&](int32_t base) {
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
  };
  load_round(rank * kPerCta);
  pdl_wait();
  int32_t bad = INT32_MAX;          // smallest failing block-table index seen
  for (int32_t base = rank * kPerCta; base < npages; base += C * kPerCta) {
    if (base != rank * kPerCta) load_round(base);
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int32_t i = base + k * kValThreads + threadIdx.x;
      if (i < npages) {
        const int32_t p = page[k];
        if (p < 0 || p >= P || tags[p] != want[k]) bad = min(bad, i);
      }
    }
  }
  bad = __reduce_min_sync(0xffffffffu, bad);
  if ((threadIdx.x & 31) == 0) warp_min[threadIdx.x >> 5] = bad;
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t m = INT32_MAX;
    for (int w = 0; w < kValThreads / 32; ++w) m = min(m, warp_min[w]);
    flag = m;
  }
  cluster.sync();
  if (rank == 0 && threadIdx.x == 0) {
    int32_t first = INT32_MAX;
    for (int r = 0; r < C; ++r) first = min(first, *cluster.map_shared_rank(&flag, r));
    const bool aborted = first != INT32_MAX;
    abort_mask[b] = aborted ? 1 : 0;
    if (first_bad != nullptr) first_bad[b] = aborted ? first : -1;
    if (n_aborted != nullptr && aborted) atomicAdd(n_aborted, 1);
  }
  cluster.sync();   // every CTA's flag stays alive until rank 0 has read it
}

cudaError_t launch_validate(const uint32_t* tags, int32_t P, const int32_t* block_table,
                            const uint32_t* expected, const int32_t* seq_lens, int32_t ps,
                            int32_t B, int32_t max_pages, uint8_t* abort_mask,
                            int32_t* n_aborted, int32_t* first_bad, cudaStream_t stream) {
  if (n_aborted != nullptr) {
    const cudaError_t e = cudaMemsetAsync(n_aborted, 0, sizeof(int32_t), stream);
    if (e != cudaSuccess) return e;
  }
  if (B == 0) return cudaSuccess;
  int C = (max_pages + kPerCta - 1) / kPerCta;
  C = C < 1 ? 1 : (C > kMaxCluster ? kMaxCluster : C);
  if (static_cast<int64_t>(B) * C > 0x7fffffff) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(B * C));
  cfg.blockDim = dim3(kValThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, validate_kernel, tags, P, block_table, expected, seq_lens, ps,
                            max_pages, abort_mask, n_aborted, first_bad);
}

cudaError_t read_and_clear_error_flags(uint32_t* flags) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(flags, g_error_flags, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_error_flags, &zero, sizeof(uint32_t));
}

}  // namespace kvq
