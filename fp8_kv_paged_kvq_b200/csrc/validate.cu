// Batched page-tag validation, run as its own launch before decode reads the
// cache (not fused into attention, where thread groups could race on it):
// "Cloudflare: Kleinere Modellbereitstellung senkt Speicherbedarf, doch
// Sicherheit wird zum Prüfstein" (remio.ai), section "Sicherheit gemeinsamer
// KV-Caches wird zum Produktionsthema"; "Cloudflare zrýchľuje inferenciu
// modelov Kimi a GLM kompresiou cache a váh" (aifeed.sk), section "Kvalita
// odpovedí a integrita spoločnej cache".
//
// Two kernels.  Batches of up to 4,096 requests run validate_flat_kernel
// (below): one small CTA per SM over all requests' entries, sized to share
// the SM with the decode launch that follows.  Larger batches run
// validate_kernel: each request gets a thread-block cluster of C <= 8 CTAs,
// enough that one round of loads covers its block-table row; CTA r checks
// entries r*kPerCta + k*kValThreads + tid (+ C*kPerCta per further round).
// The CTAs combine their flags through distributed shared memory and rank 0
// writes the request's mask byte, so no separate clear is needed.  Either
// way the cost is launch latency plus, after the sequence length, two
// dependent loads per entry: the block-table entry with its expected tag,
// then the live tag.
#include <cooperative_groups.h>

#include <mutex>

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

// ---------------------------------------------------------------------------
// The same check for batches of up to kFlatMaxB requests, sized so that it
// shares each SM with the decode kernel that follows it: one CTA of 128
// threads and at most 32 registers per SM (the decode kernel's two CTAs leave
// 4,096 registers), so the decode CTAs are resident, past their prologue and
// waiting while the check runs.  The block-table entries of all requests form
// one flat index space (request b owns [pre[b], pre[b+1])); CTA g takes the
// g-th of gridDim.x equal slices, so long and short requests cost alike.
//
// Outputs without a combining step.  Before the dependency wait (while the
// append still runs) CTA 0 writes the result of a clean call: every mask byte
// 0, every first_bad -1, n_aborted 0, and then publishes that it has done so
// for this call's epoch.  After the wait a CTA whose entries all pass simply
// exits, so a clean call ends as soon as its gathers do.  A CTA that finds a
// failing entry waits until CTA 0 has published for this epoch and then
// writes over the clean result: mask byte 1, first_bad lowered to the
// failing index (an unsigned minimum, under which -1 is the largest value),
// and n_aborted raised by one for the request's first recorded failure.
//
// The epoch comes from device memory, so CUDA graph replays of one call get
// fresh epochs: before its wait every CTA reads the epoch and takes an
// arrival ticket; the last CTA to arrive puts the ticket back to 0 and
// advances the epoch for the next call.  These words (and the per-request
// epochs that dedupe the abort count when first_bad is not requested) are
// shared by the library's calls on one device, so such calls must not run
// at the same time.
// ---------------------------------------------------------------------------
constexpr int kFlatThreads = 128;
constexpr int kFlatPer = 8;                 // entries per thread and round
constexpr int kFlatMaxB = 4096;             // prefix of B + 1 ints in (dynamic) shared memory

__device__ uint32_t g_val_epoch = 1;        // epoch of the next call (never 0)
__device__ uint32_t g_val_arrive = 0;       // CTAs of the current call that have read it
__device__ uint32_t g_val_ready = 0xFFFFFFFFu;   // epoch whose clean result CTA 0 has written
__device__ uint32_t g_val_seen[kFlatMaxB];  // epoch in which request b was last counted

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
               : "=r"(old)
               : "l"(p), "r"(v)
               : "memory");
  return old;
}

// Wait (bounded, about one second) until CTA 0 has written this call's clean
// result.  On a timeout the error word records it and the caller goes on:
// CTA 0 writes that result before its dependency wait, so it is long done.
__device__ __forceinline__ void wait_clean_result(uint32_t epoch) {
  if (ld_acquire_gpu(&g_val_ready) == epoch) return;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire_gpu(&g_val_ready) == epoch) return;
    if ((it & 255u) == 0 && globaltimer_ns() - t0 > 1000000000ull) {
      atomicOr(&g_error_flags, kErrWaitTimeout);
      return;
    }
  }
}

__global__ void __maxnreg__(32)
    validate_flat_kernel(const uint32_t* __restrict__ tags, int32_t P,
                         const int32_t* __restrict__ block_table,
                         const uint32_t* __restrict__ expected,
                         const int32_t* __restrict__ seq_lens, int32_t ps, int32_t B,
                         int32_t max_pages, uint8_t* __restrict__ abort_mask,
                         int32_t* __restrict__ n_aborted, int32_t* __restrict__ first_bad) {
  // The same programmatic-dependent-launch contract as validate_kernel: the
  // sequence lengths, block table and expected tags are read before the
  // wait, the live tags after it.  In addition the outputs are written
  // before the wait (CTA 0's clean result).
  pdl_trigger();
  extern __shared__ int32_t pre[];          // [B + 1]
  __shared__ int32_t warp_sum[kFlatThreads / 32];
  __shared__ uint32_t epoch_sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t cap = static_cast<int64_t>(max_pages) * ps;
  // pages per request, then an exclusive prefix (each thread a run of requests)
  const int per = (B + kFlatThreads - 1) / kFlatThreads;
  const int r0 = min(B, tid * per), r1 = min(B, r0 + per);
  int32_t run = 0;
  for (int b = r0; b < r1; ++b) {
    int64_t n = seq_lens[b];
    n = n < 0 ? 0 : (n > cap ? cap : n);
    pre[b] = static_cast<int32_t>((n + ps - 1) / ps);
    run += pre[b];
  }
  int32_t incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  int32_t base = incl - run;
  for (int w = 0; w < warp; ++w) base += warp_sum[w];
  for (int b = r0; b < r1; ++b) {
    const int32_t np = pre[b];
    pre[b] = base;
    base += np;
  }
  if (tid == kFlatThreads - 1) pre[B] = base;
  __syncthreads();
  const int64_t E = pre[B];
  const int32_t f0 = static_cast<int32_t>(E * blockIdx.x / gridDim.x);
  const int32_t f1 = static_cast<int32_t>(E * (blockIdx.x + 1) / gridDim.x);
  // entry f -> (request b, index i within its row): the largest b >= from
  // with pre[b] <= f, by doubling steps from `from` and then halving
  auto locate = [&](int32_t f, int from, int32_t& b, int32_t& i) {
    int lo = from, step = 1;
    while (lo + step < B && pre[lo + step] <= f) {
      lo += step;
      step <<= 1;
    }
    for (step >>= 1; step > 0; step >>= 1)
      if (lo + step < B && pre[lo + step] <= f) lo += step;
    b = lo;
    i = f - pre[lo];
  };
  // The entries, expected tags and live tags are read with an evict-last L2
  // policy: they are a few hundred KB that every step reads again, next to a
  // decode launch that streams the whole cache through L2 (evict-first).
  const uint64_t keep = l2_policy_evict_last();
  int32_t page[kFlatPer];
  uint32_t want[kFlatPer];
  auto load_round = [&](int32_t r) {
    int32_t b = 0, i;
#pragma unroll
    for (int k = 0; k < kFlatPer; ++k) {
      const int32_t f = r + k * kFlatThreads + tid;
      page[k] = 0;
      want[k] = 0;
      if (f < f1) {
        locate(f, b, b, i);                 // entries grow with k: start from the last
        const int64_t e = static_cast<int64_t>(b) * max_pages + i;
        page[k] = static_cast<int32_t>(ld_global_hint(block_table + e, keep));
        want[k] = ld_global_hint(expected + e, keep);
      }
    }
  };
  load_round(f0);
  // With the first entries' loads in flight: the call's epoch (its read comes
  // before this CTA's arrival, an acquire-release ticket; the last arrival
  // advances it) and, in CTA 0, the clean result, published for the epoch.
  if (tid == 0) {
    const uint32_t e = ld_acquire_gpu(&g_val_epoch);
    if (atom_add_acq_rel_gpu(&g_val_arrive, 1u) == gridDim.x - 1) {
      g_val_arrive = 0;                     // every CTA of this call has read the epoch
      st_release_gpu(&g_val_epoch, e + 1u == 0u ? 1u : e + 1u);
    }
    epoch_sh = e;
  }
  if (blockIdx.x == 0) {
    for (int b = tid; b < B; b += kFlatThreads) {
      abort_mask[b] = 0;
      if (first_bad != nullptr) first_bad[b] = -1;
    }
    if (tid == 0 && n_aborted != nullptr) *n_aborted = 0;
    __threadfence();
  }
  __syncthreads();                          // epoch_sh; CTA 0's clean result written
  const uint32_t epoch = epoch_sh;
  if (blockIdx.x == 0 && tid == 0) st_release_gpu(&g_val_ready, epoch);
  pdl_wait();
  for (int32_t r = f0; r < f1; r += kFlatPer * kFlatThreads) {
    if (r != f0) load_round(r);
    // every live-tag load of the round is issued before any compare; the
    // loaded tag replaces the page id, which is no longer needed
    uint32_t inb = 0;
#pragma unroll
    for (int k = 0; k < kFlatPer; ++k)
      if (page[k] >= 0 && page[k] < P) inb |= 1u << k;
#pragma unroll
    for (int k = 0; k < kFlatPer; ++k)
      page[k] = ((inb >> k) & 1u) ? static_cast<int32_t>(ld_global_hint(tags + page[k], keep)) : 0;
    uint32_t bits = 0;
#pragma unroll
    for (int k = 0; k < kFlatPer; ++k) {
      const int32_t f = r + k * kFlatThreads + tid;
      const bool in = (inb >> k) & 1u;
      if (f < f1 && (!in || static_cast<uint32_t>(page[k]) != want[k])) bits |= 1u << k;
    }
    if (bits != 0) {
      // rare: overwrite the clean result for the failing requests
      wait_clean_result(epoch);
#pragma unroll 1
      for (int k = 0; k < kFlatPer; ++k) {
        if ((bits >> k) & 1u) {
          int32_t b, i;
          locate(r + k * kFlatThreads + tid, 0, b, i);
          abort_mask[b] = 1;
          bool first;
          if (first_bad != nullptr)
            first = atomicMin(reinterpret_cast<uint32_t*>(first_bad) + b,
                              static_cast<uint32_t>(i)) == 0xFFFFFFFFu;
          else
            first = atomicExch(&g_val_seen[b], epoch) != epoch;
          if (first && n_aborted != nullptr) atomicAdd(n_aborted, 1);
        }
      }
    }
  }
}

cudaError_t launch_validate(const uint32_t* tags, int32_t P, const int32_t* block_table,
                            const uint32_t* expected, const int32_t* seq_lens, int32_t ps,
                            int32_t B, int32_t max_pages, uint8_t* abort_mask,
                            int32_t* n_aborted, int32_t* first_bad, cudaStream_t stream) {
  if (B == 0) {
    if (n_aborted == nullptr) return cudaSuccess;
    return cudaMemsetAsync(n_aborted, 0, sizeof(int32_t), stream);
  }
  if (B <= kFlatMaxB && static_cast<int64_t>(B) * max_pages <= 0x7fffffff) {
    static std::mutex mu;
    static int sms_of[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    int sms = 0;
    {
      std::lock_guard<std::mutex> lock(mu);
      if (sms_of[dev] == 0) {
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        // keep the SM's shared memory at its largest split while this runs,
        // so the decode CTAs (about 100 KB each) fit beside it
        e = prefer_max_shared(validate_flat_kernel);
        if (e != cudaSuccess) return e;
        sms_of[dev] = n;
      }
      sms = sms_of[dev];
    }
    // No more CTAs than B * max_pages entries need, and at most 7/8 of the
    // SMs: the append kernel's few CTAs occupy some SMs when this grid is
    // placed, and a full grid then doubles up on others, where two of these
    // CTAs leave no room for the second decode CTA until one exits.  One
    // round of kFlatPer loads per thread covers 1,024 entries per CTA
    // (133K entries on a 148-SM B200).
    const int64_t per_cta = static_cast<int64_t>(kFlatThreads) * kFlatPer;
    const int64_t want = (static_cast<int64_t>(B) * max_pages + per_cta - 1) / per_cta;
    const int cap = sms - sms / 8 > 0 ? sms - sms / 8 : 1;
    const int grid = static_cast<int>(want < 1 ? 1 : (want < cap ? want : cap));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kFlatThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(B + 1) * sizeof(int32_t);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, validate_flat_kernel, tags, P, block_table, expected,
                              seq_lens, ps, B, max_pages, abort_mask, n_aborted, first_bad);
  }
  if (n_aborted != nullptr) {
    const cudaError_t e = cudaMemsetAsync(n_aborted, 0, sizeof(int32_t), stream);
    if (e != cudaSuccess) return e;
  }
  int C = (max_pages + kPerCta - 1) / kPerCta;
  C = C < 1 ? 1 : (C > kMaxCluster ? kMaxCluster : C);
  if (static_cast<int64_t>(B) * C > 0x7fffffff) return cudaErrorInvalidValue;
  {
    const cudaError_t e = prefer_max_shared(validate_kernel);
    if (e != cudaSuccess) return e;
  }
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

// One thread waits, through the decode kernels' bounded mbarrier wait, on a
// barrier that nothing completes: after the wait's limit (about one second)
// it records kErrWaitTimeout, and the kernel writes 1 to *timed_out (0 if
// the wait had returned true).
__global__ void wait_timeout_check_kernel(int32_t* timed_out) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  *timed_out = mbar_wait(&bar, 0) ? 0 : 1;
}

cudaError_t launch_wait_timeout_check(int32_t* timed_out, cudaStream_t stream) {
  wait_timeout_check_kernel<<<1, 32, 0, stream>>>(timed_out);
  return cudaGetLastError();
}

cudaError_t read_and_clear_error_flags(uint32_t* flags) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(flags, g_error_flags, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_error_flags, &zero, sizeof(uint32_t));
}

}  // namespace kvq
