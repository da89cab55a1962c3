// Host/device shared declarations internal to libkvq (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kvq {

// Plain-pointer view of a kvq_cache descriptor, passed by value to kernels.
struct CacheView {
  int32_t fp8;         // 1: E4M3 codes, 0: bf16
  int32_t scale_mode;  // 0 tensor, 1 head, 2 token
  int32_t P, ps, Hkv, Dk, Dv;
  void* k_pages;
  void* v_pages;       // nullptr: V aliases the first Dv dims of K
  float* k_scale;
  float* v_scale;
  uint32_t* tags;
};

cudaError_t launch_amax(const uint16_t* x, int64_t T, int32_t H, int32_t D, int32_t per_head,
                        float* amax_io, cudaStream_t stream);
cudaError_t launch_scale_from_amax(const float* amax, float* scale, int32_t n,
                                   cudaStream_t stream);
cudaError_t launch_append(const CacheView& c, const uint16_t* k_new, const uint16_t* v_new,
                          const int32_t* slot_mapping, int32_t T, const int32_t* realloc_pages,
                          int32_t n_realloc, cudaStream_t stream);
cudaError_t launch_quantize_bits(uint32_t start, uint32_t count, float scale, uint8_t* out,
                                 cudaStream_t stream);
cudaError_t launch_encode_bits(uint32_t start, uint32_t count, uint8_t* out,
                               cudaStream_t stream);
cudaError_t launch_validate(const uint32_t* tags, int32_t P, const int32_t* block_table,
                            const uint32_t* expected, const int32_t* seq_lens, int32_t ps,
                            int32_t B, int32_t max_pages, uint8_t* abort_mask,
                            int32_t* n_aborted, int32_t* first_bad, cudaStream_t stream);
cudaError_t read_and_clear_error_flags(uint32_t* flags);
cudaError_t launch_wait_timeout_check(int32_t* timed_out, cudaStream_t stream);

// Ask for the largest shared-memory carveout for `kernel` on the current
// device (once per device).  The tag check and the wide pre-pass, which run
// beside the decode CTAs that follow them, use it, so that the SMs they
// occupy are already split for the decode CTAs' shared memory (an SM changes
// its split only when it is empty).  The append kernel keeps the default: its
// streaming loads want L1, and its CTAs exit before a decode launch that
// follows a tag check needs their SMs.
template <typename K>
cudaError_t prefer_max_shared(K* kernel);

}  // namespace kvq
