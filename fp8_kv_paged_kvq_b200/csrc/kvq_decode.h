// Decode-path declarations internal to libkvq (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "kvq_internal.h"

namespace kvq {

struct DecodeArgs {
  CacheView c;
  const uint16_t* q;   // bf16 [B][Hq][Dk]
  int32_t Hq;
  const int32_t* block_table;
  int32_t max_pages;
  const int32_t* seq_lens;
  int32_t B;
  const uint8_t* abort_mask;
  float sm_scale;
  float* out;
  float* lse;
  void* workspace;
  int32_t num_ctas;
  cudaStream_t stream;
};

// Workspace: [B+2] i32 unit prefix and the count of working CTAs | [num_ctas+1] i32 first
// unit of each working CTA, then U (8-head kernel) | [slots][G] f32 partial lse |
// [slots][G][Dv] f32 partial outputs, slots = num_ctas + B * Hkv (num_ctas counts CTA
// pairs for the wide kernel).
struct WorkspaceLayout {
  size_t off_pre, off_bounds, off_lse, off_o, off_extra, total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline WorkspaceLayout workspace_layout(int32_t B, int32_t Hkv, int32_t G, int32_t Dv,
                                        int32_t num_ctas, size_t extra_per_seq = 0) {
  WorkspaceLayout w;
  const size_t slots = static_cast<size_t>(num_ctas) + static_cast<size_t>(B) * Hkv;
  w.off_pre = 0;
  w.off_bounds = static_cast<size_t>(B + 2) * 4;
  w.off_lse = align_up(w.off_bounds + static_cast<size_t>(num_ctas + 1) * 4, 256);
  w.off_o = align_up(w.off_lse + slots * G * 4, 256);
  w.off_extra = align_up(w.off_o + slots * G * static_cast<size_t>(Dv) * 4, 256);
  w.total = align_up(w.off_extra + static_cast<size_t>(B) * extra_per_seq, 256);
  return w;
}

// Launch a kernel as a programmatic dependent of the previous kernel in the
// stream: it may start launching early, and waits (griddepcontrol.wait)
// before reading that kernel's results.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

int gqa_default_ctas(bool fp8, int D, int G, int B);
int wide_default_pairs(int B);
size_t wide_q_image_bytes();   // per sequence, in the workspace's extra region
cudaError_t launch_wide_decode(const DecodeArgs& a, const CUtensorMap& kqk, const CUtensorMap& ktail);
cudaError_t launch_lse_combine(const int32_t* ws_pre, const int32_t* ws_bounds,
                               const float* ws_lse, const float* ws_o, int32_t B, int32_t Hkv,
                               int32_t G, int32_t Hq, int32_t Dv, int32_t num_ctas, float* out,
                               float* lse, cudaStream_t stream);
void gqa_tma_box(bool fp8, int D, int* box_elems, int* swizzle_bytes);
cudaError_t launch_gqa_decode(const DecodeArgs& a, const CUtensorMap& km, const CUtensorMap& vm);

}  // namespace kvq
