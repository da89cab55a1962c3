// C ABI of libkvq.so (declared in include/kvq.h): host-side argument checks,
// TMA descriptor set-up and kernel dispatch.  No allocation, no host sync
// (except kvq_device_error), everything enqueued on the caller's stream.
#include <cudaTypedefs.h>

#include <mutex>

#include "kvq.h"
#include "kvq_decode.h"
#include "kvq_internal.h"

namespace kvq {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

kvq_status check_cache(const kvq_cache* c) {
  if (c == nullptr) return KVQ_ERR_INVALID_ARG;
  if (c->dtype != KVQ_FP8_E4M3 && c->dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
  if (c->num_pages < 1 || c->page_size < 1 || c->num_kv_heads < 1) return KVQ_ERR_INVALID_ARG;
  if (c->head_dim_k < 16 || c->head_dim_v < 16 || c->head_dim_k % 16 || c->head_dim_v % 16)
    return KVQ_ERR_INVALID_ARG;
  if (c->k_pages == nullptr || c->page_tags == nullptr) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(c->k_pages) || !aligned16(c->v_pages)) return KVQ_ERR_INVALID_ARG;
  if (c->v_pages == nullptr && c->head_dim_v > c->head_dim_k) return KVQ_ERR_INVALID_ARG;
  if (c->dtype == KVQ_FP8_E4M3) {
    if (c->scale_mode < KVQ_SCALE_TENSOR || c->scale_mode > KVQ_SCALE_TOKEN)
      return KVQ_ERR_INVALID_ARG;
    if (c->k_scale == nullptr) return KVQ_ERR_INVALID_ARG;
    if (c->v_pages != nullptr && c->v_scale == nullptr) return KVQ_ERR_INVALID_ARG;
  }
  // sizes that index with 64-bit arithmetic on the device but must fit the
  // TMA descriptor and the int32 slot space
  if (static_cast<int64_t>(c->num_pages) * c->page_size > INT32_MAX) return KVQ_ERR_UNSUPPORTED;
  return KVQ_OK;
}

CacheView view_of(const kvq_cache* c) {
  CacheView v;
  v.fp8 = c->dtype == KVQ_FP8_E4M3 ? 1 : 0;
  v.scale_mode = c->scale_mode;
  v.P = c->num_pages;
  v.ps = c->page_size;
  v.Hkv = c->num_kv_heads;
  v.Dk = c->head_dim_k;
  v.Dv = c->head_dim_v;
  v.k_pages = c->k_pages;
  v.v_pages = c->v_pages;
  v.k_scale = c->k_scale;
  v.v_scale = c->v_scale;
  v.tags = c->page_tags;
  return v;
}

kvq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

// ---- driver entry point for tensor-map encoding (no link-time libcuda) ----
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 4-D map over pages [P][Hkv][ps][D] with a box of (box_elems, 16, 1, 1).
bool make_page_map(CUtensorMap* map, void* base, bool fp8, int P, int Hkv, int ps, int D) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  int box_elems = 0, swz = 0;
  gqa_tma_box(fp8, D, &box_elems, &swz);
  const uint64_t el = fp8 ? 1 : 2;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(ps),
                              static_cast<cuuint64_t>(Hkv), static_cast<cuuint64_t>(P)};
  const cuuint64_t strides[3] = {D * el, static_cast<cuuint64_t>(ps) * D * el,
                                 static_cast<cuuint64_t>(Hkv) * ps * D * el};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(box_elems), 16, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swz == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr int32_t kMaxBatch = kGqaMaxBatch;   // unit prefix kept in shared memory

enum class Path { kNone, kGqa, kWide };

Path decode_path(const kvq_cache* c, int32_t Hq) {
  if (Hq < 1 || Hq % c->num_kv_heads) return Path::kNone;
  const int G = Hq / c->num_kv_heads;
  if (c->v_pages != nullptr && c->head_dim_k == c->head_dim_v &&
      (c->head_dim_k == 64 || c->head_dim_k == 128) && c->page_size % 16 == 0 && G <= 16)
    return Path::kGqa;
  if (c->dtype == KVQ_FP8_E4M3 && c->v_pages == nullptr && c->head_dim_k == 576 &&
      c->head_dim_v == 512 && c->num_kv_heads == 1 && Hq == 128 &&
      c->scale_mode == KVQ_SCALE_TOKEN && c->page_size % 64 == 0)
    return Path::kWide;
  return Path::kNone;
}

// Persistent CTAs (8-head kernel) or CTA pairs (wide kernel).
int32_t resolve_ctas(const kvq_cache* c, int32_t Hq, int32_t B, int32_t num_ctas) {
  if (num_ctas > 0) return num_ctas;
  if (decode_path(c, Hq) == Path::kWide) return wide_default_pairs(B);
  return gqa_default_ctas(c->dtype == KVQ_FP8_E4M3, c->head_dim_k, Hq / c->num_kv_heads, B);
}

// 4-D map over [P][Hkv][ps][D] bytes with a (box_x bytes, box_rows, 1, 1) box.
bool make_u8_map(CUtensorMap* map, void* base, int P, int Hkv, int ps, int D, int box_x,
                 int box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(ps),
                              static_cast<cuuint64_t>(Hkv), static_cast<cuuint64_t>(P)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(ps) * D,
                                 static_cast<cuuint64_t>(Hkv) * ps * D};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(box_x), static_cast<cuuint32_t>(box_rows),
                             1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

kvq_status decode_common(bool want_fp8, const kvq_cache* cache, const void* q, int32_t Hq,
                         const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens,
                         int32_t B, const uint8_t* abort_mask, float sm_scale, float* out,
                         float* lse, void* workspace, size_t workspace_bytes, int32_t num_ctas,
                         void* stream) {
  kvq_status st = check_cache(cache);
  if (st != KVQ_OK) return st;
  if ((cache->dtype == KVQ_FP8_E4M3) != want_fp8) return KVQ_ERR_INVALID_ARG;
  if (B < 0 || max_pages < 1 || num_ctas < 0) return KVQ_ERR_INVALID_ARG;
  if (Hq < 1 || Hq % cache->num_kv_heads) return KVQ_ERR_INVALID_ARG;
  if (B == 0) return KVQ_OK;
  if (q == nullptr || block_table == nullptr || seq_lens == nullptr || out == nullptr)
    return KVQ_ERR_INVALID_ARG;
  if (!aligned16(q)) return KVQ_ERR_INVALID_ARG;
  if (B > kMaxBatch) return KVQ_ERR_UNSUPPORTED;
  const Path path = decode_path(cache, Hq);
  if (path == Path::kNone) return KVQ_ERR_UNSUPPORTED;
  const int32_t ctas = resolve_ctas(cache, Hq, B, num_ctas);
  if (ctas <= 0) return KVQ_ERR_CUDA;
  const WorkspaceLayout wl =
      workspace_layout(B, cache->num_kv_heads, Hq / cache->num_kv_heads, cache->head_dim_v, ctas,
                       path == Path::kWide ? wide_q_image_bytes() : 0);
  if (workspace == nullptr || workspace_bytes < wl.total ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return KVQ_ERR_WORKSPACE;
  DecodeArgs a;
  a.c = view_of(cache);
  a.q = static_cast<const uint16_t*>(q);
  a.Hq = Hq;
  a.block_table = block_table;
  a.max_pages = max_pages;
  a.seq_lens = seq_lens;
  a.B = B;
  a.abort_mask = abort_mask;
  a.sm_scale = sm_scale;
  a.out = out;
  a.lse = lse;
  a.workspace = workspace;
  a.num_ctas = ctas;
  a.stream = static_cast<cudaStream_t>(stream);
  if (path == Path::kWide) {
    // key rows of one SM's 32-token half: 128-dim atoms (128-byte swizzle)
    // and the 64-dim tail (64-byte swizzle)
    CUtensorMap kqk, ktail;
    if (!make_u8_map(&kqk, cache->k_pages, cache->num_pages, 1, cache->page_size, 576, 128, 32,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_u8_map(&ktail, cache->k_pages, cache->num_pages, 1, cache->page_size, 576, 64, 32,
                     CU_TENSOR_MAP_SWIZZLE_64B))
      return KVQ_ERR_CUDA;
    return from_cuda(launch_wide_decode(a, kqk, ktail));
  }
  CUtensorMap km, vm;
  if (!make_page_map(&km, cache->k_pages, want_fp8, cache->num_pages, cache->num_kv_heads,
                     cache->page_size, cache->head_dim_k) ||
      !make_page_map(&vm, cache->v_pages, want_fp8, cache->num_pages, cache->num_kv_heads,
                     cache->page_size, cache->head_dim_v))
    return KVQ_ERR_CUDA;
  return from_cuda(launch_gqa_decode(a, km, vm));
}

}  // namespace
}  // namespace kvq

using namespace kvq;

extern "C" {

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "KVQ_OK";
    case KVQ_ERR_INVALID_ARG: return "KVQ_ERR_INVALID_ARG";
    case KVQ_ERR_UNSUPPORTED: return "KVQ_ERR_UNSUPPORTED";
    case KVQ_ERR_WORKSPACE: return "KVQ_ERR_WORKSPACE";
    case KVQ_ERR_CUDA: return "KVQ_ERR_CUDA";
  }
  return "KVQ_ERR_UNKNOWN";
}

kvq_status kvq_amax(const void* x, int64_t T, int32_t H, int32_t D, int32_t per_head,
                    float* amax_io, void* stream) {
  if (T < 0 || H < 1 || D < 1 || D % 8 || amax_io == nullptr) return KVQ_ERR_INVALID_ARG;
  if (T == 0) return KVQ_OK;
  if (x == nullptr || !aligned16(x)) return KVQ_ERR_INVALID_ARG;
  return from_cuda(launch_amax(static_cast<const uint16_t*>(x), T, H, D, per_head ? 1 : 0,
                               amax_io, static_cast<cudaStream_t>(stream)));
}

kvq_status kvq_scale_from_amax(const float* amax, float* scale, int32_t n, void* stream) {
  if (n < 0) return KVQ_ERR_INVALID_ARG;
  if (n == 0) return KVQ_OK;
  if (amax == nullptr || scale == nullptr) return KVQ_ERR_INVALID_ARG;
  return from_cuda(launch_scale_from_amax(amax, scale, n, static_cast<cudaStream_t>(stream)));
}

kvq_status kvq_append(const kvq_cache* cache, const void* k_new, const void* v_new,
                      const int32_t* slot_mapping, int32_t T, const int32_t* realloc_pages,
                      int32_t n_realloc, void* stream) {
  kvq_status st = check_cache(cache);
  if (st != KVQ_OK) return st;
  if (T < 0 || n_realloc < 0) return KVQ_ERR_INVALID_ARG;
  if (n_realloc > 0 && realloc_pages == nullptr) return KVQ_ERR_INVALID_ARG;
  if (T > 0) {
    if (k_new == nullptr || slot_mapping == nullptr || !aligned16(k_new)) return KVQ_ERR_INVALID_ARG;
    if (cache->v_pages != nullptr && (v_new == nullptr || !aligned16(v_new)))
      return KVQ_ERR_INVALID_ARG;
  }
  const CacheView c = view_of(cache);
  return from_cuda(launch_append(c, static_cast<const uint16_t*>(k_new),
                                 static_cast<const uint16_t*>(v_new), slot_mapping, T,
                                 realloc_pages, n_realloc, static_cast<cudaStream_t>(stream)));
}

kvq_status kvq_validate(const uint32_t* page_tags, int32_t num_pages, const int32_t* block_table,
                        const uint32_t* expected_tags, const int32_t* seq_lens,
                        int32_t page_size, int32_t B, int32_t max_pages, uint8_t* abort_mask,
                        int32_t* n_aborted, int32_t* first_bad, void* stream) {
  if (num_pages < 1 || page_size < 1 || B < 0 || max_pages < 1) return KVQ_ERR_INVALID_ARG;
  if (B > 0 && (page_tags == nullptr || block_table == nullptr || expected_tags == nullptr ||
                seq_lens == nullptr || abort_mask == nullptr))
    return KVQ_ERR_INVALID_ARG;
  return from_cuda(launch_validate(page_tags, num_pages, block_table, expected_tags, seq_lens,
                                   page_size, B, max_pages, abort_mask, n_aborted, first_bad,
                                   static_cast<cudaStream_t>(stream)));
}

size_t kvq_decode_workspace_size(const kvq_cache* cache, int32_t B, int32_t num_q_heads,
                                 int32_t num_ctas) {
  if (check_cache(cache) != KVQ_OK || B < 0 || num_ctas < 0 || num_q_heads < 1 ||
      num_q_heads % cache->num_kv_heads)
    return 0;
  if (B > kMaxBatch || decode_path(cache, num_q_heads) == Path::kNone) return 0;
  const int32_t ctas = resolve_ctas(cache, num_q_heads, B, num_ctas);
  if (ctas <= 0) return 0;
  const bool wide = decode_path(cache, num_q_heads) == Path::kWide;
  return workspace_layout(B, cache->num_kv_heads, num_q_heads / cache->num_kv_heads,
                          cache->head_dim_v, ctas, wide ? wide_q_image_bytes() : 0)
      .total;
}

kvq_status kvq_decode(const kvq_cache* cache, const void* q, int32_t num_q_heads,
                      const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens,
                      int32_t B, const uint8_t* abort_mask, float sm_scale, float* out,
                      float* lse, void* workspace, size_t workspace_bytes, int32_t num_ctas,
                      void* stream) {
  return decode_common(true, cache, q, num_q_heads, block_table, max_pages, seq_lens, B,
                       abort_mask, sm_scale, out, lse, workspace, workspace_bytes, num_ctas,
                       stream);
}

kvq_status kvq_decode_bf16(const kvq_cache* cache, const void* q, int32_t num_q_heads,
                           const int32_t* block_table, int32_t max_pages,
                           const int32_t* seq_lens, int32_t B, const uint8_t* abort_mask,
                           float sm_scale, float* out, float* lse, void* workspace,
                           size_t workspace_bytes, int32_t num_ctas, void* stream) {
  return decode_common(false, cache, q, num_q_heads, block_table, max_pages, seq_lens, B,
                       abort_mask, sm_scale, out, lse, workspace, workspace_bytes, num_ctas,
                       stream);
}

kvq_status kvq_e4m3_quantize_bits(uint32_t start, uint32_t count, float scale, uint8_t* out,
                                  void* stream) {
  if (out == nullptr || !(scale > 0.0f) || scale == __builtin_inff()) return KVQ_ERR_INVALID_ARG;
  return from_cuda(launch_quantize_bits(start, count, scale, out, static_cast<cudaStream_t>(stream)));
}

kvq_status kvq_e4m3_encode_bits(uint32_t start, uint32_t count, uint8_t* out, void* stream) {
  if (count == 0) return KVQ_OK;
  if (out == nullptr || (reinterpret_cast<uintptr_t>(out) & 3u)) return KVQ_ERR_INVALID_ARG;
  return from_cuda(launch_encode_bits(start, count, out, static_cast<cudaStream_t>(stream)));
}

kvq_status kvq_wait_timeout_check(int32_t* timed_out, void* stream) {
  if (timed_out == nullptr || (reinterpret_cast<uintptr_t>(timed_out) & 3u))
    return KVQ_ERR_INVALID_ARG;
  return from_cuda(launch_wait_timeout_check(timed_out, static_cast<cudaStream_t>(stream)));
}

kvq_status kvq_device_error(uint32_t* flags_host) {
  if (flags_host == nullptr) return KVQ_ERR_INVALID_ARG;
  return from_cuda(read_and_clear_error_flags(flags_host));
}

}  // extern "C"
