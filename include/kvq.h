/*
 * kvq — FP8 (e4m3) paged KV-cache decode path for NVIDIA B200 (sm_100a).
 *
 * C ABI of libkvq.so.  Plain pointers and sizes only.
 *
 * Sources (web pages on one engineering report, cited by page and section):
 *   [aifeed]  "Cloudflare zrýchľuje inferenciu modelov Kimi a GLM kompresiou
 *             cache a váh" (aifeed.sk)
 *   [manulx]  "Công thức của Cloudflare để phục vụ Kimi và GLM: lượng tử hóa
 *             bộ nhớ đệm KV, nén trọng số, xác minh bộ nhớ đệm" (manulx.blog)
 *   [remio]   "Cloudflare: Kleinere Modellbereitstellung senkt Speicherbedarf,
 *             doch Sicherheit wird zum Prüfstein" (remio.ai)
 *   [lens]    "Cloudflare Workers AI: Kimi および GLM の推論を大規模に最適化する"
 *             (agentlenshq.com)
 *
 * Conventions for every call:
 *   - All data pointers are DEVICE pointers owned by the caller (the library
 *     allocates nothing), unless a parameter says "host".
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; no call synchronizes with
 *     the host except kvq_device_error.
 *   - Arguments are checked on the host before anything is enqueued; a bad
 *     argument returns KVQ_ERR_INVALID_ARG (or KVQ_ERR_UNSUPPORTED for a
 *     shape the kernels do not implement) and enqueues nothing.  A failed
 *     launch returns KVQ_ERR_CUDA.  Device-resident values (slot ids, page
 *     ids, sequence lengths) cannot be checked on the host: the kernels clamp
 *     or skip them as documented below and never read or write out of the
 *     buffers described here.
 *   - Calls that share buffers must be ordered on one stream (or by events).
 *     The intended order within a decode step is
 *         kvq_append -> kvq_validate -> kvq_decode.
 *
 * E4M3: the pages only say "e4m3" ([aifeed] "Dve odlišné úzke miesta v
 * pamäti GPU"; [lens] "並行性を高めるための KV キャッシュ量子化").  This library
 * uses the OCP 8-bit floating point E4M3 encoding: bias 7, no infinities,
 * S.1111.111 = NaN, largest finite 448; conversion rounds to nearest even
 * and saturates to +-448.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1, /* null pointer, negative size, inconsistent descriptor */
  KVQ_ERR_UNSUPPORTED = 2, /* valid but not implemented (head dim, group, page size) */
  KVQ_ERR_WORKSPACE = 3,   /* workspace missing, too small or misaligned */
  KVQ_ERR_CUDA = 4         /* a CUDA launch or API call failed */
} kvq_status;

typedef enum { KVQ_FP8_E4M3 = 0, KVQ_BF16 = 1 } kvq_dtype;

/* Granularity of the FP32 dequantisation scales of an FP8 cache. */
typedef enum {
  KVQ_SCALE_TENSOR = 0, /* k_scale[1], v_scale[1] */
  KVQ_SCALE_HEAD = 1,   /* k_scale[Hkv], v_scale[Hkv] */
  KVQ_SCALE_TOKEN = 2   /* k_scale[P][Hkv][ps], v_scale[P][Hkv][ps]; written by kvq_append */
} kvq_scale_mode;

/*
 * Paged KV cache descriptor.  The cache is split into fixed-size physical
 * pages shared by all requests, and every page carries a uint32 tag that
 * changes each time the page is reallocated ([remio] "Sicherheit gemeinsamer
 * KV-Caches wird zum Produktionsthema"; [manulx] "Bảo vệ bộ nhớ đệm dùng chung").
 *
 * Layout (all row-major, device memory owned by the caller):
 *   k_pages   [P][Hkv][ps][Dk]   FP8: u8 E4M3 codes; BF16: bf16
 *   v_pages   [P][Hkv][ps][Dv]   or NULL: V is the first Dv dims of each K
 *                                row (Dv <= Dk) and shares K's scales
 *   k_scale   FP32, shape per scale_mode (FP8 only; NULL for BF16)
 *   v_scale   FP32, shape per scale_mode (NULL when v_pages is NULL or BF16)
 *   page_tags u32 [P]
 * A token at slot s (0 <= s < P*ps) lives on page s / ps at offset s % ps.
 * Dequantised value of an FP8 element: fl32(decode(code) * scale).
 * Base pointers must be 16-byte aligned.
 */
typedef struct {
  int32_t dtype;        /* kvq_dtype */
  int32_t scale_mode;   /* kvq_scale_mode; ignored for BF16 */
  int32_t num_pages;    /* P  >= 1 */
  int32_t page_size;    /* ps >= 1 tokens per page */
  int32_t num_kv_heads; /* Hkv >= 1 */
  int32_t head_dim_k;   /* Dk, multiple of 16 */
  int32_t head_dim_v;   /* Dv, multiple of 16, Dv <= Dk when v_pages == NULL */
  void* k_pages;
  void* v_pages;
  float* k_scale;
  float* v_scale;
  uint32_t* page_tags;
} kvq_cache;

/* Human-readable name of a status code (static string, never NULL). */
const char* kvq_status_string(kvq_status status);

/*
 * Fold max |x| of a BF16 tensor x[T][H][D] into amax_io (FP32): amax_io[0]
 * over everything (per_head == 0) or amax_io[h] per head (per_head != 0),
 * as amax_io = max(amax_io, max|x|).  The caller zero-initialises amax_io;
 * repeated calls over chunks of a tensor accumulate.  NaN elements are
 * ignored.  Together with kvq_scale_from_amax this gives the per-tensor /
 * per-head scale amax / 448 that maps the largest element onto the largest
 * E4M3 code.  (The pages fix no scale granularity; this is the reading that
 * the per-tensor and per-head workloads use.)
 * Requires T >= 0, H >= 1, D >= 1 and D % 8 == 0 (16-byte rows).
 */
kvq_status kvq_amax(const void* x, int64_t T, int32_t H, int32_t D, int32_t per_head,
                    float* amax_io, void* stream);

/* scale[i] = fl32(amax[i] / 448) (IEEE division), or 1 where amax[i] is 0
 * or NaN.  n >= 0.  amax and scale may alias. */
kvq_status kvq_scale_from_amax(const float* amax, float* scale, int32_t n, void* stream);

/*
 * Quantize-on-append (write path of the decode pool, where the cache is
 * stored as E4M3: [aifeed] "Kompresia sa oplatí inde pri vstupe a inde pri
 * výstupe"; [manulx] "Bộ nhớ đệm KV FP8 tăng gấp đôi dung lượng ngữ cảnh").
 *
 * 1. Tag bump: for every entry p of realloc_pages[n_realloc] (device, may be
 *    NULL when n_realloc == 0), page_tags[p] += 1 (mod 2^32), once per
 *    occurrence.  Ids outside [0, P) are skipped.
 * 2. For token t < T with slot = slot_mapping[t] (device, [T]) in [0, P*ps)
 *    and every KV head h: FP8 caches store code = E4M3(fl32(x) / s) for each
 *    element x of k_new[t][h][:] (and v_new[t][h][:]), with IEEE division
 *    and saturating round-to-nearest-even; in TOKEN mode s = fl32(amax(row)
 *    / 448) (1 if amax is 0) is computed first and stored at
 *    scale[page][h][offset].  BF16 caches store the values unchanged.
 *    Slots < 0 (padding) or >= P*ps are skipped.  Two tokens with the same
 *    slot in one call race (unspecified result).
 * k_new: bf16 [T][Hkv][Dk]; v_new: bf16 [T][Hkv][Dv], ignored (may be NULL)
 * when cache->v_pages is NULL.
 */
kvq_status kvq_append(const kvq_cache* cache, const void* k_new, const void* v_new,
                      const int32_t* slot_mapping, int32_t T, const int32_t* realloc_pages,
                      int32_t n_realloc, void* stream);

/*
 * Batched tag validation, a separate launch before decode reads the cache
 * rather than a check fused into the attention kernel ([remio] "Sicherheit
 * gemeinsamer KV-Caches wird zum Produktionsthema"; [aifeed] "Kvalita
 * odpovedí a integrita spoločnej cache"; [lens] "KV キャッシュ整合性チェック").
 *
 * For each request b < B: n = clamp(seq_lens[b], 0, max_pages*page_size),
 * abort_mask[b] = 1 if some i < ceil(n / page_size) has
 *   block_table[b][i] outside [0, num_pages) or
 *   page_tags[block_table[b][i]] != expected_tags[b][i],
 * else 0.  Entries of block_table / expected_tags beyond ceil(n/ps) are not
 * read.
 *   block_table i32 [B][max_pages]; expected_tags u32 [B][max_pages];
 *   seq_lens i32 [B]; abort_mask u8 [B] (written).
 * Optional telemetry (device pointers, NULL to skip), because the pages name
 * the mismatch rate as the quantity to watch ([remio] "Sicherheit
 * gemeinsamer KV-Caches wird zum Produktionsthema"):
 *   n_aborted   i32 [1]: set to the number of aborted requests (needs no
 *               initialisation);
 *   first_bad   i32 [B]: the smallest failing index i of each request, or -1.
 * Launched as a programmatic dependent of the previous kernel on the stream.
 * It reads seq_lens, block_table and expected_tags while that kernel may
 * still run, and page_tags only after it has finished: the kernel launched
 * just before on the same stream must not write the first three (kvq_append,
 * the usual predecessor, never does; copies and earlier kernels are
 * complete before it starts).
 * Batches of up to 4,096 requests (and B * max_pages < 2^31) run as one CTA
 * of 128 threads per SM over all requests' entries, small enough to share
 * each SM with the decode launch that follows, whose CTAs then start while
 * the check runs.  This form also writes the result of a clean check
 * (mask 0, first_bad -1, n_aborted 0) while the previous kernel may still
 * run, and only failing requests are written after it: that kernel must not
 * read or write abort_mask, n_aborted or first_bad either (kvq_append never
 * does).  Its CTAs share a few words of the library's device memory (a call
 * epoch, an arrival count, per-request epochs for the abort count): on one
 * device, such calls must not run at the same time (on different streams).
 * Larger batches use one cluster of up to 8 CTAs per request and have no
 * such restriction.
 */
kvq_status kvq_validate(const uint32_t* page_tags, int32_t num_pages, const int32_t* block_table,
                        const uint32_t* expected_tags, const int32_t* seq_lens,
                        int32_t page_size, int32_t B, int32_t max_pages, uint8_t* abort_mask,
                        int32_t* n_aborted, int32_t* first_bad, void* stream);

/*
 * Bytes of device workspace kvq_decode / kvq_decode_bf16 need for this
 * cache, batch size and query-head count, with num_ctas persistent blocks
 * (0 = the library's default for the current device).  Returns 0 for
 * invalid or unsupported arguments.
 */
size_t kvq_decode_workspace_size(const kvq_cache* cache, int32_t B, int32_t num_q_heads,
                                 int32_t num_ctas);

/*
 * Decode attention over the paged FP8 cache: each sequence's single new
 * query token attends to its cached tokens through its page table, with the
 * E4M3 codes converted to 16-bit values in registers on the way
 * ([manulx] "Bộ nhớ đệm KV FP8 tăng gấp đôi dung lượng ngữ cảnh"; [remio]
 * "Warum kleinere Cloudflare-Caches reine Geschwindigkeit schlagen").
 *
 *   q           bf16 [B][num_q_heads][Dk]; query head h reads KV head
 *               h / (num_q_heads / Hkv)
 *   block_table i32 [B][max_pages]; seq_lens i32 [B] (tokens, clamped to
 *               [0, max_pages*ps])
 *   abort_mask  u8 [B] from kvq_validate, or NULL when the check is disabled
 *               for this deployment; aborted rows read no cache bytes
 *   out         f32 [B][num_q_heads][Dv]:  sum_j softmax(s)_j * Vhat_j with
 *               s_j = sm_scale * (q . Khat_j)
 *   lse         f32 [B][num_q_heads] natural-log sum-exp of s, or NULL
 *   Aborted or empty rows: out = 0, lse = -inf.
 *   workspace   device, >= kvq_decode_workspace_size(...) bytes, 256-byte
 *               aligned; contents on entry are ignored.
 *   num_ctas    persistent blocks (0 = default); the work is split evenly
 *               over them regardless of sequence lengths (split-KV), and the
 *               partial results are merged by a log-sum-exp combine launch.
 * Page ids outside [0, P) read as zeros (no fault); run kvq_validate first
 * to abort such requests instead.  Queries must lie within the FP16 range.
 * Requires cache->dtype == KVQ_FP8_E4M3 and B <= 8,000 (larger batches return
 * KVQ_ERR_UNSUPPORTED).  Supported shapes: Dk == Dv in
 * {64, 128} with separate V pages, ps a multiple of 16 and
 * num_q_heads / Hkv <= 16; or Dk = 576, Dv = 512 with V aliasing K, one KV
 * head, 128 query heads, TOKEN scales and ps a multiple of 64.  The second
 * shape runs on the tensor cores on the stored codes: each query row is
 * scaled by a power of two to a maximum in [128, 256) and split into two
 * E4M3 terms (any BF16 range; exact for scaled elements of magnitude >= 2^-2,
 * smaller ones are rounded at the E4M3 step 2^-9); the probabilities, times
 * the token scales and a power of two per head, into three (about 2^-12
 * relative); and an E4M3 NaN code (0x7F / 0xFF, which
 * kvq_append never writes) in a cached token gives NaN there.
 * The kernels are launched as programmatic dependents of the previous work
 * on the stream.  The 8-head kernel reads seq_lens, block_table and the
 * per-tensor or per-head scales to plan its split while that work may still
 * run (the kernel launched just before must not write them; kvq_validate and
 * kvq_append never do, and kvq_scale_from_amax lets no kernel start before
 * it ends) and everything else, the abort mask included, after it has
 * finished; the wide kernels
 * wait before reading any argument.  The last kernel of the call (the
 * log-sum-exp combine) lets the next kernel on the stream start once the
 * decode kernel has finished, while it still writes out and lse: a kernel
 * that follows must wait for its predecessor before reading them.
 */
kvq_status kvq_decode(const kvq_cache* cache, const void* q, int32_t num_q_heads,
                      const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens,
                      int32_t B, const uint8_t* abort_mask, float sm_scale, float* out,
                      float* lse, void* workspace, size_t workspace_bytes, int32_t num_ctas,
                      void* stream);

/* The same decode over a BF16 cache (cache->dtype == KVQ_BF16), the format
 * the FP8 cache is compared with ([remio] "Warum kleinere Cloudflare-Caches
 * reine Geschwindigkeit schlagen").  Same arguments, shapes and rules as
 * kvq_decode for the Dk == Dv in {64, 128} family. */
kvq_status kvq_decode_bf16(const kvq_cache* cache, const void* q, int32_t num_q_heads,
                           const int32_t* block_table, int32_t max_pages,
                           const int32_t* seq_lens, int32_t B, const uint8_t* abort_mask,
                           float sm_scale, float* out, float* lse, void* workspace,
                           size_t workspace_bytes, int32_t num_ctas, void* stream);

/*
 * kvq_decode without a caller-provided workspace.  The source pages have no
 * counterpart to this call: it exists for callers that cannot allocate
 * device memory, such as a plug-in inside a host framework that owns all
 * device memory and hands out none, or a serving loop that forbids any
 * allocation after start-up.  Same arguments, rules and results as
 * kvq_decode (FP8 caches only) minus `workspace` / `workspace_bytes`.
 *
 * The scratch lives in a fixed 8 MiB array inside libkvq.so that every GPU
 * which loads the library holds until the process exits.  A batch whose
 * workspace (kvq_decode_workspace_size) exceeds 8 MiB is rejected with
 * KVQ_ERR_WORKSPACE before anything is enqueued; the allocating kvq_decode
 * has no such limit.  The call allocates nothing.  The first call on each
 * device looks up the array's device address (with that device current);
 * make that first call before any stream capture.  All calls on a device
 * share the array, so calls that overlap on the GPU (e.g. on two unordered
 * streams) race and give undefined results; order them on one stream.
 * Nothing in the array needs to start at zero.
 */
kvq_status kvq_decode_noalloc(const kvq_cache* cache, const void* q, int32_t num_q_heads,
                              const int32_t* block_table, int32_t max_pages,
                              const int32_t* seq_lens, int32_t B, const uint8_t* abort_mask,
                              float sm_scale, float* out, float* lse, int32_t num_ctas,
                              void* stream);

/*
 * Device E4M3 conversion used by kvq_append, exposed for exhaustive checks:
 * out[i] = E4M3(float with bit pattern start + i), i < count (bit patterns
 * wrap mod 2^32).  out: u8 [count].
 */
kvq_status kvq_e4m3_encode_bits(uint32_t start, uint32_t count, uint8_t* out, void* stream);

/*
 * The quantize step of kvq_append, exposed for exhaustive checks:
 * out[i] = E4M3(x / scale) for x the float with bit pattern start + i,
 * where x / scale is the IEEE binary32 quotient (round to nearest even).
 * It is computed as kvq_append computes it, which reaches that quotient
 * without a division per value where the arithmetic allows (the product
 * by the rounded reciprocal with one FMA correction) and divides elsewhere.
 * scale must be positive and finite.  out: u8 [count].
 */
kvq_status kvq_e4m3_quantize_bits(uint32_t start, uint32_t count, float scale, uint8_t* out,
                                  void* stream);

/*
 * Reads and clears the library's device-side error word on the current
 * device (synchronous).  Bit 0: a bounded wait gave up after its time limit
 * (about one second): a pipeline wait in a decode kernel (the kernel returned
 * early, so that launch's outputs are invalid), or, in kvq_validate, a
 * failing CTA's wait for the clean result of the same call (the mask bytes
 * written after it may then be overwritten by that late clean result, so
 * the call's outputs are invalid).  Bit 1: the wide-group decode kernel's
 * tensor-memory allocation (all 512 columns, so it starts at column 0) came
 * back at another address; that CTA pair did no work and the call's outputs
 * are invalid.  *flags_host receives the word.
 */
kvq_status kvq_device_error(uint32_t* flags_host);

/*
 * Exercises the error path above: one thread waits, through the bounded
 * mbarrier wait the decode kernels use, on a barrier that nothing
 * completes.  After the wait's limit (about one second) the kernel sets bit
 * 0 of the error word and writes 1 to *timed_out (device i32, 4-byte
 * aligned; 0 would mean the wait returned normally).  The context stays
 * usable; read kvq_device_error afterwards to see and clear the bit, since
 * the tensor-core decode kernel's waits give up at once while it is set.
 */
kvq_status kvq_wait_timeout_check(int32_t* timed_out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
