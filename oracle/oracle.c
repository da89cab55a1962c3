/*
 * CPU oracle for the FP8 (e4m3) paged KV-cache decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: it is used by tests/, by the smoke check and by the CPU
 * baseline leg of the benchmark.  It shares no code, header, table or
 * constant generator with the CUDA library; it is deliberately plain and
 * slow (fp64 arithmetic, one pass over each logical sequence, no blocking,
 * no splitting) so that it can be checked against the pages by eye.
 *
 * Sources (web pages on one engineering report; cited by page and section):
 *   [aifeed]  "Cloudflare zrýchľuje inferenciu modelov Kimi a GLM kompresiou
 *             cache a váh" (aifeed.sk)
 *   [manulx]  "Công thức của Cloudflare để phục vụ Kimi và GLM: lượng tử hóa
 *             bộ nhớ đệm KV, nén trọng số, xác minh bộ nhớ đệm" (manulx.blog)
 *   [remio]   "Cloudflare: Kleinere Modellbereitstellung senkt Speicherbedarf,
 *             doch Sicherheit wird zum Prüfstein" (remio.ai)
 *   [lens]    "Cloudflare Workers AI: Kimi および GLM の推論を大規模に最適化する"
 *             (agentlenshq.com)
 *
 * The pages say the cache is stored as 8-bit "e4m3" instead of BF16
 * ([aifeed] "Dve odlišné úzke miesta v pamäti GPU"; [remio] "Was Cloudflare
 * für Kimi und GLM geändert hat"; [lens] "並行性を高めるための KV キャッシュ量子化").
 * They do not spell the format out.  Reading taken: the OCP 8-bit floating
 * point E4M3 encoding (exponent bias 7, no infinities, the all-ones
 * exponent+mantissa pattern is NaN, largest finite value 448), conversion
 * by round-to-nearest-even with saturation to +-448.
 *
 * Pins (what checks this file against something other than itself) live in
 * tests/test_oracle_*.py: the codec against torch.float8_e4m3fn and exact
 * bit-level properties; attention against an independent dense brute force
 * and closed forms; validation against brute force.  No function here is
 * "parity unpinned".
 *
 * Cache layout restated here (independently of the CUDA headers):
 *   K pages  [P][Hkv][ps][Dk]  (u8 e4m3 codes, or u16 BF16 bits)
 *   V pages  [P][Hkv][ps][Dv]  (NULL: V is the first Dv dims of K)
 *   scales   TENSOR: [1]   HEAD: [Hkv]   TOKEN: [P][Hkv][ps]
 *   tags     u32 [P]
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Threads the parallel loops below may use (the CPU baseline is timed on all
 * host cores and on one).  n <= 0 keeps the current setting.  Returns the
 * setting in force. */
int oracle_set_threads(int n) {
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
}

#define ORACLE_FP8 0
#define ORACLE_BF16 1
#define ORACLE_SCALE_TENSOR 0
#define ORACLE_SCALE_HEAD 1
#define ORACLE_SCALE_TOKEN 2

/* ------------------------------------------------------------------ */
/* Number formats                                                      */
/* ------------------------------------------------------------------ */

static float bits_to_float(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t float_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* BF16 is the upper half of an IEEE binary32: widening is exact. */
float oracle_bf16_to_f32(uint16_t b) { return bits_to_float(((uint32_t)b) << 16); }

/*
 * Value of an E4M3 code, from the definition of the format:
 *   s = bit 7, e = bits 6..3, m = bits 2..0
 *   e == 15 and m == 7      -> NaN (no infinities)
 *   e == 0                  -> (-1)^s * (m/8) * 2^(1-7)      (subnormal)
 *   otherwise               -> (-1)^s * (1 + m/8) * 2^(e-7)
 */
double oracle_e4m3_decode(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m / 8.0, 1 - 7);
  else v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return s ? -v : v;
}

/* Round the non-negative integer m * 2^-sh to the nearest integer, ties to
 * even.  Exact integer arithmetic; m < 2^24. */
static uint32_t rne_shift(uint32_t m, int sh) {
  if (sh <= 0) return m << (-sh);
  if (sh >= 32) return 0;
  uint32_t q = m >> sh;
  uint32_t r = m & ((1u << sh) - 1u);
  uint32_t half = 1u << (sh - 1);
  if (r > half || (r == half && (q & 1u))) q++;
  return q;
}

/*
 * FP32 -> E4M3, round to nearest even, saturating.  Works on the bits of the
 * float: |y| = M * 2^E exactly (M the integer significand), the E4M3 grid
 * spacing at that magnitude is 2^Q, and the code's integer significand is
 * k = rne(|y| / 2^Q).  Subnormal codes use Q = -9 and code = k (k = 8 lands
 * on the smallest normal, code 0x08); normal codes with exponent e use
 * Q = e - 3 and code = (e + 7) * 8 + (k - 8), where k = 16 carries into the
 * next exponent by the same formula.
 *   NaN -> 0x7F; |y| >= 448 (inf included) -> 0x7E with the sign;
 *   zeros and values that round to zero keep their sign (-0 -> 0x80).
 */
uint8_t oracle_e4m3_encode(float y) {
  uint32_t u = float_to_bits(y);
  uint8_t sign = (uint8_t)((u >> 31) << 7);
  uint32_t a = u & 0x7FFFFFFFu;
  if (a > 0x7F800000u) return 0x7F;                  /* NaN */
  if (a >= float_to_bits(448.0f)) return sign | 0x7E; /* saturate */
  uint32_t M; int E;                                   /* |y| = M * 2^E */
  if (a >= 0x00800000u) { M = (a & 0x7FFFFFu) | 0x800000u; E = (int)(a >> 23) - 127 - 23; }
  else { M = a; E = -149; }                            /* float subnormal / zero */
  if (M == 0) return sign;
  /* unbiased exponent of |y| (floor(log2|y|)) */
  int msb = 31; while (!(M & (1u << msb))) msb--;
  int e = E + msb;
  uint32_t code;
  if (e < -6) {                                        /* E4M3 subnormal range */
    uint32_t k = rne_shift(M, -9 - E);
    code = k;                                          /* k <= 8 */
  } else {
    int Q = e - 3;
    uint32_t k = rne_shift(M, Q - E);                  /* 8 <= k <= 16 */
    code = (uint32_t)(e + 7) * 8u + (k - 8u);
  }
  return (uint8_t)(sign | code);
}

void oracle_e4m3_encode_array(const float* y, uint8_t* out, int64_t n) {
  for (int64_t i = 0; i < n; i++) out[i] = oracle_e4m3_encode(y[i]);
}

/* Encode the floats whose bit patterns are start, start+1, ..., start+count-1. */
void oracle_e4m3_encode_bits_range(uint32_t start, uint32_t count, uint8_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)count; i++)
    out[i] = oracle_e4m3_encode(bits_to_float(start + (uint32_t)i));
}

/* Codes of (float with bit pattern start + i) / scale, the quotient being
 * the IEEE binary32 division (this file is built without contraction or
 * fast math): the quantize step of the append, R3. */
void oracle_e4m3_quantize_bits_range(uint32_t start, uint32_t count, float scale, uint8_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < (int64_t)count; i++)
    out[i] = oracle_e4m3_encode(bits_to_float(start + (uint32_t)i) / scale);
}

void oracle_e4m3_decode_array(const uint8_t* c, double* out, int64_t n) {
  for (int64_t i = 0; i < n; i++) out[i] = oracle_e4m3_decode(c[i]);
}

/* ------------------------------------------------------------------ */
/* Scales: s = fl32(amax / 448), amax = 0 -> 1                          */
/* ------------------------------------------------------------------ */

float oracle_scale_from_amax(float amax) {
  if (!(amax > 0.0f)) return 1.0f;
  return amax / 448.0f;   /* IEEE binary32 division, correctly rounded */
}

/* Fold max|x| of a BF16 tensor x[T][H][D] into amax_io[1] (per_head == 0)
 * or amax_io[H] (per_head != 0); NaN elements are ignored (v > amax is
 * false for them). */
void oracle_amax(const uint16_t* x, int64_t T, int32_t H, int32_t D, int32_t per_head,
                 float* amax_io) {
  for (int64_t t = 0; t < T; t++)
    for (int32_t h = 0; h < H; h++) {
      float* a = amax_io + (per_head ? h : 0);
      for (int32_t d = 0; d < D; d++) {
        float v = fabsf(oracle_bf16_to_f32(x[(t * H + h) * D + d]));
        if (v > *a) *a = v;
      }
    }
}

/* Scales of a BF16 tensor x[T][H][D]: one over everything (per_head == 0)
 * or one per head (per_head != 0). */
void oracle_scales(const uint16_t* x, int64_t T, int32_t H, int32_t D, int32_t per_head,
                   float* scale_out) {
  int32_t nout = per_head ? H : 1;
  for (int32_t o = 0; o < nout; o++) scale_out[o] = 0.0f;
  oracle_amax(x, T, H, D, per_head, scale_out);
  for (int32_t o = 0; o < nout; o++) scale_out[o] = oracle_scale_from_amax(scale_out[o]);
}

/* ------------------------------------------------------------------ */
/* Append: tag bump on reallocation, then quantize-on-write             */
/* ------------------------------------------------------------------ */

/*
 * Every page in realloc_pages gets its tag advanced by one (mod 2^32) per
 * occurrence: the tag is a generation counter that changes whenever the
 * page is handed out again ([remio] "Sicherheit gemeinsamer KV-Caches wird
 * zum Produktionsthema"; [manulx] "Bảo vệ bộ nhớ đệm dùng chung").
 * Ids outside [0, P) are ignored.
 *
 * Then each new token t with slot = slot_mapping[t] in [0, P*ps) is written
 * at page slot/ps, offset slot%ps.  FP8: code = E(fl32(x) / s), IEEE float
 * division; TOKEN scale mode first sets s = fl32(amax(row)/448) and stores
 * it at [page][head][offset].  BF16: the bits are copied.  Slots < 0 or
 * beyond the pool are skipped.
 */
void oracle_append(int32_t dtype, int32_t scale_mode, int32_t P, int32_t ps, int32_t Hkv,
                   int32_t Dk, int32_t Dv, void* k_pages, void* v_pages, float* k_scale,
                   float* v_scale, uint32_t* tags, const uint16_t* k_new,
                   const uint16_t* v_new, const int32_t* slot_mapping, int32_t T,
                   const int32_t* realloc_pages, int32_t n_realloc) {
  for (int32_t r = 0; r < n_realloc; r++) {
    int32_t p = realloc_pages[r];
    if (p >= 0 && p < P) tags[p] = tags[p] + 1u;
  }
  /* tokens write disjoint rows (distinct slots), so they are independent */
#pragma omp parallel for schedule(static)
  for (int32_t t = 0; t < T; t++) {
    int64_t slot = slot_mapping[t];
    if (slot < 0 || slot >= (int64_t)P * ps) continue;
    int64_t p = slot / ps, o = slot % ps;
    for (int32_t h = 0; h < Hkv; h++) {
      for (int part = 0; part < 2; part++) {          /* 0: K, 1: V */
        if (part == 1 && v_pages == NULL) continue;
        int32_t D = part ? Dv : Dk;
        const uint16_t* row = (part ? v_new : k_new) + ((int64_t)t * Hkv + h) * D;
        int64_t dst = ((p * Hkv + h) * ps + o) * D;
        if (dtype == ORACLE_BF16) {
          uint16_t* pages = (uint16_t*)(part ? v_pages : k_pages);
          for (int32_t d = 0; d < D; d++) pages[dst + d] = row[d];
          continue;
        }
        float* sc = part ? v_scale : k_scale;
        float s;
        if (scale_mode == ORACLE_SCALE_TENSOR) s = sc[0];
        else if (scale_mode == ORACLE_SCALE_HEAD) s = sc[h];
        else {
          float amax = 0.0f;
          for (int32_t d = 0; d < D; d++) {
            float v = fabsf(oracle_bf16_to_f32(row[d]));
            if (v > amax) amax = v;
          }
          s = oracle_scale_from_amax(amax);
          sc[(p * Hkv + h) * ps + o] = s;
        }
        uint8_t* pages = (uint8_t*)(part ? v_pages : k_pages);
        for (int32_t d = 0; d < D; d++) {
          float x = oracle_bf16_to_f32(row[d]);
          pages[dst + d] = oracle_e4m3_encode(x / s);
        }
      }
    }
  }
}

/* ------------------------------------------------------------------ */
/* Validation                                                          */
/* ------------------------------------------------------------------ */

/* Tokens of sequence b that decode reads: seq_len clamped to [0, max_pages*ps]. */
static int64_t clamp_tokens(int32_t seq_len, int32_t max_pages, int32_t ps) {
  int64_t n = seq_len < 0 ? 0 : seq_len;
  int64_t cap = (int64_t)max_pages * ps;
  return n > cap ? cap : n;
}

/*
 * Batched check of each request's expected (page, tag) pairs against the
 * live tags, run before decode reads the cache; a mismatch aborts the
 * request instead of letting it read a page that may belong to someone else
 * ([remio] "Sicherheit gemeinsamer KV-Caches wird zum Produktionsthema";
 * [manulx] "Bảo vệ bộ nhớ đệm dùng chung"; [lens] "KV キャッシュ整合性チェック").
 * abort[b] = 1 iff some i < ceil(tokens_b/ps) has bt[b][i] outside [0, P)
 * or tags[bt[b][i]] != expected[b][i]; entries beyond are ignored.
 */
void oracle_validate(const uint32_t* tags, int32_t P, const int32_t* block_table,
                     const uint32_t* expected, const int32_t* seq_lens, int32_t ps, int32_t B,
                     int32_t max_pages, uint8_t* abort_mask, int32_t* first_bad) {
  for (int32_t b = 0; b < B; b++) {
    int64_t n = clamp_tokens(seq_lens[b], max_pages, ps);
    int64_t npages = (n + ps - 1) / ps;
    uint8_t bad = 0;
    int32_t first = -1;   /* telemetry: the first entry that fails, in index order */
    for (int64_t i = 0; i < npages; i++) {
      int32_t p = block_table[(int64_t)b * max_pages + i];
      if (p < 0 || p >= P || tags[p] != expected[(int64_t)b * max_pages + i]) {
        if (!bad) first = (int32_t)i;
        bad = 1;
      }
    }
    abort_mask[b] = bad;
    if (first_bad) first_bad[b] = first;
  }
}

/* ------------------------------------------------------------------ */
/* Decode attention                                                    */
/* ------------------------------------------------------------------ */

/* Dequantised cache value, the number both sides start from:
 * FP8: fl32(dec(code) * s) (the double product is exact, one rounding to
 * float); BF16: the stored value.  Pages outside [0, P) read as zero. */
static float cache_value(int32_t dtype, int32_t scale_mode, int32_t P, int32_t ps,
                         int32_t Hkv, int32_t D, const void* pages, const float* scale,
                         int32_t page, int32_t h, int32_t o, int32_t d) {
  if (page < 0 || page >= P) return 0.0f;
  int64_t idx = (((int64_t)page * Hkv + h) * ps + o) * D + d;
  if (dtype == ORACLE_BF16) return oracle_bf16_to_f32(((const uint16_t*)pages)[idx]);
  float s;
  if (scale_mode == ORACLE_SCALE_TENSOR) s = scale[0];
  else if (scale_mode == ORACLE_SCALE_HEAD) s = scale[h];
  else s = scale[((int64_t)page * Hkv + h) * ps + o];
  return (float)(oracle_e4m3_decode(((const uint8_t*)pages)[idx]) * (double)s);
}

/*
 * One decode step: the single new query token of each sequence attends to
 * the sequence's cached tokens, gathered through its page table, reading the
 * FP8 cache with a conversion per element ([manulx] "Bộ nhớ đệm KV FP8 tăng
 * gấp đôi dung lượng ngữ cảnh"; [remio] "Warum kleinere Cloudflare-Caches
 * reine Geschwindigkeit schlagen").  Query head h reads KV head h / (Hq/Hkv).
 * In fp64:
 *   s_j = sm_scale * sum_d q_d Khat_jd,  p = softmax(s),
 *   out = sum_j p_j Vhat_j,  lse = ln sum_j exp(s_j).
 * Aborted or empty rows: out = 0, lse = -inf.
 * rows: list of b*Hq + h to compute (NULL: all, in order); out is
 * [n_rows][Dv], lse [n_rows].
 */
void oracle_decode(int32_t dtype, int32_t scale_mode, int32_t P, int32_t ps, int32_t Hkv,
                   int32_t Dk, int32_t Dv, const void* k_pages, const void* v_pages,
                   const float* k_scale, const float* v_scale, const uint16_t* q, int32_t Hq,
                   const int32_t* block_table, int32_t max_pages, const int32_t* seq_lens,
                   int32_t B, const uint8_t* abort_mask, float sm_scale, const int32_t* rows,
                   int32_t n_rows, double* out, double* lse) {
  int32_t G = Hq / Hkv;
  int32_t total = rows ? n_rows : B * Hq;
  /* V aliasing K: V is the first Dv dims of K and uses K's scales. */
  const void* vp = v_pages ? v_pages : k_pages;
  const float* vs = v_pages ? v_scale : k_scale;
  int32_t vD = v_pages ? Dv : Dk;
#pragma omp parallel for schedule(dynamic, 1)
  for (int32_t r = 0; r < total; r++) {
    int32_t row = rows ? rows[r] : r;
    int32_t b = row / Hq, h = row % Hq, hk = h / G;
    double* o_row = out + (int64_t)r * Dv;
    for (int32_t d = 0; d < Dv; d++) o_row[d] = 0.0;
    int64_t n = clamp_tokens(seq_lens[b], max_pages, ps);
    if ((abort_mask && abort_mask[b]) || n == 0) { lse[r] = -INFINITY; continue; }
    const uint16_t* qr = q + ((int64_t)b * Hq + h) * Dk;
    double* s = (double*)malloc(sizeof(double) * (size_t)n);
    double m = -INFINITY;
    for (int64_t j = 0; j < n; j++) {
      int32_t page = block_table[(int64_t)b * max_pages + j / ps];
      int32_t off = (int32_t)(j % ps);
      double acc = 0.0;
      for (int32_t d = 0; d < Dk; d++)
        acc += (double)oracle_bf16_to_f32(qr[d]) *
               (double)cache_value(dtype, scale_mode, P, ps, Hkv, Dk, k_pages, k_scale, page,
                                   hk, off, d);
      s[j] = (double)sm_scale * acc;
      if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < n; j++) {
      double p = exp(s[j] - m);
      l += p;
      int32_t page = block_table[(int64_t)b * max_pages + j / ps];
      int32_t off = (int32_t)(j % ps);
      for (int32_t d = 0; d < Dv; d++)
        o_row[d] += p * (double)cache_value(dtype, scale_mode, P, ps, Hkv, vD, vp, vs, page,
                                            hk, off, d);
    }
    for (int32_t d = 0; d < Dv; d++) o_row[d] /= l;
    lse[r] = m + log(l);
    free(s);
  }
}
