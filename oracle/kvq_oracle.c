/*
 * kvq_oracle.c -- plain, slow CPU oracle for the rotated-INT4 paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this file's library.  It shares no
 * code, header, table or constant generator with the CUDA library; both are
 * written independently from the same sources:
 *
 *   [P1] "KVキャッシュを4ビットへ — SAW-INT4とシステムを踏まえたINT4量子化"
 *        (youngju.dev blog, explaining the SAW-INT4 preprint)
 *   [P2] "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World
 *        LLM Serving" (gist.science explainer of the same preprint)
 *   [P3] "BitDecoding-FP4:FP4 KVキャッシュのネイティブ復号" (sns.style), for the
 *        NVFP4 cache format (fmt = 1): E2M1 codes with E4M3 block scales.
 *
 * Where the pages leave a step open, the reading taken is stated beside the
 * step and collected in the design notes.  Every floating-point step below is
 * a single IEEE operation in the precision named; build with
 * -O2 -fno-fast-math -ffp-contract=off so that no multiply-add is fused.
 *
 * Parity pins (tests/test_oracle_*.py) tie each function to something other
 * than itself: the explicit Sylvester-Hadamard matrix, H.H^T = b.I, the
 * rotate/unrotate round trip, (Hq).(Hk) = q.k, closed-form rows, the
 * |x - code*s| <= s/2 bound, brute-force softmax on tiny inputs, and an index
 * round trip of the paged store.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- fp16 ---- */
/* fp16 <-> fp32 through the compiler's IEEE binary16 type (_Float16).  The
 * conversion float -> _Float16 rounds to nearest, ties to even. */
float oracle_half_to_float(uint16_t h) {
  _Float16 v;
  memcpy(&v, &h, sizeof v);
  return (float)v;
}

uint16_t oracle_float_to_half(float f) {
  _Float16 v = (_Float16)f;
  uint16_t h;
  memcpy(&h, &v, sizeof h);
  return h;
}

/* ------------------------------------------------------------ rotation ---- */
/* Normalising constant of the orthonormal Hadamard block of size b: the fp32
 * value nearest 1/sqrt(b).  [P1, "回転のトリック — ブロック対角アダマール":
 * the rotation is orthogonal, so the +-1 Sylvester matrix is scaled by
 * 1/sqrt(b).] */
float oracle_hadamard_scale_f32(int b) { return (float)(1.0 / sqrt((double)b)); }

static int is_pow2(int b) { return b > 0 && (b & (b - 1)) == 0; }

/* Block-diagonal fast Walsh-Hadamard transform in fp32, in place, on a vector
 * of n channels cut into n/b independent blocks of b channels.
 * [P1, "回転のトリック — ブロック対角アダマール": a Hadamard rotation applied
 * only inside blocks of channels.]  Fixed butterfly order (a stated reading):
 * stages h = 1, 2, 4, ..., b/2; in stage h every pair (i, i+h) with bit h of i
 * clear becomes (a + c, a - c); after the last stage every channel is
 * multiplied once by the fp32 constant nearest 1/sqrt(b).  Natural (Sylvester)
 * order, not sequency order.  Returns 0, or -1 for a bad size. */
int oracle_fwht_f32(float* x, int n, int b) {
  if (!is_pow2(b) || n <= 0 || n % b != 0) return -1;
  const float cb = oracle_hadamard_scale_f32(b);
  for (int base = 0; base < n; base += b) {
    float* y = x + base;
    for (int h = 1; h < b; h *= 2) {
      for (int i = 0; i < b; i++) {
        if (i & h) continue;
        float a = y[i];
        float c = y[i + h];
        y[i] = a + c;
        y[i + h] = a - c;
      }
    }
    for (int i = 0; i < b; i++) y[i] = y[i] * cb;
  }
  return 0;
}

/* The same transform in fp64 (used for the attention reference, whose
 * arithmetic the pages do not fix; fp64 is the exact-as-practical choice). */
int oracle_fwht_f64(double* x, int n, int b) {
  if (!is_pow2(b) || n <= 0 || n % b != 0) return -1;
  const double cb = 1.0 / sqrt((double)b);
  for (int base = 0; base < n; base += b) {
    double* y = x + base;
    for (int h = 1; h < b; h *= 2) {
      for (int i = 0; i < b; i++) {
        if (i & h) continue;
        double a = y[i];
        double c = y[i + h];
        y[i] = a + c;
        y[i + h] = a - c;
      }
    }
    for (int i = 0; i < b; i++) y[i] = y[i] * cb;
  }
  return 0;
}

/* -------------------------------------------------------- quantisation ---- */
/* Token-wise symmetric INT4 quantisation of one rotated row y[0..d).
 * [P1, "素朴なINT4はなぜ崩れるのか": one scale per token, taken the moment the
 * token's K/V is produced.]  Readings for what the pages leave open:
 *   m   = max_d |y_d| over the whole head (not per Hadamard block);
 *   s32 = m / 7 (one IEEE fp32 division);
 *   s   = s32 rounded to fp16, nearest-even; saturated to 65504 if s32 is
 *         above the fp16 range;
 *   code_d = clamp(rint(y_d / s), -8, 7), the division by the STORED fp16
 *         scale, rint with ties to even; every code 0 when s == 0.
 * Returns the fp16 bit pattern of s; writes codes[0..d). */
uint16_t oracle_quant_row(const float* y, int d, int8_t* codes) {
  float m = 0.0f;
  for (int i = 0; i < d; i++) {
    float a = fabsf(y[i]);
    if (a > m) m = a;
  }
  const float s32 = m / 7.0f;
  const uint16_t sbits = (s32 > 65504.0f) ? (uint16_t)0x7BFF : oracle_float_to_half(s32);
  const float s = oracle_half_to_float(sbits);
  for (int i = 0; i < d; i++) {
    int c = 0;
    if (s != 0.0f) {
      float t = rintf(y[i] / s);
      if (t < -8.0f) t = -8.0f;
      if (t > 7.0f) t = 7.0f;
      c = (int)t;
    }
    codes[i] = (int8_t)c;
  }
  return sbits;
}

/* Two codes per byte, low nibble = even channel, 4-bit two's complement
 * (a stated reading; the pages do not fix the nibble order). */
void oracle_pack_codes(const int8_t* codes, int d, uint8_t* out) {
  for (int j = 0; j < d / 2; j++)
    out[j] = (uint8_t)(((unsigned)codes[2 * j] & 0xFu) | (((unsigned)codes[2 * j + 1] & 0xFu) << 4));
}

/* Inverse of the packing: nibble -> signed integer in [-8, 7]. */
void oracle_unpack_codes(const uint8_t* in, int d, int8_t* codes) {
  for (int j = 0; j < d / 2; j++) {
    int lo = in[j] & 0xF, hi = (in[j] >> 4) & 0xF;
    codes[2 * j] = (int8_t)(lo >= 8 ? lo - 16 : lo);
    codes[2 * j + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
  }
}

/* --------------------------------------------------------------- NVFP4 ---- */
/* [P3, "背景と概要": NVFP4 is a 4-bit microscaling format -- 4-bit elements sharing a
 * block scale -- and "深掘り分析": its block scales are E4M3.]  The pages give no
 * formulas; the readings, for the cache format fmt = 1:
 *   element  E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; magnitudes
 *            {0, 0.5, 1, 1.5, 2, 3, 4, 6} for codes 0..7, bit 3 the sign;
 *   block    16 consecutive channels of one rotated row share one scale;
 *   scale    E4M3 (bias 7, 3 mantissa bits, no infinity, largest 448), the value
 *            amax / 6 (one fp32 division) rounded to nearest, ties to even, and
 *            saturated to 448; no second, per-tensor scale;
 *   codes    t = y * r with r = 1 / s (both fp32 operations), rounded to the nearest
 *            E2M1 magnitude (ties to the even code), saturated to 6, the sign of t
 *            kept (so -0 is code 8); every code 0 when s == 0.
 * Both roundings are written out as a search over the format's finite values, the
 * plainest statement of round-to-nearest-even. */
float oracle_e4m3_to_float(uint8_t b) {
  const int sgn = (b >> 7) & 1, e = (b >> 3) & 0xF, m = b & 7;
  double v = e == 0 ? (double)m / 8.0 * ldexp(1.0, -6) : (1.0 + (double)m / 8.0) * ldexp(1.0, e - 7);
  return (float)(sgn ? -v : v);
}

/* Nearest E4M3 code to x (x >= 0 or negative: the sign is kept), ties to the even code,
 * saturating at 448.  Codes 0..126 are the non-negative finite values in order. */
uint8_t oracle_float_to_e4m3(float x) {
  const int sgn = signbit(x) ? 1 : 0;
  const double a = fabs((double)x);
  int best = 0;
  double bestd = INFINITY;
  for (int c = 0; c <= 126; c++) {
    const double d = fabs(a - (double)oracle_e4m3_to_float((uint8_t)c));
    if (d < bestd || (d == bestd && (c & 1) == 0)) { best = c; bestd = d; }
  }
  return (uint8_t)((sgn << 7) | best);
}

float oracle_e2m1_to_float(uint8_t c) {
  static const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  const float v = mag[c & 7];
  return (c & 8) ? -v : v;
}

/* Nearest E2M1 code to x, ties to the even code, saturating at 6, sign of x kept. */
uint8_t oracle_float_to_e2m1(float x) {
  const int sgn = signbit(x) ? 1 : 0;
  const double a = fabs((double)x);
  int best = 0;
  double bestd = INFINITY;
  for (int c = 0; c < 8; c++) {
    const double d = fabs(a - (double)oracle_e2m1_to_float((uint8_t)c));
    if (d < bestd || (d == bestd && (c & 1) == 0)) { best = c; bestd = d; }
  }
  return (uint8_t)((sgn << 3) | best);
}

/* NVFP4 quantisation of one rotated row y[0..d) (d a multiple of 16): codes[0..d) (one
 * E2M1 code per byte, 0..15) and scales[0..d/16) (E4M3 bytes). */
void oracle_quant_row_nvfp4(const float* y, int d, uint8_t* codes, uint8_t* scales) {
  for (int b0 = 0; b0 < d; b0 += 16) {
    float m = 0.0f;
    for (int i = b0; i < b0 + 16; i++) {
      const float a = fabsf(y[i]);
      if (a > m) m = a;
    }
    const float s32 = m / 6.0f;
    const uint8_t sb = oracle_float_to_e4m3(s32);
    const float s = oracle_e4m3_to_float(sb);
    scales[b0 / 16] = sb;
    if (s == 0.0f) {
      for (int i = b0; i < b0 + 16; i++) codes[i] = 0;
      continue;
    }
    const float r = 1.0f / s;
    for (int i = b0; i < b0 + 16; i++) {
      const float t = y[i] * r;
      codes[i] = oracle_float_to_e2m1(t);
    }
  }
}

/* ------------------------------------------------------------- paging ---- */
/* Deterministic page assignment (a stated reading; the pages only fix
 * "fixed-size blocks plus a page table" [P1, "KVキャッシュこそが本当の
 * ボトルネックである理由"]): walk the page order (or 0..num_pages-1), giving
 * sequence b, in order of b, the next ceil(capacity_b / page_size) pages.
 * Unused table entries are -1.  Returns 0, -1 for a bad argument, -2 when a
 * sequence needs more than max_pages_per_seq pages, -3 when the pool runs out. */
int oracle_assign_pages(int batch, const int32_t* capacity, int page_size, int num_pages,
                        int max_pages_per_seq, const int32_t* page_order, int32_t* page_table) {
  if (batch < 0 || page_size <= 0 || num_pages < 0 || max_pages_per_seq < 0) return -1;
  int next = 0;
  for (int b = 0; b < batch; b++) {
    if (capacity[b] < 0) return -1;
    int need = (capacity[b] + page_size - 1) / page_size;
    if (need > max_pages_per_seq) return -2;
    for (int p = 0; p < max_pages_per_seq; p++) {
      int32_t v = -1;
      if (p < need) {
        if (next >= num_pages) return -3;
        v = page_order ? page_order[next] : next;
        next++;
      }
      page_table[(size_t)b * max_pages_per_seq + p] = v;
    }
  }
  return 0;
}

/* Byte size of one (page, head) block: K codes, V codes, K scales, V scales,
 * each for page_size tokens (a stated reading of the block layout).  A token row's
 * scales take 2 bytes (fmt 0: one fp16) or head_dim / 16 bytes (fmt 1: E4M3 per block). */
static size_t row_scale_bytes(int head_dim, int fmt) { return fmt ? (size_t)head_dim / 16 : 2; }

size_t oracle_block_bytes(int page_size, int head_dim, int fmt) {
  return (size_t)page_size * ((size_t)head_dim + 2 * row_scale_bytes(head_dim, fmt));
}

/* Offset of block (layer, page, head) in the pool.  Pool layout, outermost
 * first: layer, page, KV head; inside a block:
 *   [K codes  S x D/2 bytes][V codes  S x D/2 bytes][K scales S x sb][V scales S x sb]
 * with sb = row_scale_bytes (one fp16, or D/16 E4M3 bytes). */
static size_t block_offset(int layer, int page, int head, int num_pages, int num_kv_heads,
                           int page_size, int head_dim, int fmt) {
  return (((size_t)layer * num_pages + (size_t)page) * num_kv_heads + (size_t)head) *
         oracle_block_bytes(page_size, head_dim, fmt);
}

/* Rotate, quantise and append new tokens into the paged pool.
 * [P1, "システムこそが設計である — 融合カーネル": for every new token, K and V
 * are rotated block-diagonally, quantised token-wise and appended to the paged
 * KV blocks; past tokens are never revisited.]
 * k, v:           fp16 bit patterns, [total_new_tokens][num_kv_heads][head_dim]
 * cu_new_tokens:  [batch+1] prefix sums of new tokens per sequence
 * seq_lens:       [batch] lengths BEFORE this append
 * page_table:     [batch][max_pages_per_seq]
 * pool:           the whole pool (all layers), written in place.
 * Token i of sequence b goes to position pos = seq_lens[b] + i, page
 * page_table[b][pos / S], slot pos % S.  Returns 0, or -1 for a bad argument,
 * -4 for a page-table entry outside [0, num_pages). */
int oracle_rotate_quant_append(uint8_t* pool, int layer, int num_pages, int num_kv_heads,
                               int head_dim, int block, int page_size, int max_pages_per_seq,
                               const uint16_t* k, const uint16_t* v, const int32_t* cu_new_tokens,
                               const int32_t* seq_lens, const int32_t* page_table, int batch,
                               int fmt) {
  const int D = head_dim, S = page_size;
  if (D <= 0 || D % 2 || D % block || S <= 0 || batch < 0) return -1;
  if (fmt && D % 16) return -1;
  const size_t sb = row_scale_bytes(D, fmt);
  float* row = (float*)malloc(sizeof(float) * (size_t)D);
  int8_t* codes = (int8_t*)malloc((size_t)D);
  uint8_t* fcodes = (uint8_t*)malloc((size_t)D);
  uint8_t* fscales = (uint8_t*)malloc((size_t)D / 16 + 1);
  if (!row || !codes || !fcodes || !fscales) {
    free(row); free(codes); free(fcodes); free(fscales);
    return -1;
  }
  int rc = 0;
  for (int b = 0; b < batch && rc == 0; b++) {
    for (int t = cu_new_tokens[b]; t < cu_new_tokens[b + 1] && rc == 0; t++) {
      const int pos = seq_lens[b] + (t - cu_new_tokens[b]);
      const int lp = pos / S, slot = pos % S;
      if (pos < 0 || lp >= max_pages_per_seq) { rc = -1; break; }
      const int page = page_table[(size_t)b * max_pages_per_seq + lp];
      if (page < 0 || page >= num_pages) { rc = -4; break; }
      for (int h = 0; h < num_kv_heads; h++) {
        uint8_t* blk = pool + block_offset(layer, page, h, num_pages, num_kv_heads, S, D, fmt);
        for (int kv = 0; kv < 2; kv++) {
          const uint16_t* src = (kv == 0 ? k : v) + ((size_t)t * num_kv_heads + h) * D;
          for (int d = 0; d < D; d++) row[d] = oracle_half_to_float(src[d]);
          oracle_fwht_f32(row, D, block);
          uint8_t* cp = blk + (size_t)kv * S * (D / 2) + (size_t)slot * (D / 2);
          uint8_t* sp = blk + (size_t)S * D + (size_t)kv * S * sb + (size_t)slot * sb;
          if (fmt) {
            oracle_quant_row_nvfp4(row, D, fcodes, fscales);
            for (int j = 0; j < D / 2; j++) cp[j] = (uint8_t)(fcodes[2 * j] | (fcodes[2 * j + 1] << 4));
            memcpy(sp, fscales, sb);
          } else {
            uint16_t sbits = oracle_quant_row(row, D, codes);
            oracle_pack_codes(codes, D, cp);
            memcpy(sp, &sbits, 2);
          }
        }
      }
    }
  }
  free(row);
  free(codes);
  free(fcodes);
  free(fscales);
  return rc;
}

/* Dequantised row of the cache: code * scale in fp32 (exact: a 4-bit integer
 * times an 11-bit significand, or an E2M1 value times an E4M3 scale, 2 + 4
 * significant bits).  kv = 0 for K, 1 for V. */
int oracle_read_row(const uint8_t* pool, int layer, int num_pages, int num_kv_heads, int head_dim,
                    int page_size, int page, int head, int slot, int kv, float* out, int fmt) {
  const int D = head_dim, S = page_size;
  if (page < 0 || page >= num_pages || slot < 0 || slot >= S) return -1;
  const uint8_t* blk = pool + block_offset(layer, page, head, num_pages, num_kv_heads, S, D, fmt);
  const size_t sb = row_scale_bytes(D, fmt);
  const uint8_t* cp = blk + (size_t)kv * S * (D / 2) + (size_t)slot * (D / 2);
  const uint8_t* sp = blk + (size_t)S * D + (size_t)kv * S * sb + (size_t)slot * sb;
  if (D > 1024) return -1;
  if (fmt) {
    for (int d = 0; d < D; d++) {
      const uint8_t c = (uint8_t)((cp[d / 2] >> (4 * (d & 1))) & 0xF);
      out[d] = oracle_e2m1_to_float(c) * oracle_e4m3_to_float(sp[d / 16]);
    }
    return 0;
  }
  int8_t codes[1024];
  oracle_unpack_codes(cp, D, codes);
  uint16_t sbits;
  memcpy(&sbits, sp, 2);
  const float s = oracle_half_to_float(sbits);
  for (int d = 0; d < D; d++) out[d] = (float)codes[d] * s;
  return 0;
}

/* ----------------------------------------------------------- attention ---- */
/* Paged GQA decode attention for one (sequence b, query head hq), on the
 * dequantised cache, in fp64.  [P1, "KVキャッシュこそが本当のボトルネックで
 * ある理由": paged layout + fused attention execution.]  Readings:
 *   KV head of query head hq = hq / (num_q_heads / num_kv_heads);
 *   q' = block-diagonal orthonormal Hadamard of q (fp64);
 *   score_t = softmax_scale * sum_d q'_d * khat_{t,d};  softmax_scale 0 means
 *             1/sqrt(head_dim);
 *   p = exp(score - max) / sum exp;  o' = sum_t p_t vhat_t;
 *   o = Hadamard(o')  (the orthonormal Sylvester matrix is its own inverse).
 * An empty sequence gives zeros.  out: [head_dim] fp64.  Returns 0 or <0. */
/* Attention of one query row qrow (fp16 bits, [head_dim]) of sequence b over its
 * first L cached tokens of KV head h; the steps of oracle_decode_one below. */
static int attend_row(const uint8_t* pool, int layer, int num_pages, int num_kv_heads,
                      int head_dim, int block, int page_size, int max_pages_per_seq,
                      const uint16_t* qrow, const int32_t* page_table, int b, int L, int h,
                      double softmax_scale, double* out, int fmt) {
  const int D = head_dim, S = page_size;
  if (softmax_scale == 0.0) softmax_scale = 1.0 / sqrt((double)D);
  for (int d = 0; d < D; d++) out[d] = 0.0;
  if (L <= 0) return 0;
  if ((L + S - 1) / S > max_pages_per_seq) return -1;

  double* qr = (double*)malloc(sizeof(double) * (size_t)D);
  double* sc = (double*)malloc(sizeof(double) * (size_t)L);
  float* row = (float*)malloc(sizeof(float) * (size_t)D);
  if (!qr || !sc || !row) { free(qr); free(sc); free(row); return -1; }
  int rc = 0;

  for (int d = 0; d < D; d++) qr[d] = (double)oracle_half_to_float(qrow[d]);
  oracle_fwht_f64(qr, D, block);

  double mx = -INFINITY;
  for (int t = 0; t < L && rc == 0; t++) {
    const int page = page_table[(size_t)b * max_pages_per_seq + t / S];
    if (oracle_read_row(pool, layer, num_pages, num_kv_heads, D, S, page, h, t % S, 0, row, fmt)) {
      rc = -4;
      break;
    }
    double acc = 0.0;
    for (int d = 0; d < D; d++) acc += qr[d] * (double)row[d];
    sc[t] = softmax_scale * acc;
    if (sc[t] > mx) mx = sc[t];
  }
  double den = 0.0;
  for (int t = 0; t < L && rc == 0; t++) {
    sc[t] = exp(sc[t] - mx);
    den += sc[t];
  }
  for (int t = 0; t < L && rc == 0; t++) {
    const int page = page_table[(size_t)b * max_pages_per_seq + t / S];
    oracle_read_row(pool, layer, num_pages, num_kv_heads, D, S, page, h, t % S, 1, row, fmt);
    const double p = sc[t] / den;
    for (int d = 0; d < D; d++) out[d] += p * (double)row[d];
  }
  if (rc == 0) oracle_fwht_f64(out, D, block);
  free(qr);
  free(sc);
  free(row);
  return rc;
}

int oracle_decode_one(const uint8_t* pool, int layer, int num_pages, int num_kv_heads,
                      int num_q_heads, int head_dim, int block, int page_size,
                      int max_pages_per_seq, const uint16_t* q, const int32_t* seq_lens,
                      const int32_t* page_table, int b, int hq, double softmax_scale,
                      double* out, int fmt) {
  if (num_kv_heads <= 0 || num_q_heads % num_kv_heads) return -1;
  const int G = num_q_heads / num_kv_heads;
  return attend_row(pool, layer, num_pages, num_kv_heads, head_dim, block, page_size,
                    max_pages_per_seq, q + ((size_t)b * num_q_heads + hq) * head_dim,
                    page_table, b, seq_lens[b], hq / G, softmax_scale, out, fmt);
}

/* All (b, hq) pairs: out [batch][num_q_heads][head_dim] fp64. */
int oracle_decode_attention(const uint8_t* pool, int layer, int num_pages, int num_kv_heads,
                            int num_q_heads, int head_dim, int block, int page_size,
                            int max_pages_per_seq, const uint16_t* q, const int32_t* seq_lens,
                            const int32_t* page_table, int batch, double softmax_scale,
                            double* out, int fmt) {
  for (int b = 0; b < batch; b++)
    for (int hq = 0; hq < num_q_heads; hq++) {
      int rc = oracle_decode_one(pool, layer, num_pages, num_kv_heads, num_q_heads, head_dim,
                                 block, page_size, max_pages_per_seq, q, seq_lens, page_table, b,
                                 hq, softmax_scale,
                                 out + ((size_t)b * num_q_heads + hq) * head_dim, fmt);
      if (rc) return rc;
    }
  return 0;
}

/* Chunked-prefill attention over the paged cache, causal.  Sequence b holds
 * L_b = seq_lens[b] tokens, the last C_b = cu_q[b+1] - cu_q[b] of which are the chunk's
 * queries (already appended); query i of the chunk sits at position p = L_b - C_b + i and
 * attends positions 0..p.  [P1, "KVキャッシュこそが本当のボトルネックである理由": serving
 * engines run attention over the paged cache; a chunk of prompt tokens attending the
 * cache causally is the many-query case of the same attention (a stated reading).]
 * Each (query token, query head) is oracle_decode_one's computation over its causal
 * prefix.  q, out: [cu_q[batch]][num_q_heads][head_dim] (fp16 bits in, fp64 out). */
int oracle_prefill_attention(const uint8_t* pool, int layer, int num_pages, int num_kv_heads,
                             int num_q_heads, int head_dim, int block, int page_size,
                             int max_pages_per_seq, const uint16_t* q, const int32_t* cu_q,
                             const int32_t* seq_lens, const int32_t* page_table, int batch,
                             double softmax_scale, double* out, int fmt) {
  if (num_kv_heads <= 0 || num_q_heads % num_kv_heads) return -1;
  const int G = num_q_heads / num_kv_heads, D = head_dim;
  for (int b = 0; b < batch; b++) {
    const int C = cu_q[b + 1] - cu_q[b], L = seq_lens[b];
    if (C < 0 || C > L) return -1;
    for (int i = 0; i < C; i++) {
      const size_t tok = (size_t)cu_q[b] + i;
      const int pos = L - C + i;
      for (int hq = 0; hq < num_q_heads; hq++) {
        const int rc = attend_row(pool, layer, num_pages, num_kv_heads, D, block, page_size,
                                  max_pages_per_seq, q + (tok * num_q_heads + hq) * D,
                                  page_table, b, pos + 1, hq / G, softmax_scale,
                                  out + (tok * num_q_heads + hq) * D, fmt);
        if (rc) return rc;
      }
    }
  }
  return 0;
}

/* Exact softmax attention on UNQUANTISED fp64 inputs, for pinning the
 * attention arithmetic against a brute-force reference on tiny cases:
 * q [D], keys [L][D], values [L][D] -> out [D]; rotate = 1 runs the same
 * rotate-q / unrotate-o steps as the cache path (keys and values are then
 * taken to be already rotated). */
int oracle_attention_dense(const double* q, const double* keys, const double* values, int L,
                           int D, int block, int rotate, double softmax_scale, double* out) {
  if (softmax_scale == 0.0) softmax_scale = 1.0 / sqrt((double)D);
  double* qr = (double*)malloc(sizeof(double) * (size_t)D);
  double* sc = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
  if (!qr || !sc) { free(qr); free(sc); return -1; }
  for (int d = 0; d < D; d++) { qr[d] = q[d]; out[d] = 0.0; }
  if (rotate) oracle_fwht_f64(qr, D, block);
  if (L > 0) {
    double mx = -INFINITY;
    for (int t = 0; t < L; t++) {
      double acc = 0.0;
      for (int d = 0; d < D; d++) acc += qr[d] * keys[(size_t)t * D + d];
      sc[t] = softmax_scale * acc;
      if (sc[t] > mx) mx = sc[t];
    }
    double den = 0.0;
    for (int t = 0; t < L; t++) { sc[t] = exp(sc[t] - mx); den += sc[t]; }
    for (int t = 0; t < L; t++)
      for (int d = 0; d < D; d++) out[d] += (sc[t] / den) * values[(size_t)t * D + d];
    if (rotate) oracle_fwht_f64(out, D, block);
  }
  free(qr);
  free(sc);
  return 0;
}
