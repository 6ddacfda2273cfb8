/*
 * CSA2 decode-step oracle: a plain, slow, obviously correct CPU implementation.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this code: only the
 * tests, the smoke check and the benchmark's CPU-baseline leg load it.  It shares no
 * code, header, table or helper with the CUDA library; every format rule below is
 * written out again from the format definitions and the pages.
 *
 * Sources (web pages about the DeepSeek-V4.1-Flash technical report):
 *   P1 = "KV 캐시를 토큰당 890바이트로 압축한 552B 멀티모달 MoE, DeepSeek-V4.1-Flash"
 *        (onedev.kr paper summary)
 *   P2 = thakicloud tech blog, "DeepSeek V4.1-Flash KV compression"
 *   P3 = "100만 토큰을 0.9GB에, 딥시크 V4.1 논문이 KV 캐시를 줄인 방법" (genexis.ai)
 * A citation reads "P3 §<section heading>".
 *
 * Arithmetic: every score, logit, softmax and weighted sum is accumulated in double.
 * The packing decisions (block absmax, scale = absmax/6, x/scale) are taken in fp32,
 * the precision an NVFP4 encoder works in, so that both sides of a parity test take
 * each integer decision in the same precision.
 *
 * Parity pins for each function live in tests/test_oracle_*.py; every function here
 * has at least one pin that does not reuse its own arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_D 512   /* main-KV latent channels (P3 §레이어 40개 가운데 4개만 전역 캐시를 만듭니다) */
#define ORC_DI 128  /* indexer-key dimension (same section) */
#define ORC_KV_BYTES 288
#define ORC_IK_BYTES 68

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads.  Queries, entries and heads are independent, so every result is the same
 * whatever the thread count.  A call with at least as many queries as threads spreads
 * its queries over the threads; a call with fewer spreads the work inside each query
 * instead (the entries of a scan, the candidates of a Reindex, the heads of an attention
 * call), so a one-query sample still uses every core. */
static int orc_queries_parallel(int64_t n_queries) { return n_queries >= orc_num_threads(); }
static int orc_in_parallel(void) {
#ifdef _OPENMP
  return omp_in_parallel();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------------------
 * Element formats (P2 §KV 캐시 네 가지: "E2M1 family, shared scale";
 * P3 §4비트로 적어도 되는 이유: NVFP4 without the second-level global scale, one 8-bit
 * scale per 16 channels).  Written from the OCP microscaling format definitions.
 * ------------------------------------------------------------------------------------ */

/* E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa; no inf/NaN. */
double orc_e2m1_value(unsigned code) {
  unsigned e = (code >> 1) & 3u, f = code & 1u;
  double mag = (e == 0) ? 0.5 * f : ldexp(1.0 + 0.5 * f, (int)e - 1);
  return (code & 8u) ? -mag : mag;
}

/* Nearest E2M1 value to x; a tie goes to the code with an even mantissa bit; magnitudes
 * beyond 6 saturate to 6; the sign of x is kept (a negative value that rounds to zero
 * gives code 0x8).  Brute force over the eight magnitudes. */
unsigned orc_e2m1_encode(float x) {
  double a = fabs((double)x);
  unsigned sign = signbit(x) ? 8u : 0u;
  if (a >= 6.0) return 7u | sign;
  unsigned best = 0;
  double best_d = HUGE_VAL;
  for (unsigned m = 0; m < 8; ++m) {
    double d = fabs(a - orc_e2m1_value(m));
    if (d < best_d || (d == best_d && (m & 1u) == 0)) {
      best = m;
      best_d = d;
    }
  }
  return best | sign;
}

/* E4M3 ("fn" variant): bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa;
 * subnormals m*2^-9; 0x7F/0xFF are NaN; no infinities; largest finite 448 = 0x7E. */
double orc_e4m3_value(unsigned code) {
  unsigned e = (code >> 3) & 15u, m = code & 7u;
  if (e == 15 && m == 7) return NAN;
  double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, (int)e - 7);
  return (code & 0x80u) ? -mag : mag;
}

/* Nearest finite E4M3 value to x, ties to an even mantissa, saturating to +-448. */
unsigned orc_e4m3_encode(float x) {
  double a = fabs((double)x);
  unsigned sign = signbit(x) ? 0x80u : 0u;
  if (a >= 448.0) return 0x7Eu | sign;
  unsigned best = 0;
  double best_d = HUGE_VAL;
  for (unsigned c = 0; c <= 0x7Eu; ++c) {
    double d = fabs(a - orc_e4m3_value(c));
    if (d < best_d || (d == best_d && (c & 1u) == 0)) {
      best = c;
      best_d = d;
    }
  }
  return best | sign;
}

/* bfloat16 is the upper half of an IEEE binary32. */
float orc_bf16_value(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* ------------------------------------------------------------------------------------
 * Packing (P3 §레이어 40개 가운데 4개만 전역 캐시를 만듭니다: an entry is 288 B of
 * 512-channel FP4 main KV = 256 B values + 32 B scales, plus a 68 B 128-dim indexer
 * key; P3 §4비트로 적어도 되는 이유 for the scale granularity).
 *
 * Readings where the pages are silent:
 *  - main KV, per 16-channel block: amax = max|x| (fp32); s = E4M3(amax / 6.0f);
 *    sd = value(s); code = E2M1(x / sd) with an fp32 quotient; sd == 0 gives +0 codes.
 *  - layout: byte i (0..255) holds channel 2i in its low nibble and 2i+1 in its high
 *    nibble; byte 256+b holds the scale of channels 16b..16b+15.
 *  - indexer key: 64 B of codes in the same nibble order, then one little-endian fp32
 *    scale s = amax/6.0f over all 128 dims (64 + 4 = 68 B); code = E2M1(x / s);
 *    s == 0 gives +0 codes.
 *  - ratio 2 (encoder entries cover 2 tokens, same section): each channel is the fp32
 *    mean (a + b) * 0.5f of the two bf16 tokens before quantisation.
 * ------------------------------------------------------------------------------------ */

static void encode_kv_entry(const float* x /*[512]*/, uint8_t* out /*[288]*/) {
  memset(out, 0, ORC_KV_BYTES);
  for (int b = 0; b < ORC_D / 16; ++b) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
      float a = fabsf(x[16 * b + i]);
      if (a > amax) amax = a;
    }
    float sf = amax / 6.0f;
    unsigned s = orc_e4m3_encode(sf);
    float sd = (float)orc_e4m3_value(s);
    out[256 + b] = (uint8_t)s;
    for (int i = 0; i < 16; ++i) {
      int c = 16 * b + i;
      unsigned code = 0;
      if (sd != 0.0f) {
        float qv = x[c] / sd;
        code = orc_e2m1_encode(qv);
      }
      out[c / 2] |= (uint8_t)(code << ((c & 1) ? 4 : 0));
    }
  }
}

static void encode_ik_entry(const float* x /*[128]*/, uint8_t* out /*[68]*/) {
  memset(out, 0, ORC_IK_BYTES);
  float amax = 0.0f;
  for (int d = 0; d < ORC_DI; ++d) {
    float a = fabsf(x[d]);
    if (a > amax) amax = a;
  }
  float s = amax / 6.0f;
  for (int d = 0; d < ORC_DI; ++d) {
    unsigned code = 0;
    if (s != 0.0f) {
      float qv = x[d] / s;
      code = orc_e2m1_encode(qv);
    }
    out[d / 2] |= (uint8_t)(code << ((d & 1) ? 4 : 0));
  }
  memcpy(out + 64, &s, 4); /* little-endian host */
}

/* kv: [T][512] bf16 bits, ik: [T][128] bf16 bits; writes T/ratio contiguous entries. */
void orc_pack_kv(const uint16_t* kv, const uint16_t* ik, int64_t T, int ratio, uint8_t* kv_out,
                 uint8_t* ik_out) {
  int64_t E = T / ratio;
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < E; ++j) {
    float x[ORC_D], y[ORC_DI];
    for (int c = 0; c < ORC_D; ++c) {
      if (ratio == 1) {
        x[c] = orc_bf16_value(kv[j * ORC_D + c]);
      } else {
        float a = orc_bf16_value(kv[(2 * j) * ORC_D + c]);
        float b = orc_bf16_value(kv[(2 * j + 1) * ORC_D + c]);
        x[c] = (a + b) * 0.5f;
      }
    }
    for (int d = 0; d < ORC_DI; ++d) {
      if (ratio == 1) {
        y[d] = orc_bf16_value(ik[j * ORC_DI + d]);
      } else {
        float a = orc_bf16_value(ik[(2 * j) * ORC_DI + d]);
        float b = orc_bf16_value(ik[(2 * j + 1) * ORC_DI + d]);
        y[d] = (a + b) * 0.5f;
      }
    }
    encode_kv_entry(x, kv_out + j * ORC_KV_BYTES);
    encode_ik_entry(y, ik_out + j * ORC_IK_BYTES);
  }
}

/* ------------------------------------------------------------------------------------
 * Producer: RMSNorm + rotary position encoding, then the pack above (P3 §4비트로 적어도
 * 되는 이유: cached values are normalised and rotated before they are cached, which is
 * what bounds them by sqrt(512); the pages give no formula).
 *
 * Readings (the pages are silent; every operation is one fp32 rounding, no contraction):
 *  - RMSNorm of a 512-channel token x (bf16):  S = sum of x_c^2 by a fixed pairwise order:
 *    within each 16-channel block b, halving (element i += element i+8, then +4, +2, +1);
 *    then over the 32 block sums, halving (b += b+16, then +8, +4, +2, +1).
 *    m = S / 512;  r = 1 / sqrt(m + eps) as three rounded steps (add, sqrt, reciprocal);
 *    n_c = x_c * r, then n_c * gamma_c when a gain is given.
 *  - rotation of channel pairs (2i, 2i+1), i = 0..255, by the caller's tables at the
 *    token's position p:  c = cos[p][i], s = sin[p][i];
 *    y_2i = n_2i c - n_2i+1 s,  y_2i+1 = n_2i s + n_2i+1 c  (each product rounded).
 *  - y is rounded to bf16 (nearest, ties to even), then packed exactly as orc_pack_kv
 *    packs bf16 tokens (ratio 2: each token is normalised and rotated at its own
 *    position, the pair mean is taken from the two bf16 results).  The indexer key is
 *    packed from its own bf16 input unchanged.
 * ------------------------------------------------------------------------------------ */

/* Nearest bf16 (ties to even) of a finite fp32 value, as raw bits. */
uint16_t orc_bf16_round(float v) {
  uint32_t u;
  memcpy(&u, &v, 4);
  uint32_t lsb = (u >> 16) & 1u;
  return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
}

/* One token: x [512] bf16 bits -> y [512] fp32, normalised and rotated at position p
 * (cos_p, sin_p: that position's 256-entry table rows; gamma may be NULL). */
void orc_norm_rope_row(const uint16_t* x, const float* cos_p, const float* sin_p, const float* gamma,
                       float eps, float* y) {
  float v[ORC_D], blk[32];
  for (int c = 0; c < ORC_D; ++c) v[c] = orc_bf16_value(x[c]);
  for (int b = 0; b < 32; ++b) {
    float t[16];
    for (int i = 0; i < 16; ++i) t[i] = v[16 * b + i] * v[16 * b + i];
    for (int h = 8; h >= 1; h /= 2)
      for (int i = 0; i < h; ++i) t[i] = t[i] + t[i + h];
    blk[b] = t[0];
  }
  for (int h = 16; h >= 1; h /= 2)
    for (int b = 0; b < h; ++b) blk[b] = blk[b] + blk[b + h];
  float m = blk[0] / 512.0f;
  float r = 1.0f / sqrtf(m + eps);
  float n[ORC_D];
  for (int c = 0; c < ORC_D; ++c) {
    n[c] = v[c] * r;
    if (gamma) n[c] = n[c] * gamma[c];
  }
  for (int i = 0; i < ORC_D / 2; ++i) {
    float c = cos_p[i], s = sin_p[i];
    float a = n[2 * i], b = n[2 * i + 1];
    float ac = a * c, bs = b * s, as = a * s, bc = b * c;
    y[2 * i] = ac - bs;
    y[2 * i + 1] = as + bc;
  }
}

/* Producer: kv [T][512] raw bf16 tokens at positions pos[T] (indices into the tables,
 * rope_cos/rope_sin [n_pos][256]), ik [T][128] bf16; writes T/ratio contiguous entries.
 * A position outside [0, n_pos) leaves its entry all zero and returns nonzero. */
int orc_pack_kv_normed(const uint16_t* kv, const uint16_t* ik, int64_t T, int ratio, const int64_t* pos,
                       const float* rope_cos, const float* rope_sin, int64_t n_pos, const float* gamma,
                       float eps, uint8_t* kv_out, uint8_t* ik_out) {
  int64_t E = T / ratio;
  int bad = 0;
  uint16_t* tok = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(T > 0 ? T : 1) * ORC_D);
#pragma omp parallel for schedule(static) reduction(| : bad)
  for (int64_t t = 0; t < T; ++t) {
    float y[ORC_D];
    int64_t p = pos[t];
    if (p < 0 || p >= n_pos) {
      bad = 1;
      for (int c = 0; c < ORC_D; ++c) tok[t * ORC_D + c] = 0;
      continue;
    }
    orc_norm_rope_row(kv + t * ORC_D, rope_cos + p * (ORC_D / 2), rope_sin + p * (ORC_D / 2), gamma, eps, y);
    for (int c = 0; c < ORC_D; ++c) tok[t * ORC_D + c] = orc_bf16_round(y[c]);
  }
  orc_pack_kv(tok, ik, T, ratio, kv_out, ik_out);
  for (int64_t j = 0; j < E; ++j) {  /* entries with a bad position stay zero */
    int zero = 0;
    for (int k = 0; k < ratio; ++k) {
      int64_t p = pos[j * ratio + k];
      if (p < 0 || p >= n_pos) zero = 1;
    }
    if (zero) {
      memset(kv_out + j * ORC_KV_BYTES, 0, ORC_KV_BYTES);
      memset(ik_out + j * ORC_IK_BYTES, 0, ORC_IK_BYTES);
    }
  }
  free(tok);
  return bad;
}

/* Exact dequantisation (products of an E2M1 value and a scale are exact in double). */
void orc_dequant_kv(const uint8_t* e, double* out /*[512]*/) {
  for (int c = 0; c < ORC_D; ++c) {
    unsigned code = (e[c / 2] >> ((c & 1) ? 4 : 0)) & 15u;
    out[c] = orc_e4m3_value(e[256 + c / 16]) * orc_e2m1_value(code);
  }
}

void orc_dequant_ik(const uint8_t* e, double* out /*[128]*/) {
  float s;
  memcpy(&s, e + 64, 4);
  for (int d = 0; d < ORC_DI; ++d) {
    unsigned code = (e[d / 2] >> ((d & 1) ? 4 : 0)) & 15u;
    out[d] = (double)s * orc_e2m1_value(code);
  }
}

/* ------------------------------------------------------------------------------------
 * Indexer (P1 §무엇과 다른가: Full mode scores every causally visible entry with its own
 * indexer Q and picks Top-K; Reindex rescores with its own indexer Q).  The score
 * formula is the ReLU-weighted multi-head score the workload names:
 *     score_j = sum_h w_h * max(0, q_h . k_j),   k_j = dequantised indexer key.
 * ------------------------------------------------------------------------------------ */

static double score_one(const float* q, const float* w, int HI, const uint8_t* e) {
  double k[ORC_DI];
  orc_dequant_ik(e, k);
  double s = 0.0;
  for (int h = 0; h < HI; ++h) {
    double dot = 0.0;
    for (int d = 0; d < ORC_DI; ++d) dot += (double)q[h * ORC_DI + d] * k[d];
    s += (double)w[h] * (dot > 0.0 ? dot : 0.0);
  }
  return s;
}

void orc_index_scores(const float* q, const float* w, int HI, const uint8_t* ik_seq, int64_t n,
                      double* scores) {
#pragma omp parallel for schedule(static) if (!orc_in_parallel())
  for (int64_t j = 0; j < n; ++j) scores[j] = score_one(q, w, HI, ik_seq + j * ORC_IK_BYTES);
}

typedef struct {
  double s;
  int64_t i;
} orc_pair;

/* Descending score, then ascending index (a total order on distinct indices). */
static int cmp_pair(const void* a, const void* b) {
  const orc_pair* x = (const orc_pair*)a;
  const orc_pair* y = (const orc_pair*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->i < y->i) ? -1 : (x->i > y->i) ? 1 : 0;
}

/* Top-K of scores[0..n) (labels[i] names element i; NULL means i itself): the first
 * min(K, n) of the order above; the rest of the K slots hold -1. */
static void topk_labeled(const double* scores, const int64_t* labels, int64_t n, int K,
                         int32_t* idx_out, double* score_out) {
  orc_pair* p = (orc_pair*)malloc(sizeof(orc_pair) * (size_t)(n > 0 ? n : 1));
  for (int64_t i = 0; i < n; ++i) {
    p[i].s = scores[i];
    p[i].i = labels ? labels[i] : i;
  }
  qsort(p, (size_t)n, sizeof(orc_pair), cmp_pair);
  for (int k = 0; k < K; ++k) {
    if (k < n) {
      idx_out[k] = (int32_t)p[k].i;
      if (score_out) score_out[k] = p[k].s;
    } else {
      idx_out[k] = -1;
      if (score_out) score_out[k] = -HUGE_VAL;
    }
  }
  free(p);
}

void orc_topk(const double* scores, int64_t n, int K, int32_t* idx_out, double* score_out) {
  topk_labeled(scores, NULL, n, K, idx_out, score_out);
}

/* Flat Full-mode index: q [B][Q][HI][128], w [B][Q][HI]; entry j of sequence b is pool
 * entry seq_base[b] + j; query (b,i) sees entries [0, n_vis[b*Q+i]). */
void orc_index_full(const float* q, const float* w, const uint8_t* ik_pool, const int64_t* seq_base,
                    const int32_t* n_vis, int B, int Q, int HI, int K, int32_t* topk,
                    double* topk_score) {
#pragma omp parallel for schedule(dynamic, 1) if (orc_queries_parallel((int64_t)B * Q))
  for (int64_t bq = 0; bq < (int64_t)B * Q; ++bq) {
    int64_t b = bq / Q;
    int64_t n = n_vis[bq];
    double* sc = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    orc_index_scores(q + bq * HI * ORC_DI, w + bq * HI, HI, ik_pool + seq_base[b] * ORC_IK_BYTES, n,
                     sc);
    topk_labeled(sc, NULL, n, K, topk + bq * K, topk_score ? topk_score + bq * K : NULL);
    free(sc);
  }
}

/* Hierarchical block selection (P1 §무엇과 다른가; P3 §레이어 40개 가운데 4개만 전역
 * 캐시를 만듭니다: up to 2,048 blocks of 8 positions, a 16,384-position pool).
 * Reading: block c holds visible entries [block*c, block*c + block) of the sequence and
 * scores the max of its entries' scores; the top n_blocks blocks by (-score, c). */
void orc_index_hier(const float* q, const float* w, const uint8_t* ik_pool, const int64_t* seq_base,
                    const int32_t* n_vis, int B, int Q, int HI, int n_blocks, int block,
                    int32_t* blocks, double* block_score) {
#pragma omp parallel for schedule(dynamic, 1) if (orc_queries_parallel((int64_t)B * Q))
  for (int64_t bq = 0; bq < (int64_t)B * Q; ++bq) {
    int64_t b = bq / Q;
    int64_t n = n_vis[bq];
    int64_t nb = (n + block - 1) / block;
    double* sc = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double* bs = (double*)malloc(sizeof(double) * (size_t)(nb > 0 ? nb : 1));
    orc_index_scores(q + bq * HI * ORC_DI, w + bq * HI, HI, ik_pool + seq_base[b] * ORC_IK_BYTES, n,
                     sc);
    for (int64_t c = 0; c < nb; ++c) {
      double m = -HUGE_VAL;
      for (int64_t j = c * block; j < (c + 1) * block && j < n; ++j)
        if (sc[j] > m) m = sc[j];
      bs[c] = m;
    }
    topk_labeled(bs, NULL, nb, n_blocks, blocks + bq * n_blocks,
                 block_score ? block_score + bq * n_blocks : NULL);
    free(sc);
    free(bs);
  }
}

/* Reindex (P1 §무엇과 다른가; P3 §레이어 40개 가운데 4개만 전역 캐시를 만듭니다): the
 * layer's own q/w score only the visible entries of the given blocks (ids < 0 are
 * empty slots; ids are distinct), and the flat Top-K is taken over those candidates. */
void orc_reindex(const float* q, const float* w, const uint8_t* ik_pool, const int64_t* seq_base,
                 const int32_t* n_vis, const int32_t* blocks, int n_blocks, int block, int B, int Q,
                 int HI, int K, int32_t* topk, double* topk_score) {
#pragma omp parallel for schedule(dynamic, 1) if (orc_queries_parallel((int64_t)B * Q))
  for (int64_t bq = 0; bq < (int64_t)B * Q; ++bq) {
    int64_t b = bq / Q;
    int64_t n = n_vis[bq];
    int64_t cap = (int64_t)n_blocks * block;
    double* sc = (double*)malloc(sizeof(double) * (size_t)(cap > 0 ? cap : 1));
    int64_t* lab = (int64_t*)malloc(sizeof(int64_t) * (size_t)(cap > 0 ? cap : 1));
    int64_t m = 0;
    const uint8_t* seq = ik_pool + seq_base[b] * ORC_IK_BYTES;
    for (int s = 0; s < n_blocks; ++s) {
      int64_t c = blocks[bq * n_blocks + s];
      if (c < 0) continue;
      for (int64_t j = c * block; j < (c + 1) * block && j < n; ++j) {
        lab[m] = j;
        ++m;
      }
    }
#pragma omp parallel for schedule(static) if (!orc_in_parallel())
    for (int64_t i = 0; i < m; ++i)
      sc[i] = score_one(q + bq * HI * ORC_DI, w + bq * HI, HI, seq + lab[i] * ORC_IK_BYTES);
    topk_labeled(sc, lab, m, K, topk + bq * K, topk_score ? topk_score + bq * K : NULL);
    free(sc);
    free(lab);
  }
}

/* ------------------------------------------------------------------------------------
 * Sparse MQA attention (P1 §어떻게 동작하나: every CSA2 layer has a global branch and a
 * sliding-window branch; P3 §전역 어텐션과 지역 어텐션: the window is 128 tokens; P3
 * §4비트로 적어도 되는 이유: the window is kept in 8-bit FP; P1 §무엇과 다른가: Reuse
 * layers attend with the inherited Top-K list).
 * Reading: all H heads of a query read the same key set
 *     { dequant(KV entry j) : j in topk, j >= 0 }  U  { E4M3 window tokens u },
 * u in [max(0, t - window + 1), t] intersected with the buffer [swa_start, swa_start+S_w);
 * the dequantised latent is both key and value; logit = sm_scale * q_h . k; no
 * de-duplication between an entry and raw window tokens.  An empty key set gives
 * O = 0 and lse = -inf.
 * ------------------------------------------------------------------------------------ */
void orc_sparse_attn(const float* q /*[B][Q][H][512]*/, const uint8_t* kv_pool, const int64_t* seq_base,
                     const int32_t* topk /*[B][Q][K]*/, int K, const uint8_t* swa /*[B][S_w][512]*/,
                     int S_w, const int64_t* swa_start /*[B]*/, const int64_t* q_pos /*[B][Q]*/,
                     int window, int B, int Q, int H, double sm_scale, double* out /*[B][Q][H][512]*/,
                     double* lse /*[B][Q][H]*/) {
#pragma omp parallel for schedule(dynamic, 1) if (orc_queries_parallel((int64_t)B * Q))
  for (int64_t bq = 0; bq < (int64_t)B * Q; ++bq) {
    int64_t b = bq / Q;
    int64_t t = q_pos[bq];
    int nkeys_max = K + (S_w > 0 ? S_w : 0);
    double* keys = (double*)malloc(sizeof(double) * (size_t)(nkeys_max > 0 ? nkeys_max : 1) * ORC_D);
    int nk = 0;
    for (int k = 0; k < K; ++k) {
      int32_t j = topk[bq * K + k];
      if (j < 0) continue;
      orc_dequant_kv(kv_pool + (seq_base[b] + j) * ORC_KV_BYTES, keys + (size_t)nk * ORC_D);
      ++nk;
    }
    if (S_w > 0 && swa) {
      int64_t lo = t - window + 1;
      if (lo < 0) lo = 0;
      for (int64_t u = lo; u <= t; ++u) {
        int64_t r = u - swa_start[b];
        if (r < 0 || r >= S_w) continue;
        const uint8_t* row = swa + ((size_t)b * S_w + (size_t)r) * ORC_D;
        for (int c = 0; c < ORC_D; ++c) keys[(size_t)nk * ORC_D + c] = orc_e4m3_value(row[c]);
        ++nk;
      }
    }
#pragma omp parallel for schedule(dynamic, 1) if (!orc_in_parallel())
    for (int h = 0; h < H; ++h) {
      double* logit = (double*)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
      const float* qh = q + (bq * H + h) * ORC_D;
      double* oh = out + (bq * H + h) * ORC_D;
      if (nk == 0) {
        for (int c = 0; c < ORC_D; ++c) oh[c] = 0.0;
        lse[bq * H + h] = -HUGE_VAL;
        free(logit);
        continue;
      }
      double mx = -HUGE_VAL;
      for (int i = 0; i < nk; ++i) {
        double dot = 0.0;
        for (int c = 0; c < ORC_D; ++c) dot += (double)qh[c] * keys[(size_t)i * ORC_D + c];
        logit[i] = sm_scale * dot;
        if (logit[i] > mx) mx = logit[i];
      }
      double l = 0.0;
      for (int c = 0; c < ORC_D; ++c) oh[c] = 0.0;
      for (int i = 0; i < nk; ++i) {
        double p = exp(logit[i] - mx);
        l += p;
        for (int c = 0; c < ORC_D; ++c) oh[c] += p * keys[(size_t)i * ORC_D + c];
      }
      for (int c = 0; c < ORC_D; ++c) oh[c] /= l;
      lse[bq * H + h] = mx + log(l);
      free(logit);
    }
    free(keys);
  }
}

/* ------------------------------------------------------------------------------------
 * Context-parallel decode: the entries of one sequence split over C parts (P1 §무엇과
 * 다른가: a Full layer's Top-K is taken over everything the query sees; P3 §전역
 * 어텐션과 지역 어텐션: one softmax over the selected entries together with the window).
 * The pages describe a single device; splitting is this oracle's reading of how the same
 * results decompose, and each function below is the plain definition of one step.
 * ------------------------------------------------------------------------------------ */

/* Top-K of n labeled candidates: the order above (descending score, then ascending label)
 * over (scores[i], labels[i]); -1 fills the slots past n.  With every part's own Top-K as
 * the candidates, this is the Top-K of the union. */
void orc_topk_labeled(const double* scores, const int64_t* labels, int64_t n, int K, int32_t* idx_out,
                      double* score_out) {
  topk_labeled(scores, labels, n, K, idx_out, score_out);
}

/* Attention over the union of C disjoint key sets from each set's normalised output and
 * log-sum-exp of its logits: with M = max_c lse_c,
 *   lse = M + log(sum_c exp(lse_c - M)),   out = sum_c exp(lse_c - lse) * out_c.
 * A part with lse_c = -inf (no keys) contributes nothing; all parts empty gives out = 0,
 * lse = -inf.  out_parts [C][N][512], lse_parts [C][N]; out [N][512], lse [N]. */
void orc_attn_combine(const double* out_parts, const double* lse_parts, int C, int64_t N, double* out,
                      double* lse) {
  for (int64_t r = 0; r < N; ++r) {
    double mx = -HUGE_VAL;
    for (int c = 0; c < C; ++c)
      if (lse_parts[(int64_t)c * N + r] > mx) mx = lse_parts[(int64_t)c * N + r];
    double* o = out + r * ORC_D;
    for (int d = 0; d < ORC_D; ++d) o[d] = 0.0;
    if (mx == -HUGE_VAL) {
      lse[r] = -HUGE_VAL;
      continue;
    }
    double l = 0.0;
    for (int c = 0; c < C; ++c) {
      double wc = exp(lse_parts[(int64_t)c * N + r] - mx);
      l += wc;
      for (int d = 0; d < ORC_D; ++d) o[d] += wc * out_parts[((int64_t)c * N + r) * ORC_D + d];
    }
    for (int d = 0; d < ORC_D; ++d) o[d] /= l;
    lse[r] = mx + log(l);
  }
}
