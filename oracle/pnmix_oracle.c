/*
 * pnmix_oracle.c -- the reference oracle of the PN-Mix KV-cache path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is compiled and called by the tests, by
 * the smoke check and by the benchmark's CPU-baseline leg; the product (the
 * CUDA library and its Python binding) never loads it.  It is plain,
 * single-threaded C that states each definition directly, with no blocking,
 * fusion or reordering, so that it can be checked by eye.  It shares no code,
 * header or table with the CUDA library: the record layout is re-derived here
 * from its written definition.
 *
 * Precision.  Everything that decides a code, an index or a stored bit
 * (pair norms, scores, scales, zero points, codes) is IEEE binary32 with
 * round-to-nearest-even and one rounding per operation (build flags
 * -ffp-contract=off -fno-fast-math, SSE arithmetic).  Dequantized values and
 * attention are binary64.
 *
 * Sources of each definition:
 *  - Saliency from the query-key pair-norm product, chosen once at prefill and
 *    reused through decode: "PN-Mix: Pair-Norm Guided Mixed-Precision Key Cache
 *    Quantization for Efficient Long-Output LLM Inference", abstract, and the
 *    same page's transcript (the pairs whose query and key pair norms have a
 *    large product are the salient ones).  The exact statistic (mean query pair-norm over the
 *    last W prefill queries of the group, max key pair-norm over the prefill
 *    tokens), k, W and the half-split pairing are this library's fixed
 *    parameters.
 *  - Mixed-precision per-channel keys: PN-Mix abstract; MixKVQ abstract
 *    (precision chosen per key channel).
 *  - Per-token values: "MixKVQ: Query-Aware Mixed-Precision KV Cache
 *    Quantization for Long-Context Reasoning", abstract.
 *  - Asymmetric min-max quantizer with a float zero point (KIVI-style, as
 *    recorded in the PM-KVQ review page, "key_machinery"), fp16 scale and zero.
 *
 * Parity pins (tests/test_oracle_pins.py): closed-form top-k on Pythagorean
 * inputs with ties, outlier-union selection on the tiny workload, grid-exact
 * round trips, the s/2 round-trip bound, half-even ties, code-bit accounting,
 * fp16 rounding against numpy, layout bijection, append == bulk prefill, and
 * the 16-bit pass-through reducing to plain softmax attention; for the two-
 * precision mixing: exact means of identical rows, exact integer group scores,
 * the route against a stable sort, and the union of two equal-precision parts
 * against one cache; for query-channel pruning: the pruned pairs and the pruned
 * key slices against sorts of exact integer norms and energies, the channel-0 rule,
 * and pruned key channels that can hold anything without changing the output.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Number formats, from their IEEE-754 definitions.                    */
/* ------------------------------------------------------------------ */

/* bf16 bits -> binary32 (exact: bf16 is the top half of binary32). */
float orc_f32_from_bf16(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* binary16 bits -> binary32 (exact). */
float orc_f32_from_f16(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int m = h & 0x3FF;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + m), e - 25);     /* (1 + m/1024) * 2^(e-15) */
  return (float)(sign ? -v : v);
}

/*
 * binary32 -> binary16 bits, round to nearest, ties to even.  The value is
 * rounded to the quantum of its binade (2^(E-10) for a normal result with
 * exponent E, 2^-24 for a subnormal one); a magnitude that rounds to 2^16 or
 * more overflows to infinity.
 */
uint16_t orc_f16_from_f32(float f) {
  uint16_t sign = signbit(f) ? 0x8000u : 0u;
  double a = fabs((double)f);
  if (isnan(f)) return 0x7E00u;
  if (a == 0.0) return sign;
  int E;
  frexp(a, &E);                     /* a = fr * 2^E, 0.5 <= fr < 1, so binade exponent E-1 */
  int ex = E - 1;
  if (ex < -14) ex = -14;           /* subnormal range shares the quantum 2^-24 */
  double quantum = ldexp(1.0, ex - 10);
  double r = nearbyint(a / quantum) * quantum; /* a / quantum is exact */
  if (r >= 65536.0) return (uint16_t)(sign | 0x7C00u);
  /* encode r */
  if (r < ldexp(1.0, -14)) {
    int m = (int)(r / ldexp(1.0, -24));
    return (uint16_t)(sign | m);
  }
  int E2;
  double fr2 = frexp(r, &E2);       /* r = fr2 * 2^E2 */
  int exp_field = E2 - 1 + 15;
  int mant = (int)(fr2 * 2048.0) - 1024;
  return (uint16_t)(sign | (exp_field << 10) | mant);
}

/* ------------------------------------------------------------------ */
/* Step 1: pair saliency and top-k.                                    */
/* ------------------------------------------------------------------ */

/*
 * Scores of the 64 RoPE pairs of one KV head.
 *   qwin: bf16 [G][W][128] (the last W prefill queries of the group's heads)
 *   k:    bf16 [L][128]
 * K_p = sqrt(max_t (a*a + b*b)), (a, b) = (k[t][p], k[t][p+64]);
 * Q_p = (sum_h sum_t sqrt(a*a + b*b)) / (G*W), heads outer, tokens inner;
 * s_p = Q_p * K_p.  knorm / qnorm may be NULL.
 */
void orc_pair_scores(int G, int W, int L, const uint16_t* qwin, const uint16_t* k, float* scores,
                     float* knorm, float* qnorm) {
  for (int p = 0; p < 64; ++p) {
    float kmax2 = 0.0f;
    for (int t = 0; t < L; ++t) {
      float a = orc_f32_from_bf16(k[(size_t)t * 128 + p]);
      float b = orc_f32_from_bf16(k[(size_t)t * 128 + p + 64]);
      float aa = a * a;
      float bb = b * b;
      float n2 = aa + bb;
      if (n2 > kmax2) kmax2 = n2;
    }
    float kp = sqrtf(kmax2);
    float qsum = 0.0f;
    for (int h = 0; h < G; ++h) {
      for (int t = 0; t < W; ++t) {
        const uint16_t* row = qwin + ((size_t)h * W + t) * 128;
        float a = orc_f32_from_bf16(row[p]);
        float b = orc_f32_from_bf16(row[p + 64]);
        float aa = a * a;
        float bb = b * b;
        float n2 = aa + bb;
        qsum = qsum + sqrtf(n2);
      }
    }
    float qp = qsum / (float)(G * W);
    scores[p] = qp * kp;
    if (knorm) knorm[p] = kp;
    if (qnorm) qnorm[p] = qp;
  }
}

/*
 * Saliency scores under the three statistics the path supports (mode):
 *   0  PN-Mix: s_p = Q_p * K_p as in orc_pair_scores (query pair norm times key pair
 *      norm; PN-Mix abstract).
 *   1  key statistics only: s_p = K_p (the channel-saliency estimate of the earlier
 *      mixed-precision methods that the PN-Mix abstract contrasts with).
 *   2  quantization difficulty times query relevance (the MixKVQ abstract's two factors):
 *      D_p = sqrt(r_p*r_p + r_{p+64}*r_{p+64}) with r_c = max_t k[t][c] - min_t k[t][c],
 *      the pair norm of the two channels' ranges; s_p = Q_p * D_p.
 * Every operation is one fp32 rounding, in the order written.
 */
void orc_pair_scores_mode(int mode, int G, int W, int L, const uint16_t* qwin, const uint16_t* k,
                          float* scores) {
  float s0[64], kn[64], qn[64];
  orc_pair_scores(G, W, L, qwin, k, s0, kn, qn);
  for (int p = 0; p < 64; ++p) {
    if (mode == 0) {
      scores[p] = s0[p];
    } else if (mode == 1) {
      scores[p] = kn[p];
    } else {
      float r[2];
      for (int e = 0; e < 2; ++e) {
        const int c = p + 64 * e;
        float mn = orc_f32_from_bf16(k[c]), mx = mn;
        for (int t = 1; t < L; ++t) {
          const float x = orc_f32_from_bf16(k[(size_t)t * 128 + c]);
          if (x < mn) mn = x;
          if (x > mx) mx = x;
        }
        r[e] = mx - mn;
      }
      const float r0 = r[0] * r[0];
      const float r1 = r[1] * r[1];
      const float d = sqrtf(r0 + r1);
      scores[p] = qn[p] * d;
    }
  }
}

/*
 * The k pairs with the largest score; among equal scores the lower pair index
 * wins.  idx receives them in ascending pair order, mask has bit p set for
 * every chosen p.
 */
void orc_topk(const float* scores, int k, uint8_t* idx, uint64_t* mask) {
  int taken[64] = {0};
  uint64_t m = 0;
  for (int i = 0; i < k; ++i) {
    int best = -1;
    for (int p = 0; p < 64; ++p) {
      if (taken[p]) continue;
      if (best < 0 || scores[p] > scores[best]) best = p;
    }
    taken[best] = 1;
    m |= (uint64_t)1 << best;
  }
  int n = 0;
  for (int p = 0; p < 64; ++p)
    if (taken[p]) idx[n++] = (uint8_t)p;
  *mask = m;
}

/*
 * Position order of the 128 key channels: the channels of the salient pairs
 * {p, p+64} in ascending channel order, then every other channel ascending.
 * perm[j] = channel at position j.  Returns the number of salient channels.
 */
int orc_position_order(uint64_t mask, uint8_t* perm) {
  int n = 0;
  for (int c = 0; c < 128; ++c)
    if ((mask >> (c & 63)) & 1) perm[n++] = (uint8_t)c;
  int nhi = n;
  for (int c = 0; c < 128; ++c)
    if (!((mask >> (c & 63)) & 1)) perm[n++] = (uint8_t)c;
  return nhi;
}

/* ------------------------------------------------------------------ */
/* Step 2/3: the asymmetric min-max quantizer.                         */
/* ------------------------------------------------------------------ */

/*
 * Quantize n values to `bits`-bit codes.
 *   s16 = fp16((mx - mn) / (2^bits - 1)), z16 = fp16(mn),
 *   code = clamp(rint((x - z) / s), 0, 2^bits - 1) with s, z the fp32 values
 *   of s16, z16; all codes are 0 when s16 is zero.
 */
void orc_minmax_quant(const float* x, int n, int bits, uint16_t* s16, uint16_t* z16,
                      uint8_t* codes) {
  float mn = x[0], mx = x[0];
  for (int i = 1; i < n; ++i) {
    if (x[i] < mn) mn = x[i];
    if (x[i] > mx) mx = x[i];
  }
  float levels = (float)((1 << bits) - 1);
  float range = mx - mn;
  float s32 = range / levels;
  uint16_t sh = orc_f16_from_f32(s32);
  uint16_t zh = orc_f16_from_f32(mn);
  float s = orc_f32_from_f16(sh);
  float z = orc_f32_from_f16(zh);
  for (int i = 0; i < n; ++i) {
    int code = 0;
    if (s != 0.0f) {
      float d = x[i] - z;
      float qv = d / s;
      float r = rintf(qv);
      if (r < 0.0f) r = 0.0f;
      if (r > levels) r = levels;
      code = (int)r;
    }
    codes[i] = (uint8_t)code;
  }
  *s16 = sh;
  *z16 = zh;
}

/*
 * Keys of one 32-token group: every position j quantizes channel perm[j] over
 * the 32 tokens, with b_hi bits for j < nhi and b_lo bits otherwise.
 *   rows: bf16 [32][128] (natural channel order)
 *   codes: [32 tokens][128 positions]; s16, z16: [128 positions]
 * bits 16 is the pass-through setting: nothing is stored (used only by the
 * exact-attention check, see orc_attend_unit).
 */
void orc_key_group(const uint16_t* rows, const uint8_t* perm, int nhi, int bhi, int blo,
                   uint8_t* codes, uint16_t* s16, uint16_t* z16) {
  for (int j = 0; j < 128; ++j) {
    float x[32];
    uint8_t c[32];
    int bits = j < nhi ? bhi : blo;
    for (int t = 0; t < 32; ++t) x[t] = orc_f32_from_bf16(rows[t * 128 + perm[j]]);
    orc_minmax_quant(x, 32, bits, &s16[j], &z16[j], c);
    for (int t = 0; t < 32; ++t) codes[t * 128 + j] = c[t];
  }
}

/* Values of one token: four 32-channel groups of `bits`-bit codes. */
void orc_value_token(const uint16_t* row, int bits, uint8_t* codes, uint16_t* s16,
                     uint16_t* z16) {
  for (int jg = 0; jg < 4; ++jg) {
    float x[32];
    for (int i = 0; i < 32; ++i) x[i] = orc_f32_from_bf16(row[32 * jg + i]);
    orc_minmax_quant(x, 32, bits, &s16[jg], &z16[jg], codes + 32 * jg);
  }
}

/* ------------------------------------------------------------------ */
/* The group record layout.                                             */
/* ------------------------------------------------------------------ */

/* Words per lane of the hi and lo key blocks; -1 if not whole. */
static int orc_block_words(int nslices, int bits) {
  if ((nslices * bits) % 2) return -1;
  return nslices * bits / 2;
}

/* Bytes of one record, 0 if the parameters do not give whole words. */
long orc_record_bytes(int k, int bhi, int blo) {
  if (k < 0 || k > 64 || (2 * k) % 16) return 0;
  int nhs = 2 * k / 16;
  int wh = orc_block_words(nhs, bhi), wl = orc_block_words(8 - nhs, blo);
  if (wh < 0 || wl < 0) return 0;
  return 128L * (wh + wl) + 2048L;
}

static void put32(uint8_t* p, uint32_t v) {
  p[0] = (uint8_t)v;
  p[1] = (uint8_t)(v >> 8);
  p[2] = (uint8_t)(v >> 16);
  p[3] = (uint8_t)(v >> 24);
}
static uint32_t get32(const uint8_t* p) {
  return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
static void put16(uint8_t* p, uint16_t v) {
  p[0] = (uint8_t)v;
  p[1] = (uint8_t)(v >> 8);
}
static uint16_t get16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* fp16 element index of key position j in the scale (and zero) array: the 16 bytes of
   (tq, slice pair) hold the pairs (even slice e=0, odd slice e=0, even slice e=1, odd
   slice e=1). */
static int orc_kscale_index(int j) {
  int sigma = j / 16, e = (j % 16) / 8, tq = (j % 8) / 2, v = j % 2;
  return ((tq * 4 + sigma / 2) * 4 + 2 * e + sigma % 2) * 2 + v;
}

/* fp16 element index of the value scale of (token t, channel group jg). */
static int orc_vscale_index(int t, int jg) { return ((t / 2) * 4 + jg) * 2 + (t % 2); }

/* fp16 element index of the value zero point of (token t, channel group jg): token pair
   tp = t/2 sits in the 16 bytes of (tp mod 4, jg), which hold tp, tp+8, tp+4, tp+12. */
static int orc_vzero_index(int t, int jg) {
  int tp = t / 2;
  return (((tp % 4) * 4 + jg) * 4 + tp / 8 + 2 * ((tp / 4) % 2)) * 2 + (t % 2);
}

/* Byte offset of the key-code word w (lane-local) of lane L. */
static long orc_kword_offset(int w, int L) { return ((long)w * 32 + L) * 4; }

/* Byte offset of value-code word m of lane L. */
static long orc_vword_offset(int m, int L) { return ((long)(m >> 2) * 32 + L) * 16 + (m & 3) * 4; }

/*
 * Location of the key code of (token tau, position j): lane-local word index w,
 * lane L and bit.  Derived from the slot definition: position j lies in slice
 * sigma = j/16 with j = 16*sigma + 2*tq + 8*c + half; token tau = gq + 8*u.
 */
static void orc_key_code_loc(int tau, int j, int nhs, int bhi, int blo, int* w, int* L, int* bit,
                             int* bits) {
  int sigma = j / 16, rem = j % 16;
  int c = rem / 8, tq = (rem % 8) / 2, half = rem % 2;
  int gq = tau % 8, u = tau / 8;
  int hi = sigma < nhs;
  int b = hi ? bhi : blo;
  int m = 16 / b;
  int n = ((hi ? sigma : sigma - nhs) * 8) + c * 4 + u;
  int base = hi ? 0 : orc_block_words(nhs, bhi);
  *w = base + n / m;
  *L = gq * 4 + tq;
  *bit = 16 * half + b * (n % m);
  *bits = b;
}

/* Location of the value code of (token t, channel ch). */
static void orc_value_code_loc(int t, int ch, int* m, int* L, int* bit) {
  int tq = (t % 8) / 2, p = t / 8, second = t % 2;
  int mm = ch / 16, rem = ch % 16;
  int r = rem / 8, gq = rem % 8;
  int q = r * 4 + p;
  *m = mm;
  *L = gq * 4 + tq;
  *bit = 16 * second + 2 * q;
}

/*
 * Pack one record.
 *   kcodes [32][128 positions], ks/kz [128 positions] (fp16 bits),
 *   vcodes [32][128 channels], vs/vz [32 tokens][4 groups] (fp16 bits).
 */
int orc_pack_record(int k, int bhi, int blo, const uint8_t* kcodes, const uint16_t* ks,
                    const uint16_t* kz, const uint8_t* vcodes, const uint16_t* vs,
                    const uint16_t* vz, uint8_t* rec) {
  long R = orc_record_bytes(k, bhi, blo);
  if (!R) return 1;
  memset(rec, 0, (size_t)R);
  int nhs = 2 * k / 16;
  long KC = R - 2048;
  for (int tau = 0; tau < 32; ++tau) {
    for (int j = 0; j < 128; ++j) {
      int w, L, bit, bits;
      orc_key_code_loc(tau, j, nhs, bhi, blo, &w, &L, &bit, &bits);
      uint8_t* p = rec + orc_kword_offset(w, L);
      uint32_t code = kcodes[tau * 128 + j] & ((1u << bits) - 1u);
      put32(p, get32(p) | (code << bit));
    }
  }
  for (int j = 0; j < 128; ++j) {
    put16(rec + KC + 2 * orc_kscale_index(j), ks[j]);
    put16(rec + KC + 256 + 2 * orc_kscale_index(j), kz[j]);
  }
  uint8_t* vc = rec + KC + 512;
  for (int t = 0; t < 32; ++t) {
    for (int ch = 0; ch < 128; ++ch) {
      int m, L, bit;
      orc_value_code_loc(t, ch, &m, &L, &bit);
      uint8_t* p = vc + orc_vword_offset(m, L);
      put32(p, get32(p) | ((uint32_t)(vcodes[t * 128 + ch] & 3u) << bit));
    }
  }
  uint8_t* vsb = rec + KC + 1536;
  for (int t = 0; t < 32; ++t) {
    for (int jg = 0; jg < 4; ++jg) {
      put16(vsb + 2 * orc_vscale_index(t, jg), vs[t * 4 + jg]);
      put16(vsb + 256 + 2 * orc_vzero_index(t, jg), vz[t * 4 + jg]);
    }
  }
  return 0;
}

/* Inverse of orc_pack_record. */
int orc_unpack_record(int k, int bhi, int blo, const uint8_t* rec, uint8_t* kcodes, uint16_t* ks,
                      uint16_t* kz, uint8_t* vcodes, uint16_t* vs, uint16_t* vz) {
  long R = orc_record_bytes(k, bhi, blo);
  if (!R) return 1;
  int nhs = 2 * k / 16;
  long KC = R - 2048;
  for (int tau = 0; tau < 32; ++tau) {
    for (int j = 0; j < 128; ++j) {
      int w, L, bit, bits;
      orc_key_code_loc(tau, j, nhs, bhi, blo, &w, &L, &bit, &bits);
      uint32_t word = get32(rec + orc_kword_offset(w, L));
      kcodes[tau * 128 + j] = (uint8_t)((word >> bit) & ((1u << bits) - 1u));
    }
  }
  for (int j = 0; j < 128; ++j) {
    ks[j] = get16(rec + KC + 2 * orc_kscale_index(j));
    kz[j] = get16(rec + KC + 256 + 2 * orc_kscale_index(j));
  }
  const uint8_t* vc = rec + KC + 512;
  for (int t = 0; t < 32; ++t) {
    for (int ch = 0; ch < 128; ++ch) {
      int m, L, bit;
      orc_value_code_loc(t, ch, &m, &L, &bit);
      uint32_t word = get32(vc + orc_vword_offset(m, L));
      vcodes[t * 128 + ch] = (uint8_t)((word >> bit) & 3u);
    }
  }
  const uint8_t* vsb = rec + KC + 1536;
  for (int t = 0; t < 32; ++t) {
    for (int jg = 0; jg < 4; ++jg) {
      vs[t * 4 + jg] = get16(vsb + 2 * orc_vscale_index(t, jg));
      vz[t * 4 + jg] = get16(vsb + 256 + 2 * orc_vzero_index(t, jg));
    }
  }
  return 0;
}

/*
 * Equivalent right shift (PM-KVQ review page, the bit-width shrinking step of its
 * progressive quantization): a 2b-bit code X becomes the b-bit code
 *   X_b = ((2^(2b) - 2^b + 1) * (X + 2^(b-1))) >> 3b,
 * the integer form of round(X / (2^b + 1)), with the scale multiplied by 2^b + 1 and the
 * zero point kept.
 */
uint32_t orc_ers(uint32_t x, int b) {
  const uint32_t mul = (1u << (2 * b)) - (1u << b) + 1u;
  return (mul * (x + (1u << (b - 1)))) >> (3 * b);
}

/*
 * Shrink one record of the (bhi, blo, k) layout to the (bhi, blo, 0) layout (every
 * position at blo = bhi / 2 bits, same position order): the codes of the salient
 * positions [0, 2k) go through orc_ers with b = blo and their scale becomes
 * fp16(fl(s * (2^blo + 1))); every other byte is carried over.
 */
int orc_shrink_record(int k, int bhi, int blo, const uint8_t* src, uint8_t* dst) {
  if (bhi != 2 * blo) return 1;
  uint8_t kcodes[32 * 128], vcodes[32 * 128];
  uint16_t ks[128], kz[128], vs[32 * 4], vz[32 * 4];
  if (orc_unpack_record(k, bhi, blo, src, kcodes, ks, kz, vcodes, vs, vz)) return 1;
  const int nhi = 2 * k;
  const float mul = (float)((1 << blo) + 1);
  for (int j = 0; j < nhi; ++j) {
    for (int t = 0; t < 32; ++t) kcodes[t * 128 + j] = (uint8_t)orc_ers(kcodes[t * 128 + j], blo);
    const float s = orc_f32_from_f16(ks[j]) * mul;
    ks[j] = orc_f16_from_f32(s);
  }
  return orc_pack_record(0, bhi, blo, kcodes, ks, kz, vcodes, vs, vz, dst);
}

/* Quantize 32 K rows and 32 V rows (bf16 [32][128] each) into one record. */
int orc_make_record(int k, int bhi, int blo, int bv, const uint8_t* perm, const uint16_t* krows,
                    const uint16_t* vrows, uint8_t* rec) {
  uint8_t kcodes[32 * 128], vcodes[32 * 128];
  uint16_t ks[128], kz[128], vs[32 * 4], vz[32 * 4];
  orc_key_group(krows, perm, 2 * k, bhi, blo, kcodes, ks, kz);
  for (int t = 0; t < 32; ++t)
    orc_value_token(vrows + t * 128, bv, vcodes + t * 128, vs + t * 4, vz + t * 4);
  return orc_pack_record(k, bhi, blo, kcodes, ks, kz, vcodes, vs, vz, rec);
}

/* ------------------------------------------------------------------ */
/* Prefill and append of one (sequence, KV head).                      */
/* ------------------------------------------------------------------ */

/*
 * Prefill of one (b, h): tokens [0, 32*floor(L/32)) become records 0..,
 * the last L % 32 rows go to residual slots (token % 32).
 *   k, v: bf16 [L][128]; records: [>= L/32][R]; resid_k, resid_v: [32][128].
 */
int orc_prefill_unit(int k, int bhi, int blo, int bv, const uint8_t* perm, int L,
                     const uint16_t* kin, const uint16_t* vin, uint8_t* records,
                     uint16_t* resid_k, uint16_t* resid_v) {
  long R = orc_record_bytes(k, bhi, blo);
  if (!R) return 1;
  int ng = L / 32;
  for (int g = 0; g < ng; ++g) {
    int rc = orc_make_record(k, bhi, blo, bv, perm, kin + (size_t)g * 32 * 128,
                             vin + (size_t)g * 32 * 128, records + (size_t)g * R);
    if (rc) return rc;
  }
  for (int t = ng * 32; t < L; ++t) {
    memcpy(resid_k + (t % 32) * 128, kin + (size_t)t * 128, 256);
    memcpy(resid_v + (t % 32) * 128, vin + (size_t)t * 128, 256);
  }
  return 0;
}

/*
 * Append one token to one (b, h) holding `len` tokens: the row goes to
 * residual slot len % 32; when that is slot 31 the 32 residual rows become
 * record len / 32.  Returns the new length.
 */
int orc_append_unit(int k, int bhi, int blo, int bv, const uint8_t* perm, int len,
                    const uint16_t* knew, const uint16_t* vnew, uint8_t* records,
                    uint16_t* resid_k, uint16_t* resid_v) {
  long R = orc_record_bytes(k, bhi, blo);
  int slot = len % 32;
  memcpy(resid_k + slot * 128, knew, 256);
  memcpy(resid_v + slot * 128, vnew, 256);
  if (slot == 31)
    orc_make_record(k, bhi, blo, bv, perm, resid_k, resid_v, records + (size_t)(len / 32) * R);
  return len + 1;
}

/* ------------------------------------------------------------------ */
/* Attention.                                                           */
/* ------------------------------------------------------------------ */

/* Dequantized K and V rows (binary64, natural channel order) of one record. */
static void orc_dequant_record(int k, int bhi, int blo, const uint8_t* perm, const uint8_t* rec,
                               double* khat, double* vhat) {
  uint8_t kc[32 * 128], vc[32 * 128];
  uint16_t ks[128], kz[128], vs[128], vz[128];
  orc_unpack_record(k, bhi, blo, rec, kc, ks, kz, vc, vs, vz);
  for (int t = 0; t < 32; ++t) {
    for (int j = 0; j < 128; ++j)
      khat[t * 128 + perm[j]] =
          (double)kc[t * 128 + j] * (double)orc_f32_from_f16(ks[j]) + (double)orc_f32_from_f16(kz[j]);
    for (int c = 0; c < 128; ++c)
      vhat[t * 128 + c] = (double)vc[t * 128 + c] * (double)orc_f32_from_f16(vs[t * 4 + c / 32]) +
                          (double)orc_f32_from_f16(vz[t * 4 + c / 32]);
  }
}

/*
 * Softmax attention of G query rows over n dequantized tokens:
 *   out[h] = sum_t exp(l_t - max l) v_t / sum_t exp(l_t - max l),
 *   l_t = scale * sum_c q[h][c] * khat[t][c].
 * khat, vhat: binary64 [n][128]; q: binary64 [G][128]; out: [G][128].
 * With n == 0 the output is 0.
 */
void orc_attention_core(int G, const double* q, const double* khat, const double* vhat, long n,
                        double scale, double* out) {
  for (int h = 0; h < G; ++h) {
    double* o = out + (size_t)h * 128;
    for (int c = 0; c < 128; ++c) o[c] = 0.0;
    if (n == 0) continue;
    double* logit = (double*)malloc(sizeof(double) * (size_t)n);
    double mx = -INFINITY;
    for (long t = 0; t < n; ++t) {
      double acc = 0.0;
      for (int c = 0; c < 128; ++c) acc += q[h * 128 + c] * khat[t * 128 + c];
      logit[t] = acc * scale;
      if (logit[t] > mx) mx = logit[t];
    }
    double den = 0.0;
    for (long t = 0; t < n; ++t) {
      double w = exp(logit[t] - mx);
      den += w;
      for (int c = 0; c < 128; ++c) o[c] += w * vhat[t * 128 + c];
    }
    for (int c = 0; c < 128; ++c) o[c] /= den;
    free(logit);
  }
}

/*
 * Decode attention of one (b, KV head): the G query rows q (bf16 [G][128])
 * attend over the n_groups records and the n_resid residual rows.
 * bhi == 16 selects the pass-through setting: records are ignored and
 * k_pass / v_pass (bf16 [n_groups*32][128]) are used as the dequantized keys
 * and values, so the result is plain softmax attention over bf16 K and V.
 */
int orc_attend_unit(int G, const uint16_t* q, double scale, int k, int bhi, int blo,
                    const uint8_t* perm, const uint8_t* records, int n_groups,
                    const uint16_t* resid_k, const uint16_t* resid_v, int n_resid,
                    const uint16_t* k_pass, const uint16_t* v_pass, double* out) {
  long R = bhi == 16 ? 0 : orc_record_bytes(k, bhi, blo);
  if (bhi != 16 && !R) return 1;
  long n = (long)n_groups * 32 + n_resid;
  double* khat = (double*)malloc(sizeof(double) * 128 * (size_t)(n > 0 ? n : 1));
  double* vhat = (double*)malloc(sizeof(double) * 128 * (size_t)(n > 0 ? n : 1));
  double qd[8 * 128];
  if (!khat || !vhat || G > 8) {
    free(khat);
    free(vhat);
    return 2;
  }
  for (int i = 0; i < G * 128; ++i) qd[i] = (double)orc_f32_from_bf16(q[i]);
  for (int g = 0; g < n_groups; ++g) {
    if (bhi == 16) {
      for (int i = 0; i < 32 * 128; ++i) {
        khat[(size_t)g * 4096 + i] = (double)orc_f32_from_bf16(k_pass[(size_t)g * 4096 + i]);
        vhat[(size_t)g * 4096 + i] = (double)orc_f32_from_bf16(v_pass[(size_t)g * 4096 + i]);
      }
    } else {
      orc_dequant_record(k, bhi, blo, perm, records + (size_t)g * R, khat + (size_t)g * 4096,
                         vhat + (size_t)g * 4096);
    }
  }
  for (int r = 0; r < n_resid; ++r) {
    long t = (long)n_groups * 32 + r;
    for (int c = 0; c < 128; ++c) {
      khat[t * 128 + c] = (double)orc_f32_from_bf16(resid_k[r * 128 + c]);
      vhat[t * 128 + c] = (double)orc_f32_from_bf16(resid_v[r * 128 + c]);
    }
  }
  orc_attention_core(G, qd, khat, vhat, n, scale, out);
  free(khat);
  free(vhat);
  return 0;
}

/*
 * Several query rows per (b, KV head), each over its own prefix of the cache: row r
 * (bf16 q[r][128]) attends over the first n_visible[r] of the n_groups*32 + n_resid
 * tokens (the cache dequantized as in orc_attend_unit).  A verify or chunked decode step
 * appends T new tokens first; its query j then sees len - T + 1 + j tokens (causal among
 * the new ones).  A row that sees no token gets zeros.
 */
int orc_attend_unit_rows(int rows, const uint16_t* q, double scale, int k, int bhi, int blo,
                         const uint8_t* perm, const uint8_t* records, int n_groups,
                         const uint16_t* resid_k, const uint16_t* resid_v, int n_resid,
                         const int* n_visible, double* out) {
  long R = orc_record_bytes(k, bhi, blo);
  if (!R) return 1;
  long n = (long)n_groups * 32 + n_resid;
  double* khat = (double*)malloc(sizeof(double) * 128 * (size_t)(n > 0 ? n : 1));
  double* vhat = (double*)malloc(sizeof(double) * 128 * (size_t)(n > 0 ? n : 1));
  if (!khat || !vhat) {
    free(khat);
    free(vhat);
    return 2;
  }
  for (int g = 0; g < n_groups; ++g)
    orc_dequant_record(k, bhi, blo, perm, records + (size_t)g * R, khat + (size_t)g * 4096,
                       vhat + (size_t)g * 4096);
  for (int r = 0; r < n_resid; ++r) {
    long t = (long)n_groups * 32 + r;
    for (int c = 0; c < 128; ++c) {
      khat[t * 128 + c] = (double)orc_f32_from_bf16(resid_k[r * 128 + c]);
      vhat[t * 128 + c] = (double)orc_f32_from_bf16(resid_v[r * 128 + c]);
    }
  }
  for (int r = 0; r < rows; ++r) {
    double qd[128];
    for (int c = 0; c < 128; ++c) qd[c] = (double)orc_f32_from_bf16(q[r * 128 + c]);
    long nv = n_visible[r] < 0 ? 0 : (n_visible[r] > n ? n : n_visible[r]);
    if (nv == 0) {
      for (int c = 0; c < 128; ++c) out[r * 128 + c] = 0.0;
      continue;
    }
    orc_attention_core(1, qd, khat, vhat, nv, scale, out + (size_t)r * 128);
  }
  free(khat);
  free(vhat);
  return 0;
}

/*
 * Dynamic query-channel pruning (the Dual-QK abstract's query-channel pruning, at the
 * RoPE-pair level of PN-Mix): for one query row q (bf16 [128]) the n_prune pairs with
 * the smallest squared pair norm n2_p = fl(fl(a*a) + fl(b*b)), (a, b) = (q[p], q[p+64]),
 * are pruned, pair 0 never (the abstract's channel-0 protection); among equal norms the
 * higher pair index is pruned first.  Returns the mask of pruned pairs.
 */
uint64_t orc_pruned_pairs(const uint16_t* q, int n_prune) {
  float n2[64];
  for (int p = 0; p < 64; ++p) {
    const float a = orc_f32_from_bf16(q[p]);
    const float b = orc_f32_from_bf16(q[p + 64]);
    const float aa = a * a;
    const float bb = b * b;
    n2[p] = aa + bb;
  }
  uint64_t mask = 0;
  for (int i = 0; i < n_prune && i < 63; ++i) {
    int best = -1;
    for (int p = 63; p >= 1; --p) {   /* scan high to low: ties keep the higher p */
      if ((mask >> p) & 1ull) continue;
      if (best < 0 || n2[p] < n2[best]) best = p;
    }
    mask |= 1ull << best;
  }
  return mask;
}

/* Copy of the query rows q (bf16 [rows][128]) with the channels of the pairs each row
 * prunes (orc_pruned_pairs) set to zero: attention with that copy drops exactly their
 * contributions, q_c * k_c = 0 for every token. */
void orc_prune_queries(int rows, const uint16_t* q, int n_prune, uint16_t* out) {
  for (int r = 0; r < rows; ++r) {
    const uint64_t mask = orc_pruned_pairs(q + (size_t)r * 128, n_prune);
    for (int c = 0; c < 128; ++c)
      out[(size_t)r * 128 + c] = ((mask >> (c & 63)) & 1ull) ? 0 : q[(size_t)r * 128 + c];
  }
}

/*
 * Key-slice pruning (the Dual-QK abstract's query-channel pruning, taken at the
 * granularity the packed record reads keys in, so that a pruned block of channels is a
 * block of key codes left unread).  The unit is one (sequence, KV head) and all `rows`
 * query rows that attend it (bf16 [rows][128]): they read the same key codes, so they
 * share one decision.  Candidates are the position slices of the low-precision block
 * (sigma in [2k/16, 8), positions 16*sigma .. 16*sigma+15 of the order perm) that hold
 * neither channel 0 nor channel 64 (the abstract's channel-0 protection, kept for the
 * RoPE pair 0).  The energy of a slice is
 *     E_sigma = sum over rows v (ascending) of e_{sigma,v},
 *     e_{sigma,v} = sum over its 16 positions j (ascending) of q_v[perm[j]]^2,
 * every square and every partial sum rounded to fp32.  The n_prune candidates of least
 * energy are pruned (all candidates when there are fewer), the higher slice first among
 * equal energies.  Returns the mask of pruned slices (bit sigma).
 */
uint32_t orc_pruned_slices(int rows, const uint16_t* q, const uint8_t* perm, int k, int n_prune) {
  const int nhs = 2 * k / 16;
  float E[8];
  int cand[8];
  for (int sigma = 0; sigma < 8; ++sigma) {
    E[sigma] = 0.0f;
    cand[sigma] = sigma >= nhs;
    for (int j = 16 * sigma; j < 16 * sigma + 16; ++j)
      if ((perm[j] & 63) == 0) cand[sigma] = 0;
    if (!cand[sigma]) continue;
    for (int v = 0; v < rows; ++v) {
      float e = 0.0f;
      for (int j = 16 * sigma; j < 16 * sigma + 16; ++j) {
        const float x = orc_f32_from_bf16(q[(size_t)v * 128 + perm[j]]);
        const float sq = x * x;
        e = e + sq;
      }
      E[sigma] = E[sigma] + e;
    }
  }
  uint32_t mask = 0;
  for (int i = 0; i < n_prune; ++i) {
    int best = -1;
    for (int sigma = 7; sigma >= 0; --sigma) {   /* high to low: ties keep the higher slice */
      if (!cand[sigma] || ((mask >> sigma) & 1u)) continue;
      if (best < 0 || E[sigma] < E[best]) best = sigma;
    }
    if (best < 0) break;
    mask |= 1u << best;
  }
  return mask;
}

/* Copy of the unit's query rows with the channels of its pruned slices
 * (orc_pruned_slices) set to zero in every row. */
void orc_prune_query_slices(int rows, const uint16_t* q, const uint8_t* perm, int k, int n_prune,
                            uint16_t* out) {
  const uint32_t mask = orc_pruned_slices(rows, q, perm, k, n_prune);
  int pruned[128] = {0};
  for (int j = 0; j < 128; ++j)
    if ((mask >> (j / 16)) & 1u) pruned[perm[j]] = 1;
  for (int v = 0; v < rows; ++v)
    for (int c = 0; c < 128; ++c)
      out[(size_t)v * 128 + c] = pruned[c] ? 0 : q[(size_t)v * 128 + c];
}

/* Plain softmax attention over unquantized bf16 K and V ([n][128]). */
void orc_exact_attention(int G, const uint16_t* q, const uint16_t* kin, const uint16_t* vin,
                         long n, double scale, double* out) {
  double* khat = (double*)malloc(sizeof(double) * 128 * (size_t)(n > 0 ? n : 1));
  double* vhat = (double*)malloc(sizeof(double) * 128 * (size_t)(n > 0 ? n : 1));
  double qd[8 * 128];
  for (int i = 0; i < G * 128; ++i) qd[i] = (double)orc_f32_from_bf16(q[i]);
  for (long i = 0; i < n * 128; ++i) {
    khat[i] = (double)orc_f32_from_bf16(kin[i]);
    vhat[i] = (double)orc_f32_from_bf16(vin[i]);
  }
  orc_attention_core(G, qd, khat, vhat, n, scale, out);
  free(khat);
  free(vhat);
}

/* Average stored key code bits per value implied by the record layout. */
double orc_key_code_bits(int k, int bhi, int blo) {
  long R = orc_record_bytes(k, bhi, blo);
  if (!R) return 0.0;
  return (double)(R - 2048) * 8.0 / (32.0 * 128.0);
}

/* ------------------------------------------------------------------ */
/* Token-level two-precision mixing (SemKV).                           */
/* ------------------------------------------------------------------ */
/*
 * "SemKV: Semantic Mixed-Precision KV Cache Quantization Guided by the Quality Cliff for
 * Long-Context LLM Inference", abstract: every token is kept, tokens are ranked by a
 * model-internal score, and two adjacent precisions are assigned by rank.  In this path
 * the unit of assignment is a 32-token group (its tokens share the per-channel key
 * statistics), the two precisions are two salient-pair counts k_hi > k_lo of the same bit
 * pair, and the score of a group is the largest logit that the mean query of the saliency
 * window gives one of its tokens.
 */

/*
 * Mean query of one KV head's saliency window: qbar[c] = (sum_h sum_t q[h][t][c]) / (G*W),
 * heads outer, tokens inner, one fp32 rounding per operation.  qwin: bf16 [G][W][128].
 */
void orc_mean_query(int G, int W, const uint16_t* qwin, float* qbar) {
  for (int c = 0; c < 128; ++c) {
    float s = 0.0f;
    for (int h = 0; h < G; ++h)
      for (int t = 0; t < W; ++t) s = s + orc_f32_from_bf16(qwin[((size_t)h * W + t) * 128 + c]);
    qbar[c] = s / (float)(G * W);
  }
}

/*
 * Group scores of the L / 32 full groups of k (bf16 [L][128]):
 *   l_t = sum_c qbar[c] * k[t][c], channels 0..127 in order, one fp32 rounding per
 *         product and per sum;
 *   score[g] = max over t in [32g, 32g + 32) of l_t.
 */
void orc_group_scores(const float* qbar, int L, const uint16_t* k, float* score) {
  for (int g = 0; g < L / 32; ++g) {
    float best = -INFINITY;
    for (int t = 32 * g; t < 32 * g + 32; ++t) {
      float acc = 0.0f;
      for (int c = 0; c < 128; ++c) {
        float p = qbar[c] * orc_f32_from_bf16(k[(size_t)t * 128 + c]);
        acc = acc + p;
      }
      if (acc > best) best = acc;
    }
    score[g] = best;
  }
}

/*
 * Route of ng groups: group g ranks r_g = #{g' : score[g'] > score[g], or equal with
 * g' < g}; it takes the high precision (route[g] = 1) when r_g < n_hi, else 0.
 */
void orc_route_groups(int ng, const float* score, int n_hi, uint8_t* route) {
  for (int g = 0; g < ng; ++g) {
    int r = 0;
    for (int o = 0; o < ng; ++o)
      if (score[o] > score[g] || (score[o] == score[g] && o < g)) ++r;
    route[g] = (uint8_t)(r < n_hi);
  }
}

/*
 * Decode attention of one (b, KV head) over a two-precision cache: the G query rows q
 * (bf16 [G][128]) attend over the union of the n_hi records of the high-precision part
 * (k_hi salient pairs, permutation perm_hi), the n_lo records of the low-precision part
 * (k_lo, perm_lo) and the n_resid bf16 residual rows: plain softmax attention over all
 * of these tokens (its value does not depend on their order).
 */
int orc_attend_two(int G, const uint16_t* q, double scale, int bhi, int blo, int k_hi,
                   const uint8_t* perm_hi, const uint8_t* rec_hi, int n_hi, int k_lo,
                   const uint8_t* perm_lo, const uint8_t* rec_lo, int n_lo,
                   const uint16_t* resid_k, const uint16_t* resid_v, int n_resid, double* out) {
  long Rh = orc_record_bytes(k_hi, bhi, blo), Rl = orc_record_bytes(k_lo, bhi, blo);
  if (!Rh || !Rl || G > 8) return 1;
  long n = (long)(n_hi + n_lo) * 32 + n_resid;
  double* khat = (double*)malloc(sizeof(double) * 128 * (size_t)(n > 0 ? n : 1));
  double* vhat = (double*)malloc(sizeof(double) * 128 * (size_t)(n > 0 ? n : 1));
  double qd[8 * 128];
  if (!khat || !vhat) {
    free(khat);
    free(vhat);
    return 2;
  }
  for (int i = 0; i < G * 128; ++i) qd[i] = (double)orc_f32_from_bf16(q[i]);
  for (int g = 0; g < n_hi; ++g)
    orc_dequant_record(k_hi, bhi, blo, perm_hi, rec_hi + (size_t)g * Rh, khat + (size_t)g * 4096,
                       vhat + (size_t)g * 4096);
  for (int g = 0; g < n_lo; ++g)
    orc_dequant_record(k_lo, bhi, blo, perm_lo, rec_lo + (size_t)g * Rl,
                       khat + (size_t)(n_hi + g) * 4096, vhat + (size_t)(n_hi + g) * 4096);
  for (int r = 0; r < n_resid; ++r) {
    long t = (long)(n_hi + n_lo) * 32 + r;
    for (int c = 0; c < 128; ++c) {
      khat[t * 128 + c] = (double)orc_f32_from_bf16(resid_k[r * 128 + c]);
      vhat[t * 128 + c] = (double)orc_f32_from_bf16(resid_v[r * 128 + c]);
    }
  }
  orc_attention_core(G, qd, khat, vhat, n, scale, out);
  free(khat);
  free(vhat);
  return 0;
}
