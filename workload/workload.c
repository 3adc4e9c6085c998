/*
 * workload.c -- seeded synthetic Q/K/V rows for the PN-Mix KV-cache path.
 *
 * This module only makes inputs.  It holds none of the method's arithmetic
 * (no norms, scores, quantizers or attention); the CUDA library and the CPU
 * oracle both read the bytes it writes.
 *
 * Recipe (the synthetic stand-in for the RoPE decoder layers the PN-Mix
 * abstract evaluates on):
 *   - every element is N(0,1), drawn by Box-Muller from a counter-based
 *     SplitMix64 stream (Steele, Lea and Flood, "Fast splittable pseudorandom
 *     number generators", OOPSLA 2014; the 64-bit finaliser constants of that
 *     generator), keyed by (seed, tensor, batch row, head, token);
 *   - per (batch row, KV head) four key channel pairs are scaled by key_scale
 *     and four independently drawn query pairs by query_scale (both channels of
 *     each pair, every query head of the group), before RoPE;
 *   - Q and K are then rotated by half-split RoPE at their true positions
 *     (pair i = channels (i, i+64), frequency theta^(-i/64));
 *   - V has no outliers and no RoPE;
 *   - each value is rounded once from double to bf16, round-to-nearest-even.
 * Draw i of a row uses the two 64-bit outputs 2i and 2i+1 of the row's stream;
 * its cosine branch goes to channel i and its sine branch to channel i+64.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define WL_GOLDEN 0x9E3779B97F4A7C15ULL

enum { WL_Q = 0, WL_K = 1, WL_V = 2, WL_KOUT = 3, WL_QOUT = 4 };

static uint64_t wl_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Stream key of one row: a chain of SplitMix64 finalisations. */
uint64_t wl_row_key(uint64_t seed, int tensor, int b, int head, int64_t t) {
  uint64_t h = wl_mix64(seed + WL_GOLDEN * (uint64_t)(tensor + 1));
  h = wl_mix64(h + WL_GOLDEN * (uint64_t)(b + 1));
  h = wl_mix64(h + WL_GOLDEN * (uint64_t)(head + 1));
  h = wl_mix64(h + WL_GOLDEN * (uint64_t)(t + 1));
  return h;
}

/* Output i of a stream. */
uint64_t wl_draw(uint64_t key, uint64_t i) { return wl_mix64(key + WL_GOLDEN * (i + 1)); }

/* The four outlier pairs of (b, kv head): partial Fisher-Yates over 0..63. */
void wl_outlier_pairs(uint64_t seed, int which_query, int b, int kv_head, int32_t* out4) {
  int arr[64];
  for (int i = 0; i < 64; ++i) arr[i] = i;
  uint64_t key = wl_row_key(seed, which_query ? WL_QOUT : WL_KOUT, b, kv_head, 0);
  for (int j = 0; j < 4; ++j) {
    int r = (int)(wl_draw(key, (uint64_t)j) % (uint64_t)(64 - j));
    int tmp = arr[j];
    arr[j] = arr[j + r];
    arr[j + r] = tmp;
    out4[j] = arr[j];
  }
}

/* Round a double to the nearest bf16 (ties to even) and return its bits. */
uint16_t wl_bf16_from_double(double x) {
  if (x == 0.0) return signbit(x) ? 0x8000u : 0u;
  if (isnan(x)) return 0x7FC0u;
  int e;
  double f = frexp(x, &e);          /* x = f * 2^e, 0.5 <= |f| < 1 */
  if (e < -125) {                   /* below the normal range: quantum 2^-133 */
    double r = nearbyint(ldexp(x, 133));
    float v = (float)ldexp(r, -133);
    uint32_t u;
    memcpy(&u, &v, 4);
    return (uint16_t)(u >> 16);
  }
  double r = nearbyint(ldexp(f, 8)); /* 8 significant bits, ties to even */
  double y = ldexp(r, e - 8);
  float v = (float)y;               /* exact: y has 8 significant bits */
  uint32_t u;
  memcpy(&u, &v, 4);
  if (isinf(v)) return (uint16_t)(x > 0 ? 0x7F80u : 0xFF80u);
  return (uint16_t)(u >> 16);
}

typedef struct {
  uint64_t seed;
  int tensor;      /* WL_Q, WL_K or WL_V */
  int G;           /* query heads per KV head (Q only) */
  double theta;
  double key_scale, query_scale;
} wl_params;

/* One row of 128 values at position pos of (b, head); head is a query head for Q. */
static void wl_one_row(const wl_params* P, int b, int head, int64_t pos, uint16_t* out) {
  double x[128];
  uint64_t key = wl_row_key(P->seed, P->tensor, b, head, pos);
  for (int i = 0; i < 64; ++i) {
    uint64_t a = wl_draw(key, 2 * (uint64_t)i);
    uint64_t c = wl_draw(key, 2 * (uint64_t)i + 1);
    double u1 = ((double)(a >> 11) + 1.0) * 0x1.0p-53; /* (0, 1] */
    double u2 = (double)(c >> 11) * 0x1.0p-53;         /* [0, 1) */
    double r = sqrt(-2.0 * log(u1));
    double ang = 2.0 * M_PI * u2;
    x[i] = r * cos(ang);
    x[i + 64] = r * sin(ang);
  }
  if (P->tensor == WL_K || P->tensor == WL_Q) {
    int32_t pairs[4];
    int kvh = P->tensor == WL_K ? head : head / P->G;
    double sc = P->tensor == WL_K ? P->key_scale : P->query_scale;
    wl_outlier_pairs(P->seed, P->tensor == WL_Q, b, kvh, pairs);
    for (int j = 0; j < 4; ++j) {
      x[pairs[j]] *= sc;
      x[pairs[j] + 64] *= sc;
    }
    for (int i = 0; i < 64; ++i) {
      double f = pow(P->theta, -(double)i / 64.0);
      double ang = (double)pos * f;
      double cs = cos(ang), sn = sin(ang);
      double a = x[i], c = x[i + 64];
      x[i] = a * cs - c * sn;
      x[i + 64] = c * cs + a * sn;
    }
  }
  for (int c = 0; c < 128; ++c) out[c] = wl_bf16_from_double(x[c]);
}

/* Pre-RoPE (unrotated) row, for the norm-invariance pin. */
void wl_row_unrotated(uint64_t seed, int tensor, int G, double key_scale, double query_scale,
                      int b, int head, int64_t pos, double* out128) {
  uint64_t key = wl_row_key(seed, tensor, b, head, pos);
  for (int i = 0; i < 64; ++i) {
    uint64_t a = wl_draw(key, 2 * (uint64_t)i);
    uint64_t c = wl_draw(key, 2 * (uint64_t)i + 1);
    double u1 = ((double)(a >> 11) + 1.0) * 0x1.0p-53;
    double u2 = (double)(c >> 11) * 0x1.0p-53;
    double r = sqrt(-2.0 * log(u1));
    double ang = 2.0 * M_PI * u2;
    out128[i] = r * cos(ang);
    out128[i + 64] = r * sin(ang);
  }
  if (tensor == WL_K || tensor == WL_Q) {
    int32_t pairs[4];
    int kvh = tensor == WL_K ? head : head / G;
    double sc = tensor == WL_K ? key_scale : query_scale;
    wl_outlier_pairs(seed, tensor == WL_Q, b, kvh, pairs);
    for (int j = 0; j < 4; ++j) {
      out128[pairs[j]] *= sc;
      out128[pairs[j] + 64] *= sc;
    }
  }
}

/* Rotated row in double (before bf16 rounding), for the norm-invariance pin. */
void wl_row_double(uint64_t seed, int tensor, int G, double theta, double key_scale,
                   double query_scale, int b, int head, int64_t pos, double* out128) {
  wl_row_unrotated(seed, tensor, G, key_scale, query_scale, b, head, pos, out128);
  if (tensor == WL_K || tensor == WL_Q) {
    for (int i = 0; i < 64; ++i) {
      double f = pow(theta, -(double)i / 64.0);
      double ang = (double)pos * f;
      double cs = cos(ang), sn = sin(ang);
      double a = out128[i], c = out128[i + 64];
      out128[i] = a * cs - c * sn;
      out128[i + 64] = c * cs + a * sn;
    }
  }
}

typedef struct {
  wl_params P;
  int b0, h0;      /* first batch row and head of the block */
  int B, H, n;
  int64_t t0;
  int64_t ld;      /* rows between consecutive heads in out */
  uint16_t* out;
  int64_t first, last; /* [first, last) over the B*H*n rows */
} wl_job;

static void* wl_worker(void* arg) {
  wl_job* J = (wl_job*)arg;
  for (int64_t r = J->first; r < J->last; ++r) {
    int64_t bh = r / J->n;
    int64_t t = r % J->n;
    int b = (int)(bh / J->H), h = (int)(bh % J->H);
    wl_one_row(&J->P, J->b0 + b, J->h0 + h, J->t0 + t, J->out + (bh * J->ld + t) * 128);
  }
  return NULL;
}

/*
 * Fill out[b][h][t][128] (head stride ld rows) with the rows of positions
 * t0 .. t0+n-1 of batch rows b0 .. b0+B-1 and heads h0 .. h0+H-1, using nthreads
 * threads.  tensor: 0 = Q (heads are query heads), 1 = K, 2 = V.
 */
int wl_fill_block(uint64_t seed, int tensor, int b0, int B, int h0, int H, int G, int64_t t0, int n,
                  int64_t ld, double theta, double key_scale, double query_scale, uint16_t* out,
                  int nthreads) {
  if (B <= 0 || H <= 0 || n <= 0 || ld < n || G <= 0 || !out || b0 < 0 || h0 < 0) return 1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  int64_t rows = (int64_t)B * H * n;
  if (rows < 4096) nthreads = 1;
  wl_job jobs[256];
  pthread_t th[256];
  for (int i = 0; i < nthreads; ++i) {
    wl_job* J = &jobs[i];
    J->P.seed = seed;
    J->P.tensor = tensor;
    J->P.G = G;
    J->P.theta = theta;
    J->P.key_scale = key_scale;
    J->P.query_scale = query_scale;
    J->b0 = b0;
    J->h0 = h0;
    J->B = B;
    J->H = H;
    J->n = n;
    J->t0 = t0;
    J->ld = ld;
    J->out = out;
    J->first = rows * i / nthreads;
    J->last = rows * (i + 1) / nthreads;
  }
  if (nthreads == 1) {
    wl_worker(&jobs[0]);
    return 0;
  }
  for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, wl_worker, &jobs[i]);
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  return 0;
}

/* The whole batch from row 0 and head 0. */
int wl_fill(uint64_t seed, int tensor, int B, int H, int G, int64_t t0, int n, int64_t ld,
            double theta, double key_scale, double query_scale, uint16_t* out, int nthreads) {
  return wl_fill_block(seed, tensor, 0, B, 0, H, G, t0, n, ld, theta, key_scale, query_scale, out,
                       nthreads);
}
