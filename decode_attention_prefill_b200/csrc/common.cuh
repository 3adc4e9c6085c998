// common.cuh -- device-side helpers shared by the pnmix kernels (not by the oracle).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pnmix.h"

namespace pnmix {

constexpr int kHeadDim = 128;
constexpr int kGroup = 32;      // tokens per key group / value records
constexpr int kMaxG = 8;        // query heads per KV head
constexpr int kMaxRows = 64;    // query rows per KV head in one decode launch (G x queries)

// Geometry derived from a validated pnmix_config (host computes, kernels read by value).
struct Geometry {
  int B, Hq, Hkv, G;
  int k;          // salient pairs
  int nhi;        // salient positions = 2k
  int nhs;        // hi slices = nhi / 16
  int bhi, blo, bv;
  int wh, wl;     // key-code words per lane, hi / lo block
  int kc_bytes;   // key-code bytes per record = 128 * (wh + wl)
  int record_bytes;
  int capacity;   // tokens per sequence
  int gcap;       // records per (b, h) = capacity / 32
  float scale;    // softmax scale
  int score;      // saliency statistic, PNMIX_SCORE_*
  int n_prune;    // decode: query pairs each query row drops (0: none)
  int n_prune_slices;   // decode: low-precision key slices each unit drops (0: none)
  int tq;         // decode queries per sequence (1, or T of a multi-query step)
  int rows;       // query rows per (b, KV head) in decode: G * tq (row v = query v / G, head v % G)
  int kernel;     // decode kernel, PNMIX_DECODE_*
  uint32_t wait_limit;   // decode: try_wait rounds before a staging wait gives up
  int skip_unit;         // decode test hook: the unit whose records are never staged (-1: none)
  int append;            // decode: the launch first appends one K/V row per sequence (fused)
  int lead;              // decode partition: work items counted at the start of every unit for
                         // its fixed cost (setup, merge, combine), with no work of their own
  int resid_w;           // decode partition: items the residual window counts for (>= 1)
};

// try_wait rounds before a decode staging wait gives up (each round may suspend the warp
// for a while); a wait that runs out sets PNMIX_DEVERR_TIMEOUT and the kernel stops
// consuming.
constexpr uint32_t kDecodeWaitLimit = 1u << 22;

// Record part offsets.
__host__ __device__ __forceinline__ int rec_kscale(const Geometry& g) { return g.kc_bytes; }
__host__ __device__ __forceinline__ int rec_kzero(const Geometry& g) { return g.kc_bytes + 256; }
__host__ __device__ __forceinline__ int rec_vcode(const Geometry& g) { return g.kc_bytes + 512; }
__host__ __device__ __forceinline__ int rec_vscale(const Geometry& g) { return g.kc_bytes + 1536; }
__host__ __device__ __forceinline__ int rec_vzero(const Geometry& g) { return g.kc_bytes + 1792; }

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// fp16 element index of key position j in the scale / zero arrays: one 16-byte chunk per
// (tq, slice pair) holds (even slice e=0, odd slice e=0, even slice e=1, odd slice e=1).
__host__ __device__ __forceinline__ int kscale_index(int j) {
  int sigma = j >> 4, e = (j >> 3) & 1, tq = (j >> 1) & 3, v = j & 1;
  return ((tq * 4 + (sigma >> 1)) * 4 + 2 * e + (sigma & 1)) * 2 + v;
}

// fp16 element index of the value scale of (token t, channel group jg).
__host__ __device__ __forceinline__ int vscale_index(int t, int jg) {
  return ((t >> 1) * 4 + jg) * 2 + (t & 1);
}

// fp16 element index of the value zero point of (token t, channel group jg): the token
// pair tp = t / 2 of group jg sits in the 16-byte chunk (tp % 4, jg) at slot
// tp / 8 + 2 * ((tp / 4) % 2), i.e. the chunk holds tp, tp + 8, tp + 4, tp + 12.
__host__ __device__ __forceinline__ int vzero_index(int t, int jg) {
  const int tp = t >> 1;
  return ((((tp & 3) * 4 + jg) * 4) + ((tp >> 3) & 1) + 2 * ((tp >> 2) & 1)) * 2 + (t & 1);
}

// Byte offset (inside the value-code area) of value word m of lane L.
__host__ __device__ __forceinline__ int vword_offset(int m, int L) {
  return ((m >> 2) * 32 + L) * 16 + (m & 3) * 4;
}

// Location of the key code of (token tau, position j): byte offset of its 32-bit
// word in the record and its bit.  Follows the slot definition of pnmix.h.
__device__ __forceinline__ void key_code_loc(const Geometry& g, int tau, int j, int& byte_off,
                                             int& bit, int& bits) {
  int sigma = j >> 4, rem = j & 15;
  int c = rem >> 3, tq = (rem & 7) >> 1, half = rem & 1;
  int gq = tau & 7, u = tau >> 3;
  bool hi = sigma < g.nhs;
  bits = hi ? g.bhi : g.blo;
  int m = 16 / bits;
  int n = (hi ? sigma : sigma - g.nhs) * 8 + c * 4 + u;
  int w = (hi ? 0 : g.wh) + n / m;
  int L = gq * 4 + tq;
  byte_off = (w * 32 + L) * 4;
  bit = 16 * half + bits * (n % m);
}

// Location of the value code of (token t, channel ch).
__device__ __forceinline__ void value_code_loc(int t, int ch, int& byte_off, int& bit) {
  int tq = (t & 7) >> 1, p = t >> 3, second = t & 1;
  int m = ch >> 4, rem = ch & 15, r = rem >> 3, gq = rem & 7;
  int q = r * 4 + p;
  byte_off = vword_offset(m, gq * 4 + tq);
  bit = 16 * second + 2 * q;
}

// The min-max quantizer parameters, bit-exact with the reference definition:
// s16 = fp16(fl(mx - mn) / (2^b - 1)), z16 = fp16(mn).
struct QParams {
  float s, z;
  uint16_t s16, z16;
};

__device__ __forceinline__ QParams quant_params(float mn, float mx, int bits) {
  float levels = static_cast<float>((1 << bits) - 1);
  float range = __fsub_rn(mx, mn);
  float s32 = __fdiv_rn(range, levels);
  __half hs = __float2half_rn(s32);
  __half hz = __float2half_rn(mn);
  QParams q;
  q.s16 = __half_as_ushort(hs);
  q.z16 = __half_as_ushort(hz);
  q.s = __half2float(hs);
  q.z = __half2float(hz);
  return q;
}

// The code of the reference definition, code = clamp(rint(fl(fl(x - z) / s)), 0, 2^b - 1)
// (0 when s == 0, handled by the callers), with one multiply by the correctly rounded
// reciprocal inv = rcp_rn(s) in place of the division.  t = fl(d * inv) differs from d / s by at most |d / s| * 2^-23
// (two roundings of 2^-24).  Only quotients below 16 decide a code (beyond, the clamp
// does), and there t and the rounded quotient fl(d / s) differ by less than 2^-18, so rint
// gives the same integer for both unless t lies within that distance of a half-integer.
// Elements with |t - rint(t)| >= 0.5 - 2^-17 take the exact division instead.  rint is
// formed by adding and removing 1.5 * 2^23 (round-to-nearest-even in the add), whose low
// bits are then the integer.  Needs s > 0.
__device__ __forceinline__ uint32_t quant_code_rcp(float x, float z, float s, float inv, int levels) {
  constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
  const float d = __fsub_rn(x, z);
  const float t = __fmul_rn(d, inv);
  const float y = __fadd_rn(t, kMagic);
  const float r = __fsub_rn(y, kMagic);
  int code;
  if (fabsf(__fsub_rn(t, r)) < 0.5f - 0x1p-17f) {
    code = __float_as_int(y) - 0x4B400000;
  } else {
    const float e = fminf(fmaxf(rintf(__fdiv_rn(d, s)), -1.0f), static_cast<float>(levels + 1));
    code = static_cast<int>(e);
  }
  return static_cast<uint32_t>(min(max(code, 0), levels));
}

// Squared pair norm fl(fl(a*a) + fl(b*b)).
__device__ __forceinline__ float pair_norm2(float a, float b) {
  return __fadd_rn(__fmul_rn(a, a), __fmul_rn(b, b));
}

// Pointer helpers.
__device__ __forceinline__ size_t unit_index(const Geometry& g, int b, int h) {
  return static_cast<size_t>(b) * g.Hkv + h;
}
__device__ __forceinline__ uint8_t* record_ptr(const Geometry& g, uint8_t* records, int b, int h,
                                               int grp) {
  return records + (unit_index(g, b, h) * g.gcap + grp) * static_cast<size_t>(g.record_bytes);
}

// Scratch regions inside pnmix_cache::scratch.
__host__ __device__ __forceinline__ size_t scratch_kmax_offset() { return 0; }
__host__ __device__ __forceinline__ size_t scratch_select_ticket_offset(int B, int Hkv) {
  return static_cast<size_t>(B) * Hkv * 64;
}
__host__ __device__ __forceinline__ size_t scratch_append_ticket_offset(int B, int Hkv) {
  return static_cast<size_t>(B) * Hkv * 65;
}
// per unit, ordered-key images of the channel minima [128] then maxima [128] (the
// range statistic of pnmix_select_pairs)
__host__ __device__ __forceinline__ size_t scratch_range_offset(int B, int Hkv) {
  return static_cast<size_t>(B) * Hkv * 65 + B;
}
// one word: the grid ticket of a fused append + decode launch (its last CTA advances len)
__host__ __device__ __forceinline__ size_t scratch_fused_ticket_offset(int B, int Hkv) {
  return static_cast<size_t>(B) * Hkv * (65 + 256) + B;
}
__host__ __device__ __forceinline__ size_t scratch_words(int B, int Hkv) {
  return static_cast<size_t>(B) * Hkv * (65 + 256) + B + 1;
}

// Launchers (one translation unit each).
cudaError_t launch_select_pairs(const Geometry& g, const uint16_t* q_window, int n_window,
                                const uint16_t* k, int L, int ld, const pnmix_cache& c,
                                cudaStream_t s);
cudaError_t launch_quantize_keys(const Geometry& g, const uint16_t* k, int L, int ld,
                                 const pnmix_cache& c, cudaStream_t s);
cudaError_t launch_quantize_values(const Geometry& g, const uint16_t* v, int L, int ld,
                                   const pnmix_cache& c, cudaStream_t s);
cudaError_t launch_append(const Geometry& g, const uint16_t* k_new, const uint16_t* v_new,
                          const pnmix_cache& c, cudaStream_t s);

// Decode: host-side validation of a decode call's arguments (everything but the
// workspace), the workspace a batch / context bound needs, the byte offset of its ticket
// words (the only part that must be zero before a launch), and the launch.
pnmix_status check_decode_args(const pnmix_config* cfg, const uint16_t* q, const pnmix_cache* cache,
                               int max_context, const float* out, Geometry* g);
size_t decode_workspace_bytes(const Geometry& g, int max_context);
size_t decode_ticket_offset(const Geometry& g, int max_context);
// Optional parts of a decode launch: the log-sum-exp output and the merge with an earlier
// attention over other tokens (the two parts of a two-precision cache; see combine_segment
// in decode_common.cuh), and the rows of a fused append (Geometry::append).
struct DecodeMerge {
  float* lse_out = nullptr;
  const float* prior_out = nullptr;
  const float* prior_lse = nullptr;
  const uint16_t* k_new = nullptr;
  const uint16_t* v_new = nullptr;
};
cudaError_t launch_decode(const Geometry& g, const uint16_t* q, const pnmix_cache& c,
                          int max_context, float* out, void* ws, cudaStream_t s,
                          const DecodeMerge& merge = DecodeMerge());

}  // namespace pnmix
