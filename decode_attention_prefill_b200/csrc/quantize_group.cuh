// quantize_group.cuh -- the key and value quantizers of one staged 32-token group
// (shared by the prefill / append kernels of quantize.cu and the fused append + decode
// kernel of decode_mma.cu).  A CTA of kQuantThreads threads calls them together.
//
// Keys: per channel over the 32 tokens, channels of the salient pairs at b_hi bits and
// the rest at b_lo bits; values: per token over 32-channel groups at b_v bits.  Both use
// the asymmetric min-max code with fp16 scale and zero point in fp32 with one rounding per
// operation (common.cuh), so the codes are bit-exact with the reference definition.
#pragma once

#include "common.cuh"

namespace pnmix {
namespace {

constexpr int kQuantThreads = 128;
constexpr int kTileStride = kHeadDim + 8;   // bf16 elements per shared row (+16 B pad)

struct GroupSmem {
  uint16_t tile[kGroup][kTileStride];
  uint32_t vcodes[kGroup][8];   // value codes of token t, channels 16i .. 16i+15 in word i
  uint8_t perm[kHeadDim];
};

// Stage 32 rows of 128 bf16 (row stride `ld_elems`) into shared memory: every thread's
// four 16-byte loads are issued before their stores.
__device__ __forceinline__ void load_tile(GroupSmem& sm, const uint16_t* src, size_t ld_elems) {
  constexpr int kPer = kGroup * 16 / kQuantThreads;
  uint4 v[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int i = threadIdx.x + k * kQuantThreads, r = i >> 4, c = i & 15;
    v[k] = __ldg(reinterpret_cast<const uint4*>(src + r * ld_elems) + c);
  }
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int i = threadIdx.x + k * kQuantThreads, r = i >> 4, c = i & 15;
    *reinterpret_cast<uint4*>(&sm.tile[r][c * 8]) = v[k];
  }
}

// Keys of the staged group -> key part of `rec`.  Thread j owns position j (channel
// perm[j]) and its 32 tokens.  Its codes go to the words of the 8 lanes gq (tokens
// gq + 8u, u = 0..3, in consecutive slots of one word); the positions sharing a word
// (the two halves, and the two 8-position blocks c of a slice at 2 bits, or also the two
// slices at 1 bit) are 1, 8 and 16 threads apart, so the words are completed with warp
// shuffles and every word is stored once, by one of the threads that hold it.
__device__ void quantize_key_group(const Geometry& g, GroupSmem& sm, uint8_t* rec) {
  const int j = threadIdx.x;
  const int ch = sm.perm[j];
  const bool hi = j < g.nhi;
  const int bits = hi ? g.bhi : g.blo;
  const int levels = (1 << bits) - 1;
  float x[kGroup];
#pragma unroll
  for (int t = 0; t < kGroup; ++t) x[t] = bf16_bits_to_float(sm.tile[t][ch]);
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int t = 1; t < kGroup; ++t) {
    mn = fminf(mn, x[t]);
    mx = fmaxf(mx, x[t]);
  }
  const QParams q = quant_params(mn, mx, bits);
  uint16_t* ks = reinterpret_cast<uint16_t*>(rec + rec_kscale(g));
  uint16_t* kz = reinterpret_cast<uint16_t*>(rec + rec_kzero(g));
  ks[kscale_index(j)] = q.s16;
  kz[kscale_index(j)] = q.z16;

  // slot of (token gq + 8u) in this position's word: n = 8 * slice + 4 * c + u
  const int sigma = j >> 4, rem = j & 15, cc = rem >> 3, tq = (rem & 7) >> 1, half = rem & 1;
  const int sl = hi ? sigma : sigma - g.nhs;
  const int m = 16 / bits;
  const int n0 = sl * 8 + cc * 4;
  const int w = (hi ? 0 : g.wh) + n0 / m;
  const int shift0 = 16 * half + bits * (n0 % m);
  uint32_t pw[8];
  if (q.s == 0.0f) {
#pragma unroll
    for (int gq = 0; gq < 8; ++gq) pw[gq] = 0u;
  } else {
    const float inv = __frcp_rn(q.s);
#pragma unroll
    for (int gq = 0; gq < 8; ++gq) {
      uint32_t word = 0u;
#pragma unroll
      for (int u = 0; u < 4; ++u)
        word |= quant_code_rcp(x[gq + 8 * u], q.z, q.s, inv, levels) << (shift0 + bits * u);
      pw[gq] = word;
    }
  }
  const bool join8 = bits <= 2, join16 = bits == 1;
  const bool any8 = __any_sync(0xffffffffu, join8), any16 = __any_sync(0xffffffffu, join16);
#pragma unroll
  for (int gq = 0; gq < 8; ++gq) pw[gq] |= __shfl_xor_sync(0xffffffffu, pw[gq], 1);
  if (any8) {
#pragma unroll
    for (int gq = 0; gq < 8; ++gq) {
      const uint32_t o = __shfl_xor_sync(0xffffffffu, pw[gq], 8);
      if (join8) pw[gq] |= o;
    }
  }
  if (any16) {
#pragma unroll
    for (int gq = 0; gq < 8; ++gq) {
      const uint32_t o = __shfl_xor_sync(0xffffffffu, pw[gq], 16);
      if (join16) pw[gq] |= o;
    }
  }
  // holders of a word: 2 (4-bit), 4 (2-bit) or 8 (1-bit) threads; holder `rank` stores
  // the words of the lanes gq = rank (mod holders)
  const int holders = bits == 4 ? 2 : (bits == 2 ? 4 : 8);
  const int rank = half + (bits <= 2 ? 2 * cc : 0) + (bits == 1 ? 4 * (sl & 1) : 0);
  uint32_t* kw = reinterpret_cast<uint32_t*>(rec);
#pragma unroll
  for (int gq = 0; gq < 8; ++gq)
    if ((gq & (holders - 1)) == rank) kw[w * 32 + gq * 4 + tq] = pw[gq];
}

// Values of the staged group -> value part of `rec`.  Thread (t, jg) quantizes token t
// over channels 32 jg .. 32 jg + 31 and keeps the 2-bit codes as two 16-channel words;
// then every thread assembles two record words from those.
__device__ void quantize_value_group(const Geometry& g, GroupSmem& sm, uint8_t* rec) {
  {
    const int t = threadIdx.x >> 2, jg = threadIdx.x & 3;
    float x[32];
    const uint4* row = reinterpret_cast<const uint4*>(&sm.tile[t][32 * jg]);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 v = row[k];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[8 * k + 2 * e] = __uint_as_float(w[e] << 16);
        x[8 * k + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
    float mn = x[0], mx = x[0];
#pragma unroll
    for (int i = 1; i < 32; ++i) {
      mn = fminf(mn, x[i]);
      mx = fmaxf(mx, x[i]);
    }
    const QParams q = quant_params(mn, mx, g.bv);
    const int levels = (1 << g.bv) - 1;
    uint32_t cw[2] = {0u, 0u};
    if (q.s != 0.0f) {
      const float inv = __frcp_rn(q.s);
#pragma unroll
      for (int i = 0; i < 32; ++i) cw[i >> 4] |= quant_code_rcp(x[i], q.z, q.s, inv, levels) << (2 * (i & 15));
    }
    sm.vcodes[t][2 * jg] = cw[0];
    sm.vcodes[t][2 * jg + 1] = cw[1];
    uint16_t* vs = reinterpret_cast<uint16_t*>(rec + rec_vscale(g));
    uint16_t* vz = reinterpret_cast<uint16_t*>(rec + rec_vzero(g));
    vs[vscale_index(t, jg)] = q.s16;
    vz[vzero_index(t, jg)] = q.z16;
  }
  __syncthreads();
  // word (m, L): slot q = 4r + p holds channel 16m + gq + 8r of tokens 2tq + 8p (+1)
  uint8_t* vc = rec + rec_vcode(g);
  for (int i = threadIdx.x; i < 8 * 32; i += kQuantThreads) {
    const int m = i >> 5, L = i & 31;
    const int gq = L >> 2, tq = L & 3;
    uint32_t word = 0;
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const uint32_t v = sm.vcodes[2 * tq + 8 * p + hf][m] >> (2 * gq);
        word |= (v & 3u) << (2 * p + 16 * hf);
        word |= ((v >> 16) & 3u) << (2 * (4 + p) + 16 * hf);
      }
    *reinterpret_cast<uint32_t*>(vc + vword_offset(m, L)) = word;
  }
}


}  // namespace
}  // namespace pnmix
