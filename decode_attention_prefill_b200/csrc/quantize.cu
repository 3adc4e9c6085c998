// quantize.cu -- prefill key/value quantization and the streaming append.
//
// Keys: per channel over 32-token groups, channels of the salient pairs at b_hi bits and
// the rest at b_lo bits (PN-Mix abstract: mixed-precision key cache with higher precision
// for the salient RoPE pairs).  Values: per token over 32-channel groups at 2 bits
// (MixKVQ abstract: per-token value quantization).  Both use the asymmetric min-max code
// with fp16 scale and zero point, in fp32 with one rounding per operation so the codes
// are bit-exact with the reference definition.
//
// One CTA of 128 threads quantizes one 32-token group of one (b, KV head): the 8 KB bf16
// tile is staged in shared memory with 16-byte loads, thread j owns key position j (or
// value (token, channel group) pair), codes go to a shared byte array and are then
// packed into the record words of the layout in pnmix.h with coalesced 32-bit stores.
#include "common.cuh"

namespace pnmix {
namespace {

constexpr int kThreads = 128;
constexpr int kTileStride = kHeadDim + 8;   // bf16 elements per shared row (+16 B pad)

struct GroupSmem {
  uint16_t tile[kGroup][kTileStride];
  uint8_t codes[kGroup][kHeadDim];
  uint8_t perm[kHeadDim];
};

// Stage 32 rows of 128 bf16 (row stride `ld_elems`) into shared memory.
__device__ __forceinline__ void load_tile(GroupSmem& sm, const uint16_t* src, size_t ld_elems) {
  for (int i = threadIdx.x; i < kGroup * 16; i += kThreads) {
    int r = i >> 4, c = i & 15;
    uint4 v = __ldg(reinterpret_cast<const uint4*>(src + r * ld_elems) + c);
    *reinterpret_cast<uint4*>(&sm.tile[r][c * 8]) = v;
  }
}

// Keys of the staged group -> key part of `rec`.
__device__ void quantize_key_group(const Geometry& g, GroupSmem& sm, uint8_t* rec) {
  const int j = threadIdx.x;   // position
  {
    const int ch = sm.perm[j];
    const int bits = j < g.nhi ? g.bhi : g.blo;
    float mn = bf16_bits_to_float(sm.tile[0][ch]), mx = mn;
#pragma unroll 8
    for (int t = 1; t < kGroup; ++t) {
      float x = bf16_bits_to_float(sm.tile[t][ch]);
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    QParams q = quant_params(mn, mx, bits);
#pragma unroll 8
    for (int t = 0; t < kGroup; ++t)
      sm.codes[t][j] = static_cast<uint8_t>(quant_code(bf16_bits_to_float(sm.tile[t][ch]), q, bits));
    uint16_t* ks = reinterpret_cast<uint16_t*>(rec + rec_kscale(g));
    uint16_t* kz = reinterpret_cast<uint16_t*>(rec + rec_kzero(g));
    ks[kscale_index(j)] = q.s16;
    kz[kscale_index(j)] = q.z16;
  }
  __syncthreads();
  // pack: word (w, L) for every lane L and lane-local word w
  const int words = (g.wh + g.wl) * 32;
  uint32_t* kw = reinterpret_cast<uint32_t*>(rec);
  for (int i = threadIdx.x; i < words; i += kThreads) {
    const int w = i >> 5, L = i & 31;
    const int gq = L >> 2, tq = L & 3;
    const bool hi = w < g.wh;
    const int bits = hi ? g.bhi : g.blo;
    const int m = 16 / bits;
    const int wl = hi ? w : w - g.wh;
    const int sigma0 = hi ? 0 : g.nhs;
    uint32_t word = 0;
    for (int r = 0; r < m; ++r) {
      const int n = wl * m + r;
      const int sigma = sigma0 + (n >> 3), cc = (n >> 2) & 1, u = n & 3;
      const int p0 = 16 * sigma + 2 * tq + 8 * cc;
      const int tau = gq + 8 * u;
      word |= static_cast<uint32_t>(sm.codes[tau][p0]) << (bits * r);
      word |= static_cast<uint32_t>(sm.codes[tau][p0 + 1]) << (16 + bits * r);
    }
    kw[i] = word;
  }
}

// Values of the staged group -> value part of `rec`.
__device__ void quantize_value_group(const Geometry& g, GroupSmem& sm, uint8_t* rec) {
  {
    const int t = threadIdx.x >> 2, jg = threadIdx.x & 3;
    // the thread's 32 channels with four 16-byte loads
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
    QParams q = quant_params(mn, mx, g.bv);
    uint32_t packed[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      uint32_t wv = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) wv |= quant_code(x[4 * k + e], q, g.bv) << (8 * e);
      packed[k] = wv;
    }
    uint4* crow = reinterpret_cast<uint4*>(&sm.codes[t][32 * jg]);
    crow[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    crow[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    uint16_t* vs = reinterpret_cast<uint16_t*>(rec + rec_vscale(g));
    uint16_t* vz = reinterpret_cast<uint16_t*>(rec + rec_vzero(g));
    vs[vscale_index(t, jg)] = q.s16;
    vz[vscale_index(t, jg)] = q.z16;
  }
  __syncthreads();
  uint8_t* vc = rec + rec_vcode(g);
  for (int i = threadIdx.x; i < 8 * 32; i += kThreads) {
    const int m = i >> 5, L = i & 31;
    const int gq = L >> 2, tq = L & 3;
    uint32_t word = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int r = q >> 2, p = q & 3;
      const int ch = 16 * m + gq + 8 * r;
      const int t0 = 2 * tq + 8 * p;
      word |= static_cast<uint32_t>(sm.codes[t0][ch]) << (2 * q);
      word |= static_cast<uint32_t>(sm.codes[t0 + 1][ch]) << (16 + 2 * q);
    }
    *reinterpret_cast<uint32_t*>(vc + vword_offset(m, L)) = word;
  }
}

// Copy rows [32*ng, L) of one unit into its residual window (slot = token % 32).
__device__ void copy_tail(const uint16_t* src, int first, int L, uint16_t* resid) {
  const int n = L - first;
  for (int i = threadIdx.x; i < n * 16; i += kThreads) {
    int r = i >> 4, c = i & 15;
    int t = first + r;
    reinterpret_cast<uint4*>(resid + (t & 31) * kHeadDim)[c] =
        __ldg(reinterpret_cast<const uint4*>(src + static_cast<size_t>(t) * kHeadDim) + c);
  }
}

template <bool kKeys>
__global__ void __launch_bounds__(kThreads)
quantize_prefill_kernel(Geometry g, const uint16_t* __restrict__ x, int L, int ld, pnmix_cache c) {
  __shared__ GroupSmem sm;
  const int grp = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int ng = L / kGroup;
  const uint16_t* src = x + unit_index(g, b, h) * static_cast<size_t>(ld) * kHeadDim;
  if (grp == 0 && h == 0 && threadIdx.x == 0) c.len[b] = L;
  if (grp >= ng) {   // the tail CTA
    uint16_t* resid = (kKeys ? c.k_resid : c.v_resid) + unit_index(g, b, h) * kGroup * kHeadDim;
    copy_tail(src, ng * kGroup, L, resid);
    return;
  }
  if (kKeys) sm.perm[threadIdx.x] = c.perm[unit_index(g, b, h) * kHeadDim + threadIdx.x];
  load_tile(sm, src + static_cast<size_t>(grp) * kGroup * kHeadDim, kHeadDim);
  __syncthreads();
  uint8_t* rec = record_ptr(g, c.records, b, h, grp);
  if (kKeys)
    quantize_key_group(g, sm, rec);
  else
    quantize_value_group(g, sm, rec);
}

// One CTA per (b, KV head): write the new row into residual slot len % 32; when that
// is slot 31, quantize the 32 residual rows into record len / 32.  The last CTA of a
// sequence (atomic ticket, taken after every CTA of that sequence has read len[b])
// advances len[b].
__global__ void __launch_bounds__(kThreads)
append_kernel(Geometry g, const uint16_t* __restrict__ k_new, const uint16_t* __restrict__ v_new,
              pnmix_cache c) {
  __shared__ GroupSmem sm;
  const int h = blockIdx.x, b = blockIdx.y;
  const int n = c.len[b];
  if (n >= g.capacity) {
    if (h == 0 && threadIdx.x == 0) atomicOr(c.error, PNMIX_DEVERR_APPEND_FULL);
    return;
  }
  const size_t u = unit_index(g, b, h);
  const int slot = n & 31;
  uint16_t* rk = c.k_resid + u * kGroup * kHeadDim;
  uint16_t* rv = c.v_resid + u * kGroup * kHeadDim;
  if (threadIdx.x < 16) {
    reinterpret_cast<uint4*>(rk + slot * kHeadDim)[threadIdx.x] =
        __ldg(reinterpret_cast<const uint4*>(k_new + u * kHeadDim) + threadIdx.x);
  } else if (threadIdx.x < 32) {
    reinterpret_cast<uint4*>(rv + slot * kHeadDim)[threadIdx.x - 16] =
        __ldg(reinterpret_cast<const uint4*>(v_new + u * kHeadDim) + threadIdx.x - 16);
  }
  if (slot == kGroup - 1) {
    __syncthreads();
    uint8_t* rec = record_ptr(g, c.records, b, h, n / kGroup);
    sm.perm[threadIdx.x] = c.perm[u * kHeadDim + threadIdx.x];
    for (int i = threadIdx.x; i < kGroup * 16; i += kThreads) {
      int r = i >> 4, cc = i & 15;
      *reinterpret_cast<uint4*>(&sm.tile[r][cc * 8]) = reinterpret_cast<const uint4*>(rk + r * kHeadDim)[cc];
    }
    __syncthreads();
    quantize_key_group(g, sm, rec);
    __syncthreads();
    for (int i = threadIdx.x; i < kGroup * 16; i += kThreads) {
      int r = i >> 4, cc = i & 15;
      *reinterpret_cast<uint4*>(&sm.tile[r][cc * 8]) = reinterpret_cast<const uint4*>(rv + r * kHeadDim)[cc];
    }
    __syncthreads();
    quantize_value_group(g, sm, rec);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    uint32_t* ticket = c.scratch + scratch_append_ticket_offset(g.B, g.Hkv) + b;
    if (atomicAdd(ticket, 1u) == static_cast<unsigned>(g.Hkv - 1)) {
      c.len[b] = n + 1;
      *ticket = 0u;
    }
  }
}

}  // namespace

cudaError_t launch_quantize_keys(const Geometry& g, const uint16_t* k, int L, int ld,
                                 const pnmix_cache& c, cudaStream_t s) {
  const int ng = L / kGroup;
  dim3 grid(ng + ((L % kGroup) ? 1 : 0) + (L == 0 ? 1 : 0), g.Hkv, g.B);
  quantize_prefill_kernel<true><<<grid, kThreads, 0, s>>>(g, k, L, ld, c);
  return cudaGetLastError();
}

cudaError_t launch_quantize_values(const Geometry& g, const uint16_t* v, int L, int ld,
                                   const pnmix_cache& c, cudaStream_t s) {
  const int ng = L / kGroup;
  dim3 grid(ng + ((L % kGroup) ? 1 : 0) + (L == 0 ? 1 : 0), g.Hkv, g.B);
  quantize_prefill_kernel<false><<<grid, kThreads, 0, s>>>(g, v, L, ld, c);
  return cudaGetLastError();
}

cudaError_t launch_append(const Geometry& g, const uint16_t* k_new, const uint16_t* v_new,
                          const pnmix_cache& c, cudaStream_t s) {
  dim3 grid(g.Hkv, g.B);
  append_kernel<<<grid, kThreads, 0, s>>>(g, k_new, v_new, c);
  return cudaGetLastError();
}

}  // namespace pnmix
