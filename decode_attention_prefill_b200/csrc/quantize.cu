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
#include "quantize_group.cuh"

namespace pnmix {
namespace {

constexpr int kThreads = 128;
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
  if (kKeys) sm.perm[threadIdx.x] = c.perm[unit_index(g, b, h) * kHeadDim + threadIdx.x] & (kHeadDim - 1);
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
  if (n < 0 || n >= g.capacity) {
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
    sm.perm[threadIdx.x] = c.perm[u * kHeadDim + threadIdx.x] & (kHeadDim - 1);
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
