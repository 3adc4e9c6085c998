// shrink.cu -- bit-width shrinking of the salient key positions (the equivalent right
// shift of the PM-KVQ review page, the step of its progressive quantization that halves a
// cache's bit width in place of re-quantizing from full precision).
//
// A cache of (b_hi, b_lo = b_hi / 2, k salient pairs) becomes a cache of (b_hi, b_lo, 0):
// every position at b_lo bits, in the same position order.  For the salient positions
// [0, 2k) the code X becomes ((2^(2b) - 2^b + 1) * (X + 2^(b-1))) >> 3b with b = b_lo,
// i.e. round(X / (2^b + 1)), and the scale becomes fp16(fl(s * (2^b + 1))); zero points,
// the other positions' codes, the value part, the residual window, lengths, permutation
// and scores are carried over.  The result is read by the ordinary decode kernels.
//
// One CTA of 128 threads per group record: the source record is staged in shared memory
// with 16-byte loads, thread j takes position j of the 32 tokens from there, the codes meet
// in shared memory, and the destination words (the all-b_lo layout of include/pnmix.h) are
// assembled from there and written with coalesced stores.
#include "common.cuh"

namespace pnmix {
namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ uint32_t ers(uint32_t x, int b) {
  const uint32_t mul = (1u << (2 * b)) - (1u << b) + 1u;
  return (mul * (x + (1u << (b - 1)))) >> (3 * b);
}

__global__ void __launch_bounds__(kThreads)
shrink_kernel(Geometry gs, Geometry gd, pnmix_cache src, pnmix_cache dst) {
  constexpr int kMaxRecord = 4096;   // 4/2-bit keys with every pair salient
  __shared__ __align__(16) uint8_t rec[kMaxRecord];
  __shared__ uint8_t codes[kGroup][kHeadDim];
  const int grp = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  if (grp >= src.len[b] / kGroup) return;
  const uint4* rs = reinterpret_cast<const uint4*>(record_ptr(gs, src.records, b, h, grp));
  uint8_t* rd = record_ptr(gd, dst.records, b, h, grp);
  for (int i = threadIdx.x; i < gs.record_bytes / 16; i += kThreads)
    reinterpret_cast<uint4*>(rec)[i] = rs[i];
  __syncthreads();
  const int j = threadIdx.x;
  const bool hi = j < gs.nhi;
  const int lo_bits = gs.blo;
  // ---- codes of position j, shifted down where salient
  for (int tau = 0; tau < kGroup; ++tau) {
    int off, bit, bits;
    key_code_loc(gs, tau, j, off, bit, bits);
    uint32_t c = (*reinterpret_cast<const uint32_t*>(rec + off) >> bit) & ((1u << bits) - 1u);
    codes[tau][j] = static_cast<uint8_t>(hi ? ers(c, lo_bits) : c);
  }
  // ---- scale and zero point of position j (same index in both layouts)
  const uint16_t* ss = reinterpret_cast<const uint16_t*>(rec + rec_kscale(gs));
  const uint16_t* zs = reinterpret_cast<const uint16_t*>(rec + rec_kzero(gs));
  uint16_t* sd = reinterpret_cast<uint16_t*>(rd + rec_kscale(gd));
  uint16_t* zd = reinterpret_cast<uint16_t*>(rd + rec_kzero(gd));
  const int si = kscale_index(j);
  uint16_t s16 = ss[si];
  if (hi) {
    const float s = __fmul_rn(__half2float(__ushort_as_half(s16)), static_cast<float>((1 << lo_bits) + 1));
    s16 = __half_as_ushort(__float2half_rn(s));
  }
  sd[si] = s16;
  zd[si] = zs[si];
  // ---- the value part (codes, scales, zero points) as is
  const uint4* vs = reinterpret_cast<const uint4*>(rec + rec_vcode(gs));
  uint4* vd = reinterpret_cast<uint4*>(rd + rec_vcode(gd));
  for (int i = threadIdx.x; i < 1536 / 16; i += kThreads) vd[i] = vs[i];
  __syncthreads();
  // ---- destination key words: all positions in the b_lo block (no salient slice)
  const int m = 16 / lo_bits;   // slots per half-word
  uint32_t* kw = reinterpret_cast<uint32_t*>(rd);
  for (int i = threadIdx.x; i < gd.wl * 32; i += kThreads) {
    const int w = i >> 5, L = i & 31;
    const int gq = L >> 2, tq = L & 3;
    uint32_t word = 0;
    for (int r = 0; r < m; ++r) {
      const int n = w * m + r;
      const int sigma = n >> 3, cc = (n >> 2) & 1, u = n & 3;
      const int p0 = 16 * sigma + 2 * tq + 8 * cc;
      const int tau = gq + 8 * u;
      word |= static_cast<uint32_t>(codes[tau][p0]) << (lo_bits * r);
      word |= static_cast<uint32_t>(codes[tau][p0 + 1]) << (16 + lo_bits * r);
    }
    kw[i] = word;
  }
}

}  // namespace

cudaError_t launch_shrink(const Geometry& gs, const Geometry& gd, const pnmix_cache& src,
                          const pnmix_cache& dst, cudaStream_t s) {
  const size_t units = static_cast<size_t>(gs.B) * gs.Hkv;
  cudaError_t e;
  // the regions that carry over; the salient set of the result is empty
  if ((e = cudaMemcpyAsync(dst.len, src.len, sizeof(int32_t) * gs.B, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
    return e;
  const size_t resid = units * kGroup * kHeadDim * sizeof(uint16_t);
  if ((e = cudaMemcpyAsync(dst.k_resid, src.k_resid, resid, cudaMemcpyDeviceToDevice, s)) != cudaSuccess) return e;
  if ((e = cudaMemcpyAsync(dst.v_resid, src.v_resid, resid, cudaMemcpyDeviceToDevice, s)) != cudaSuccess) return e;
  if ((e = cudaMemcpyAsync(dst.perm, src.perm, units * kHeadDim, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
    return e;
  if ((e = cudaMemcpyAsync(dst.pair_scores, src.pair_scores, units * 64 * sizeof(float), cudaMemcpyDeviceToDevice,
                           s)) != cudaSuccess)
    return e;
  if ((e = cudaMemsetAsync(dst.pair_idx, 0, units * 64, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dst.pair_mask, 0, units * sizeof(uint64_t), s)) != cudaSuccess) return e;
  if (gs.gcap == 0) return cudaSuccess;
  if (gs.record_bytes > 4096 || gs.record_bytes % 16) return cudaErrorInvalidValue;
  dim3 grid(gs.gcap, gs.Hkv, gs.B);
  shrink_kernel<<<grid, kThreads, 0, s>>>(gs, gd, src, dst);
  return cudaGetLastError();
}

}  // namespace pnmix
