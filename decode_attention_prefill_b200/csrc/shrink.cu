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
// One warp per group record, four records per CTA.  The packed layout makes this a
// per-lane word map: destination word w of lane L (in the low block of the new layout) is
// built from source words 2w and 2w + 1 of the same lane, because a 2b-bit word holds half
// as many slots as a b-bit word and slot r of source word 2w + p lands in destination slot
// (16 / 2b) p + r.  The shift itself runs on all fields of a word at once: the fields are
// spread one per byte (b = 2) or one per nibble (b = 1), where (2^(2b) - 2^b + 1)(X + 2^(b-1))
// stays below the lane's width, so one 32-bit multiply serves four or eight fields.  The low
// block, zero points and the value part are copied; the first CTA of each (sequence, KV
// head) also copies its residual window, permutation and scores, so one launch does all.
#include "common.cuh"

namespace pnmix {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;

// The equivalent right shift of every 2b-bit field of w, the result field of slot r placed
// at the low bits of that slot.
template <int B>
__device__ __forceinline__ uint32_t ers_fields(uint32_t w);

template <>
__device__ __forceinline__ uint32_t ers_fields<2>(uint32_t w) {   // 4-bit fields, 2-bit results
  constexpr uint32_t kMul = 16u - 4u + 1u;                         // 2^(2b) - 2^b + 1
  const uint32_t e = w & 0x0F0F0F0Fu, o = (w >> 4) & 0x0F0F0F0Fu;  // one field per byte
  const uint32_t ye = (((e + 0x02020202u) * kMul) >> 6) & 0x03030303u;
  const uint32_t yo = (((o + 0x02020202u) * kMul) >> 6) & 0x03030303u;
  return ye | (yo << 4);
}

template <>
__device__ __forceinline__ uint32_t ers_fields<1>(uint32_t w) {   // 2-bit fields, 1-bit results
  constexpr uint32_t kMul = 4u - 2u + 1u;
  const uint32_t e = w & 0x33333333u, o = (w >> 2) & 0x33333333u;  // one field per nibble
  const uint32_t ye = (((e + 0x11111111u) * kMul) >> 3) & 0x11111111u;
  const uint32_t yo = (((o + 0x11111111u) * kMul) >> 3) & 0x11111111u;
  return ye | (yo << 2);
}

// Close up the b-bit results (one per 2b-bit slot) into the low 8 bits of each half-word.
template <int B>
__device__ __forceinline__ uint32_t compress_fields(uint32_t y);

template <>
__device__ __forceinline__ uint32_t compress_fields<2>(uint32_t y) {
  y = (y | (y >> 2)) & 0x0F0F0F0Fu;
  return (y | (y >> 4)) & 0x00FF00FFu;
}

template <>
__device__ __forceinline__ uint32_t compress_fields<1>(uint32_t y) {
  y = (y | (y >> 1)) & 0x33333333u;
  y = (y | (y >> 2)) & 0x0F0F0F0Fu;
  return (y | (y >> 4)) & 0x00FF00FFu;
}

template <int B>
__global__ void __launch_bounds__(kThreads)
shrink_kernel(Geometry gs, Geometry gd, pnmix_cache src, pnmix_cache dst) {
  const int warp = threadIdx.x >> 5, L = threadIdx.x & 31;
  const int grp = blockIdx.x * kWarps + warp, h = blockIdx.y, b = blockIdx.z;
  if (blockIdx.x == 0) {
    // the unit's state that carries over (residual window, permutation, scores); its
    // salient set becomes empty
    const size_t u = unit_index(gs, b, h);
    constexpr int kResid16 = kGroup * kHeadDim * 2 / 16;
    const uint4* rk = reinterpret_cast<const uint4*>(src.k_resid) + u * kResid16;
    const uint4* rv = reinterpret_cast<const uint4*>(src.v_resid) + u * kResid16;
    uint4* dk = reinterpret_cast<uint4*>(dst.k_resid) + u * kResid16;
    uint4* dv = reinterpret_cast<uint4*>(dst.v_resid) + u * kResid16;
    for (int i = threadIdx.x; i < kResid16; i += kThreads) {
      dk[i] = rk[i];
      dv[i] = rv[i];
    }
    if (threadIdx.x < kHeadDim / 16)
      reinterpret_cast<uint4*>(dst.perm + u * kHeadDim)[threadIdx.x] =
          reinterpret_cast<const uint4*>(src.perm + u * kHeadDim)[threadIdx.x];
    if (threadIdx.x < 64) dst.pair_scores[u * 64 + threadIdx.x] = src.pair_scores[u * 64 + threadIdx.x];
    if (threadIdx.x < 64) dst.pair_idx[u * 64 + threadIdx.x] = 0;
    if (threadIdx.x == 0) dst.pair_mask[u] = 0;
    if (threadIdx.x == 0 && h == 0) dst.len[b] = src.len[b];
  }
  const int n = src.len[b];
  if (grp >= (n < 0 ? 0 : (n > gs.capacity ? gs.capacity : n)) / kGroup) return;
  const uint32_t* ws = reinterpret_cast<const uint32_t*>(record_ptr(gs, src.records, b, h, grp));
  uint32_t* wd = reinterpret_cast<uint32_t*>(record_ptr(gd, dst.records, b, h, grp));
  // ---- key words: the salient block shrinks, the low block moves down unchanged.  All
  //      loads of the record are issued before the first store (at most 16 salient and
  //      8 low words per lane).
  const int wh_d = gs.wh / 2;
  uint32_t hw[16], lw[8];
#pragma unroll
  for (int w = 0; w < 16; ++w)
    if (w < gs.wh) hw[w] = ws[w * 32 + L];
#pragma unroll
  for (int w = 0; w < 8; ++w)
    if (w < gs.wl) lw[w] = ws[(gs.wh + w) * 32 + L];
  // ---- scales (x (2^b + 1) where salient) and zero points: lane L holds the four fp16
  //      entries 4L .. 4L + 3, i.e. the fp16x2 words 2L (slice 2 * ((L >> 1) & 3)) and
  //      2L + 1 (the next slice)
  const uint2 sc = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(ws) + rec_kscale(gs) + 8 * L);
  const uint2 zr = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(ws) + rec_kzero(gs) + 8 * L);
  const uint4* vs = reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(ws) + rec_vcode(gs));
  uint4 vv[3];
#pragma unroll
  for (int i = 0; i < 3; ++i) vv[i] = vs[L + 32 * i];   // 1536 B = 3 x 32 x 16 B
#pragma unroll
  for (int w = 0; w < 8; ++w)
    if (w < wh_d)
      wd[w * 32 + L] = compress_fields<B>(ers_fields<B>(hw[2 * w])) |
                       (compress_fields<B>(ers_fields<B>(hw[2 * w + 1])) << 8);
#pragma unroll
  for (int w = 0; w < 8; ++w)
    if (w < gs.wl) wd[(wh_d + w) * 32 + L] = lw[w];
  uint2 so = sc;
  {
    const float mul = static_cast<float>((1 << B) + 1);
    uint32_t v[2] = {sc.x, sc.y};
    for (int i = 0; i < 2; ++i) {
      if (2 * ((L >> 1) & 3) + i >= gs.nhs) continue;   // slice not salient: scale kept
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&v[i]));
      const __half lo = __float2half_rn(__fmul_rn(f.x, mul)), hi = __float2half_rn(__fmul_rn(f.y, mul));
      v[i] = static_cast<uint32_t>(__half_as_ushort(lo)) | (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
    }
    so = make_uint2(v[0], v[1]);
  }
  *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(wd) + rec_kscale(gd) + 8 * L) = so;
  *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(wd) + rec_kzero(gd) + 8 * L) = zr;
  // ---- the value part (codes, scales, zero points) as is
  uint4* vd = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(wd) + rec_vcode(gd));
#pragma unroll
  for (int i = 0; i < 3; ++i) vd[L + 32 * i] = vv[i];
}

}  // namespace

cudaError_t launch_shrink(const Geometry& gs, const Geometry& gd, const pnmix_cache& src,
                          const pnmix_cache& dst, cudaStream_t s) {
  if (gs.bhi != 2 * gs.blo || gd.wl != gs.wh / 2 + gs.wl || gs.wh > 16 || gs.wl > 8)
    return cudaErrorInvalidValue;
  if (gs.B == 0) return cudaSuccess;
  dim3 grid(gs.gcap > 0 ? (gs.gcap + kWarps - 1) / kWarps : 1, gs.Hkv, gs.B);
  if (gs.blo == 2)
    shrink_kernel<2><<<grid, kThreads, 0, s>>>(gs, gd, src, dst);
  else
    shrink_kernel<1><<<grid, kThreads, 0, s>>>(gs, gd, src, dst);
  return cudaGetLastError();
}

}  // namespace pnmix
