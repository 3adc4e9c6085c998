// decode_frag.cuh -- pieces shared by the tensor-core decode kernels: PTX wrappers
// (fp16x2 arithmetic, m16n8k16 MMA, mbarriers, bulk copies), the key-code fragment
// builders of the packed record layout (include/pnmix.h) and the CUDA-core attention of
// the bf16 residual window.
#pragma once

#include "common.cuh"
#include "decode_common.cuh"

namespace pnmix {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// Key-code bytes of a record (32 lanes x (WH + WL) words) for a kernel instance: NHS hi
// slices of BHI bits, 8 - NHS lo slices of BLO bits.  The record adds 2048 bytes of key
// scales and zeros, value codes, value scales and zeros.
template <int BHI, int BLO, int NHS>
__host__ __device__ constexpr int key_code_bytes() {
  return 128 * (NHS * BHI / 2 + (8 - NHS) * BLO / 2);
}
template <int BHI, int BLO, int NHS>
__host__ __device__ constexpr int record_bytes_of() {
  return key_code_bytes<BHI, BLO, NHS>() + 2048;
}
constexpr int kResidKStride = kHeadDim + 8;   // bf16 per staged K row (+16 B: no bank conflicts)

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// (lo, hi) fp32 -> f16x2 with lo in the low half.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
// 2^x with the hardware approximation (MUFU.EX2, ~2 ulp; inputs here are <= 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// The same product without `volatile`: the compiler may then reorder it against other
// inline assembly, which helped the warp-pair kernel (its two roles' instruction streams
// interleave more freely) and did not help the one-role kernel, which keeps the form above.
__device__ __forceinline__ void mma16816_free(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
// One staged group (a TMA bulk copy, no multicast): the issuing lane orders the warp's
// earlier shared-memory reads of the slot before the copy's writes (fence.proxy.async),
// arms the slot's barrier with the byte count and starts the copy.  Every lane executes
// it; only `leader` acts (predicated, so the warp does not branch).
__device__ __forceinline__ void stage_group(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                            bool leader) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.u32 p, %4, 0;\n"
      " @p fence.proxy.async.shared::cta;\n"
      " @p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%3], %2;\n"
      " @p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n}"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "r"(static_cast<uint32_t>(leader))
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t phase) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(phase) : "memory");
  return ok != 0;
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }


// Codes as fp16 subnormals.  A code pair sitting at bit offset e of both 16-bit halves of
// a word becomes an exact fp16x2 of (code * 2^(e-24)) with one AND: the exponent field
// stays zero.  The tensor cores take subnormal fp16 operands exactly, so the bit offset
// only scales the product, and the kernel removes that power of two afterwards.
__device__ __forceinline__ uint32_t sub_pair(uint32_t w, uint32_t mask) { return w & mask; }

// Bit offset of token row u (0..3) of a BITS-bit key slice in the A registers below.
template <int BITS>
__host__ __device__ constexpr int key_row_shift(int u) {
  return BITS == 4 ? 4 * (u & 1) : (BITS == 2 ? 2 * u : u);
}

// A fragments (2 M-tiles x 4 registers) of one key slice from its code word(s).
//   4-bit: words w0 (c = 0), w1 (c = 1); token rows u = 0,1 in bits 0-7, rows 2,3 in 8-15.
//   2-bit: word w; c = 0 in bits 0-7, c = 1 in bits 8-15, row u at 2u.
//   1-bit: word w holds two slices; the slice of parity o and half c sit at 4*(2o+c), row u at u.
template <int BITS>
__device__ __forceinline__ void key_slice_frags(uint32_t w0, uint32_t w1, int parity, uint32_t (&A)[2][4]) {
  if constexpr (BITS == 4) {
    const uint32_t s0 = w0 >> 8, s1 = w1 >> 8;
    A[0][0] = sub_pair(w0, 0x000F000Fu); A[0][1] = sub_pair(w0, 0x00F000F0u);
    A[1][0] = sub_pair(s0, 0x000F000Fu); A[1][1] = sub_pair(s0, 0x00F000F0u);
    A[0][2] = sub_pair(w1, 0x000F000Fu); A[0][3] = sub_pair(w1, 0x00F000F0u);
    A[1][2] = sub_pair(s1, 0x000F000Fu); A[1][3] = sub_pair(s1, 0x00F000F0u);
  } else if constexpr (BITS == 2) {
    const uint32_t s = w0 >> 8;
    A[0][0] = sub_pair(w0, 0x00030003u); A[0][1] = sub_pair(w0, 0x000C000Cu);
    A[1][0] = sub_pair(w0, 0x00300030u); A[1][1] = sub_pair(w0, 0x00C000C0u);
    A[0][2] = sub_pair(s, 0x00030003u);  A[0][3] = sub_pair(s, 0x000C000Cu);
    A[1][2] = sub_pair(s, 0x00300030u);  A[1][3] = sub_pair(s, 0x00C000C0u);
  } else {
    const uint32_t a = parity ? (w0 >> 8) : w0;     // half c = 0
    const uint32_t b = parity ? (w0 >> 12) : (w0 >> 4);   // half c = 1
    A[0][0] = sub_pair(a, 0x00010001u); A[0][1] = sub_pair(a, 0x00020002u);
    A[1][0] = sub_pair(a, 0x00040004u); A[1][1] = sub_pair(a, 0x00080008u);
    A[0][2] = sub_pair(b, 0x00010001u); A[0][3] = sub_pair(b, 0x00020002u);
    A[1][2] = sub_pair(b, 0x00040004u); A[1][3] = sub_pair(b, 0x00080008u);
  }
}

// The query constants of one lane, per slice pair c (entries 2*sigma + e of the pair):
// X = (0 | q) and Y = (q | -q) on (even | odd) B columns, fp16x2; z: the B operand of the
// pair's zero-point product where a kernel uses one (see decode_mma.cu).
template <int NT>
struct QFrags {
  uint4 x[NT][4], y[NT][4];
  uint2 z[NT][4];
};

// The unit's query rows (unscaled fp32, natural channel order, rows >= g.rows zero) and
// its position order into shared memory, every load of the CTA issued in one round:
// thread i < 128 takes 16-byte chunk i (row i / 16), threads < 8 the order.  Needs a CTA
// of at least 128 threads.
__device__ __forceinline__ void load_query_rows(const Geometry& g, const uint16_t* q, const uint8_t* cperm, int b,
                                                int h, int unit, float* qnat, uint8_t* perm, int tid) {
  static_assert(kMaxG * (kHeadDim / 8) == 128, "one 16-byte chunk per thread");
  const int hh = tid >> 4;
  uint4 v = make_uint4(0u, 0u, 0u, 0u), pv = make_uint4(0u, 0u, 0u, 0u);
  if (tid < 128 && hh < g.rows) v = __ldg(reinterpret_cast<const uint4*>(q + row_offset(g, b, h, hh)) + (tid & 15));
  if (tid < kHeadDim / 16) pv = __ldg(reinterpret_cast<const uint4*>(cperm + static_cast<size_t>(unit) * kHeadDim) + tid);
  if (tid < 128) {
    float4* dst = reinterpret_cast<float4*>(qnat + tid * 8);
    dst[0] = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                         __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u));
    dst[1] = make_float4(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xFFFF0000u),
                         __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xFFFF0000u));
  }
  if (tid < kHeadDim / 16) reinterpret_cast<uint4*>(perm)[tid] = pv;
}

// Dynamic query-channel pruning of the unit's query rows in shared memory (qnat, fp32
// [kMaxG][128], natural channel order): row v drops the g.n_prune pairs of smallest
// squared pair norm fl(fl(a*a) + fl(b*b)), never pair 0, the higher pair index first among
// equal norms, by zeroing both channels.  Warp w handles rows w, w + nwarps, ...; lane l
// ranks pairs l and l + 32 against all 63 candidates with shuffles.
__device__ __forceinline__ void prune_query_rows(const Geometry& g, float* qnat, int warp, int nwarps) {
  const int lane = threadIdx.x & 31;
  for (int v = warp; v < g.rows; v += nwarps) {
    float* row = qnat + v * kHeadDim;
    float n2[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) n2[e] = pair_norm2(row[lane + 32 * e], row[lane + 32 * e + 64]);
    // pair p is pruned when fewer than n_prune candidates (pairs 1..63) precede it in the
    // order (norm ascending, index descending)
    int before[2] = {0, 0};
#pragma unroll 4
    for (int src = 0; src < 32; ++src) {
#pragma unroll
      for (int e2 = 0; e2 < 2; ++e2) {
        const float o = __shfl_sync(0xffffffffu, n2[e2], src);
        const int po = src + 32 * e2;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int p = lane + 32 * e;
          before[e] += (po >= 1 && po != p && (o < n2[e] || (o == n2[e] && po > p))) ? 1 : 0;
        }
      }
    }
    __syncwarp();
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int p = lane + 32 * e;
      if (p >= 1 && before[e] < g.n_prune) {
        row[p] = 0.f;
        row[p + 64] = 0.f;
      }
    }
  }
}

// Key-slice pruning of a unit's query rows (qnat fp32 [g.rows][128], natural channel order;
// perm the unit's position order): the g.n_prune_slices slices of the low-precision block of
// least energy sum_v sum_{j in slice} q_v[perm[j]]^2 (rows ascending, positions ascending,
// each square and partial sum rounded to fp32), among those holding neither channel 0 nor
// channel 64, the higher slice first among equal energies.  Every warp computes the decision
// (the same one) with lane = 4 * slice + row-in-block; the caller zeroes the channels with
// zero_pruned_slices after a barrier.  Returns the pruned-slice mask (bit sigma).
__device__ __forceinline__ uint32_t pruned_slices(const Geometry& g, const float* qnat, const uint8_t* perm) {
  const int lane = threadIdx.x & 31;
  const int sl = lane >> 2, rl = lane & 3;
  const int nls = 8 - g.nhs, sigma = g.nhs + sl;
  const bool live = sl < nls;
  int chan[16];
  bool protect = false;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    chan[j] = live ? (perm[16 * sigma + j] & (kHeadDim - 1)) : 0;
    protect |= (chan[j] & 63) == 0;
  }
  float E = 0.f;   // lanes rl == 0: the slice's energy, rows in order
  for (int v0 = 0; v0 < g.rows; v0 += 4) {
    const int v = v0 + rl;
    float e = 0.f;
    if (live && v < g.rows) {
      const float* row = qnat + v * kHeadDim;
#pragma unroll
      for (int j = 0; j < 16; ++j) e = __fadd_rn(e, __fmul_rn(row[chan[j]], row[chan[j]]));
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float er = __shfl_sync(0xffffffffu, e, (lane & ~3) | r);
      if (v0 + r < g.rows) E = __fadd_rn(E, er);
    }
  }
  const bool cand = live && !protect;
  int before = 0;   // candidates pruned ahead of this slice: (energy, higher slice first)
#pragma unroll
  for (int o = 0; o < 8; ++o) {
    const float Eo = __shfl_sync(0xffffffffu, E, 4 * o);
    const bool co = __shfl_sync(0xffffffffu, cand, 4 * o);
    before += (co && o != sl && (Eo < E || (Eo == E && o > sl))) ? 1 : 0;
  }
  const uint32_t ball = __ballot_sync(0xffffffffu, cand && before < g.n_prune_slices && rl == 0);
  uint32_t mask = 0;
#pragma unroll
  for (int o = 0; o < 8; ++o)
    if ((ball >> (4 * o)) & 1u) mask |= 1u << (g.nhs + o);
  return mask;
}

// Zero the channels of the pruned slices (mask from pruned_slices) in every query row.
__device__ __forceinline__ void zero_pruned_slices(const Geometry& g, float* qnat, const uint8_t* perm, uint32_t mask,
                                                   int tid, int nthreads) {
  for (int i = tid; i < g.rows * kHeadDim; i += nthreads) {
    const int j = i & (kHeadDim - 1);
    if ((mask >> (j >> 4)) & 1u) qnat[(i >> 7) * kHeadDim + (perm[j] & (kHeadDim - 1))] = 0.f;
  }
}

// The residual item: up to 31 bf16 tokens staged in shared memory, with CUDA cores, heads
// h0, h0 + hstep, ... one at a time (few registers).  Lane = token for the logit (its K
// row, q in natural channel order), lane = channel for the values.  Writes one partial
// per head into `slot`.
__device__ __noinline__ void residual_partial(const Geometry& g, const uint16_t* rk, const uint16_t* rv,
                                              int nr, const float* qnat, float qscale, float* slot, int h0,
                                              int hstep, int tok0, int vis_base, int kstride = kResidKStride) {
  const int lane = threadIdx.x & 31;
  const uint4* row = reinterpret_cast<const uint4*>(rk + (lane < nr ? lane : 0) * kstride);
#pragma unroll 1
  for (int hh = h0; hh < g.rows; hh += hstep) {
    // residual row `lane` is token tok0 + lane; row hh sees tokens below vis_base + hh / G
    const bool vis = lane < nr && tok0 + lane < vis_base + hh / g.G;
    const float* qh = qnat + hh * kHeadDim;
    float lg = 0.f;
#pragma unroll 4
    for (int c8 = 0; c8 < 16; ++c8) {
      const uint4 kv = row[c8];
      const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float k = __uint_as_float((e & 1) ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16));
        lg = fmaf(qh[c8 * 8 + e], k, lg);
      }
    }
    lg = vis ? lg * qscale : -INFINITY;
    float m = lg;
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float pw = vis ? exp2f(lg - m) : 0.f;   // (m = -inf only when no token is visible)
    float l = pw;
#pragma unroll
    for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int t = 0; t < nr; ++t) {
      const float pt = __shfl_sync(0xffffffffu, pw, t);
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = fmaf(pt, bf16_bits_to_float(rv[t * kHeadDim + lane + 32 * i]), acc[i]);
    }
    float* s = slot + hh * kPartialStride;
    if (lane == 0) {
      s[0] = m;
      s[1] = l;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) s[2 + lane + 32 * i] = acc[i];
  }
}

}  // namespace
}  // namespace pnmix
