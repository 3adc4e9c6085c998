// mix.cu -- token-level two-precision mixing ("SemKV: Semantic Mixed-Precision KV Cache
// Quantization Guided by the Quality Cliff for Long-Context LLM Inference", abstract:
// every token is kept, tokens are ranked by a model-internal score and take one of two
// adjacent precisions by rank).
//
// In this path the unit of assignment is a 32-token group, because the tokens of a group
// share the per-channel key statistics.  The score of a group is the largest logit that the
// mean query of the saliency window gives one of its tokens:
//   qbar[c]  = (sum over the G heads and the window tokens of q[c]) / (G * W'),
//              heads outer, tokens inner;
//   l_t      = sum_c qbar[c] * k[t][c], channels in order;
//   score[g] = max over the group's tokens of l_t, first occurrence kept;
// every operation one fp32 rounding (explicit _rn intrinsics, no contraction), so the
// scores, and the route they decide, are bit-exact with the plain definition.  The best
// n_hi groups (rank by score, ties to the lower index) form the high-precision part, the
// others and the ragged tail the low-precision part; each part's K / V rows are gathered in
// ascending token order into its own buffers, ready for the ordinary quantizers.
//
// route_kernel: one CTA of 256 threads per (sequence, KV head).  The token logits run one
// token per thread (eight groups per pass, one warp per group), the group maxima one thread
// per group over the staged logits, and the ranking one thread per group over all of the
// unit's scores (ng^2 comparisons: a prefill-time cost).
// split_kernel: one CTA per (group, KV head, sequence), plus one per unit for the tail.
#include "common.cuh"

namespace pnmix {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kSplitThreads = 128;

__global__ void __launch_bounds__(kRouteThreads)
route_kernel(int G, int Hq, int Hkv, const uint16_t* __restrict__ qwin, int nw, const uint16_t* __restrict__ k,
             int L, int ld, int n_hi, float* scores, uint8_t* route, int32_t* dest) {
  __shared__ float qbar[kHeadDim];
  __shared__ float logit[kRouteThreads];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int ng = L / kGroup;
  const size_t u = static_cast<size_t>(b) * Hkv + h;

  // ---- mean query of the unit's saliency window
  if (tid < kHeadDim) {
    float s = 0.f;
    for (int hh = 0; hh < G; ++hh) {
      const uint16_t* col = qwin + ((static_cast<size_t>(b) * Hq + h * G + hh) * nw) * kHeadDim + tid;
      for (int t = 0; t < nw; ++t) s = __fadd_rn(s, bf16_bits_to_float(col[static_cast<size_t>(t) * kHeadDim]));
    }
    qbar[tid] = __fdiv_rn(s, static_cast<float>(G * nw));
  }
  __syncthreads();

  // ---- group scores: 256 tokens (8 groups) per pass
  float* sc = scores + u * ng;
  const uint16_t* ku = k + u * static_cast<size_t>(ld) * kHeadDim;
  for (int base = 0; base < ng * kGroup; base += kRouteThreads) {
    const int t = base + tid;
    float acc = 0.f;
    if (t < ng * kGroup) {
      const uint4* row = reinterpret_cast<const uint4*>(ku + static_cast<size_t>(t) * kHeadDim);
      for (int c8 = 0; c8 < kHeadDim / 8; ++c8) {
        const uint4 w = row[c8];
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {   // channel c8*8 + 2e in the low half, + 1 in the high half
          acc = __fadd_rn(acc, __fmul_rn(qbar[c8 * 8 + 2 * e], __uint_as_float(wv[e] << 16)));
          acc = __fadd_rn(acc, __fmul_rn(qbar[c8 * 8 + 2 * e + 1], __uint_as_float(wv[e] & 0xFFFF0000u)));
        }
      }
    }
    logit[tid] = acc;
    __syncthreads();
    if (tid < kRouteThreads / kGroup) {
      const int g = base / kGroup + tid;
      if (g < ng) {
        float best = -INFINITY;
        for (int i = 0; i < kGroup; ++i) {
          const float x = logit[tid * kGroup + i];
          if (x > best) best = x;
        }
        sc[g] = best;
      }
    }
    __syncthreads();
  }

  // ---- rank and route (the block's own score writes are visible after the barrier)
  for (int g = tid; g < ng; g += kRouteThreads) {
    const float s = sc[g];
    int r = 0;
    for (int o = 0; o < ng; ++o) {
      const float x = sc[o];
      r += (x > s || (x == s && o < g)) ? 1 : 0;
    }
    route[u * ng + g] = r < n_hi ? 1 : 0;
  }
  __syncthreads();
  // ---- place of each group inside its part: earlier groups with the same route
  for (int g = tid; g < ng; g += kRouteThreads) {
    const uint8_t mine = route[u * ng + g];
    int d = 0;
    for (int o = 0; o < g; ++o) d += route[u * ng + o] == mine ? 1 : 0;
    dest[u * ng + g] = d;
  }
}

__global__ void __launch_bounds__(kSplitThreads)
split_kernel(int Hkv, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v, int L, int ld, int n_hi,
             const uint8_t* __restrict__ route, const int32_t* __restrict__ dest, uint16_t* k_hi, uint16_t* v_hi,
             uint16_t* k_lo, uint16_t* v_lo) {
  const int item = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int ng = L / kGroup, L_hi = kGroup * n_hi, L_lo = L - L_hi;
  const size_t u = static_cast<size_t>(b) * Hkv + h;
  bool hi;
  int src0, rows, dst0;
  if (item < ng) {   // a full group goes to its part at its place
    hi = route[u * ng + item] != 0;
    src0 = kGroup * item;
    rows = kGroup;
    dst0 = kGroup * dest[u * ng + item];
  } else {           // the ragged tail ends the low part
    hi = false;
    src0 = kGroup * ng;
    rows = L - kGroup * ng;
    dst0 = kGroup * (ng - n_hi);
  }
  if (rows == 0) return;
  const int Lp = hi ? L_hi : L_lo;
  uint4* kd = reinterpret_cast<uint4*>((hi ? k_hi : k_lo) + (u * Lp + dst0) * kHeadDim);
  uint4* vd = reinterpret_cast<uint4*>((hi ? v_hi : v_lo) + (u * Lp + dst0) * kHeadDim);
  const uint4* ks = reinterpret_cast<const uint4*>(k + (u * ld + src0) * kHeadDim);
  const uint4* vs = reinterpret_cast<const uint4*>(v + (u * ld + src0) * kHeadDim);
  for (int i = threadIdx.x; i < rows * (kHeadDim / 8); i += kSplitThreads) {
    kd[i] = ks[i];
    vd[i] = vs[i];
  }
}

}  // namespace

cudaError_t launch_split_groups(const Geometry& g, const uint16_t* q_window, int nw, const uint16_t* k,
                                const uint16_t* v, int L, int ld, int n_hi, float* scores, uint8_t* route,
                                int32_t* dest, uint16_t* k_hi, uint16_t* v_hi, uint16_t* k_lo, uint16_t* v_lo,
                                cudaStream_t s) {
  if (g.B == 0) return cudaSuccess;
  const int ng = L / kGroup;
  if (ng > 0) {
    route_kernel<<<dim3(g.Hkv, g.B), kRouteThreads, 0, s>>>(g.G, g.Hq, g.Hkv, q_window, nw, k, L, ld, n_hi, scores,
                                                           route, dest);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  split_kernel<<<dim3(ng + 1, g.Hkv, g.B), kSplitThreads, 0, s>>>(g.Hkv, k, v, L, ld, n_hi, route, dest, k_hi, v_hi,
                                                                  k_lo, v_lo);
  return cudaGetLastError();
}

}  // namespace pnmix
