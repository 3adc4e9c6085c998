// decode_common.cuh -- split-K workspace and the fused combine of the decode kernels.
//
// Every CTA of a (b, KV head) writes one partial (m, l, acc[128]) per query head of the
// group; m is the running max in the log2 domain, l the sum of 2^(logit - m) and acc the
// matching weighted sum of values.  The CTA that takes the last ticket of its unit merges
// the S partials:  m* = max m_s,  out = sum_s acc_s 2^(m_s - m*) / sum_s l_s 2^(m_s - m*).
// Nothing waits: the other CTAs simply exit after taking their ticket.
#pragma once

#include "common.cuh"

namespace pnmix {

constexpr int kPartialStride = 2 + kHeadDim;   // m, l, acc[128]

struct DecodeWs {
  float* part;         // [units][S][G][kPartialStride]
  uint32_t* tickets;   // [units], zero between calls
};

__host__ __device__ __forceinline__ size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ __forceinline__ size_t decode_partial_bytes(int units, int S, int G) {
  return align256(sizeof(float) * static_cast<size_t>(units) * S * G * kPartialStride);
}

__device__ __forceinline__ void write_partial(const DecodeWs& ws, int unit, int split, int S, int G,
                                              int hh, int c, float m, float l, float acc) {
  float* p = ws.part + ((static_cast<size_t>(unit) * S + split) * G + hh) * kPartialStride;
  if (c == 0) {
    p[0] = m;
    p[1] = l;
  }
  p[2 + c] = acc;
}

// Called by every thread of a CTA after its partials are written.  out_unit points at
// out[b][h*G][0] (G rows of 128 floats).
__device__ __forceinline__ void combine_if_last(const DecodeWs& ws, int unit, int split, int S, int G,
                                                float* out_unit) {
  __shared__ int is_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(ws.tickets + unit, 1u) == static_cast<unsigned>(S - 1));
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  const float* base = ws.part + static_cast<size_t>(unit) * S * G * kPartialStride;
  for (int i = threadIdx.x; i < G * kHeadDim; i += blockDim.x) {
    const int hh = i / kHeadDim, c = i % kHeadDim;
    float m = -INFINITY;
    for (int s = 0; s < S; ++s) m = fmaxf(m, __ldcg(base + (static_cast<size_t>(s) * G + hh) * kPartialStride));
    float den = 0.0f, num = 0.0f;
    if (m != -INFINITY) {
      for (int s = 0; s < S; ++s) {
        const float* p = base + (static_cast<size_t>(s) * G + hh) * kPartialStride;
        float ms = __ldcg(p);
        if (ms == -INFINITY) continue;
        float f = exp2f(ms - m);
        den = fmaf(__ldcg(p + 1), f, den);
        num = fmaf(__ldcg(p + 2 + c), f, num);
      }
    }
    out_unit[static_cast<size_t>(hh) * kHeadDim + c] = den > 0.0f ? num / den : 0.0f;
  }
  if (threadIdx.x == 0) ws.tickets[unit] = 0u;
}

cudaError_t launch_decode_simt(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int S,
                               float* out, DecodeWs ws, cudaStream_t s);

}  // namespace pnmix
