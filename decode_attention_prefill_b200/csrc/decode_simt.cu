// decode_simt.cu -- plain CUDA-core decode attention over the packed cache.
//
// The straightforward formulation, kept as the readable baseline of the tensor-core
// kernel in decode_mma.cu (selected with decode_kernel = PNMIX_DECODE_SIMT in the
// config): lane = token for q.k^, lane = channel for p.v^, fp32 online softmax per warp.  Same work partition and
// fused combine as the tensor-core kernel (decode_common.cuh).
#include "common.cuh"
#include "decode_common.cuh"

namespace pnmix {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

struct WarpState {
  float m[kMaxG], l[kMaxG], acc[kMaxG][4];
};

// Online-softmax update with this lane's logits (log2 domain) for token `lane`;
// `vhat(t, i)` returns the dequantized value of token t, channel lane + 32*i.
template <typename VFn>
__device__ __forceinline__ void absorb(WarpState& st, int G, float (&lg)[kMaxG], int ntok, VFn vhat) {
  float p[kMaxG];
#pragma unroll
  for (int hh = 0; hh < kMaxG; ++hh) {
    if (hh >= G) break;
    float gm = warp_max(lg[hh]);
    float mn = fmaxf(st.m[hh], gm);
    float alpha = exp2f(st.m[hh] - mn);
    p[hh] = exp2f(lg[hh] - mn);
    st.l[hh] = st.l[hh] * alpha + warp_sum(p[hh]);
#pragma unroll
    for (int i = 0; i < 4; ++i) st.acc[hh][i] *= alpha;
    st.m[hh] = mn;
  }
  for (int t = 0; t < ntok; ++t) {
    float v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = vhat(t, i);
#pragma unroll
    for (int hh = 0; hh < kMaxG; ++hh) {
      if (hh >= G) break;
      float pt = __shfl_sync(0xffffffffu, p[hh], t);
#pragma unroll
      for (int i = 0; i < 4; ++i) st.acc[hh][i] = fmaf(pt, v[i], st.acc[hh][i]);
    }
  }
}

__global__ void __launch_bounds__(kThreads)
decode_simt_kernel(Geometry g, const uint16_t* __restrict__ q, pnmix_cache c, float* __restrict__ out,
                   DecodeWs ws) {
  const int G = g.G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  __shared__ float qs[kMaxG][kHeadDim];
  __shared__ uint8_t perm_s[kHeadDim];
  __shared__ float part[kWarps][kMaxG][2 + kHeadDim];

  for_each_segment(g, c.len, ws.N, [&](const Segment& s) {
    const int b = s.b, h = s.h, unit = s.unit;
    perm_s[tid] = c.perm[static_cast<size_t>(unit) * kHeadDim + tid] & (kHeadDim - 1);
    __syncthreads();
    const float qscale = g.scale * 1.4426950408889634f;   // logits in the log2 domain
    for (int i = tid; i < G * kHeadDim; i += kThreads) {
      int hh = i / kHeadDim, j = i % kHeadDim;
      qs[hh][j] = bf16_bits_to_float(q[(static_cast<size_t>(b) * g.Hq + h * G + hh) * kHeadDim + perm_s[j]]) * qscale;
    }
    __syncthreads();

    WarpState st;
#pragma unroll
    for (int hh = 0; hh < kMaxG; ++hh) {
      st.m[hh] = -INFINITY;
      st.l[hh] = 0.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i) st.acc[hh][i] = 0.0f;
    }

    const int gend = s.hi < s.ng ? s.hi : s.ng;
    for (int grp = s.lo + warp; grp < gend; grp += kWarps) {
      const uint8_t* rec = record_ptr(g, c.records, b, h, grp);
      const uint16_t* ks = reinterpret_cast<const uint16_t*>(rec + rec_kscale(g));
      const uint16_t* kz = reinterpret_cast<const uint16_t*>(rec + rec_kzero(g));
      float lg[kMaxG];
#pragma unroll
      for (int hh = 0; hh < kMaxG; ++hh) lg[hh] = 0.0f;
      for (int j = 0; j < kHeadDim; ++j) {
        int off, bit, bits;
        key_code_loc(g, lane, j, off, bit, bits);
        uint32_t word = *reinterpret_cast<const uint32_t*>(rec + off);
        float code = static_cast<float>((word >> bit) & ((1u << bits) - 1u));
        int si = kscale_index(j);
        float khat = fmaf(code, __half2float(__ushort_as_half(ks[si])), __half2float(__ushort_as_half(kz[si])));
#pragma unroll
        for (int hh = 0; hh < kMaxG; ++hh)
          if (hh < G) lg[hh] = fmaf(qs[hh][j], khat, lg[hh]);
      }
      const uint8_t* vc = rec + rec_vcode(g);
      const uint16_t* vs = reinterpret_cast<const uint16_t*>(rec + rec_vscale(g));
      const uint16_t* vz = reinterpret_cast<const uint16_t*>(rec + rec_vzero(g));
      absorb(st, G, lg, kGroup, [&](int t, int i) {
        int ch = lane + 32 * i;
        int off, bit;
        value_code_loc(t, ch, off, bit);
        uint32_t word = *reinterpret_cast<const uint32_t*>(vc + off);
        float code = static_cast<float>((word >> bit) & 3u);
        return fmaf(code, __half2float(__ushort_as_half(vs[vscale_index(t, i)])),
                    __half2float(__ushort_as_half(vz[vzero_index(t, i)])));
      });
    }

    // the residual item, if this segment holds it, goes to the warp next in turn
    if (s.hi > s.ng && s.nr > 0 && warp == ((s.ng - s.lo) & (kWarps - 1))) {
      const uint16_t* rk = c.k_resid + static_cast<size_t>(unit) * kGroup * kHeadDim;
      const uint16_t* rv = c.v_resid + static_cast<size_t>(unit) * kGroup * kHeadDim;
      const int nr = s.nr;
      float lg[kMaxG];
#pragma unroll
      for (int hh = 0; hh < kMaxG; ++hh) lg[hh] = 0.0f;
      if (lane < nr) {
        for (int j = 0; j < kHeadDim; ++j) {
          float khat = bf16_bits_to_float(rk[lane * kHeadDim + perm_s[j]]);
#pragma unroll
          for (int hh = 0; hh < kMaxG; ++hh)
            if (hh < G) lg[hh] = fmaf(qs[hh][j], khat, lg[hh]);
        }
      } else {
#pragma unroll
        for (int hh = 0; hh < kMaxG; ++hh) lg[hh] = -INFINITY;
      }
      absorb(st, G, lg, nr, [&](int t, int i) { return bf16_bits_to_float(rv[t * kHeadDim + lane + 32 * i]); });
    }

    // merge the warps of this CTA into the segment's partial
    if (lane == 0) {
      for (int hh = 0; hh < G; ++hh) {
        part[warp][hh][0] = st.m[hh];
        part[warp][hh][1] = st.l[hh];
      }
    }
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int i = 0; i < 4; ++i) part[warp][hh][2 + lane + 32 * i] = st.acc[hh][i];
    __syncthreads();
    float* slot = partial_slot(ws, unit, G);
    for (int hh = 0; hh < G; ++hh) {
      float m = -INFINITY;
      for (int w = 0; w < kWarps; ++w) m = fmaxf(m, part[w][hh][0]);
      float l = 0.0f, a = 0.0f;
      if (m != -INFINITY) {
        for (int w = 0; w < kWarps; ++w) {
          if (part[w][hh][0] == -INFINITY) continue;
          float f = exp2f(part[w][hh][0] - m);
          l += part[w][hh][1] * f;
          a += part[w][hh][2 + tid] * f;
        }
      }
      float* p = slot + hh * kPartialStride;
      if (tid == 0) {
        p[0] = m;
        p[1] = l;
      }
      p[2 + tid] = a;
    }
    combine_segment(ws, s, G, out, g);   // one query per sequence here (g.tq == 1)
  });
}

}  // namespace

cudaError_t launch_decode_simt(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax,
                               float* out, DecodeWs ws, cudaStream_t s) {
  int dev = 0, sms = 148, occ = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_simt_kernel, kThreads, 0);
  int n = sms * (occ > 0 ? occ : 1);
  ws.N = n < nmax ? n : nmax;
  decode_simt_kernel<<<ws.N, kThreads, 0, s>>>(g, q, c, out, ws);
  return cudaGetLastError();
}

}  // namespace pnmix
