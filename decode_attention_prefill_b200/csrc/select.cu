// select.cu -- prefill pair saliency and top-k selection (PN-Mix abstract: salient RoPE
// channel pairs are those with a large query pair-norm x key pair-norm product; they are
// picked once at prefill and reused for the whole decode).
//
// One launch, grid (splits, B*Hkv):
//   every CTA reduces max_t (k_{t,p}^2 + k_{t,p+64}^2) over its token slice with 16-byte
//   loads and merges it into a per-unit scratch array with atomicMax on the float bits
//   (non-negative floats order like their bit patterns, and max is order-free, so the
//   split is exact); for the range statistic it also reduces every channel's min and max
//   (atomicMax on an order-preserving integer image of the float, and on its complement
//   for the minimum, so that zero means "no value" for both);
//   the last CTA of a unit (atomic ticket, no waiting) forms the query pair norms of the
//   G x W window, sums them sequentially in the reference order (heads outer, tokens
//   inner), builds the scores of the configured statistic, selects the top k with warp
//   shuffles and sets the unit's accumulators and ticket back to zero, so a call needs no
//   clearing beforehand (the cache starts zero-filled).
#include <atomic>

#include "common.cuh"

namespace pnmix {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerIter = kThreads / 8;   // 8 threads per 128-channel row

// Pair norms of 8 consecutive pairs p = 8*c .. 8*c+7 of one row, from the two 16-byte
// chunks (channels 8c..8c+7 and 64+8c..64+8c+7); with RANGE also the 16 channel values.
template <bool RANGE = false>
__device__ __forceinline__ void chunk_pair_norm2(const uint4& lo, const uint4& hi, float out[8],
                                                 float* mn = nullptr, float* mx = nullptr) {
  const uint16_t* a = reinterpret_cast<const uint16_t*>(&lo);
  const uint16_t* b = reinterpret_cast<const uint16_t*>(&hi);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float x = bf16_bits_to_float(a[i]), y = bf16_bits_to_float(b[i]);
    out[i] = pair_norm2(x, y);
    if constexpr (RANGE) {
      mn[i] = fminf(mn[i], x);
      mx[i] = fmaxf(mx[i], x);
      mn[8 + i] = fminf(mn[8 + i], y);
      mx[8 + i] = fmaxf(mx[8 + i], y);
    }
  }
}
constexpr int kRowUnroll = 4;   // rows per thread per pass: 8 independent 16-byte loads in flight
constexpr int kQnRows = 3 * kRowsPerIter;   // query-window rows per round of the last CTA

// Order-preserving map of non-NaN floats to unsigned integers (and back), so that
// integer atomics compute float min / max.
__device__ __forceinline__ uint32_t ordered_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ordered_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <int SCORE>
__global__ void __launch_bounds__(kThreads)
select_pairs_kernel(Geometry g, const uint16_t* __restrict__ q_window, int n_window,
                    const uint16_t* __restrict__ k, int L, int ld, pnmix_cache c) {
  constexpr bool RANGE = SCORE == PNMIX_SCORE_RANGE_QUERY;
  const int unit = blockIdx.y;
  const int b = unit / g.Hkv, h = unit % g.Hkv;
  const int nsplit = gridDim.x, split = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cidx = tid & 7;          // chunk index: pairs 8*cidx .. 8*cidx+7
  const int rsub = tid >> 3;         // row within an iteration

  __shared__ float red[kThreads / 32][64];
  __shared__ float qn[kQnRows][64];
  __shared__ float score_s[64];
  __shared__ float rmin[RANGE ? kThreads / 32 : 1][128], rmax[RANGE ? kThreads / 32 : 1][128];
  __shared__ int is_last;

  uint32_t* kmax = c.scratch + scratch_kmax_offset() + static_cast<size_t>(unit) * 64;
  uint32_t* ticket = c.scratch + scratch_select_ticket_offset(g.B, g.Hkv) + unit;
  uint32_t* cmin = c.scratch + scratch_range_offset(g.B, g.Hkv) + static_cast<size_t>(unit) * 256;
  uint32_t* cmax = cmin + 128;

  // ---- key pair-norm max (and channel min / max) over this split's tokens
  const int t0 = static_cast<int>(static_cast<long long>(L) * split / nsplit);
  const int t1 = static_cast<int>(static_cast<long long>(L) * (split + 1) / nsplit);
  const uint16_t* kbase = k + unit_index(g, b, h) * static_cast<size_t>(ld) * kHeadDim;
  float m8[8];
  float mn16[RANGE ? 16 : 1], mx16[RANGE ? 16 : 1];
#pragma unroll
  for (int i = 0; i < 8; ++i) m8[i] = 0.0f;
  if constexpr (RANGE) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      mn16[i] = INFINITY;
      mx16[i] = -INFINITY;
    }
  }
  for (int t = t0 + rsub; t < t1; t += kRowUnroll * kRowsPerIter) {
    uint4 lo[kRowUnroll], hi[kRowUnroll];
#pragma unroll
    for (int u = 0; u < kRowUnroll; ++u) {   // all loads of the pass first
      const int tt = t + u * kRowsPerIter;
      if (tt < t1) {
        const uint4* row = reinterpret_cast<const uint4*>(kbase + static_cast<size_t>(tt) * kHeadDim);
        lo[u] = __ldg(row + cidx);
        hi[u] = __ldg(row + 8 + cidx);
      }
    }
#pragma unroll
    for (int u = 0; u < kRowUnroll; ++u) {
      if (t + u * kRowsPerIter < t1) {
        float n2[8];
        chunk_pair_norm2<RANGE>(lo[u], hi[u], n2, mn16, mx16);
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = fmaxf(m8[i], n2[i]);
      }
    }
  }
  // lanes with the same cidx: xor 8, 16
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    m8[i] = fmaxf(m8[i], __shfl_xor_sync(0xffffffffu, m8[i], 8));
    m8[i] = fmaxf(m8[i], __shfl_xor_sync(0xffffffffu, m8[i], 16));
  }
  if constexpr (RANGE) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      mn16[i] = fminf(mn16[i], __shfl_xor_sync(0xffffffffu, mn16[i], 8));
      mn16[i] = fminf(mn16[i], __shfl_xor_sync(0xffffffffu, mn16[i], 16));
      mx16[i] = fmaxf(mx16[i], __shfl_xor_sync(0xffffffffu, mx16[i], 8));
      mx16[i] = fmaxf(mx16[i], __shfl_xor_sync(0xffffffffu, mx16[i], 16));
    }
    if (lane < 8) {   // channels 8*lane + i and 64 + 8*lane + i
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        rmin[warp][8 * lane + i] = mn16[i];
        rmax[warp][8 * lane + i] = mx16[i];
        rmin[warp][64 + 8 * lane + i] = mn16[8 + i];
        rmax[warp][64 + 8 * lane + i] = mx16[8 + i];
      }
    }
  }
  if (lane < 8) {
#pragma unroll
    for (int i = 0; i < 8; ++i) red[warp][8 * lane + i] = m8[i];
  }
  __syncthreads();
  if (tid < 64) {
    float v = 0.0f;
    for (int w = 0; w < kThreads / 32; ++w) v = fmaxf(v, red[w][tid]);
    atomicMax(kmax + tid, __float_as_uint(v));
  }
  if constexpr (RANGE) {
    if (tid < 128 && t1 > t0) {
      float lo = INFINITY, hi = -INFINITY;
      for (int w = 0; w < kThreads / 32; ++w) {
        lo = fminf(lo, rmin[w][tid]);
        hi = fmaxf(hi, rmax[w][tid]);
      }
      atomicMax(cmin + tid, ~ordered_key(lo));   // the complement: zero is "no value yet"
      atomicMax(cmax + tid, ordered_key(hi));
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = (atomicAdd(ticket, 1u) == static_cast<unsigned>(nsplit - 1));
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // ---- query pair norms, summed in the reference order: kQnRows window rows per round,
  // all of a round's loads issued together (the G heads' windows are consecutive rows:
  // row i = head i / n_window, token i % n_window)
  float qsum = 0.0f;   // meaningful for tid < 64
  const int rows = g.G * n_window;
  const uint16_t* qrows = q_window + (static_cast<size_t>(b) * g.Hq + h * g.G) * n_window * kHeadDim;
  for (int r0 = 0; r0 < rows; r0 += kQnRows) {
    uint4 lo[kQnRows / kRowsPerIter], hi[kQnRows / kRowsPerIter];
#pragma unroll
    for (int u = 0; u < kQnRows / kRowsPerIter; ++u) {
      const int r = r0 + rsub + u * kRowsPerIter;
      if (r < rows) {
        const uint4* row = reinterpret_cast<const uint4*>(qrows + static_cast<size_t>(r) * kHeadDim);
        lo[u] = __ldg(row + cidx);
        hi[u] = __ldg(row + 8 + cidx);
      }
    }
#pragma unroll
    for (int u = 0; u < kQnRows / kRowsPerIter; ++u) {
      if (r0 + rsub + u * kRowsPerIter < rows) {
        float n2[8];
        chunk_pair_norm2(lo[u], hi[u], n2);
#pragma unroll
        for (int i = 0; i < 8; ++i) qn[rsub + u * kRowsPerIter][8 * cidx + i] = __fsqrt_rn(n2[i]);
      }
    }
    __syncthreads();
    if (tid < 64) {
      const int nr = min(kQnRows, rows - r0);
#pragma unroll 8
      for (int i = 0; i < nr; ++i) qsum = __fadd_rn(qsum, qn[i][tid]);
    }
    __syncthreads();
  }
  if (tid < 64) {
    float kp = __fsqrt_rn(__uint_as_float(__ldcg(kmax + tid)));
    float qp = __fdiv_rn(qsum, static_cast<float>(rows));
    float s;
    if constexpr (SCORE == PNMIX_SCORE_KEY_ONLY) {
      s = kp;
    } else if constexpr (RANGE) {
      const float r0 = __fsub_rn(ordered_value(__ldcg(cmax + tid)), ordered_value(~__ldcg(cmin + tid)));
      const float r1 = __fsub_rn(ordered_value(__ldcg(cmax + 64 + tid)), ordered_value(~__ldcg(cmin + 64 + tid)));
      s = __fmul_rn(qp, __fsqrt_rn(__fadd_rn(__fmul_rn(r0, r0), __fmul_rn(r1, r1))));
    } else {
      s = __fmul_rn(qp, kp);
    }
    score_s[tid] = s;
    c.pair_scores[static_cast<size_t>(unit) * 64 + tid] = s;
  }
  __syncthreads();
  // leave the unit's accumulators and ticket at zero for the next call (every CTA of the
  // unit has added to them, and the scores above have read them)
  if (tid < 64) kmax[tid] = 0u;
  if constexpr (RANGE) {
    cmin[tid] = 0u;   // 256 threads: 128 minima then 128 maxima
  }
  if (tid == 0) *ticket = 0u;

  // ---- top k by (score desc, pair asc): rank of every pair, by warp shuffles
  if (warp == 0) {
    // key = (score bits << 8) | (63 - p): unique, larger key = better
    unsigned long long key0 =
        (static_cast<unsigned long long>(__float_as_uint(score_s[lane])) << 8) | (63 - lane);
    unsigned long long key1 =
        (static_cast<unsigned long long>(__float_as_uint(score_s[lane + 32])) << 8) | (31 - lane);
    int rank0 = 0, rank1 = 0;
    for (int i = 0; i < 32; ++i) {
      unsigned long long o0 = __shfl_sync(0xffffffffu, key0, i);
      unsigned long long o1 = __shfl_sync(0xffffffffu, key1, i);
      rank0 += (o0 > key0) + (o1 > key0);
      rank1 += (o0 > key1) + (o1 > key1);
    }
    unsigned sel_lo = __ballot_sync(0xffffffffu, rank0 < g.k);
    unsigned sel_hi = __ballot_sync(0xffffffffu, rank1 < g.k);
    unsigned long long mask = (static_cast<unsigned long long>(sel_hi) << 32) | sel_lo;
    if (lane == 0) c.pair_mask[unit] = mask;
    // pair indices (salient pairs ascending, then zeros) and the position order (salient
    // channels ascending, then the others ascending): every lane places its own entries,
    // the position of each from a population count of the mask below it
    uint8_t* idx = c.pair_idx + static_cast<size_t>(unit) * 64;
    uint8_t* perm = c.perm + static_cast<size_t>(unit) * 128;
    const int k = __popcll(mask);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int p = lane + 32 * e;
      const int below = __popcll(mask & ((1ull << p) - 1ull));   // salient pairs below p
      if ((mask >> p) & 1ull) idx[below] = static_cast<uint8_t>(p);
      if (p >= k) idx[p] = 0;   // entries k..63: zero (none of them is a salient slot)
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int ch = lane + 32 * e, p = ch & 63;
      const int below = __popcll(mask & ((1ull << p) - 1ull)) + (ch >= 64 ? k : 0);   // salient channels below ch
      const int pos = ((mask >> p) & 1ull) ? below : 2 * k + (ch - below);
      perm[pos] = static_cast<uint8_t>(ch);
    }
  }
}

// Resident CTAs of one full wave of a select instance on the current device (the occupancy
// query runs once per instance and device).
template <typename K>
cudaError_t resident_ctas(K kern, int* out) {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> cache[3][kMaxDevices];
  const int which = kern == select_pairs_kernel<PNMIX_SCORE_KEY_ONLY> ? 1
                    : kern == select_pairs_kernel<PNMIX_SCORE_RANGE_QUERY> ? 2 : 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cacheable = dev >= 0 && dev < kMaxDevices;
  int v = cacheable ? cache[which][dev].load(std::memory_order_relaxed) : 0;
  if (v == 0) {
    int sms = 0, occ = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, 0);
    if (e != cudaSuccess) return e;
    v = sms * (occ > 0 ? occ : 1);
    if (cacheable) cache[which][dev].store(v, std::memory_order_relaxed);
  }
  *out = v;
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_select_pairs(const Geometry& g, const uint16_t* q_window, int n_window,
                                const uint16_t* k, int L, int ld, const pnmix_cache& c,
                                cudaStream_t s) {
  const int units = g.B * g.Hkv;
  // one wave: as many token splits per unit as the resident CTAs allow (the max pass then
  // ends together on every SM), with >= 256 tokens per CTA (two passes of kRowUnroll rows
  // per thread)
  auto kern = select_pairs_kernel<PNMIX_SCORE_PNMIX>;
  if (g.score == PNMIX_SCORE_KEY_ONLY) kern = select_pairs_kernel<PNMIX_SCORE_KEY_ONLY>;
  if (g.score == PNMIX_SCORE_RANGE_QUERY) kern = select_pairs_kernel<PNMIX_SCORE_RANGE_QUERY>;
  int resident = 0;
  cudaError_t e = resident_ctas(kern, &resident);
  if (e != cudaSuccess) return e;
  int want = resident / units;
  int max_split = (L + 255) / 256;
  int nsplit = want < max_split ? want : max_split;
  if (nsplit < 1) nsplit = 1;
  if (nsplit > 512) nsplit = 512;
  dim3 grid(nsplit, units);
  kern<<<grid, kThreads, 0, s>>>(g, q_window, n_window, k, L, ld, c);
  return cudaGetLastError();
}

}  // namespace pnmix
