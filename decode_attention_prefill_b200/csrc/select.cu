// select.cu -- prefill pair saliency and top-k selection (PN-Mix abstract: salient RoPE
// channel pairs are those with a large query pair-norm x key pair-norm product; they are
// picked once at prefill and reused for the whole decode).
//
// One launch, grid (splits, B*Hkv):
//   every CTA reduces max_t (k_{t,p}^2 + k_{t,p+64}^2) over its token slice with 16-byte
//   loads and merges it into a per-unit scratch array with atomicMax on the float bits
//   (non-negative floats order like their bit patterns, and max is order-free, so the
//   split is exact);
//   the last CTA of a unit (atomic ticket, no waiting) forms the query pair norms of the
//   G x W window, sums them sequentially in the reference order (heads outer, tokens
//   inner), builds the scores and selects the top k with warp shuffles.
#include "common.cuh"

namespace pnmix {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerIter = kThreads / 8;   // 8 threads per 128-channel row

// Pair norms of 8 consecutive pairs p = 8*c .. 8*c+7 of one row, from the two 16-byte
// chunks (channels 8c..8c+7 and 64+8c..64+8c+7).
__device__ __forceinline__ void row_pair_norm2(const uint16_t* row, int c, float out[8]) {
  uint4 lo = __ldg(reinterpret_cast<const uint4*>(row) + c);
  uint4 hi = __ldg(reinterpret_cast<const uint4*>(row) + 8 + c);
  const uint16_t* a = reinterpret_cast<const uint16_t*>(&lo);
  const uint16_t* b = reinterpret_cast<const uint16_t*>(&hi);
#pragma unroll
  for (int i = 0; i < 8; ++i) out[i] = pair_norm2(bf16_bits_to_float(a[i]), bf16_bits_to_float(b[i]));
}

__global__ void __launch_bounds__(kThreads)
select_pairs_kernel(Geometry g, const uint16_t* __restrict__ q_window, int n_window,
                    const uint16_t* __restrict__ k, int L, int ld, pnmix_cache c) {
  const int unit = blockIdx.y;
  const int b = unit / g.Hkv, h = unit % g.Hkv;
  const int nsplit = gridDim.x, split = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cidx = tid & 7;          // chunk index: pairs 8*cidx .. 8*cidx+7
  const int rsub = tid >> 3;         // row within an iteration

  __shared__ float red[kThreads / 32][64];
  __shared__ float qn[kRowsPerIter][64];
  __shared__ float score_s[64];
  __shared__ int is_last;

  uint32_t* kmax = c.scratch + scratch_kmax_offset() + static_cast<size_t>(unit) * 64;
  uint32_t* ticket = c.scratch + scratch_select_ticket_offset(g.B, g.Hkv) + unit;

  // ---- key pair-norm max over this split's tokens
  const int t0 = static_cast<int>(static_cast<long long>(L) * split / nsplit);
  const int t1 = static_cast<int>(static_cast<long long>(L) * (split + 1) / nsplit);
  const uint16_t* kbase = k + unit_index(g, b, h) * static_cast<size_t>(ld) * kHeadDim;
  float m8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m8[i] = 0.0f;
  for (int t = t0 + rsub; t < t1; t += kRowsPerIter) {
    float n2[8];
    row_pair_norm2(kbase + static_cast<size_t>(t) * kHeadDim, cidx, n2);
#pragma unroll
    for (int i = 0; i < 8; ++i) m8[i] = fmaxf(m8[i], n2[i]);
  }
  // lanes with the same cidx: xor 8, 16
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    m8[i] = fmaxf(m8[i], __shfl_xor_sync(0xffffffffu, m8[i], 8));
    m8[i] = fmaxf(m8[i], __shfl_xor_sync(0xffffffffu, m8[i], 16));
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
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = (atomicAdd(ticket, 1u) == static_cast<unsigned>(nsplit - 1));
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // ---- query pair norms, summed in the reference order
  float qsum = 0.0f;   // meaningful for tid < 64
  const int rows = g.G * n_window;   // row i = head (i / n_window), token (i % n_window)
  for (int r0 = 0; r0 < rows; r0 += kRowsPerIter) {
    int r = r0 + rsub;
    if (r < rows) {
      int hh = r / n_window, tt = r % n_window;
      const uint16_t* row =
          q_window + ((static_cast<size_t>(b) * g.Hq + h * g.G + hh) * n_window + tt) * kHeadDim;
      float n2[8];
      row_pair_norm2(row, cidx, n2);
#pragma unroll
      for (int i = 0; i < 8; ++i) qn[rsub][8 * cidx + i] = __fsqrt_rn(n2[i]);
    }
    __syncthreads();
    if (tid < 64) {
      int nr = min(kRowsPerIter, rows - r0);
      for (int i = 0; i < nr; ++i) qsum = __fadd_rn(qsum, qn[i][tid]);
    }
    __syncthreads();
  }
  if (tid < 64) {
    float kp = __fsqrt_rn(__uint_as_float(__ldcg(kmax + tid)));
    float qp = __fdiv_rn(qsum, static_cast<float>(rows));
    float s = __fmul_rn(qp, kp);
    score_s[tid] = s;
    c.pair_scores[static_cast<size_t>(unit) * 64 + tid] = s;
  }
  __syncthreads();

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
    if (lane == 0) {
      c.pair_mask[unit] = mask;
      uint8_t* idx = c.pair_idx + static_cast<size_t>(unit) * 64;
      int n = 0;
      for (int p = 0; p < 64; ++p)
        if ((mask >> p) & 1ull) idx[n++] = static_cast<uint8_t>(p);
      for (; n < 64; ++n) idx[n] = 0;
      uint8_t* perm = c.perm + static_cast<size_t>(unit) * 128;
      n = 0;
      for (int ch = 0; ch < 128; ++ch)
        if ((mask >> (ch & 63)) & 1ull) perm[n++] = static_cast<uint8_t>(ch);
      for (int ch = 0; ch < 128; ++ch)
        if (!((mask >> (ch & 63)) & 1ull)) perm[n++] = static_cast<uint8_t>(ch);
    }
  }
}

}  // namespace

cudaError_t launch_select_pairs(const Geometry& g, const uint16_t* q_window, int n_window,
                                const uint16_t* k, int L, int ld, const pnmix_cache& c,
                                cudaStream_t s) {
  const int units = g.B * g.Hkv;
  // scratch (max-norm accumulators and tickets) starts at zero for every call
  cudaError_t e = cudaMemsetAsync(c.scratch, 0, sizeof(uint32_t) * static_cast<size_t>(units) * 65, s);
  if (e != cudaSuccess) return e;
  // about eight CTAs per SM so the max pass balances, with >= 128 tokens per CTA
  int want = (8 * 148 + units - 1) / units;
  int max_split = (L + 127) / 128;
  int nsplit = want < max_split ? want : max_split;
  if (nsplit < 1) nsplit = 1;
  if (nsplit > 512) nsplit = 512;
  dim3 grid(nsplit, units);
  select_pairs_kernel<<<grid, kThreads, 0, s>>>(g, q_window, n_window, k, L, ld, c);
  return cudaGetLastError();
}

}  // namespace pnmix
