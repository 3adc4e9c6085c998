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
// score_kernel: grid (chunks, KV heads, sequences); a CTA rebuilds the unit's mean query
// (the same sequential sums everywhere, so every CTA gets the same bits) and scores a run
// of groups (one wave of CTAs in all), one token per thread for the logits (rows staged
// through shared memory by coalesced loads) and one thread per group for the maxima.
// route_kernel: one CTA per (sequence, KV head).  The n_hi best groups are those whose key
// (score, then lower index) is at least the n_hi-th largest key, found by a radix select
// over the order-preserving bits of the score (four 8-bit digits, most significant
// first) and then, among the groups whose score equals the threshold, the lowest
// indices; a group's place inside its part is the count of earlier groups with the same
// route (a block-wide prefix sum).  O(ng) work per pass instead of ng^2 comparisons.
// split_kernel: one CTA per (group, KV head, sequence), plus one per unit for the tail.
#include <atomic>

#include "common.cuh"

namespace pnmix {
namespace {

constexpr int kScoreThreads = 128;
constexpr int kScoreMinGroups = 4;     // groups scored by one CTA at least (one pass)
constexpr int kStageRow = 272;         // bytes per staged key row (256 + 16 of padding)
constexpr int kRouteThreads = 1024;
constexpr int kSplitThreads = 128;

constexpr int kScoreStageBytes = (kScoreThreads / 32) * 2 * 32 * kStageRow;   // two stages per warp
static_assert(kScoreThreads == kHeadDim, "one score thread per channel for the mean query");

__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src), "r"(src_bytes)
               : "memory");
}

__global__ void __launch_bounds__(kScoreThreads)
score_kernel(int G, int Hq, int Hkv, const uint16_t* __restrict__ qwin, int nw, const uint16_t* __restrict__ k,
             int L, int ld, int gpc, float* scores) {
  __shared__ __align__(16) float qbar[kHeadDim];
  __shared__ float logit[kScoreThreads];
  extern __shared__ __align__(16) uint8_t stage[];   // [warps][2][32 rows][kStageRow]
  const int h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int ng = L / kGroup;
  const int gbeg = blockIdx.x * gpc;
  const int gend = min(ng, gbeg + gpc);
  const size_t u = static_cast<size_t>(b) * Hkv + h;
  float* sc = scores + u * ng;
  const uint16_t* ku = k + u * static_cast<size_t>(ld) * kHeadDim;
  const int lane = tid & 31, warp = tid >> 5;
  const int first = gbeg * kGroup, tend = gend * kGroup;

  // ---- key rows, 128 tokens (4 groups) per pass, warp w taking tokens 32w .. 32w+31 of the
  // pass: the warp copies its 32 rows (8 KB) into shared memory with coalesced 16-byte
  // asynchronous copies (one 512-byte stretch per instruction; rows past the end are
  // zero-filled), rows padded to 272 bytes so that the row-per-lane reads hit distinct
  // banks.  Two stages: the next pass's rows are in flight while this pass is summed.
  uint8_t* wst = stage + warp * 2 * 32 * kStageRow;
  auto issue = [&](int base, int buf) {
    const int t0 = base + 32 * warp;
    uint8_t* dst = wst + buf * 32 * kStageRow;
#pragma unroll
    for (int i = 0; i < 16; ++i) {   // rows 2i + (lane >> 4), chunk lane & 15
      const int r = 2 * i + (lane >> 4), t = t0 + r;
      const bool ok = t < tend;
      cp_async16(dst + r * kStageRow + (lane & 15) * 16,
                 ku + static_cast<size_t>(ok ? t : first) * kHeadDim + (lane & 15) * 8, ok ? 16 : 0);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // ---- mean query of the unit's saliency window (heads outer, tokens inner).  The G heads'
  // windows are consecutive rows (row r = head r / nw, token r % nw); they are copied into
  // the stage in rounds of as many rows as it holds (coalesced 16-byte copies), and thread c
  // sums column c over each round in row order
  {
    const int rows = G * nw;
    const uint16_t* qbase = qwin + (static_cast<size_t>(b) * Hq + h * G) * nw * kHeadDim;
    constexpr int kCap = kScoreStageBytes / (kHeadDim * 2);   // window rows per round
    float s = 0.f;
    for (int r0 = 0; r0 < rows; r0 += kCap) {
      const int nr = min(kCap, rows - r0);
      for (int i = tid; i < nr * 16; i += kScoreThreads)
        cp_async16(stage + i * 16, qbase + static_cast<size_t>(r0) * kHeadDim + i * 8, 16);
      asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      __syncthreads();
      const uint16_t* col = reinterpret_cast<const uint16_t*>(stage) + tid;
#pragma unroll 16
      for (int r = 0; r < nr; ++r) s = __fadd_rn(s, bf16_bits_to_float(col[r * kHeadDim]));
      __syncthreads();
    }
    qbar[tid] = __fdiv_rn(s, static_cast<float>(rows));
  }
  __syncthreads();
  if (first < tend) issue(first, 0);

  // ---- group scores: lane l sums row l of its warp's stage in channel order
  const float4* qbar4 = reinterpret_cast<const float4*>(qbar);
  int buf = 0;
  for (int base = first; base < tend; base += kScoreThreads, buf ^= 1) {
    if (base + kScoreThreads < tend)
      issue(base + kScoreThreads, buf ^ 1);
    else
      asm volatile("cp.async.commit_group;" ::: "memory");   // an empty group keeps the count
    asm volatile("cp.async.wait_group 1;" ::: "memory");     // this pass's rows have landed
    __syncwarp();
    const int t0 = base + 32 * warp;
    float acc = 0.f;
    if (t0 + lane < tend) {
      const uint8_t* row = wst + buf * 32 * kStageRow + lane * kStageRow;
#pragma unroll
      for (int c8 = 0; c8 < kHeadDim / 8; ++c8) {
        const uint4 w = *reinterpret_cast<const uint4*>(row + c8 * 16);
        const float4 qa = qbar4[2 * c8], qb = qbar4[2 * c8 + 1];
        const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {   // channel c8*8 + 2e in the low half, + 1 in the high half
          acc = __fadd_rn(acc, __fmul_rn(qv[2 * e], __uint_as_float(wv[e] << 16)));
          acc = __fadd_rn(acc, __fmul_rn(qv[2 * e + 1], __uint_as_float(wv[e] & 0xFFFF0000u)));
        }
      }
    }
    __syncwarp();   // this stage is free for the copies two passes on
    logit[tid] = acc;
    __syncthreads();
    if (tid < kScoreThreads / kGroup) {
      const int g = base / kGroup + tid;
      if (g < gend) {
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
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Order-preserving unsigned image of a float; -0 and +0 map to the same value, as they
// compare equal.
__device__ __forceinline__ uint32_t ordered_bits(float x) {
  uint32_t v = __float_as_uint(x);
  if (v == 0x80000000u) v = 0u;
  return (v & 0x80000000u) ? ~v : (v | 0x80000000u);
}

// Block-wide exclusive prefix sum of `x` over the CTA's threads in thread order; returns
// this thread's prefix and writes the block total.
__device__ __forceinline__ int block_exclusive_scan(int x, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int v = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  if (lane == 31) warp_sums[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (kRouteThreads >> 5) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;   // inclusive prefix of the warp totals
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + v - x;
  *total = warp_sums[(kRouteThreads >> 5) - 1];
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(kRouteThreads)
route_kernel(int Hkv, int L, int n_hi, const float* __restrict__ scores, uint8_t* route, int32_t* dest) {
  __shared__ int hist[256];
  __shared__ int warp_sums[32];
  __shared__ uint32_t sel_prefix;
  __shared__ int sel_rank;
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int ng = L / kGroup;
  const size_t u = static_cast<size_t>(b) * Hkv + h;
  const float* sc = scores + u * ng;
  uint8_t* ru = route + u * ng;
  int32_t* du = dest + u * ng;

  // ---- radix select of the n_hi-th largest score image: prefix/mask of the bits fixed
  // so far; `rank` = how many of the keys sharing the prefix are still to be taken
  uint32_t prefix = 0, mask = 0;
  int rank = n_hi;   // 1-based rank of the threshold among the keys with the prefix
  if (n_hi > 0 && n_hi < ng) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kRouteThreads) hist[i] = 0;
      __syncthreads();
      for (int g = tid; g < ng; g += kRouteThreads) {
        const uint32_t v = ordered_bits(sc[g]);
        if ((v & mask) == prefix) atomicAdd(&hist[(v >> shift) & 255u], 1);
      }
      __syncthreads();
      if (tid == 0) {   // walk the digits from the top until the rank falls in one
        int r = rank, d = 255;
        for (; d > 0; --d) {
          if (r <= hist[d]) break;
          r -= hist[d];
        }
        sel_prefix = prefix | (static_cast<uint32_t>(d) << shift);
        sel_rank = r;
      }
      __syncthreads();
      prefix = sel_prefix;
      rank = sel_rank;
      mask |= 255u << shift;
      __syncthreads();
    }
  }
  // threshold image T = prefix: groups above T are taken, and of the groups equal to T the
  // `rank` lowest indices (rank = n_hi minus the count above T)
  int eq_before = 0;   // groups equal to T with a lower index, over the earlier chunks
  int hi_before = 0, lo_before = 0;
  for (int base = 0; base < ng; base += kRouteThreads) {
    const int g = base + tid;
    uint32_t v = 0;
    bool above = false, equal = false;
    if (g < ng) {
      v = ordered_bits(sc[g]);
      if (n_hi >= ng) above = true;
      else if (n_hi > 0) {
        above = v > prefix;
        equal = v == prefix;
      }
    }
    int eq_total;
    const int eq_rank = eq_before + block_exclusive_scan(equal ? 1 : 0, warp_sums, &eq_total);
    eq_before += eq_total;
    const bool r1 = above || (equal && eq_rank < rank);
    int n_hi_chunk;
    const int hi_rank = hi_before + block_exclusive_scan(r1 ? 1 : 0, warp_sums, &n_hi_chunk);
    if (g < ng) {
      ru[g] = r1 ? 1 : 0;
      du[g] = r1 ? hi_rank : lo_before + (tid - (hi_rank - hi_before));
    }
    hi_before += n_hi_chunk;
    lo_before += min(kRouteThreads, ng - base) - n_hi_chunk;
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

// Resident score CTAs of one full wave on the current device (queried once per device).
cudaError_t score_resident_ctas(int* out) {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cacheable = dev >= 0 && dev < kMaxDevices;
  int v = cacheable ? cache[dev].load(std::memory_order_relaxed) : 0;
  if (v == 0) {
    int sms = 0, occ = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kScoreStageBytes);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, score_kernel, kScoreThreads, kScoreStageBytes);
    if (e != cudaSuccess) return e;
    v = sms * (occ > 0 ? occ : 1);
    if (cacheable) cache[dev].store(v, std::memory_order_relaxed);
  }
  *out = v;
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_split_groups(const Geometry& g, const uint16_t* q_window, int nw, const uint16_t* k,
                                const uint16_t* v, int L, int ld, int n_hi, float* scores, uint8_t* route,
                                int32_t* dest, uint16_t* k_hi, uint16_t* v_hi, uint16_t* k_lo, uint16_t* v_lo,
                                cudaStream_t s) {
  if (g.B == 0) return cudaSuccess;
  const int ng = L / kGroup;
  if (ng > 0) {
    // one wave of CTAs: the key rows are read with enough loads in flight only when every
    // resident slot holds a CTA
    int resident = 0;
    cudaError_t e = score_resident_ctas(&resident);
    if (e != cudaSuccess) return e;
    const long long units = static_cast<long long>(g.B) * g.Hkv;
    long long per_unit = resident / units;
    if (per_unit < 1) per_unit = 1;
    int gpc = static_cast<int>((ng + per_unit - 1) / per_unit);
    if (gpc < kScoreMinGroups) gpc = kScoreMinGroups;
    const int chunks = (ng + gpc - 1) / gpc;
    score_kernel<<<dim3(chunks, g.Hkv, g.B), kScoreThreads, kScoreStageBytes, s>>>(g.G, g.Hq, g.Hkv, q_window, nw,
                                                                                    k, L, ld, gpc, scores);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    route_kernel<<<dim3(g.Hkv, g.B), kRouteThreads, 0, s>>>(g.Hkv, L, n_hi, scores, route, dest);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  split_kernel<<<dim3(ng + 1, g.Hkv, g.B), kSplitThreads, 0, s>>>(g.Hkv, k, v, L, ld, n_hi, route, dest, k_hi, v_hi,
                                                                  k_lo, v_lo);
  return cudaGetLastError();
}

}  // namespace pnmix
