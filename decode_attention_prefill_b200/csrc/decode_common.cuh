// decode_common.cuh -- work partition, split-K workspace and fused combine of the decode
// kernels.
//
// Work items.  Unit u = (b, h) owns len[b]/32 full-group items followed by one residual
// item (the len[b] % 32 bf16 tokens, possibly none); len[b] is taken clamped to
// [0, capacity].  Items are numbered b-major, then h,
// then item, T in total.  A grid of N CTAs splits [0, T) evenly: CTA i takes
// [floor(i*T/N), floor((i+1)*T/N)).  Every CTA computes T from len[] itself, so the grid
// is balanced for any mix of lengths without the host knowing them.
//
// Partials.  The piece of unit u that CTA i covers (a "segment") produces one partial
// (m, l, acc[128]) per query head: m is the running max in the log2 domain, l the sum of
// 2^(logit - m) and acc the matching weighted sum of values.  It goes to slot i + u; the
// slots of u are contiguous and disjoint from other units'.  The CTA that takes the last
// ticket of u (the partition tells how many segments u has) merges them:
//     m* = max m_s,  out = sum_s acc_s 2^(m_s - m*) / sum_s l_s 2^(m_s - m*).
// Nothing waits: the other CTAs take their ticket and move on.
#pragma once

#include "common.cuh"

namespace pnmix {

constexpr int kPartialStride = 2 + kHeadDim;   // m, l, acc[128]
constexpr int kMaxDecodeCtas = 1024;           // grid cap of the decode kernels
constexpr unsigned kMaxCombineSegs = 32;       // segments merged per pass of the combine

struct DecodeWs {
  float* part;         // [slots][G][kPartialStride]
  uint32_t* tickets;   // [units], zero between calls
  int N;               // CTAs of the launch
  // Optional outputs / inputs of the final combine (all indexed like `out` by row_offset,
  // one float per row for the log-sum-exps):
  float* lse_out;            // if set: log2 sum_t 2^(logit_t) of every output row
  const float* prior_out;    // if set: merge with an earlier attention over other tokens,
  const float* prior_lse;    //   given by its normalised output and log-sum-exp
  // fused append (Geometry::append): the new K / V rows, bf16 [B][Hkv][128]
  const uint16_t* k_new;
  const uint16_t* v_new;
};

__host__ __device__ __forceinline__ size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ __forceinline__ size_t decode_partial_bytes(int slots, int G) {
  return align256(sizeof(float) * static_cast<size_t>(slots) * G * kPartialStride);
}

// CTA that owns item x.
__device__ __forceinline__ int cta_of(long long x, long long T, int N) {
  return static_cast<int>(((x + 1) * N - 1) / T);
}

// Whether a fused append adds a token to a sequence holding `raw` tokens (as pnmix_append:
// only while there is room).
__device__ __forceinline__ bool appends(const Geometry& g, int raw) {
  return g.append && raw >= 0 && raw < g.capacity;
}

// Length of sequence b as the partition uses it: len[b] clamped to [0, capacity], so a
// length array holding anything else (stale memory, a caller's ordering mistake) cannot
// send a record read outside the cache; plus the token a fused append adds.
__device__ __forceinline__ int seq_len(const Geometry& g, const int32_t* len, int b) {
  const int raw = len[b];
  return min(max(raw, 0), g.capacity) + (appends(g, raw) ? 1 : 0);
}

// Work items of a unit holding lb tokens: g.lead items for its fixed cost (a CTA whose slice
// starts a unit takes fewer groups), its lb / 32 groups, and for the residual window
// g.resid_w items (one when it is empty), taken whole by the CTA whose slice holds the first.
__device__ __forceinline__ long long unit_items(const Geometry& g, int lb) {
  return static_cast<long long>(g.lead) + lb / kGroup + (lb % kGroup ? g.resid_w : 1);
}

__device__ __forceinline__ long long total_items(const Geometry& g, const int32_t* len) {
  long long T = 0;
  for (int b = 0; b < g.B; ++b) T += static_cast<long long>(g.Hkv) * unit_items(g, seq_len(g, len, b));
  return T;
}

struct Segment {
  int b, h, unit;
  int lo, hi;          // groups [lo, min(hi, ng)) of the unit; hi > ng: with the residual
                       // window; lo >= hi: nothing (a slice of lead items only)
  int ng, nr;          // full groups and residual tokens of the unit
  int first, last;     // CTAs covering the unit
  int app_slot;        // fused append: residual slot of the new token (31: it completes
                       // group ng - 1), or -1 when nothing is appended
};

// Calls fn(seg) for every segment of this CTA, in item order.  All threads of the CTA
// call it with the same arguments (the loop is uniform across the block).
template <typename F>
__device__ __forceinline__ void for_each_segment(const Geometry& g, const int32_t* len, int grid, F&& fn) {
  const long long T = total_items(g, len);
  // with more CTAs than items the surplus CTAs sit out, so every CTA of [0, N) owns >= 1 item
  const int N = T < grid ? static_cast<int>(T) : grid;
  const int i = blockIdx.x;
  if (i >= N) return;
  const long long a = T * i / N, e = T * (i + 1) / N;
  long long cum = 0;   // first item of batch row b
  int b = 0;
  long long x = a;
  while (x < e) {
    int lb = seq_len(g, len, b);
    long long per_b = static_cast<long long>(g.Hkv) * unit_items(g, lb);
    while (b < g.B - 1 && cum + per_b <= x) {
      cum += per_b;
      ++b;
      lb = seq_len(g, len, b);
      per_b = static_cast<long long>(g.Hkv) * unit_items(g, lb);
    }
    const long long items = unit_items(g, lb);
    const int h = static_cast<int>((x - cum) / items);
    const long long ustart = cum + static_cast<long long>(h) * items;
    const long long uend = ustart + items;
    const long long x_lo = x - ustart, x_hi = (uend < e ? uend : e) - ustart;   // unit-local items
    const long long ng = lb / kGroup, rfirst = g.lead + ng;                    // first residual item
    Segment s;
    s.b = b;
    s.h = h;
    s.unit = b * g.Hkv + h;
    s.lo = static_cast<int>(min(max(x_lo - g.lead, 0ll), ng));
    s.hi = (x_lo <= rfirst && x_hi > rfirst) ? static_cast<int>(ng) + 1
                                              : static_cast<int>(min(max(x_hi - g.lead, 0ll), ng));
    s.ng = lb / kGroup;
    s.nr = lb % kGroup;
    s.app_slot = appends(g, len[b]) ? (lb - 1) % kGroup : -1;
    s.first = cta_of(ustart, T, N);
    s.last = cta_of(uend - 1, T, N);
    fn(s);
    x = ustart + x_hi;
  }
}

__device__ __forceinline__ float* partial_slot(const DecodeWs& ws, int unit, int G) {
  return ws.part + static_cast<size_t>(blockIdx.x + unit) * G * kPartialStride;
}

// Query row v of unit (b, h) is query v / G of sequence b, head h*G + v % G; q and out
// are [B][tq][Hq][128] (tq = 1: [B][Hq][128]).
__device__ __forceinline__ size_t row_offset(const Geometry& g, int b, int h, int v) {
  const int j = v / g.G, hg = v - j * g.G;
  return ((static_cast<size_t>(b) * g.tq + j) * g.Hq + h * g.G + hg) * kHeadDim;
}

// Tokens visible to query row v: a multi-query step appended its tq tokens before
// attending, and query j sees the cache up to its own token (len - tq + 1 + j).
__device__ __forceinline__ int visible_tokens(const Geometry& g, int len, int v) {
  return len - g.tq + 1 + v / g.G;
}

// Called by every thread of the CTA after the segment's partials are in its slot: the
// CTA that takes the unit's last ticket writes the unit's G = g.rows output rows.  With
// ws.lse_out it also writes each row's log-sum-exp L = m* + log2(sum_s l_s 2^(m_s - m*))
// (log2 domain of the scaled logits; -inf for a row that sees no token).  With
// ws.prior_out / prior_lse the row is merged with an attention over other tokens:
//   out = (2^(L0 - M) o0 + 2^(L - M) o) / (2^(L0 - M) + 2^(L - M)),  M = max(L0, L),
// and the log-sum-exp written is that of the union, M + log2(2^(L0 - M) + 2^(L - M)).
// Shared memory of the combine: the weights of a chunk of segments per row, each row's m*
// and denominator, the mixing weights of a merge with a prior part, the ticket verdict.
template <int MAXR>
struct CombineScratch {
  float w[MAXR][kMaxCombineSegs];
  float mstar[MAXR], den[MAXR];
  float mix[MAXR][2];   // weights of the prior row and of this one
  int is_last;
};

// EXT: the caller passes the scratch (a region of its dynamic shared memory that is idle
// while the combine runs) instead of the combine declaring it statically.
template <int MAXR = kMaxG, bool EXT = false>   // the most rows a launch has (G <= MAXR)
__device__ __forceinline__ void combine_segment(const DecodeWs& ws, const Segment& s, int G, float* out,
                                                const Geometry& geo, CombineScratch<MAXR>* ext = nullptr) {
  CombineScratch<MAXR>* sc;
  if constexpr (EXT) {
    sc = ext;
  } else {
    __shared__ CombineScratch<MAXR> own;
    sc = &own;
  }
  auto& wsh = sc->w;
  auto& mstar_sh = sc->mstar;
  auto& den_sh = sc->den;
  auto& mix_sh = sc->mix;
  int& is_last = sc->is_last;
  __threadfence();
  __syncthreads();
  const unsigned nseg = static_cast<unsigned>(s.last - s.first + 1);
  if (threadIdx.x == 0) is_last = (atomicAdd(ws.tickets + s.unit, 1u) == nseg - 1);
  __syncthreads();
  if (is_last) {
    __threadfence();
    // (1) per head, one warp: every lane loads the (m, l) pairs of its segments once (one
    // round), the largest reference m* and the denominator follow by shuffles and the
    // weights 2^(m_s - m*) of the first chunk go to shared memory; (2) per chunk of up to 32
    // segments, every thread sums its (head, channel) pairs with four loads in flight
    constexpr int kLaneSegs = 4;         // segments per lane held in registers (128 per head)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const float* base = ws.part + static_cast<size_t>(s.first + s.unit) * G * kPartialStride;
    const size_t seg_stride = static_cast<size_t>(G) * kPartialStride;
    for (int hh = warp; hh < G; hh += nwarps) {
      float2 ml[kLaneSegs];
#pragma unroll
      for (int r = 0; r < kLaneSegs; ++r) {
        const unsigned k = lane + 32u * r;
        ml[r] = k < nseg ? __ldcg(reinterpret_cast<const float2*>(base + k * seg_stride + hh * kPartialStride))
                         : make_float2(-INFINITY, 0.f);
      }
      float m = -INFINITY;
#pragma unroll
      for (int r = 0; r < kLaneSegs; ++r) m = fmaxf(m, ml[r].x);
      for (unsigned k = lane + 32u * kLaneSegs; k < nseg; k += 32)   // beyond 128 segments: reload
        m = fmaxf(m, __ldcg(base + k * seg_stride + hh * kPartialStride));
#pragma unroll
      for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float den = 0.f;
#pragma unroll
      for (int r = 0; r < kLaneSegs; ++r) {
        const float f = (ml[r].x == -INFINITY || m == -INFINITY) ? 0.f : exp2f(ml[r].x - m);
        den = fmaf(ml[r].y, f, den);
        if (r == 0 && static_cast<unsigned>(lane) < nseg) wsh[hh][lane] = f;
      }
      for (unsigned k = lane + 32u * kLaneSegs; k < nseg; k += 32) {
        const float2 v = __ldcg(reinterpret_cast<const float2*>(base + k * seg_stride + hh * kPartialStride));
        den = fmaf(v.y, (v.x == -INFINITY || m == -INFINITY) ? 0.f : exp2f(v.x - m), den);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
      if (lane == 0) {
        mstar_sh[hh] = m;
        den_sh[hh] = den;
        if (ws.lse_out || ws.prior_out) {
          const size_t row = row_offset(geo, s.b, s.h, hh) / kHeadDim;
          float L = den > 0.f ? m + log2f(den) : -INFINITY;
          float w0 = 0.f, w1 = den > 0.f ? 1.f : 0.f;
          if (ws.prior_out) {
            const float L0 = ws.prior_lse[row];
            const float M = fmaxf(L0, L);
            w0 = L0 == -INFINITY ? 0.f : exp2f(L0 - M);
            w1 = L == -INFINITY ? 0.f : exp2f(L - M);
            const float t = w0 + w1;
            L = t > 0.f ? M + log2f(t) : -INFINITY;
            w0 = t > 0.f ? w0 / t : 0.f;
            w1 = t > 0.f ? w1 / t : 0.f;
          }
          mix_sh[hh][0] = w0;
          mix_sh[hh][1] = w1;
          if (ws.lse_out) ws.lse_out[row] = L;
        }
      }
    }
    __syncthreads();
    for (unsigned chunk = 0; chunk < nseg; chunk += kMaxCombineSegs) {
      const unsigned n = nseg - chunk < kMaxCombineSegs ? nseg - chunk : kMaxCombineSegs;
      const bool last_chunk = chunk + n == nseg;
      if (chunk > 0) {   // the weights of a later chunk
        for (int hh = warp; hh < G; hh += nwarps) {
          if (static_cast<unsigned>(lane) < n) {
            const float ms = __ldcg(base + (chunk + lane) * seg_stride + hh * kPartialStride);
            const float m = mstar_sh[hh];
            wsh[hh][lane] = (ms == -INFINITY || m == -INFINITY) ? 0.f : exp2f(ms - m);
          }
        }
        __syncthreads();
      }
      for (int i = threadIdx.x; i < G * kHeadDim; i += blockDim.x) {
        const int hh = i / kHeadDim, c = i % kHeadDim;
        const size_t off = row_offset(geo, s.b, s.h, hh);
        float* out_row = out + off;
        const float* col = base + static_cast<size_t>(hh) * kPartialStride + 2 + c;
        float num = chunk == 0 ? 0.f : out_row[c];
        unsigned k = 0;
        for (; k + 4 <= n; k += 4) {   // four segments' values in flight
          const float a0 = __ldcg(col + (chunk + k) * seg_stride), a1 = __ldcg(col + (chunk + k + 1) * seg_stride);
          const float a2 = __ldcg(col + (chunk + k + 2) * seg_stride), a3 = __ldcg(col + (chunk + k + 3) * seg_stride);
          num = fmaf(a0, wsh[hh][k], num);
          num = fmaf(a1, wsh[hh][k + 1], num);
          num = fmaf(a2, wsh[hh][k + 2], num);
          num = fmaf(a3, wsh[hh][k + 3], num);
        }
        for (; k < n; ++k) num = fmaf(__ldcg(col + (chunk + k) * seg_stride), wsh[hh][k], num);
        if (last_chunk) {
          float o = den_sh[hh] > 0.f ? num / den_sh[hh] : 0.f;
          if (ws.prior_out) o = fmaf(mix_sh[hh][0], ws.prior_out[off + c], mix_sh[hh][1] * o);
          out_row[c] = o;
        } else {
          out_row[c] = num;
        }
      }
      __syncthreads();
    }
    if (threadIdx.x == 0) ws.tickets[s.unit] = 0u;
  }
  __syncthreads();
}

// Host side: CTAs a decode launch may use for this shape (the workspace is sized for it)
// and the slots that gives.
__host__ __forceinline__ int decode_max_ctas(const Geometry& g, int max_context) {
  const long long units = static_cast<long long>(g.B) * g.Hkv;
  const long long items = units * ((max_context > 0 ? max_context : 0) / kGroup + 1);
  long long n = items < kMaxDecodeCtas ? items : kMaxDecodeCtas;
  return static_cast<int>(n < 1 ? 1 : n);
}

cudaError_t launch_decode_simt(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax,
                               float* out, DecodeWs ws, cudaStream_t s);
cudaError_t launch_decode_mma(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax,
                              float* out, DecodeWs ws, cudaStream_t s);
cudaError_t launch_decode_ws(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax,
                             float* out, DecodeWs ws, cudaStream_t s);
cudaError_t launch_decode_tc(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax,
                             float* out, DecodeWs ws, cudaStream_t s);
// query rows per KV head the tcgen05 kernel takes (one per TMEM lane); the 8-row-warp
// kernels stop at kMaxRows
constexpr int kMaxTcRows = 128;
cudaError_t launch_decode_rows(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax,
                               float* out, DecodeWs ws, cudaStream_t s);

}  // namespace pnmix
