// decode_ws.cu -- warp-specialized tensor-core decode attention over the packed cache.
//
// One CTA = one split of the work partition (decode_common.cuh), 8 warps in 4 pairs.  In a
// pair, the QK warp turns each 32-token group record into logits and softmax weights, and
// the PV warp folds the weights into the value sum; the two run concurrently on different
// groups and meet in shared memory:
//
//   ring slot (TMA bulk copy of one record, mbarrier "full")
//       QK warp: codes x (q s) + z x q -> logits -> running max -> p = 2^(logit - m)
//                p (fp16, already in the PV B-fragment order) + rescale factors -> P buffer
//       PV warp: P buffer -> value codes x (p s_v) + z_v x p, then refills the ring slot
//
// The arithmetic of each product is the one of decode_mma.cu (fragment-ordered codes as
// exact fp16 subnormals, the query as exact fp16 with the product q s carried in two
// columns per head, log2-domain softmax).  What changes is the schedule: a warp carries
// either the key-side or the value-side state (no warp holds both), so twice as many
// warps fit per SM and one pair's key and value work overlap.  The running max is raised
// lazily (only when a group's max exceeds it by more than kLazyMax, i.e. p may reach
// 2^kLazyMax), so the value accumulators are rescaled a few times per segment instead of
// at every increase.
//
// Every wait is bounded (Geometry::wait_limit rounds); a wait that runs out sets PNMIX_DEVERR_TIMEOUT and a
// shared flag that makes every warp of the CTA stop consuming.
#include <atomic>

#include "common.cuh"
#include "decode_common.cuh"
#include "decode_frag.cuh"

namespace pnmix {
namespace {

constexpr int kPairs = 4;
constexpr int kWsWarps = 2 * kPairs;   // QK warps 0..3, PV warps 4..7
constexpr int kWsThreads = kWsWarps * 32;
constexpr float kLazyMax = 4.f;        // p <= 2^4 between rescales
constexpr int kPBufBytes = 512 + 64;   // P fragments (32 lanes x 16 B), flag + factors
constexpr int kStageBudget = 78848;    // ring bytes per CTA (two CTAs per SM)

// Ring slots per pair: as many as fit the budget (less the larger query sets of NT = 2),
// at most 6.
template <int BHI, int BLO, int NT, int NHS>
__host__ __device__ constexpr int ws_stages() {
  return (kStageBudget - (NT - 1) * 4096) / (kPairs * record_bytes_of<BHI, BLO, NHS>()) < 6
             ? (kStageBudget - (NT - 1) * 4096) / (kPairs * record_bytes_of<BHI, BLO, NHS>())
             : 6;
}

struct WsSmem {
  int qsets;   // [NT][2 sets][4 slice pairs][32 lanes][16 B]
  int qnat;    // fp32 [kMaxG][128], natural channel order, unscaled
  int perm;    // 128 bytes
  int resid;   // fp32 [kMaxG][kPartialStride]: partial of the residual item
  int rrows;   // bf16 residual K rows [32][kResidKStride] then V rows [32][128]
  int bars;    // per pair: full[S], pfull[2], pempty[2]
  int pbuf;    // per pair: 2 x kPBufBytes
  int stages;  // per pair: S x R
  int part;    // fp32 [kPairs][kMaxG][kPartialStride], aliases the stages
  int total;
};

__host__ __device__ __forceinline__ WsSmem ws_smem(int NT, int R, int S) {
  WsSmem m;
  m.qsets = 0;
  m.qnat = NT * 2 * 4 * 32 * 16;
  m.perm = m.qnat + kMaxG * kHeadDim * 4;
  m.resid = m.perm + 128;
  m.rrows = m.resid + kMaxG * kPartialStride * 4;
  m.bars = m.rrows + kGroup * kResidKStride * 2 + kGroup * kHeadDim * 2;
  m.pbuf = m.bars + ((kPairs * (S + 4) * 8 + 127) / 128) * 128;
  m.stages = m.pbuf + kPairs * 2 * kPBufBytes;
  const int stage_bytes = kPairs * S * R;
  const int part_bytes = kPairs * kMaxG * kPartialStride * 4;
  m.part = m.stages;
  m.total = m.stages + (stage_bytes > part_bytes ? stage_bytes : part_bytes);
  return m;
}

// Bounded wait on phase `parity` of `bar`.  Returns false (and raises the CTA's stop flag
// and the cache error word) when the wait runs out or another warp already stopped.
__device__ __forceinline__ bool ws_wait(uint64_t* bar, uint32_t parity, volatile int* stop, uint32_t* err,
                                       uint32_t limit) {
  uint32_t spins = 0;
  while (!mbar_try_wait(bar, parity)) {
    if (*stop) return false;
    if (++spins >= limit) {
      *stop = 1;
      if ((threadIdx.x & 31) == 0) atomicOr(err, PNMIX_DEVERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Logits of one group for the heads of this lane (log2 domain): lane (gq, tq) gets head
// 4*nt + tq at tokens gq + 8u, u = 0..3.
template <int BHI, int BLO, int NT, int NHS, bool QREG, bool MQ>
__device__ __forceinline__ void group_logits(const Geometry& g, const uint8_t* rec, const QFrags<NT>& qf,
                                             const uint4* qsets, float qscale, int tok0, int vis_base,
                                             float (&lg)[NT][4]) {
  constexpr int WH = NHS * BHI / 2;
  constexpr int kc = key_code_bytes<BHI, BLO, NHS>();
  const int lane = threadIdx.x & 31;
  const int tq = lane & 3;
  float acc_hi[NT][2][4], acc_lo[NT][2][4], dz[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc_hi[nt][0][i] = acc_hi[nt][1][i] = 0.f;
      acc_lo[nt][0][i] = acc_lo[nt][1][i] = 0.f;
      dz[nt][i] = 0.f;
    }
  const uint32_t* kw = reinterpret_cast<const uint32_t*>(rec);
  uint4 s4, z4;
#pragma unroll
  for (int sigma = 0; sigma < 8; ++sigma) {
    const int par = sigma & 1;
    if (par == 0) {
      s4 = reinterpret_cast<const uint4*>(rec + kc + tq * 64)[sigma >> 1];
      z4 = reinterpret_cast<const uint4*>(rec + kc + 256 + tq * 64)[sigma >> 1];
    }
    const bool hi = sigma < NHS;
    uint32_t A[2][4];
    if (hi) {
      if constexpr (BHI == 4)
        key_slice_frags<4>(kw[(2 * sigma) * 32 + lane], kw[(2 * sigma + 1) * 32 + lane], 0, A);
      else
        key_slice_frags<BHI>(kw[sigma * 32 + lane], 0u, 0, A);
    } else {
      const int sl = sigma - NHS;
      if constexpr (BLO == 2)
        key_slice_frags<2>(kw[(WH + sl) * 32 + lane], 0u, 0, A);
      else
        key_slice_frags<1>(kw[(WH + (sl >> 1)) * 32 + lane], 0u, par, A);
    }
    // scale / zero chunk of a slice pair: (even e=0, odd e=0, even e=1, odd e=1)
    const uint32_t s0 = par ? s4.y : s4.x, s1 = par ? s4.w : s4.z;
    const uint32_t z0 = par ? z4.y : z4.x, z1 = par ? z4.w : z4.z;
    uint32_t qxs[NT][2];   // this slice's X registers of each tile (for the zero-point term)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      uint4 X, Y;
      if constexpr (QREG) {
        X = qf.x[nt][sigma >> 1];
        Y = qf.y[nt][sigma >> 1];
      } else {
        X = qsets[((nt * 2 + 0) * 4 + (sigma >> 1)) * 32 + lane];
        Y = qsets[((nt * 2 + 1) * 4 + (sigma >> 1)) * 32 + lane];
      }
      const uint32_t qx0 = par ? X.z : X.x, qx1 = par ? X.w : X.y;
      const uint32_t qy0 = par ? Y.z : Y.x, qy1 = par ? Y.w : Y.y;
      const uint32_t b0 = hfma2(qx0, s0, hmul2(qy0, s0));
      const uint32_t b1 = hfma2(qx1, s1, hmul2(qy1, s1));
      if (hi) {
        mma16816_free(acc_hi[nt][0], A[0][0], A[0][1], A[0][2], A[0][3], b0, b1);
        mma16816_free(acc_hi[nt][1], A[1][0], A[1][1], A[1][2], A[1][3], b0, b1);
      } else {
        mma16816_free(acc_lo[nt][0], A[0][0], A[0][1], A[0][2], A[0][3], b0, b1);
        mma16816_free(acc_lo[nt][1], A[1][0], A[1][1], A[1][2], A[1][3], b0, b1);
      }
      qxs[nt][0] = qx0;
      qxs[nt][1] = qx1;
    }
    if constexpr (NT == 1) {
      mma16816_free(dz[0], z0, z0, z1, z1, qxs[0][0], qxs[0][1]);
    } else {
      // zero-point term of both tiles in one product: A = X transposed (row = query column:
      // rows gq and gq + 8 are column gq of tile 0 and tile 1, exactly this lane's X
      // registers), B = z (the same in every column).  Row c of the result is
      // sum_p X[p][c] z_p.
      mma16816_free(dz[0], qxs[0][0], qxs[1][0], qxs[0][1], qxs[1][1], z0, z1);
    }
  }
  // zero-point sums per head: columns 2tq and 2tq+1 of each tile
  float zsum[NT];
  if constexpr (NT == 1) {
    zsum[0] = dz[0][0] + dz[0][1];
  } else {
    // row c of the transposed product sits in lanes 4c .. 4c+3 (c < 8: element 0, tile 0;
    // element 2: tile 1)
    const int src0 = (2 * tq) * 4, src1 = (2 * tq + 1) * 4;
    zsum[0] = __shfl_sync(0xffffffffu, dz[0][0], src0) + __shfl_sync(0xffffffffu, dz[0][0], src1);
    zsum[1] = __shfl_sync(0xffffffffu, dz[0][2], src0) + __shfl_sync(0xffffffffu, dz[0][2], src1);
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float zb = zsum[nt] * qscale;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int mt = u >> 1, r = 2 * (u & 1);
      const float fh = __int_as_float((127 + 24 - key_row_shift<BHI>(u)) << 23) * qscale;
      const float fl = __int_as_float((127 + 24 - key_row_shift<BLO>(u)) << 23) * qscale;
      const float vhi = acc_hi[nt][mt][r] + acc_hi[nt][mt][r + 1];
      const float vlo = acc_lo[nt][mt][r] + acc_lo[nt][mt][r + 1];
      lg[nt][u] = fmaf(vhi, fh, fmaf(vlo, fl, zb));
    }
  }
  // multi-query steps: row v sees tokens below vis_base + v / G (only a group that
  // reaches the newest tokens of its unit takes this branch)
  if (MQ && tok0 + kGroup > vis_base) {
    const int gq = lane >> 2;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int lim = vis_base + (4 * nt + tq) / g.G;
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (tok0 + gq + 8 * u >= lim) lg[nt][u] = -INFINITY;
    }
  }
}

// Value side of one group: acc (channels 16m + gq (+8), heads 2tq, 2tq+1) and the zero-point
// sums, from the P fragments p16[4] (tokens 2tq + 8i (+1) of head gq).
template <int kc>
__device__ __forceinline__ void group_values(const uint8_t* rec, const uint4& p4, float (&pv)[8][4],
                                             float (&bias)[4]) {
  const int lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const uint32_t p16[4] = {p4.x, p4.y, p4.z, p4.w};
  const int vs_off = kc + 1536, vz_off = kc + 1792;
  uint32_t vsr[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = *reinterpret_cast<const uint4*>(rec + vs_off + (tq + 4 * i) * 16);
    vsr[i][0] = v.x; vsr[i][1] = v.y; vsr[i][2] = v.z; vsr[i][3] = v.w;
  }
  {
    // zero-point chunk (tq, j): token pairs tq, tq + 8, tq + 4, tq + 12 of channel group j
    const int j = gq & 3;
    const uint4 zc = *reinterpret_cast<const uint4*>(rec + vz_off + (tq * 4 + j) * 16);
    uint32_t vz[4] = {zc.x, zc.z, zc.y, zc.w};   // token pairs tq + 4i
#pragma unroll
    for (int i = 0; i < 4; ++i) vz[i] = gq < 4 ? vz[i] : 0u;
    mma16816_free(bias, vz[0], 0u, vz[1], 0u, p16[0], p16[1]);
    mma16816_free(bias, vz[2], 0u, vz[3], 0u, p16[2], p16[3]);
  }
  // slot (r, p) of value word m sits at bits 8r + 2p and is taken in place from w >> 8r,
  // so token block p carries 2^(2p); its B rows are scaled by 2^(2 - 2p)
  const uint32_t bp0 = hmul2(p16[0], 0x44004400u);   // x 4
  const uint32_t bp2 = hmul2(p16[2], 0x34003400u);   // x 1/4
  const uint32_t bp3 = hmul2(p16[3], 0x2C002C00u);   // x 1/16
  const uint4 vw0 = *reinterpret_cast<const uint4*>(rec + kc + 512 + lane * 16);
  const uint4 vw1 = *reinterpret_cast<const uint4*>(rec + kc + 512 + (32 + lane) * 16);
  const uint32_t vw[8] = {vw0.x, vw0.y, vw0.z, vw0.w, vw1.x, vw1.y, vw1.z, vw1.w};
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int j = m >> 1;
    const uint32_t w = vw[m], w8 = w >> 8;
    const uint32_t k0a0 = sub_pair(w, 0x00030003u), k0a2 = sub_pair(w, 0x000C000Cu);
    const uint32_t k1a0 = sub_pair(w, 0x00300030u), k1a2 = sub_pair(w, 0x00C000C0u);
    const uint32_t k0a1 = sub_pair(w8, 0x00030003u), k0a3 = sub_pair(w8, 0x000C000Cu);
    const uint32_t k1a1 = sub_pair(w8, 0x00300030u), k1a3 = sub_pair(w8, 0x00C000C0u);
    const uint32_t b00 = hmul2(bp0, vsr[0][j]), b01 = hmul2(p16[1], vsr[1][j]);
    const uint32_t b10 = hmul2(bp2, vsr[2][j]), b11 = hmul2(bp3, vsr[3][j]);
    mma16816_free(pv[m], k0a0, k0a1, k0a2, k0a3, b00, b01);
    mma16816_free(pv[m], k1a0, k1a1, k1a2, k1a3, b10, b11);
  }
}

// MQ: several queries per sequence (rows = G * tq) with the causal mask on the newest
// tokens; a separate instance so the one-query kernel carries none of it.
template <int BHI, int BLO, int NT, int NHS, bool MQ>
__global__ void __launch_bounds__(kWsThreads, 2)
decode_ws_kernel(Geometry g, const uint16_t* __restrict__ q, pnmix_cache c, float* __restrict__ out,
                 DecodeWs ws) {
  constexpr int R = record_bytes_of<BHI, BLO, NHS>();
  constexpr int S = ws_stages<BHI, BLO, NT, NHS>();
  constexpr bool QREG = NT == 1;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int stop_flag;
  const int G = g.rows;   // query rows per unit
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool is_qk = warp < kPairs;
  const int pair = is_qk ? warp : warp - kPairs;
  const WsSmem sm = ws_smem(NT, R, S);
  uint32_t* qsets = reinterpret_cast<uint32_t*>(smem + sm.qsets);
  float* qnat = reinterpret_cast<float*>(smem + sm.qnat);
  uint8_t* perm = smem + sm.perm;
  float* rslot = reinterpret_cast<float*>(smem + sm.resid);
  uint16_t* rrk = reinterpret_cast<uint16_t*>(smem + sm.rrows);
  uint16_t* rrv = rrk + kGroup * kResidKStride;
  float* part = reinterpret_cast<float*>(smem + sm.part);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sm.bars) + pair * (S + 4);
  uint64_t* full = bars;
  uint64_t* pfull = bars + S;
  uint64_t* pempty = bars + S + 2;
  uint8_t* pbuf = smem + sm.pbuf + pair * 2 * kPBufBytes;
  uint8_t* ring = smem + sm.stages + pair * S * R;
  volatile int* stop = &stop_flag;

  // barriers, and P buffers zeroed once (columns of absent heads stay zero)
  if (tid == 0) stop_flag = 0;
  if (!is_qk && lane == 0) {
    for (int k = 0; k < S; ++k) mbar_init(full + k, 1);
    for (int k = 0; k < 2; ++k) {
      mbar_init(pfull + k, 32);
      mbar_init(pempty + k, 32);
    }
    fence_mbar_init();
  }
  for (int i = tid; i < kPairs * 2 * kPBufBytes / 4; i += kWsThreads)
    reinterpret_cast<uint32_t*>(smem + sm.pbuf)[i] = 0u;
  __syncthreads();

  uint32_t ord_base = 0;   // ordinal of the pair's first group of the current segment

  for_each_segment(g, c.len, ws.N, [&](const Segment& seg) {
    const int b = seg.b, h = seg.h, unit = seg.unit;
    const int vis_base = seg.ng * kGroup + seg.nr - g.tq + 1;   // tokens row 0 sees
    const int gend = seg.hi < seg.ng ? seg.hi : seg.ng;
    const int my_first = seg.lo + pair;
    const int my_count = my_first < gend ? (gend - my_first + kPairs - 1) / kPairs : 0;
    const uint8_t* unit_rec = record_ptr(g, c.records, b, h, 0);
    auto rec_src = [&](int i) { return unit_rec + static_cast<size_t>(my_first + i * kPairs) * R; };

    // the PV warp owns the pair's ring: stage the first groups right away (nothing once a
    // wait of this CTA has run out, or for the unit the timeout test hook leaves unstaged)
    const bool stage = unit != g.skip_unit;
    int issued = 0;
    if (!is_qk && stage && !*stop) {
      const int n0 = my_count < S ? my_count : S;
      for (; issued < n0; ++issued) {
        const uint32_t o = ord_base + issued;
        stage_group(ring + (o % S) * R, rec_src(issued), static_cast<uint32_t>(R), full + o % S, lane == 0);
      }
    }

    // ---- query (unscaled fp32, natural order), residual rows, then the X / Y sets
    load_query_rows(g, q, c.perm, b, h, unit, qnat, perm, tid);
    const float qscale = g.scale * kLog2e;
    const bool seg_resid = seg.hi > seg.ng && seg.nr > 0;
    if (seg_resid) {
      const uint4* gk = reinterpret_cast<const uint4*>(c.k_resid + static_cast<size_t>(unit) * kGroup * kHeadDim);
      const uint4* gv = reinterpret_cast<const uint4*>(c.v_resid + static_cast<size_t>(unit) * kGroup * kHeadDim);
      for (int i = tid; i < seg.nr * 16; i += kWsThreads) {
        const int r = i >> 4, cc = i & 15;
        reinterpret_cast<uint4*>(rrk + r * kResidKStride)[cc] = __ldg(gk + i);
        reinterpret_cast<uint4*>(rrv)[i] = __ldg(gv + i);
      }
    }
    if (g.n_prune > 0) {   // dynamic query-channel pruning of the staged query rows
      __syncthreads();
      prune_query_rows(g, qnat, warp, kWsWarps);
    }
    if (g.n_prune_slices > 0) {   // key-slice pruning of the staged query rows
      __syncthreads();
      const uint32_t pmask = pruned_slices(g, qnat, perm);
      __syncthreads();
      zero_pruned_slices(g, qnat, perm, pmask, tid, kWsThreads);
    }
    __syncthreads();
    if (is_qk) {   // QK warp w builds slice pair w of the sets
      const int tq = lane & 3, gq = lane >> 2, chunk = warp;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int col = gq + 8 * nt, hh = col >> 1, hl = col & 1;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int idx = chunk * 4 + i, sigma = idx >> 1, e = idx & 1;
          const int p0 = 16 * sigma + 8 * e + 2 * tq;
          uint32_t sets[2][2];
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            // bf16 -> fp16 is exact in fp16's normal range (queries are assumed < 65504)
            const float x = hh < G ? qnat[hh * kHeadDim + perm[p0 + v]] : 0.f;
            const uint32_t qb = __half_as_ushort(__float2half_rn(x));
            sets[0][v] = hl ? qb : 0u;
            sets[1][v] = hl ? (qb ^ 0x8000u) : qb;
          }
#pragma unroll
          for (int s = 0; s < 2; ++s)
            qsets[(((nt * 2 + s) * 4 + chunk) * 32 + lane) * 4 + i] = sets[s][0] | (sets[s][1] << 16);
        }
      }
    }
    __syncthreads();

    const int gq = lane >> 2, tq = lane & 3;
    const int h0 = 2 * tq, h1 = 2 * tq + 1;   // PV warp: heads of this lane's columns
    float m_ref[NT], lsum[NT];                  // QK warp: lazy running max, partial sums
    float pv[8][4], bias[4];                    // PV warp: value and zero-point sums
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m_ref[nt] = -INFINITY;
      lsum[nt] = 0.f;
    }
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int i = 0; i < 4; ++i) pv[m][i] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) bias[i] = 0.f;

    if (is_qk) {
      // ================================================================ QK warp
      QFrags<NT> qf;
      if constexpr (QREG) {
#pragma unroll
        for (int cp = 0; cp < 4; ++cp) {
          qf.x[0][cp] = reinterpret_cast<const uint4*>(qsets)[(0 * 4 + cp) * 32 + lane];
          qf.y[0][cp] = reinterpret_cast<const uint4*>(qsets)[(1 * 4 + cp) * 32 + lane];
        }
      }
      for (int i = 0; i < my_count; ++i) {
        const uint32_t o = ord_base + i;
        if (!__all_sync(0xffffffffu, ws_wait(full + o % S, (o / S) & 1, stop, c.error, g.wait_limit))) break;
        float lg[NT][4];
        group_logits<BHI, BLO, NT, NHS, QREG, MQ>(g, ring + (o % S) * R, qf, reinterpret_cast<const uint4*>(qsets),
                                             qscale, (my_first + i * kPairs) * kGroup, vis_base, lg);
        // lazy running max per head (4*nt + tq), over the group's 32 tokens
        bool raise = false;
        float mx[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float v = fmaxf(fmaxf(lg[nt][0], lg[nt][1]), fmaxf(lg[nt][2], lg[nt][3]));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
          mx[nt] = v;
          raise |= v > m_ref[nt] + kLazyMax;
        }
        const bool any_raise = __any_sync(0xffffffffu, raise);
        const uint32_t pb = o & 1;
        uint8_t* P = pbuf + pb * kPBufBytes;
        // the P buffer's previous use (ordinal o - 2) must have been read by the PV warp
        if (o >= 2 && !__all_sync(0xffffffffu, ws_wait(pempty + pb, ((o >> 1) + 1) & 1, stop, c.error, g.wait_limit))) break;
        if (any_raise) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const float mn = mx[nt] > m_ref[nt] + kLazyMax ? mx[nt] : m_ref[nt];
            const float alpha = ex2(m_ref[nt] - mn);   // 0 from -inf, 1 when unchanged
            lsum[nt] *= alpha;
            m_ref[nt] = mn;
            const int hh = 4 * nt + tq;
            if (gq == 0 && hh < G) reinterpret_cast<float*>(P + 512 + 16)[hh] = alpha;
          }
        }
        if (lane == 0) *reinterpret_cast<int*>(P + 512) = any_raise ? 1 : 0;
        // p in the PV B-fragment order: token t = gq + 8u of head n -> lane n*4 + (gq >> 1),
        // register u, half gq & 1
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int n = 4 * nt + tq;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float p = ex2(lg[nt][u] - m_ref[nt]);
            lsum[nt] += p;
            if (n < G)
              reinterpret_cast<__half*>(P)[((n * 4 + (gq >> 1)) * 4 + u) * 2 + (gq & 1)] = __float2half_rn(p);
          }
        }
        mbar_arrive(pfull + pb);
      }
    } else {
      // ================================================================ PV warp
      if (seg_resid) {
        residual_partial(g, rrk, rrv, seg.nr, qnat, qscale, rslot, pair, kPairs, seg.ng * kGroup, vis_base);
      } else if (pair == 0 && lane < G) {
        rslot[lane * kPartialStride + 0] = -INFINITY;
        rslot[lane * kPartialStride + 1] = 0.f;
      }
      int consumed = 0;
      for (int i = 0; i < my_count; ++i) {
        const uint32_t o = ord_base + i;
        const uint32_t pb = o & 1;
        const uint8_t* P = pbuf + pb * kPBufBytes;
        if (!__all_sync(0xffffffffu, ws_wait(pfull + pb, (o >> 1) & 1, stop, c.error, g.wait_limit))) break;
        if (!__all_sync(0xffffffffu, ws_wait(full + o % S, (o / S) & 1, stop, c.error, g.wait_limit))) break;
        const uint4 p4 = reinterpret_cast<const uint4*>(P)[lane];
        const int rescale = *reinterpret_cast<const volatile int*>(P + 512);
        float a0 = 1.f, a1 = 1.f;
        if (rescale) {
          const float* al = reinterpret_cast<const float*>(P + 512 + 16);
          a0 = h0 < G ? al[h0] : 1.f;
          a1 = h1 < G ? al[h1] : 1.f;
        }
        mbar_arrive(pempty + pb);
        if (rescale) {
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            pv[m][0] *= a0;
            pv[m][1] *= a1;
            pv[m][2] *= a0;
            pv[m][3] *= a1;
          }
          bias[0] *= a0;
          bias[1] *= a1;
          bias[2] *= a0;
          bias[3] *= a1;
        }
        group_values<key_code_bytes<BHI, BLO, NHS>()>(ring + (o % S) * R, p4, pv, bias);
        consumed = i + 1;
        __syncwarp();
        if (issued < my_count && stage && !*stop) {
          const uint32_t on = ord_base + issued;
          stage_group(ring + (on % S) * R, rec_src(issued), static_cast<uint32_t>(R), full + on % S, lane == 0);
          ++issued;
        }
      }
      if (consumed < my_count) {
        // stopped early: let the copies issued and not yet taken land before the shared
        // memory is reused
        for (int k = consumed; k < issued; ++k) {
          const uint32_t o = ord_base + k;
          for (uint32_t spins = 0; spins < g.wait_limit && !mbar_try_wait(full + o % S, (o / S) & 1); ++spins) {
          }
        }
      }
    }
    __syncthreads();   // every ring is idle: the partials may alias them

    float* wp = part + pair * kMaxG * kPartialStride;
    if (is_qk) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float v = lsum[nt];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        const int hh = 4 * nt + tq;
        if (gq == 0 && hh < G) {
          wp[hh * kPartialStride + 0] = my_count ? m_ref[nt] : -INFINITY;
          wp[hh * kPartialStride + 1] = my_count ? v : 0.f;
        }
      }
    } else {
      float bz[4][2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bz[j][0] = __shfl_sync(0xffffffffu, bias[0], j * 4 + tq);
        bz[j][1] = __shfl_sync(0xffffffffu, bias[1], j * 4 + tq);
      }
      const float pv_scale = 4194304.0f;   // 2^22: the codes' 2^-24 and the blocks' 2^2
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int j = m >> 1;
        const int c0 = 16 * m + gq, c1 = c0 + 8;
        if (h0 < G) {
          wp[h0 * kPartialStride + 2 + c0] = fmaf(pv[m][0], pv_scale, bz[j][0]);
          wp[h0 * kPartialStride + 2 + c1] = fmaf(pv[m][2], pv_scale, bz[j][0]);
        }
        if (h1 < G) {
          wp[h1 * kPartialStride + 2 + c0] = fmaf(pv[m][1], pv_scale, bz[j][1]);
          wp[h1 * kPartialStride + 2 + c1] = fmaf(pv[m][3], pv_scale, bz[j][1]);
        }
      }
    }
    ord_base += my_count;
    __syncthreads();

    // ---- CTA merge (thread = (head parity, channel)) into the segment's partial slot
    float* slot = partial_slot(ws, unit, G);
    const int ch = tid & 127;
    for (int hh = tid >> 7; hh < G; hh += 2) {
      float m = rslot[hh * kPartialStride];
#pragma unroll
      for (int w = 0; w < kPairs; ++w) m = fmaxf(m, part[(w * kMaxG + hh) * kPartialStride]);
      float l = 0.f, a = 0.f;
      if (m != -INFINITY) {
#pragma unroll
        for (int w = 0; w <= kPairs; ++w) {
          const float* p = w < kPairs ? part + (w * kMaxG + hh) * kPartialStride : rslot + hh * kPartialStride;
          if (p[0] == -INFINITY) continue;
          const float f = exp2f(p[0] - m);
          l = fmaf(p[1], f, l);
          a = fmaf(p[2 + ch], f, a);
        }
      }
      float* o = slot + hh * kPartialStride;
      if (ch == 0) {
        o[0] = m;
        o[1] = l;
      }
      o[2 + ch] = a;
    }
    combine_segment(ws, seg, G, out, g);
  });
}

constexpr int kMaxDevices = 64;

template <int BHI, int BLO, int NT, int NHS, bool MQ>
cudaError_t launch_ws_t(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax, float* out,
                        DecodeWs ws, cudaStream_t s) {
  constexpr int R = record_bytes_of<BHI, BLO, NHS>();
  constexpr int S = ws_stages<BHI, BLO, NT, NHS>();
  static_assert(S >= 2, "ring too shallow");
  static std::atomic<int> wave_cache[kMaxDevices];   // resident CTAs of a full wave, 0 until known
  if (g.record_bytes != R) return cudaErrorInvalidValue;
  const WsSmem sm = ws_smem(NT, R, S);
  auto kern = decode_ws_kernel<BHI, BLO, NT, NHS, MQ>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cacheable = dev >= 0 && dev < kMaxDevices;
  int wave = cacheable ? wave_cache[dev].load(std::memory_order_relaxed) : 0;
  if (wave == 0) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sm.total);
    if (e != cudaSuccess) return e;
    int sms = 148, occ = 1;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kWsThreads, sm.total);
    if (e != cudaSuccess) return e;
    wave = sms * (occ > 0 ? occ : 1);
    if (cacheable) wave_cache[dev].store(wave, std::memory_order_relaxed);
  }
  ws.N = wave < nmax ? wave : nmax;
  kern<<<ws.N, kWsThreads, sm.total, s>>>(g, q, c, out, ws);
  return cudaGetLastError();
}

template <int BHI, int BLO, int NT, bool MQ>
cudaError_t launch_ws_nhs(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax, float* out,
                          DecodeWs ws, cudaStream_t s) {
  switch (g.nhs) {
    case 0: return launch_ws_t<BHI, BLO, NT, 0, MQ>(g, q, c, nmax, out, ws, s);
    case 2: return launch_ws_t<BHI, BLO, NT, 2, MQ>(g, q, c, nmax, out, ws, s);
    case 4: return launch_ws_t<BHI, BLO, NT, 4, MQ>(g, q, c, nmax, out, ws, s);
    case 8: return launch_ws_t<BHI, BLO, NT, 8, MQ>(g, q, c, nmax, out, ws, s);
    default: break;
  }
  if constexpr (BLO == 2) {   // one salient slice (k = 8) only exists with 2-bit lo words
    if (g.nhs == 1) return launch_ws_t<BHI, BLO, NT, 1, MQ>(g, q, c, nmax, out, ws, s);
  }
  return cudaErrorInvalidValue;
}

template <int BHI, int BLO, int NT>
cudaError_t launch_ws_mq(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax, float* out,
                         DecodeWs ws, cudaStream_t s) {
  return g.tq > 1 ? launch_ws_nhs<BHI, BLO, NT, true>(g, q, c, nmax, out, ws, s)
                  : launch_ws_nhs<BHI, BLO, NT, false>(g, q, c, nmax, out, ws, s);
}

}  // namespace

cudaError_t launch_decode_ws(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax,
                             float* out, DecodeWs ws, cudaStream_t s) {
  const bool nt2 = g.rows > 4;
  if (g.bhi == 4 && g.blo == 2)
    return nt2 ? launch_ws_mq<4, 2, 2>(g, q, c, nmax, out, ws, s) : launch_ws_mq<4, 2, 1>(g, q, c, nmax, out, ws, s);
  if (g.bhi == 2 && g.blo == 1)
    return nt2 ? launch_ws_mq<2, 1, 2>(g, q, c, nmax, out, ws, s) : launch_ws_mq<2, 1, 1>(g, q, c, nmax, out, ws, s);
  return cudaErrorInvalidValue;
}

}  // namespace pnmix
