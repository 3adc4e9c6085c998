// decode_mma.cu -- tensor-core decode attention over the packed cache, one role per warp.
//
// One CTA = one slice of the work partition (decode_common.cuh), 4 warps.  Every warp
// takes a contiguous run of each segment's 32-token group records, stages them two
// records per TMA bulk copy into its own shared-memory ring of record pairs, and keeps its
// own online softmax.  Per group:
//
//   logits  q . k^_t = sum_p q_p (s_p code_{p,t} + z_p)
//          = [codes (32 tok x 128 pos)] x [q_p s_p]  +  [z] x [q]
//   The codes become exact fp16 A fragments in registers: an AND leaves them as fp16
//   subnormals code * 2^(offset-24), which the tensor cores multiply exactly.  The bf16
//   query is exact in fp16; the product q_p s_p (19 significant bits) is carried exactly
//   by two interleaved B columns (head h -> columns 2h, 2h+1): fp16(q s) and its rounding
//   error fma(q, s, -fp16(q s)).  One lane-uniform sequence b = fma(X, s, fp16(Y s)) with
//   per-lane constants (X, Y) = (0, q) on even columns and (q, -q) on odd ones gives both.
//   The zero-point term is one more MMA per slice PAIR whose A operand is the 16-byte
//   zero-point chunk of the pair exactly as loaded (rows 0-7 carry the even slice's zeros,
//   rows 8-15 the odd slice's, see the key scale order in include/pnmix.h) and whose B
//   operand carries q of the even slice on the odd columns and q of the odd slice on the
//   even columns: rows 0-7 of a head's odd column and rows 8-15 of its even column are the
//   two slices' sums.  The softmax scale is applied to the fp32 logits.
//   out     sum_t p_t v^_t = sum_t (p_t s_{t,j}) code_{t,c} + sum_t p_t z_{t,j}
//          = [codes^T (channels x tokens)] x [p s]  +  [z rows] x [p]
//   with p rounded to fp16 once (fp32 accumulation); the value zero-point chunk of a lane
//   likewise serves both 16-token halves of a group from one load.
//
// The online softmax keeps a lazy reference m per head: a group pair only takes the
// cross-lane max when one of its logits exceeds m, and then sets m = max + kHeadroom, so
// p = 2^(logit - m) <= 1 and the accumulators are rescaled a few times per segment.
//
// The bit placement of the record (include/pnmix.h) is the fragment ownership of the
// m16n8k16 tiles, so a lane's code words are exactly its A registers.  Splits merge
// through decode_common.cuh (fused combine, no waiting).  The bf16 residual window is
// attended with CUDA cores by the CTA whose slice holds it (one query row per warp).
#include <atomic>

#include "common.cuh"
#include "decode_common.cuh"
#include "decode_frag.cuh"
#include "quantize_group.cuh"

namespace pnmix {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
// Headroom (log2 domain) the lazy softmax reference keeps above the largest logit seen.
constexpr float kHeadroom = 4.f;
// Work-partition weights (decode_common.cuh, unit_items), in group items: the fixed cost of
// a unit's segment and the residual window's CUDA-core pass.
constexpr int kLeadItems = 40;
constexpr int kResidItems = 8;
// Fused append, flush step: the quantizers' staging tile sits in the (then idle) ring.
static_assert(sizeof(GroupSmem) <= 4 * 2 * 2 * 3072, "the quantizers' tile must fit the staging ring");
// Staging ring per warp: 2 record pairs (4 records), three CTAs per SM.
template <int NT>
__host__ __device__ constexpr int pair_slots() { return 2; }

// ------------------------------------------------------------------ shared memory map

struct SmemMap {
  int qsets;     // [NT][2 sets (X, Y)][4 slice pairs][32 lanes][4 words]
  int qnat;      // fp32 [kMaxG][128], natural channel order, unscaled
  int perm;      // 128 bytes
  int resid;     // fp32 [kMaxG][kPartialStride]: partial of the residual item
  int bars;      // uint64 [kWarps][slots] mbarriers
  int stages;    // [kWarps][slots][2 R]
  int part;      // fp32 [kWarps][kMaxG][kPartialStride], aliases the stages
  int total;
};

__host__ __device__ __forceinline__ SmemMap smem_map(int NT, int R) {
  const int nsl = NT == 1 ? pair_slots<1>() : pair_slots<2>();
  SmemMap m;
  m.qsets = 0;
  m.qnat = NT * 2 * 4 * 32 * 16;
  m.perm = m.qnat + kMaxG * kHeadDim * 4;
  m.resid = m.perm + 128;
  m.bars = m.resid + kMaxG * kPartialStride * 4;
  m.stages = m.bars + ((kWarps * nsl * 8 + 127) / 128) * 128;
  int stage_bytes = kWarps * nsl * 2 * R;
  int part_bytes = kWarps * kMaxG * kPartialStride * 4;
  m.part = m.stages;
  m.total = m.stages + (stage_bytes > part_bytes ? stage_bytes : part_bytes);
  return m;
}

// ------------------------------------------------------------------ per-warp state

template <int NT>
struct WarpAcc {
  float m[NT];          // lazy softmax reference (log2 domain) of head 4*nt + tq
  float l[NT];          // this lane's partial sum of 2^(logit - m)
  float pv[8][4];       // P.V accumulators: channels 16m + gq (+8), heads 2tq, 2tq+1
  float bias[2][4];     // zero-point term: [0] rows 0-7 (first 16 tokens of each group),
                        // [1] rows 8-15 (last 16); row gq = channel group, heads 2tq, 2tq+1
};

// Logit scale factors: a row-u token's key products carry 2^(shift(u) - 24).
template <int BHI, int BLO>
struct RowScale {
  float hi[4], lo[4];
  __device__ __forceinline__ explicit RowScale(float qscale) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      hi[u] = __int_as_float((127 + 24 - key_row_shift<BHI>(u)) << 23) * qscale;
      lo[u] = __int_as_float((127 + 24 - key_row_shift<BLO>(u)) << 23) * qscale;
    }
  }
};

// Key side of NG group records: the log2-domain logits lg[gi][nt][u] of head 4*nt + tq at
// tokens gq + 8u of group gi.  With NG = 2 the two groups' MMA chains interleave.
template <int BHI, int BLO, int NT, int NHS, int NG, bool MQ>
__device__ __forceinline__ void group_logits(const Geometry& g, const uint8_t* const (&recs)[NG],
                                             const QFrags<NT>& qf, float qscale, const RowScale<BHI, BLO>& rs,
                                             const int (&tok0)[NG], int vis_base, float (&lg)[NG][NT][4]) {
  constexpr int WH = NHS * BHI / 2;   // key-code words per lane of the salient block
  constexpr int kc = key_code_bytes<BHI, BLO, NHS>();
  const int lane = threadIdx.x & 31;
  const int tq = lane & 3;

  // key-code products, kept apart per block because the two blocks' token-row bit
  // offsets differ; the zero-point term (normal fp16 scale), one product per slice pair
  float acc_hi[NG][NT][2][4], acc_lo[NG][NT][2][4], dz[NG][NT][4];
#pragma unroll
  for (int gi = 0; gi < NG; ++gi)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        dz[gi][nt][i] = 0.f;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          acc_hi[gi][nt][x][i] = 0.f;
          acc_lo[gi][nt][x][i] = 0.f;
        }
      }

#pragma unroll
  for (int sp = 0; sp < 4; ++sp) {
    // this lane's scale / zero chunk of slice pair sp: (even e=0, odd e=0, even e=1, odd e=1)
    uint4 s4[NG], z4[NG];
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
      s4[gi] = reinterpret_cast<const uint4*>(recs[gi] + kc + tq * 64)[sp];
      z4[gi] = reinterpret_cast<const uint4*>(recs[gi] + kc + 256 + tq * 64)[sp];
    }
#pragma unroll
    for (int par = 0; par < 2; ++par) {
      const int sigma = 2 * sp + par;
      const bool hi = sigma < NHS;
#pragma unroll
      for (int gi = 0; gi < NG; ++gi) {
        // ---- A fragments of this slice (2 M-tiles x 4 registers)
        const uint32_t* kw = reinterpret_cast<const uint32_t*>(recs[gi]);
        uint32_t A[2][4];
        if (hi) {
          if constexpr (BHI == 4)
            key_slice_frags<4>(kw[(2 * sigma) * 32 + lane], kw[(2 * sigma + 1) * 32 + lane], 0, A);
          else
            key_slice_frags<BHI>(kw[sigma * 32 + lane], 0u, 0, A);
        } else {
          const int sl = sigma - NHS;   // slice inside the lo block
          if constexpr (BLO == 2)
            key_slice_frags<2>(kw[(WH + sl) * 32 + lane], 0u, 0, A);
          else   // two slices per word; NHS is even, so sl % 2 == sigma % 2
            key_slice_frags<1>(kw[(WH + (sl >> 1)) * 32 + lane], 0u, par, A);
        }
        const uint32_t s0 = par ? s4[gi].y : s4[gi].x, s1 = par ? s4[gi].w : s4[gi].z;
        // ---- B fragments: fp16(q s) on even columns, its rounding error on odd ones;
        // X alone (q on odd columns) for the zero-point term
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint4& X = qf.x[nt][sp];
          const uint4& Y = qf.y[nt][sp];
          const uint32_t qx0 = par ? X.z : X.x, qx1 = par ? X.w : X.y;
          const uint32_t qy0 = par ? Y.z : Y.x, qy1 = par ? Y.w : Y.y;
          const uint32_t b0 = hfma2(qx0, s0, hmul2(qy0, s0));
          const uint32_t b1 = hfma2(qx1, s1, hmul2(qy1, s1));
          if (hi) {
            mma16816(acc_hi[gi][nt][0], A[0][0], A[0][1], A[0][2], A[0][3], b0, b1);
            mma16816(acc_hi[gi][nt][1], A[1][0], A[1][1], A[1][2], A[1][3], b0, b1);
          } else {
            mma16816(acc_lo[gi][nt][0], A[0][0], A[0][1], A[0][2], A[0][3], b0, b1);
            mma16816(acc_lo[gi][nt][1], A[1][0], A[1][1], A[1][2], A[1][3], b0, b1);
          }
          if (par == 0) mma16816(dz[gi][nt], z4[gi].x, z4[gi].y, z4[gi].z, z4[gi].w, qf.z[nt][sp].x, qf.z[nt][sp].y);
        }
      }
    }
  }

  // ---- logits (log2 domain): lane holds head 4*nt + tq at tokens gq + 8*u, u = 0..3; the
  // zero-point sum of the head: rows 0-7 (even slices) of its odd column plus rows 8-15
  // (odd slices) of its even column
#pragma unroll
  for (int gi = 0; gi < NG; ++gi)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float zb = (dz[gi][nt][1] + dz[gi][nt][2]) * qscale;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int mt = u >> 1, r = 2 * (u & 1);
        const float vhi = acc_hi[gi][nt][mt][r] + acc_hi[gi][nt][mt][r + 1];
        const float vlo = acc_lo[gi][nt][mt][r] + acc_lo[gi][nt][mt][r + 1];
        if constexpr (NHS == 0)
          lg[gi][nt][u] = fmaf(vlo, rs.lo[u], zb);
        else if constexpr (NHS == 8)
          lg[gi][nt][u] = fmaf(vhi, rs.hi[u], zb);
        else
          lg[gi][nt][u] = fmaf(vhi, rs.hi[u], fmaf(vlo, rs.lo[u], zb));
      }
    }

  // ---- multi-query steps: row v sees tokens below vis_base + v / G (only the newest
  // tokens of a unit can be hidden, so only a group reaching them takes this branch)
  if constexpr (MQ) {
    const int gq = lane >> 2;
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
      if (tok0[gi] + kGroup > vis_base) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int lim = vis_base + (4 * nt + tq) / g.G;
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (tok0[gi] + gq + 8 * u >= lim) lg[gi][nt][u] = -INFINITY;
        }
      }
    }
  }
}

// Multiply the value-side accumulators by the per-head factors alpha (lane holds heads tq
// and 4 + tq in alpha[0], alpha[1]; the accumulator columns are heads 2tq, 2tq+1).
template <int NT>
__device__ __forceinline__ void rescale_values(WarpAcc<NT>& st, const float (&alpha)[NT]) {
  const int lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int h0 = 2 * tq, h1 = 2 * tq + 1;
  float a0 = __shfl_sync(0xffffffffu, alpha[0], gq * 4 + (h0 & 3));
  float a1 = __shfl_sync(0xffffffffu, alpha[0], gq * 4 + (h1 & 3));
  if constexpr (NT == 2) {
    const float b0 = __shfl_sync(0xffffffffu, alpha[1], gq * 4 + (h0 & 3));
    const float b1 = __shfl_sync(0xffffffffu, alpha[1], gq * 4 + (h1 & 3));
    if (h0 >= 4) a0 = b0;
    if (h1 >= 4) a1 = b1;
  }
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    st.pv[m][0] *= a0;
    st.pv[m][1] *= a1;
    st.pv[m][2] *= a0;
    st.pv[m][3] *= a1;
  }
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    st.bias[x][0] *= a0;
    st.bias[x][1] *= a1;
    st.bias[x][2] *= a0;
    st.bias[x][3] *= a1;
  }
}

// Value side of NG group records with their logits: lazy online softmax update, P as B
// fragments, P x V into the warp's accumulators.
template <int NT, int NG, bool MQ>
__device__ __forceinline__ void group_softmax_values(const Geometry& g, const uint8_t* const (&recs)[NG],
                                                     const float (&lg)[NG][NT][4], WarpAcc<NT>& st, int kc) {
  const int lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;

  // ---- lazy reference: the cross-lane max only when a logit exceeds the reference
  float mloc[NT];
  bool raise = false;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float mx = -INFINITY;
#pragma unroll
    for (int gi = 0; gi < NG; ++gi)
      mx = fmaxf(mx, fmaxf(fmaxf(lg[gi][nt][0], lg[gi][nt][1]), fmaxf(lg[gi][nt][2], lg[gi][nt][3])));
    mloc[nt] = mx;
    raise |= mx > st.m[nt];
  }
  if (__any_sync(0xffffffffu, raise)) {
    float alpha[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float mx = mloc[nt];
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float mnew = mx > st.m[nt] ? mx + kHeadroom : st.m[nt];
      alpha[nt] = mnew == st.m[nt] ? 1.f : ex2(st.m[nt] - mnew);   // 0 from -inf
      st.l[nt] *= alpha[nt];
      st.m[nt] = mnew;
    }
    rescale_values<NT>(st, alpha);
  }

  const int srcA = (2 * tq) * 4 + (gq & 3), srcB = (2 * tq + 1) * 4 + (gq & 3);
  const bool col_ok = gq < g.rows;
  const uint32_t four2 = 0x44004400u;   // fp16x2 (4, 4)
#pragma unroll
  for (int gi = 0; gi < NG; ++gi) {
    const uint8_t* rec = recs[gi];
    float p[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if constexpr (MQ)   // a head that sees no token yet keeps m = -inf: its masked logits give 0
          p[nt][i] = lg[gi][nt][i] == -INFINITY ? 0.f : ex2(lg[gi][nt][i] - st.m[nt]);
        else
          p[nt][i] = ex2(lg[gi][nt][i] - st.m[nt]);
        st.l[nt] += p[nt][i];
      }
    }
    // ---- P as B fragments: column gq = head gq, tokens 2tq + {0,1} (+8, +16, +24)
    float pa[4], pb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      pa[i] = __shfl_sync(0xffffffffu, p[0][i], srcA);
      pb[i] = __shfl_sync(0xffffffffu, p[0][i], srcB);
    }
    if constexpr (NT == 2) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float xa = __shfl_sync(0xffffffffu, p[1][i], srcA);
        const float xb = __shfl_sync(0xffffffffu, p[1][i], srcB);
        if (gq >= 4) {
          pa[i] = xa;
          pb[i] = xb;
        }
      }
    }
    uint32_t p16[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) p16[i] = col_ok ? pack_f16x2(pa[i], pb[i]) : 0u;

    // value scales: token pairs tq + 4i, four channel groups each
    const int vs_off = kc + 1536, vz_off = kc + 1792;
    uint32_t vsr[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(rec + vs_off + (tq + 4 * i) * 16);
      vsr[i][0] = v.x; vsr[i][1] = v.y; vsr[i][2] = v.z; vsr[i][3] = v.w;
    }
    // zero-point term: A rows = channel groups (row gq holds group gq & 3; rows 4-7 repeat
    // them and are not read), k = tokens.  The chunk (tq, j) holds the zero pairs of token
    // pairs tq, tq + 8, tq + 4, tq + 12: as one A operand its rows 0-7 are the first 16
    // tokens (with P of tokens 0-15) and its rows 8-15 the last 16 (with P of tokens 16-31).
    {
      const uint4 zc = *reinterpret_cast<const uint4*>(rec + vz_off + (tq * 4 + (gq & 3)) * 16);
      mma16816(st.bias[0], zc.x, zc.y, zc.z, zc.w, p16[0], p16[1]);
      mma16816(st.bias[1], zc.x, zc.y, zc.z, zc.w, p16[2], p16[3]);
    }
    // value codes: words 0..7 of this lane (two 16-byte chunks).  Slot (r, p) of word m
    // sits at bits 8r + 2p; it is taken in place from w >> 8r, so token block p carries
    // 2^(2p).  The B rows of block p are scaled by 2^(2 - 2p) to leave a uniform 2^2.
    const uint32_t bp0 = hmul2(p16[0], four2);                 // x 4
    const uint32_t bp2 = hmul2(p16[2], 0x34003400u);           // x 1/4
    const uint32_t bp3 = hmul2(p16[3], 0x2C002C00u);           // x 1/16
    const uint4 vw0 = *reinterpret_cast<const uint4*>(rec + kc + 512 + lane * 16);
    const uint4 vw1 = *reinterpret_cast<const uint4*>(rec + kc + 512 + (32 + lane) * 16);
    const uint32_t vw[8] = {vw0.x, vw0.y, vw0.z, vw0.w, vw1.x, vw1.y, vw1.z, vw1.w};
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int j = m >> 1;
      const uint32_t w = vw[m], w8 = w >> 8;
      // (r, p) -> k-step p >> 1, register r + 2*(p & 1)
      const uint32_t k0a0 = sub_pair(w, 0x00030003u), k0a2 = sub_pair(w, 0x000C000Cu);
      const uint32_t k1a0 = sub_pair(w, 0x00300030u), k1a2 = sub_pair(w, 0x00C000C0u);
      const uint32_t k0a1 = sub_pair(w8, 0x00030003u), k0a3 = sub_pair(w8, 0x000C000Cu);
      const uint32_t k1a1 = sub_pair(w8, 0x00300030u), k1a3 = sub_pair(w8, 0x00C000C0u);
      const uint32_t b00 = hmul2(bp0, vsr[0][j]), b01 = hmul2(p16[1], vsr[1][j]);
      const uint32_t b10 = hmul2(bp2, vsr[2][j]), b11 = hmul2(bp3, vsr[3][j]);
      mma16816(st.pv[m], k0a0, k0a1, k0a2, k0a3, b00, b01);
      mma16816(st.pv[m], k1a0, k1a1, k1a2, k1a3, b10, b11);
    }
  }
}

template <int BHI, int BLO, int NT, int NHS, int NG, bool MQ>
__device__ __forceinline__ void process_groups(const Geometry& g, const uint8_t* const (&recs)[NG],
                                               const QFrags<NT>& qf, float qscale, const RowScale<BHI, BLO>& rs,
                                               const int (&tok0)[NG], int vis_base, WarpAcc<NT>& st) {
  float lg[NG][NT][4];
  group_logits<BHI, BLO, NT, NHS, NG, MQ>(g, recs, qf, qscale, rs, tok0, vis_base, lg);
  group_softmax_values<NT, NG, MQ>(g, recs, lg, st, key_code_bytes<BHI, BLO, NHS>());
}

// MQ: several queries per sequence (rows = G * tq), with the causal mask on the newest
// tokens; a separate instance so the one-query kernel carries none of it.
template <int BHI, int BLO, int NT, int NHS, bool MQ>
__global__ void __launch_bounds__(kThreads, 3)
decode_mma_kernel(Geometry g, const uint16_t* __restrict__ q, pnmix_cache c, float* __restrict__ out,
                  DecodeWs ws) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int R = record_bytes_of<BHI, BLO, NHS>();
  constexpr int kSlots = pair_slots<NT>();
  const int G = g.rows;   // query rows per unit
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const SmemMap sm = smem_map(NT, R);
  uint32_t* qsets = reinterpret_cast<uint32_t*>(smem + sm.qsets);
  float* qnat = reinterpret_cast<float*>(smem + sm.qnat);
  uint8_t* perm = smem + sm.perm;
  float* rslot = reinterpret_cast<float*>(smem + sm.resid);
  float* part = reinterpret_cast<float*>(smem + sm.part);
  uint8_t* ring = smem + sm.stages + warp * kSlots * 2 * R;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sm.bars) + warp * kSlots;
  if (lane == 0) {
    for (int k = 0; k < kSlots; ++k) mbar_init(bars + k, 1);
    fence_mbar_init();
  }
  __syncwarp();
  // The ring is used in order across the warp's segments: pairs are issued into slot
  // `iss_slot` and taken from slot `use_slot`, whose barrier completes phase `use_phase`.
  int iss_slot = 0, use_slot = 0;
  uint32_t use_phase = 0;
  bool failed = false;   // a staging wait ran out: stage and consume nothing more
  const float qscale = g.scale * kLog2e;
  const RowScale<BHI, BLO> rs(qscale);

  for_each_segment(g, c.len, ws.N, [&](const Segment& seg) {
    const int b = seg.b, h = seg.h, unit = seg.unit;
    if (seg.lo >= seg.hi) {   // a slice of lead items only: an empty partial for the combine
      float* o = partial_slot(ws, unit, G);
      for (int hh = 0; hh < G; ++hh) {
        if (tid == 0) {
          o[hh * kPartialStride] = -INFINITY;
          o[hh * kPartialStride + 1] = 0.f;
        }
        o[hh * kPartialStride + 2 + tid] = 0.f;
      }
      combine_segment(ws, seg, G, out, g);
      return;
    }
    const int vis_base = seg.ng * kGroup + seg.nr - g.tq + 1;   // tokens row 0 sees
    // ---- this warp's contiguous run [g0, g0 + my_count) of the segment's groups, taken
    // as pairs of consecutive records (a last single record when the count is odd)
    // fused append: on a flush step the new token completes group seg.ng - 1, whose record
    // this launch builds; the CTA owning that item quantizes it first (staging tile in the
    // idle ring), stores it, and then stages it like every other record
    const int gf = seg.ng - 1;
    const bool own_flush = seg.app_slot == kGroup - 1 && gf >= seg.lo && gf < seg.hi;
    const int gend = seg.hi < seg.ng ? seg.hi : seg.ng;
    const int n = gend > seg.lo ? gend - seg.lo : 0;
    const int g0 = seg.lo + (n * warp) / kWarps;
    const int my_count = seg.lo + (n * (warp + 1)) / kWarps - g0;
    const int my_pairs = (my_count + 1) >> 1;
    const uint8_t* unit_rec = record_ptr(g, c.records, b, h, 0);
    const bool stage = unit != g.skip_unit;   // false only under the timeout test hook
    int issued = 0;     // pairs of this segment handed to the copy engine
    int consumed = 0;   // pairs of this segment taken from the ring
    // Issue the warp's pairs [issued, upto).  A pair may only be issued into a slot whose
    // previous pair has been consumed, which the callers keep (upto <= consumed + kSlots).
    auto issue_upto = [&](int upto) {
      const int last = upto < my_pairs ? upto : my_pairs;
      if (failed || !stage) return;
      for (; issued < last; ++issued) {
        const int gi = 2 * issued;
        const uint32_t bytes = static_cast<uint32_t>(gi + 1 < my_count ? 2 * R : R);
        stage_group(ring + iss_slot * 2 * R, unit_rec + static_cast<size_t>(g0 + gi) * R, bytes, bars + iss_slot,
                    lane == 0);
        iss_slot = iss_slot + 1 == kSlots ? 0 : iss_slot + 1;
      }
    };
    // wait until the next pair has landed; returns its slot (or nullptr after a timeout)
    auto acquire = [&]() -> const uint8_t* {
      uint32_t spins = 0;
      while (!failed && !mbar_try_wait(bars + use_slot, use_phase)) {
        if (++spins >= g.wait_limit) {
          failed = true;
          if (lane == 0) atomicOr(c.error, PNMIX_DEVERR_TIMEOUT);
        }
      }
      failed = __any_sync(0xffffffffu, failed);   // keep the warp's control flow uniform
      if (failed) return nullptr;
      const uint8_t* r = ring + use_slot * 2 * R;
      if (++use_slot == kSlots) {
        use_slot = 0;
        use_phase ^= 1u;
      }
      ++consumed;
      return r;
    };
    // ---- fused append, flush step: quantize the 31 residual rows and the new row into the
    // record of group gf and store it (the bit-exact quantizers of quantize_group.cuh, the
    // staging tile in this CTA's ring, idle between segments), before any copy is issued
    if (own_flush) {
      __syncthreads();   // every warp of the CTA is past its previous segment's ring use
      GroupSmem& gs = *reinterpret_cast<GroupSmem*>(smem + sm.stages);
      gs.perm[tid] = c.perm[static_cast<size_t>(unit) * kHeadDim + tid] & (kHeadDim - 1);
      const uint16_t* rows[2] = {c.k_resid + static_cast<size_t>(unit) * kGroup * kHeadDim,
                                 c.v_resid + static_cast<size_t>(unit) * kGroup * kHeadDim};
      const uint16_t* fresh[2] = {ws.k_new + static_cast<size_t>(unit) * kHeadDim,
                                  ws.v_new + static_cast<size_t>(unit) * kHeadDim};
      uint8_t* frec = record_ptr(g, c.records, b, h, gf);
#pragma unroll 1
      for (int part = 0; part < 2; ++part) {
        for (int i = tid; i < kGroup * 16; i += kThreads) {
          const int r = i >> 4, cc = i & 15;
          const uint4* src = r == kGroup - 1 ? reinterpret_cast<const uint4*>(fresh[part]) + cc
                                             : reinterpret_cast<const uint4*>(rows[part]) + i;
          *reinterpret_cast<uint4*>(&gs.tile[r][cc * 8]) = __ldg(src);
        }
        __syncthreads();
        if (part == 0)
          quantize_key_group(g, gs, frec);
        else
          quantize_value_group(g, gs, frec);
        __syncthreads();
      }
      // the record was written through the generic proxy; the bulk copy that stages it
      // reads through the async proxy
      __threadfence();
      asm volatile("fence.proxy.async.global;" ::: "memory");
      __syncthreads();
    }
    issue_upto(kSlots);

    // ---- query: unscaled fp32 in natural channel order, then the X / Y fp16 column sets
    // in position order
    load_query_rows(g, q, c.perm, b, h, unit, qnat, perm, tid);
    const bool seg_resid = seg.hi > seg.ng && seg.nr > 0;
    uint16_t* rk = c.k_resid + static_cast<size_t>(unit) * kGroup * kHeadDim;
    uint16_t* rv = c.v_resid + static_cast<size_t>(unit) * kGroup * kHeadDim;
    if (seg_resid && seg.app_slot >= 0 && tid < 32) {
      // fused append: the new row goes into residual slot app_slot (< 31) of the cache;
      // the residual partial below reads the window from there (plain loads, after the
      // barrier)
      const int cc = tid & 15;
      const uint16_t* src = (tid < 16 ? ws.k_new : ws.v_new) + static_cast<size_t>(unit) * kHeadDim;
      uint16_t* dst = (tid < 16 ? rk : rv) + seg.app_slot * kHeadDim;
      reinterpret_cast<uint4*>(dst)[cc] = __ldg(reinterpret_cast<const uint4*>(src) + cc);
    }
    if (g.n_prune > 0) {   // dynamic query-channel pruning of the staged query rows
      __syncthreads();
      prune_query_rows(g, qnat, warp, kWarps);
    }
    __syncthreads();
    {
      const int L = lane, chunk = warp;   // entries 4*chunk .. 4*chunk+3 (= sigma*2 + e)
      const int tq = L & 3, gq = L >> 2;
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
            sets[0][v] = hl ? qb : 0u;              // X
            sets[1][v] = hl ? (qb ^ 0x8000u) : qb;  // Y
          }
#pragma unroll
          for (int s = 0; s < 2; ++s)
            qsets[(((nt * 2 + s) * 4 + chunk) * 32 + L) * 4 + i] = sets[s][0] | (sets[s][1] << 16);
        }
      }
    }
    __syncthreads();

    // ---- the residual item (CUDA cores, rows read from the cache): warp w takes heads w, w + 4
    if (seg_resid) {
      residual_partial(g, rk, rv, seg.nr, qnat, qscale, rslot, warp, kWarps, seg.ng * kGroup, vis_base, kHeadDim);
    } else if (warp == 0 && lane < G) {
      rslot[lane * kPartialStride + 0] = -INFINITY;
      rslot[lane * kPartialStride + 1] = 0.f;
    }

    // ---- the warp's groups; the query constants stay in registers for the segment
    QFrags<NT> qf;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int cp = 0; cp < 4; ++cp) {
        qf.x[nt][cp] = reinterpret_cast<const uint4*>(qsets)[((nt * 2 + 0) * 4 + cp) * 32 + lane];
        qf.y[nt][cp] = reinterpret_cast<const uint4*>(qsets)[((nt * 2 + 1) * 4 + cp) * 32 + lane];
        // zero-point B operand of slice pair cp: q of the even slice on odd columns (X), q of
        // the odd slice on even columns (Y holds q there)
        const bool odd_col = (lane >> 2) & 1;
        qf.z[nt][cp] = odd_col ? make_uint2(qf.x[nt][cp].x, qf.x[nt][cp].y) : make_uint2(qf.y[nt][cp].z, qf.y[nt][cp].w);
      }
    WarpAcc<NT> st;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      st.m[nt] = -INFINITY;
      st.l[nt] = 0.f;
    }
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int i = 0; i < 4; ++i) st.pv[m][i] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      st.bias[0][i] = 0.f;
      st.bias[1][i] = 0.f;
    }

    for (int i = 0; i < my_pairs; ++i) {
      issue_upto(i + kSlots);
      const uint8_t* slot = acquire();
      if (slot == nullptr) break;   // warp-uniform
      const int ga = g0 + 2 * i;
      if (2 * i + 1 < my_count) {
        const uint8_t* const recs[2] = {slot, slot + R};
        const int tok[2] = {ga * kGroup, (ga + 1) * kGroup};
        if constexpr (NT == 1) {
          process_groups<BHI, BLO, NT, NHS, 2, MQ>(g, recs, qf, qscale, rs, tok, vis_base, st);
        } else {   // two tiles of query columns: one group at a time
          const uint8_t* const r0[1] = {recs[0]};
          const uint8_t* const r1[1] = {recs[1]};
          const int t0[1] = {tok[0]}, t1[1] = {tok[1]};
          process_groups<BHI, BLO, NT, NHS, 1, MQ>(g, r0, qf, qscale, rs, t0, vis_base, st);
          process_groups<BHI, BLO, NT, NHS, 1, MQ>(g, r1, qf, qscale, rs, t1, vis_base, st);
        }
      } else {
        const uint8_t* const recs[1] = {slot};
        const int tok[1] = {ga * kGroup};
        process_groups<BHI, BLO, NT, NHS, 1, MQ>(g, recs, qf, qscale, rs, tok, vis_base, st);
      }
      __syncwarp();
    }
    if (failed) {   // let the pairs issued and not yet taken land before the shared memory is reused
      for (; consumed < issued; ++consumed) {
        for (uint32_t spins = 0; spins < g.wait_limit && !mbar_try_wait(bars + use_slot, use_phase); ++spins) {
        }
        if (++use_slot == kSlots) {
          use_slot = 0;
          use_phase ^= 1u;
        }
      }
    }
    __syncthreads();   // every ring is idle: the merge area may alias them

    // ---- warp partials into shared memory
    {
      const int gq = lane >> 2, tq = lane & 3;
      float lsum[NT];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float v = st.l[nt];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        lsum[nt] = v;
      }
      float* wp = part + warp * kMaxG * kPartialStride;
      const bool any = consumed > 0;
      if (gq == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int hh = 4 * nt + tq;
          if (hh < G) {
            wp[hh * kPartialStride + 0] = any ? st.m[nt] : -INFINITY;
            wp[hh * kPartialStride + 1] = any ? lsum[nt] : 0.f;
          }
        }
      }
      // zero-point term of channel group j for heads 2tq, 2tq+1: rows j (first 16 tokens)
      // and 8 + j (last 16) of lane (j, tq)
      const float zs0 = st.bias[0][0] + st.bias[1][2], zs1 = st.bias[0][1] + st.bias[1][3];
      float bz[4][2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bz[j][0] = __shfl_sync(0xffffffffu, zs0, j * 4 + tq);
        bz[j][1] = __shfl_sync(0xffffffffu, zs1, j * 4 + tq);
      }
      const int h0 = 2 * tq, h1 = 2 * tq + 1;
      const float pv_scale = 4194304.0f;   // 2^22: the codes' 2^-24 and the pairs' 2^2
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int j = m >> 1;
        const int c0 = 16 * m + gq, c1 = c0 + 8;
        if (h0 < G) {
          wp[h0 * kPartialStride + 2 + c0] = fmaf(st.pv[m][0], pv_scale, bz[j][0]);
          wp[h0 * kPartialStride + 2 + c1] = fmaf(st.pv[m][2], pv_scale, bz[j][0]);
        }
        if (h1 < G) {
          wp[h1 * kPartialStride + 2 + c0] = fmaf(st.pv[m][1], pv_scale, bz[j][1]);
          wp[h1 * kPartialStride + 2 + c1] = fmaf(st.pv[m][3], pv_scale, bz[j][1]);
        }
      }
    }
    __syncthreads();

    // ---- CTA merge (thread = channel) into the segment's partial slot
    float* slotp = partial_slot(ws, unit, G);
    for (int hh = 0; hh < G; ++hh) {
      float m = rslot[hh * kPartialStride];
#pragma unroll
      for (int w = 0; w < kWarps; ++w) m = fmaxf(m, part[(w * kMaxG + hh) * kPartialStride]);
      float l = 0.f, a = 0.f;
      if (m != -INFINITY) {
#pragma unroll
        for (int w = 0; w <= kWarps; ++w) {
          const float* p = w < kWarps ? part + (w * kMaxG + hh) * kPartialStride : rslot + hh * kPartialStride;
          if (p[0] == -INFINITY) continue;
          const float f = exp2f(p[0] - m);
          l = fmaf(p[1], f, l);
          a = fmaf(p[2 + tid], f, a);
        }
      }
      float* o = slotp + hh * kPartialStride;
      if (tid == 0) {
        o[0] = m;
        o[1] = l;
      }
      o[2 + tid] = a;
    }
    combine_segment(ws, seg, G, out, g);
  });

  // ---- fused append: the grid's last CTA (every CTA has read len[] by now) advances the
  // lengths, as pnmix_append does; a full sequence keeps its length and raises the error bit
  if (g.append) {
    __shared__ int last_cta;
    uint32_t* ticket = c.scratch + scratch_fused_ticket_offset(g.B, g.Hkv);
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      last_cta = atomicAdd(ticket, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (last_cta) {
      __threadfence();
      for (int bb = tid; bb < g.B; bb += kThreads) {
        const int raw = c.len[bb];
        if (appends(g, raw))
          c.len[bb] = raw + 1;
        else
          atomicOr(c.error, PNMIX_DEVERR_APPEND_FULL);
      }
      if (tid == 0) *ticket = 0u;
    }
  }
}

// Resident CTAs of one full wave of a kernel instance, per device: the shared-memory
// attribute and the occupancy query run once per (instance, device), not on every decode
// step (they cost more host time than a small launch's kernel).  The record size is fixed
// by the instance's bit widths, so the shared-memory footprint is too.
constexpr int kMaxDevices = 64;

template <int BHI, int BLO, int NT, int NHS, bool MQ>
cudaError_t launch_mma_t(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax, float* out,
                         DecodeWs ws, cudaStream_t s) {
  static std::atomic<int> wave_cache[kMaxDevices];   // 0 until known
  if (g.record_bytes != record_bytes_of<BHI, BLO, NHS>()) return cudaErrorInvalidValue;
  const SmemMap sm = smem_map(NT, g.record_bytes);
  auto kern = decode_mma_kernel<BHI, BLO, NT, NHS, MQ>;
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
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, sm.total);
    if (e != cudaSuccess) return e;
    wave = sms * (occ > 0 ? occ : 1);
    if (cacheable) wave_cache[dev].store(wave, std::memory_order_relaxed);
  }
  ws.N = wave < nmax ? wave : nmax;
  // partition weights: a unit's fixed cost (query setup, merge, combine) and its residual
  // window (CUDA cores, rows read from L2), in 32-token group items, measured on B200 at 32K
  Geometry gw = g;
  gw.lead = kLeadItems;
  gw.resid_w = kResidItems;
  kern<<<ws.N, kThreads, sm.total, s>>>(gw, q, c, out, ws);
  return cudaGetLastError();
}

template <int BHI, int BLO, int NT, bool MQ>
cudaError_t launch_mma_nhs(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax, float* out,
                           DecodeWs ws, cudaStream_t s) {
  switch (g.nhs) {
    case 0: return launch_mma_t<BHI, BLO, NT, 0, MQ>(g, q, c, nmax, out, ws, s);
    case 2: return launch_mma_t<BHI, BLO, NT, 2, MQ>(g, q, c, nmax, out, ws, s);
    case 4: return launch_mma_t<BHI, BLO, NT, 4, MQ>(g, q, c, nmax, out, ws, s);
    case 8: return launch_mma_t<BHI, BLO, NT, 8, MQ>(g, q, c, nmax, out, ws, s);
    default: break;
  }
  if constexpr (BLO == 2) {   // one salient slice (k = 8) only exists with 2-bit lo words
    if (g.nhs == 1) return launch_mma_t<BHI, BLO, NT, 1, MQ>(g, q, c, nmax, out, ws, s);
  }
  return cudaErrorInvalidValue;
}

template <int BHI, int BLO, int NT>
cudaError_t launch_mma_mq(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax, float* out,
                          DecodeWs ws, cudaStream_t s) {
  return g.tq > 1 ? launch_mma_nhs<BHI, BLO, NT, true>(g, q, c, nmax, out, ws, s)
                  : launch_mma_nhs<BHI, BLO, NT, false>(g, q, c, nmax, out, ws, s);
}

}  // namespace

cudaError_t launch_decode_mma(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax,
                              float* out, DecodeWs ws, cudaStream_t s) {
  const bool nt2 = g.rows > 4;
  if (g.bhi == 4 && g.blo == 2)
    return nt2 ? launch_mma_mq<4, 2, 2>(g, q, c, nmax, out, ws, s) : launch_mma_mq<4, 2, 1>(g, q, c, nmax, out, ws, s);
  if (g.bhi == 2 && g.blo == 1)
    return nt2 ? launch_mma_mq<2, 1, 2>(g, q, c, nmax, out, ws, s) : launch_mma_mq<2, 1, 1>(g, q, c, nmax, out, ws, s);
  return cudaErrorInvalidValue;
}

}  // namespace pnmix
