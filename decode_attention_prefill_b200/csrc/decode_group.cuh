// decode_group.cuh -- the per-group work of the tensor-core decode kernels (decode_mma.cu,
// decode_rows.cu): the key side (q . k^ over one or two 32-token group records with m16n8k16
// MMAs on codes taken as exact fp16 subnormals), the lazy online softmax, and the value side
// (P . v^), for one warp and the query rows it holds (4 per 8-column tile of the key side,
// heads 4*nt + tq of the lane; the value side's columns are rows gq).  See decode_mma.cu for
// the formulation.
#pragma once

#include "common.cuh"
#include "decode_common.cuh"
#include "decode_frag.cuh"

namespace pnmix {
namespace {

// Headroom (log2 domain) the lazy softmax reference keeps above the largest logit seen.
constexpr float kHeadroom = 4.f;

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
                                             const int (&tok0)[NG], int vis_base, int row0, float (&lg)[NG][NT][4]) {
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
          const int lim = vis_base + (row0 + 4 * nt + tq) / g.G;
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
                                                     const float (&lg)[NG][NT][4], WarpAcc<NT>& st, int kc,
                                                     int row0) {
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
  const bool col_ok = gq < g.rows - row0;
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

// Key and value side of NG group records for the query rows row0 .. row0 + 4 NT - 1 of a
// unit (the lane's columns), folded into the warp's state.
template <int BHI, int BLO, int NT, int NHS, int NG, bool MQ>
__device__ __forceinline__ void process_groups(const Geometry& g, const uint8_t* const (&recs)[NG],
                                               const QFrags<NT>& qf, float qscale, const RowScale<BHI, BLO>& rs,
                                               const int (&tok0)[NG], int vis_base, int row0, WarpAcc<NT>& st) {
  float lg[NG][NT][4];
  group_logits<BHI, BLO, NT, NHS, NG, MQ>(g, recs, qf, qscale, rs, tok0, vis_base, row0, lg);
  group_softmax_values<NT, NG, MQ>(g, recs, lg, st, key_code_bytes<BHI, BLO, NHS>(), row0);
}

}  // namespace
}  // namespace pnmix
