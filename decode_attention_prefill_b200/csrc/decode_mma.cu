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
#include "decode_group.cuh"
#include "quantize_group.cuh"

namespace pnmix {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
// Work-partition weights (decode_common.cuh, unit_items), in group items: the fixed cost of
// a unit's segment and the residual window's CUDA-core pass.
constexpr int kLeadItems = 28;
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
    if (g.n_prune_slices > 0) {   // key-slice pruning of the staged query rows
      __syncthreads();
      const uint32_t pmask = pruned_slices(g, qnat, perm);
      __syncthreads();
      zero_pruned_slices(g, qnat, perm, pmask, tid, kThreads);
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
          process_groups<BHI, BLO, NT, NHS, 2, MQ>(g, recs, qf, qscale, rs, tok, vis_base, 0, st);
        } else {   // two tiles of query columns: one group at a time
          const uint8_t* const r0[1] = {recs[0]};
          const uint8_t* const r1[1] = {recs[1]};
          const int t0[1] = {tok[0]}, t1[1] = {tok[1]};
          process_groups<BHI, BLO, NT, NHS, 1, MQ>(g, r0, qf, qscale, rs, t0, vis_base, 0, st);
          process_groups<BHI, BLO, NT, NHS, 1, MQ>(g, r1, qf, qscale, rs, t1, vis_base, 0, st);
        }
      } else {
        const uint8_t* const recs[1] = {slot};
        const int tok[1] = {ga * kGroup};
        process_groups<BHI, BLO, NT, NHS, 1, MQ>(g, recs, qf, qscale, rs, tok, vis_base, 0, st);
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
