// decode_rows.cu -- tensor-core decode attention for many query rows per KV head: a
// multi-token step (speculative verify, chunked decode) with rows = G * T from 9 to 64.
//
// The one-role kernel (decode_mma.cu) holds all of a unit's rows in every warp, which
// stops at 8 rows (two 8-column tiles of the key side).  Here the rows are split across
// warps instead: warp w holds rows 8w .. 8w + 7 (two key-side tiles of 4 rows with the
// exact two-column q.s split, one value-side tile of 8 rows) and every warp of the CTA goes
// over every group record of the segment.  The records are staged once per CTA, two per
// TMA bulk copy, into a shared ring: a slot's full barrier completes when its copy lands,
// its empty barrier when every warp is done with it, and warp 0 refills a slot only after
// that.  So the packed cache is read once per step for all T queries, and the per-group
// work per row is that of the one-role kernel (decode_group.cuh) minus nothing: the code
// unpacking is repeated per warp, the price of keeping each warp's accumulators in its
// registers.
//
// Causal mask: row v (query v / G) sees the first len - T + 1 + v / G tokens; only groups
// that reach the newest tokens take the masking branch.  Split-K over the context and the
// fused combine as in the other kernels (decode_common.cuh), with up to 64 rows.
#include <atomic>

#include "common.cuh"
#include "decode_common.cuh"
#include "decode_frag.cuh"
#include "decode_group.cuh"

namespace pnmix {
namespace {

constexpr int kRowsPerWarp = 8;
constexpr int kRowWarps = kMaxRows / kRowsPerWarp;   // at most 8 warps
constexpr int kRowSlots = 4;                          // ring of record pairs

// Shared memory of a launch with `nrows` rows per unit (rounded up to whole warps of 8), so
// that small launches fit several CTAs per SM.
struct RowsSmem {
  int qnat;    // fp32 [rows][128], natural channel order, unscaled
  int perm;    // 128 bytes
  int resid;   // fp32 [rows][kPartialStride]: partial of the residual item
  int bars;    // uint64 full[kRowSlots], empty[kRowSlots]
  int ring;    // [kRowSlots][2 R]
  int part;    // fp32 [rows][kPartialStride], each warp's rows, aliases the ring
  int total;
};

__host__ __device__ __forceinline__ RowsSmem rows_smem(int R, int nrows) {
  const int rows = (nrows + kRowsPerWarp - 1) / kRowsPerWarp * kRowsPerWarp;
  RowsSmem m;
  m.qnat = 0;
  m.perm = m.qnat + rows * kHeadDim * 4;
  m.resid = m.perm + 128;
  m.bars = m.resid + (rows * kPartialStride * 4 + 15) / 16 * 16;
  m.ring = m.bars + 256;
  const int ring_bytes = kRowSlots * 2 * R, part_bytes = rows * kPartialStride * 4;
  m.part = m.ring;
  m.total = m.ring + (ring_bytes > part_bytes ? ring_bytes : part_bytes);
  return m;
}

__device__ __forceinline__ void mbar_arrive_cta(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// The query constants of a warp's two tiles (rows row0 .. row0 + 7), built in registers from
// the unit's rows in shared memory: X = (0 | q) and Y = (q | -q) on even | odd columns, z the
// zero-point operand (q of the even slice on odd columns, of the odd slice on even ones).
__device__ __forceinline__ void build_qfrags(const float* qnat, const uint8_t* perm, int row0, int rows,
                                             QFrags<2>& qf) {
  const int lane = threadIdx.x & 31, tq = lane & 3, gq = lane >> 2;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const int col = gq + 8 * nt, hh = col >> 1, hl = col & 1;
    const int row = row0 + hh;
#pragma unroll
    for (int cp = 0; cp < 4; ++cp) {
      uint32_t xs[4], ys[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int idx = cp * 4 + i, sigma = idx >> 1, e = idx & 1;
        const int p0 = 16 * sigma + 8 * e + 2 * tq;
        uint32_t sets[2][2];
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const float x = row < rows ? qnat[row * kHeadDim + perm[p0 + v]] : 0.f;
          const uint32_t qb = __half_as_ushort(__float2half_rn(x));
          sets[0][v] = hl ? qb : 0u;
          sets[1][v] = hl ? (qb ^ 0x8000u) : qb;
        }
        xs[i] = sets[0][0] | (sets[0][1] << 16);
        ys[i] = sets[1][0] | (sets[1][1] << 16);
      }
      qf.x[nt][cp] = make_uint4(xs[0], xs[1], xs[2], xs[3]);
      qf.y[nt][cp] = make_uint4(ys[0], ys[1], ys[2], ys[3]);
      qf.z[nt][cp] = (gq & 1) ? make_uint2(xs[0], xs[1]) : make_uint2(ys[2], ys[3]);
    }
  }
}

template <int BHI, int BLO, int NHS>
__global__ void __launch_bounds__(kRowWarps * 32)
decode_rows_kernel(Geometry g, const uint16_t* __restrict__ q, pnmix_cache c, float* __restrict__ out,
                   DecodeWs ws) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int R = record_bytes_of<BHI, BLO, NHS>();
  const int G = g.rows;
  const int nwarps = blockDim.x >> 5;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row0 = warp * kRowsPerWarp;
  const RowsSmem sm = rows_smem(R, G);
  float* qnat = reinterpret_cast<float*>(smem + sm.qnat);
  uint8_t* perm = smem + sm.perm;
  float* rslot = reinterpret_cast<float*>(smem + sm.resid);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + sm.bars);
  uint64_t* empty = full + kRowSlots;
  uint8_t* ring = smem + sm.ring;
  float* part = reinterpret_cast<float*>(smem + sm.part);
  __shared__ int stop_flag;
  if (tid == 0) {
    stop_flag = 0;
    for (int k = 0; k < kRowSlots; ++k) {
      mbar_init(full + k, 1);
      mbar_init(empty + k, nwarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* stop = &stop_flag;
  // Pairs of records are numbered in order across the CTA's segments: pair n lives in slot
  // n % S; its copy completes phase n / S of full[slot], and its release by every warp
  // completes phase n / S of empty[slot].  Warp 0 issues (nis = pairs issued so far) and
  // may refill a slot only after the release of the pair it held; every warp consumes in
  // order (ncons = pairs consumed so far, the same in every warp while nothing stops).
  uint32_t nis = 0, ncons = 0;
  const float qscale = g.scale * kLog2e;
  const RowScale<BHI, BLO> rs(qscale);
  // bounded wait on phase `parity` of `bar`; on running out, stop the CTA
  auto wait_bar = [&](uint64_t* bar, uint32_t parity) -> bool {
    uint32_t spins = 0;
    while (!mbar_try_wait(bar, parity)) {
      if (*stop) return false;
      if (++spins >= g.wait_limit) {
        *stop = 1;
        if (lane == 0) atomicOr(c.error, PNMIX_DEVERR_TIMEOUT);
        return false;
      }
    }
    return true;
  };

  for_each_segment(g, c.len, ws.N, [&](const Segment& seg) {
    const int b = seg.b, h = seg.h, unit = seg.unit;
    const int vis_base = seg.ng * kGroup + seg.nr - g.tq + 1;   // tokens row 0 sees
    const int gend = seg.hi < seg.ng ? seg.hi : seg.ng;
    const int ngr = gend > seg.lo ? gend - seg.lo : 0;
    const int npairs = (ngr + 1) >> 1;
    const uint8_t* unit_rec = record_ptr(g, c.records, b, h, 0);
    const bool stage = unit != g.skip_unit;   // false only under the timeout test hook
    int issued = 0;                          // pairs of the segment issued (warp 0)
    // warp 0: copy the segment's next pair into its slot, after the slot's previous pair
    // was released by every warp
    auto issue_next = [&]() {
      if (*stop || !stage || issued >= npairs) return;
      const uint32_t n = nis, slot = n % kRowSlots;
      bool ok = true;
      if (lane == 0 && n >= static_cast<uint32_t>(kRowSlots)) ok = wait_bar(empty + slot, ((n / kRowSlots) - 1) & 1u);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok || *stop) return;
      const int gi = seg.lo + 2 * issued;
      const uint32_t bytes = static_cast<uint32_t>(gi + 1 < gend ? 2 * R : R);
      stage_group(ring + slot * 2 * R, unit_rec + static_cast<size_t>(gi) * R, bytes, full + slot, lane == 0);
      ++nis;
      ++issued;
    };
    if (warp == 0)
      for (int k = 0; k < kRowSlots; ++k) issue_next();

    // ---- query rows and order
    for (int i = tid; i < nwarps * kRowsPerWarp * (kHeadDim / 8); i += blockDim.x) {
      const int hh = i >> 4;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (hh < G) v = __ldg(reinterpret_cast<const uint4*>(q + row_offset(g, b, h, hh)) + (i & 15));
      float4* dst = reinterpret_cast<float4*>(qnat + i * 8);
      dst[0] = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                           __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u));
      dst[1] = make_float4(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xFFFF0000u),
                           __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xFFFF0000u));
    }
    if (tid < kHeadDim / 16)
      reinterpret_cast<uint4*>(perm)[tid] =
          __ldg(reinterpret_cast<const uint4*>(c.perm + static_cast<size_t>(unit) * kHeadDim) + tid);
    __syncthreads();
    if (g.n_prune > 0) {
      prune_query_rows(g, qnat, warp, nwarps);
      __syncthreads();
    }
    if (g.n_prune_slices > 0) {   // key-slice pruning of the staged query rows
      const uint32_t pmask = pruned_slices(g, qnat, perm);
      __syncthreads();
      zero_pruned_slices(g, qnat, perm, pmask, tid, blockDim.x);
      __syncthreads();
    }
    const bool seg_resid = seg.hi > seg.ng && seg.nr > 0;
    if (seg_resid) {   // the residual window on CUDA cores, rows spread over the warps
      residual_partial(g, c.k_resid + static_cast<size_t>(unit) * kGroup * kHeadDim,
                       c.v_resid + static_cast<size_t>(unit) * kGroup * kHeadDim, seg.nr, qnat, qscale, rslot, warp,
                       nwarps, seg.ng * kGroup, vis_base, kHeadDim);
    } else {
      for (int hh = tid; hh < G; hh += blockDim.x) {
        rslot[hh * kPartialStride + 0] = -INFINITY;
        rslot[hh * kPartialStride + 1] = 0.f;
      }
    }
    QFrags<2> qf;
    build_qfrags(qnat, perm, row0, G, qf);
    WarpAcc<2> st;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
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

    // ---- every warp over every pair of the segment
    int consumed = 0;
    for (int i = 0; i < npairs; ++i) {
      const uint32_t n = ncons, slot = n % kRowSlots;
      bool ok = true;
      if (lane == 0) ok = wait_bar(full + slot, (n / kRowSlots) & 1u);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      const uint8_t* rp = ring + slot * 2 * R;
      const int ga = seg.lo + 2 * i;
      if (row0 < G) {
        const uint8_t* const r0[1] = {rp};
        const int t0[1] = {ga * kGroup};
        process_groups<BHI, BLO, 2, NHS, 1, true>(g, r0, qf, qscale, rs, t0, vis_base, row0, st);
        if (ga + 1 < gend) {
          const uint8_t* const r1[1] = {rp + R};
          const int t1[1] = {(ga + 1) * kGroup};
          process_groups<BHI, BLO, 2, NHS, 1, true>(g, r1, qf, qscale, rs, t1, vis_base, row0, st);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cta(empty + slot);
      ++ncons;
      ++consumed;
      if (warp == 0) issue_next();
    }
    // after a stop: let the copies warp 0 issued and did not take land before the shared
    // memory is reused (a later pair's phase cannot complete: nothing more is issued)
    if (*stop && warp == 0 && lane == 0) {
      for (uint32_t n = ncons; n < nis; ++n) {
        const uint32_t slot = n % kRowSlots;
        for (uint32_t spins = 0; spins < g.wait_limit && !mbar_try_wait(full + slot, (n / kRowSlots) & 1u); ++spins) {
        }
      }
    }
    __syncthreads();   // the ring is idle: the partials may alias it

    // ---- this warp's rows: group partial into shared memory (the ring is idle now)
    {
      const int gq = lane >> 2, tq = lane & 3;
      float lsum[2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        float v = st.l[nt];
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        lsum[nt] = v;
      }
      const bool any = consumed > 0;
      if (gq == 0) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const int hh = row0 + 4 * nt + tq;
          if (hh < G) {
            part[hh * kPartialStride + 0] = any ? st.m[nt] : -INFINITY;
            part[hh * kPartialStride + 1] = any ? lsum[nt] : 0.f;
          }
        }
      }
      const float zs0 = st.bias[0][0] + st.bias[1][2], zs1 = st.bias[0][1] + st.bias[1][3];
      float bz[4][2];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bz[j][0] = __shfl_sync(0xffffffffu, zs0, j * 4 + tq);
        bz[j][1] = __shfl_sync(0xffffffffu, zs1, j * 4 + tq);
      }
      const int h0 = row0 + 2 * tq, h1 = h0 + 1;
      const float pv_scale = 4194304.0f;   // 2^22: the codes' 2^-24 and the pairs' 2^2
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int j = m >> 1;
        const int c0 = 16 * m + gq, c1 = c0 + 8;
        if (h0 < G) {
          part[h0 * kPartialStride + 2 + c0] = fmaf(st.pv[m][0], pv_scale, bz[j][0]);
          part[h0 * kPartialStride + 2 + c1] = fmaf(st.pv[m][2], pv_scale, bz[j][0]);
        }
        if (h1 < G) {
          part[h1 * kPartialStride + 2 + c0] = fmaf(st.pv[m][1], pv_scale, bz[j][1]);
          part[h1 * kPartialStride + 2 + c1] = fmaf(st.pv[m][3], pv_scale, bz[j][1]);
        }
      }
    }
    __syncthreads();
    // ---- merge with the residual partial, row by row, into the segment's slot
    float* slotp = partial_slot(ws, unit, G);
    for (int hh = warp; hh < G; hh += nwarps) {
      // a part with m = -inf holds nothing (its sums may be unset): it takes no term at all
      const float mg = part[hh * kPartialStride], mr = rslot[hh * kPartialStride];
      const float m = fmaxf(mg, mr);
      const bool has_g = mg != -INFINITY, has_r = mr != -INFINITY;
      const float fg = has_g ? exp2f(mg - m) : 0.f, fr = has_r ? exp2f(mr - m) : 0.f;
      float* o = slotp + hh * kPartialStride;
      if (lane == 0) {
        o[0] = m;
        o[1] = (has_g ? part[hh * kPartialStride + 1] * fg : 0.f) + (has_r ? rslot[hh * kPartialStride + 1] * fr : 0.f);
      }
      for (int cc = lane; cc < kHeadDim; cc += 32)
        o[2 + cc] = (has_g ? part[hh * kPartialStride + 2 + cc] * fg : 0.f) +
                    (has_r ? rslot[hh * kPartialStride + 2 + cc] * fr : 0.f);
    }
    combine_segment<kMaxRows>(ws, seg, G, out, g);
  });
}

constexpr int kMaxDevices = 64;

template <int BHI, int BLO, int NHS>
cudaError_t launch_rows_t(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax, float* out,
                          DecodeWs ws, cudaStream_t s) {
  // resident CTAs of a full wave, per device and warp count (2 .. 8 warps of 8 rows)
  static std::atomic<int> wave_cache[kMaxDevices][kRowWarps + 1];
  if (g.record_bytes != record_bytes_of<BHI, BLO, NHS>()) return cudaErrorInvalidValue;
  const RowsSmem sm = rows_smem(g.record_bytes, g.rows);
  auto kern = decode_rows_kernel<BHI, BLO, NHS>;
  const int nwarps = (g.rows + kRowsPerWarp - 1) / kRowsPerWarp;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cacheable = dev >= 0 && dev < kMaxDevices;
  int wave = cacheable ? wave_cache[dev][nwarps].load(std::memory_order_relaxed) : 0;
  if (wave == 0) {
    // the attribute for the largest map this kernel instance can get (64 rows)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             rows_smem(g.record_bytes, kMaxRows).total);
    if (e != cudaSuccess) return e;
    int sms = 148, occ = 1;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, nwarps * 32, sm.total);
    if (e != cudaSuccess) return e;
    wave = sms * (occ > 0 ? occ : 1);
    if (cacheable) wave_cache[dev][nwarps].store(wave, std::memory_order_relaxed);
  }
  ws.N = wave < nmax ? wave : nmax;
  kern<<<ws.N, nwarps * 32, sm.total, s>>>(g, q, c, out, ws);
  return cudaGetLastError();
}

template <int BHI, int BLO>
cudaError_t launch_rows_nhs(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax, float* out,
                            DecodeWs ws, cudaStream_t s) {
  switch (g.nhs) {
    case 0: return launch_rows_t<BHI, BLO, 0>(g, q, c, nmax, out, ws, s);
    case 2: return launch_rows_t<BHI, BLO, 2>(g, q, c, nmax, out, ws, s);
    case 4: return launch_rows_t<BHI, BLO, 4>(g, q, c, nmax, out, ws, s);
    case 8: return launch_rows_t<BHI, BLO, 8>(g, q, c, nmax, out, ws, s);
    default: break;
  }
  if constexpr (BLO == 2) {
    if (g.nhs == 1) return launch_rows_t<BHI, BLO, 1>(g, q, c, nmax, out, ws, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_rows(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax, float* out,
                               DecodeWs ws, cudaStream_t s) {
  if (g.rows < 1 || g.rows > kMaxRows) return cudaErrorInvalidValue;
  if (g.bhi == 4 && g.blo == 2) return launch_rows_nhs<4, 2>(g, q, c, nmax, out, ws, s);
  if (g.bhi == 2 && g.blo == 1) return launch_rows_nhs<2, 1>(g, q, c, nmax, out, ws, s);
  return cudaErrorInvalidValue;
}

}  // namespace pnmix
