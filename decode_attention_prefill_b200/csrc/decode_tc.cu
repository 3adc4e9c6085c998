// decode_tc.cu -- decode attention on the 5th-generation tensor cores (tcgen05, TMEM) for
// many query rows per KV head: a multi-token step (speculative verify, chunked decode) with
// up to 64 rows = G * T.
//
// One CTA (one warpgroup, 128 threads) per slice of the work partition (decode_common.cuh);
// thread r owns query row r, which is TMEM lane r of every accumulator (rows >= G are
// zero).  Per 32-token group record:
//
//   logits  S = Q x K^T:  A = the unit's query rows, fp16 (exact from bf16), 128 x 128
//           positions, written once per segment; B = the group's keys as two fp16 tiles,
//           hi = fp16(x) and lo = fp16(x - hi) of x = code * s + z in fp32 (32 tokens x
//           128 positions), so that hi + lo carries x to 22 bits; 16 MMAs of K = 16
//           (8 slices x hi, lo) accumulate the 128 x 32 fp32 logits in TMEM.
//   softmax each thread loads its row's 32 logits (tcgen05.ld), applies the softmax scale
//           and the causal mask, and keeps a lazy online reference m per row (raised to
//           max + 4 only when a logit exceeds it, so p = 2^(logit - m) <= 1); a raise
//           rescales the row's value accumulator in TMEM (load, scale, store).
//   values  O += P x V:  A = P (fp16, 128 rows x 32 tokens), B = the dequantized values as
//           hi / lo fp16 tiles (128 channels x 32 tokens); 4 MMAs of K = 16 accumulate the
//           128 x 128 fp32 output rows in TMEM.
//
// The bf16 residual window takes the same path as one more group (its keys and values
// split into hi / lo exactly, the tokens past it masked).  One thread issues every MMA
// (tcgen05.mma, operands from shared memory, K-major, no swizzle) and commits each batch
// to an mbarrier; the records arrive by TMA bulk copy (no multicast) into a ring of three.
// Every wait is bounded.  At the end of a segment each thread writes its row's partial
// (m, l, O) for the fused combine.
#include <atomic>

#include "common.cuh"
#include "decode_common.cuh"
#include "decode_frag.cuh"

namespace pnmix {
namespace {

constexpr int kTcThreads = 128;   // one warpgroup: TMEM lanes 0 .. 127
constexpr int kTcSlots = 3;       // record ring
constexpr int kTmemCols = 256;    // logits in columns 0 .. 31, outputs in 128 .. 255
constexpr int kTmemOut = 128;

// Byte offset of element (row r, k) of an operand tile of `rows` rows in the K-major
// no-swizzle layout: K = 16 steps of rows x 32 bytes; inside a step, 8-row core matrices of
// 8 rows x 16 bytes, the two 8-element halves of K 128 bytes apart, row groups 256 apart.
__device__ __forceinline__ int tile_off(int rows, int r, int k) {
  return (k >> 4) * rows * 32 + (r >> 3) * 256 + ((k >> 3) & 1) * 128 + (r & 7) * 16 + (k & 7) * 2;
}
// Shared-memory matrix descriptor of one K = 16 step (no swizzle, version 1).
__device__ __forceinline__ uint64_t tile_desc(const void* step_base) {
  const uint32_t a = smem_u32(step_base);
  return static_cast<uint64_t>((a >> 4) & 0x3FFFu) | (static_cast<uint64_t>(128u >> 4) << 16) |
         (static_cast<uint64_t>(256u >> 4) << 32) | (1ull << 46);
}
// Instruction descriptor: fp16 A and B, fp32 D, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t mma_idesc(int n) {
  return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | ((128u >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate ? 1u : 0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane (warp-collective).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])),
        "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
        "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
        "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
        "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
        "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
        "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
        "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
        "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// x split into two fp16 whose sum is x to 22 bits, packed (hi, lo) for two adjacent K.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
  const __half l0 = __float2half_rn(x0 - __half2float(h0)), l1 = __float2half_rn(x1 - __half2float(h1));
  hi = static_cast<uint32_t>(__half_as_ushort(h0)) | (static_cast<uint32_t>(__half_as_ushort(h1)) << 16);
  lo = static_cast<uint32_t>(__half_as_ushort(l0)) | (static_cast<uint32_t>(__half_as_ushort(l1)) << 16);
}

struct TcSmem {
  int aq;      // fp16 [128 rows][128 positions]
  int bk_hi;   // fp16 [32 tokens][128 positions]
  int bk_lo;
  int ap;      // fp16 [128 rows][32 tokens]
  int bv_hi;   // fp16 [128 channels][32 tokens]
  int bv_lo;
  int qnat;    // fp32 [64 rows][128], aliases bk_hi .. bv_lo (segment setup only)
  int ring;    // [kTcSlots][R]
  int perm;    // 128 bytes
  int bars;    // uint64 full[kTcSlots], mma_k, mma_v; uint32 TMEM address
  int total;
};

__host__ __device__ __forceinline__ TcSmem tc_smem(int R) {
  TcSmem m;
  m.aq = 0;
  m.bk_hi = m.aq + 128 * 128 * 2;
  m.bk_lo = m.bk_hi + 32 * 128 * 2;
  m.ap = m.bk_lo + 32 * 128 * 2;
  m.bv_hi = m.ap + 128 * 32 * 2;
  m.bv_lo = m.bv_hi + 128 * 32 * 2;
  m.qnat = m.bk_hi;   // 32 KB inside the 40 KB of tiles
  m.ring = m.bv_lo + 128 * 32 * 2;
  m.perm = m.ring + kTcSlots * ((R + 127) / 128 * 128);
  m.bars = m.perm + 128;
  m.total = m.bars + 128;
  return m;
}

template <int BHI, int BLO, int NHS>
__global__ void __launch_bounds__(kTcThreads, 2)
decode_tc_kernel(Geometry g, const uint16_t* __restrict__ q, pnmix_cache c, float* __restrict__ out, DecodeWs ws) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int R = record_bytes_of<BHI, BLO, NHS>();
  constexpr int WH = NHS * BHI / 2;                   // key-code words per lane, salient block
  constexpr int NW = WH + (8 - NHS) * BLO / 2;        // key-code words per lane
  constexpr int KC = key_code_bytes<BHI, BLO, NHS>();
  const TcSmem sm = tc_smem(R);
  const int G = g.rows;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint8_t* aq = smem + sm.aq;
  uint8_t* bkh = smem + sm.bk_hi;
  uint8_t* bkl = smem + sm.bk_lo;
  uint8_t* ap = smem + sm.ap;
  uint8_t* bvh = smem + sm.bv_hi;
  uint8_t* bvl = smem + sm.bv_lo;
  float* qnat = reinterpret_cast<float*>(smem + sm.qnat);
  uint8_t* perm = smem + sm.perm;
  constexpr int kSlotBytes = (R + 127) / 128 * 128;
  uint8_t* ring = smem + sm.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + sm.bars);
  uint64_t* bar_k = full + kTcSlots;
  uint64_t* bar_v = bar_k + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_v + 1);
  __shared__ int fail_sh;

  if (tid == 0) {
    fail_sh = 0;
    for (int k = 0; k < kTcSlots; ++k) mbar_init(full + k, 1);
    mbar_init(bar_k, 1);
    mbar_init(bar_v, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;   // this warp's TMEM lanes
  const uint32_t t_logit = tmem + lane_base, t_out = tmem + lane_base + kTmemOut;
  volatile int* fail = &fail_sh;
  const float qscale = g.scale * kLog2e;
  constexpr uint32_t kIdescK = mma_idesc(32), kIdescV = mma_idesc(128);
  // records staged so far / taken so far (ring position), MMA batches committed so far
  uint32_t nis = 0, ncons = 0, nk = 0, nv = 0;
  // bounded wait for phase `parity` of `bar`; gives up (error bit, CTA-wide stop) after
  // `limit` rounds: g.wait_limit for the staged records, kDecodeWaitLimit for the tensor
  // cores' commits (they always arrive; the bound only guards against a hang, and a product
  // still in flight must not outlive the TMEM it writes)
  auto wait_bar = [&](uint64_t* bar, uint32_t parity, uint32_t limit) -> bool {
    uint32_t spins = 0;
    while (!mbar_try_wait(bar, parity)) {
      if (++spins >= limit) {
        *fail = 1;
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
    const bool seg_resid = seg.hi > seg.ng && seg.nr > 0;
    const uint8_t* unit_rec = record_ptr(g, c.records, b, h, 0);
    const bool stage = unit != g.skip_unit;   // false only under the timeout test hook
    int issued = 0;
    // thread 0: stage the segment's next record into its slot (the slot's previous record
    // has been consumed: records are taken in order and a slot is refilled after its
    // record's tiles were built)
    auto issue_next = [&]() {
      if (*fail || !stage || issued >= ngr) return;
      const uint32_t slot = nis % kTcSlots;
      stage_group(ring + slot * kSlotBytes, unit_rec + static_cast<size_t>(seg.lo + issued) * R, R, full + slot, true);
      ++nis;
      ++issued;
    };
    if (tid == 0)
      for (int k = 0; k < kTcSlots; ++k) issue_next();

    // ---- query rows (fp32, natural order) and the position order; pruning as elsewhere
    for (int i = tid; i < kMaxRows * (kHeadDim / 8); i += kTcThreads) {
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
      prune_query_rows(g, qnat, warp, kTcThreads / 32);
      __syncthreads();
    }
    if (g.n_prune_slices > 0) {
      const uint32_t pmask = pruned_slices(g, qnat, perm);
      __syncthreads();
      zero_pruned_slices(g, qnat, perm, pmask, tid, kTcThreads);
      __syncthreads();
    }
    // A = Q (row tid, positions in order; bf16 -> fp16 is exact in fp16's normal range)
    {
      const int r = tid;
#pragma unroll 4
      for (int j = 0; j < kHeadDim; j += 2) {
        const float x0 = r < G ? qnat[r * kHeadDim + (perm[j] & (kHeadDim - 1))] : 0.f;
        const float x1 = r < G ? qnat[r * kHeadDim + (perm[j + 1] & (kHeadDim - 1))] : 0.f;
        const uint32_t w = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(x0))) |
                           (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(x1))) << 16);
        *reinterpret_cast<uint32_t*>(aq + tile_off(128, r, j)) = w;
      }
    }
    proxy_fence();
    __syncthreads();   // qnat (aliasing the tiles) is no longer needed

    float m_row = -INFINITY, l_row = 0.f;
    bool out_live = false;   // the TMEM output rows hold a value MMA's result
    const int nitems = ngr + (seg_resid ? 1 : 0);
    for (int it = 0; it < nitems && !*fail; ++it) {
      const bool resid_item = it == ngr;
      const int tok0 = resid_item ? seg.ng * kGroup : (seg.lo + it) * kGroup;
      const int ntok = resid_item ? seg.nr : kGroup;
      const uint8_t* rec = nullptr;
      if (!resid_item) {
        if (tid == 0) wait_bar(full + (ncons % kTcSlots), (ncons / kTcSlots) & 1u, g.wait_limit);
        __syncthreads();
        if (*fail) break;
        rec = ring + (ncons % kTcSlots) * kSlotBytes;
      }
      // ---- key tiles: x = code * s + z (or the bf16 residual key), split hi / lo
      if (!resid_item) {
        const uint16_t* ks = reinterpret_cast<const uint16_t*>(rec + KC);
        const uint16_t* kz = reinterpret_cast<const uint16_t*>(rec + KC + 256);
        for (int item = tid; item < NW * 32; item += kTcThreads) {
          const int w = item >> 5, L = item & 31, gq = L >> 2, tq = L & 3;
          const bool hiw = w < WH;
          constexpr int kBitsHi = BHI, kBitsLo = BLO;
          const int bits = hiw ? kBitsHi : kBitsLo, mslots = 16 / bits, cmask = (1 << bits) - 1;
          const uint32_t word = reinterpret_cast<const uint32_t*>(rec)[w * 32 + L];
          const int n0 = (hiw ? w : w - WH) * mslots;
          for (int i = 0; i < mslots; ++i) {
            const int n = n0 + i, u = n & 3, cc = (n >> 2) & 1;
            const int sigma = (n >> 3) + (hiw ? 0 : NHS);
            const int p0 = 16 * sigma + 2 * tq + 8 * cc, tau = gq + 8 * u;
            const float c0 = static_cast<float>((word >> (bits * i)) & cmask);
            const float c1 = static_cast<float>((word >> (16 + bits * i)) & cmask);
            const int si = kscale_index(p0);   // p0 + 1 is element si + 1
            const float x0 = fmaf(c0, __half2float(__ushort_as_half(ks[si])), __half2float(__ushort_as_half(kz[si])));
            const float x1 =
                fmaf(c1, __half2float(__ushort_as_half(ks[si + 1])), __half2float(__ushort_as_half(kz[si + 1])));
            uint32_t hi, lo;
            split_pair(x0, x1, hi, lo);
            *reinterpret_cast<uint32_t*>(bkh + tile_off(32, tau, p0)) = hi;
            *reinterpret_cast<uint32_t*>(bkl + tile_off(32, tau, p0)) = lo;
          }
        }
      } else {
        const uint16_t* rk = c.k_resid + static_cast<size_t>(unit) * kGroup * kHeadDim;
        for (int item = tid; item < kGroup * (kHeadDim / 2); item += kTcThreads) {
          const int tau = item >> 6, p0 = 2 * (item & 63);
          float x0 = 0.f, x1 = 0.f;
          if (tau < ntok) {
            x0 = bf16_bits_to_float(rk[tau * kHeadDim + (perm[p0] & (kHeadDim - 1))]);
            x1 = bf16_bits_to_float(rk[tau * kHeadDim + (perm[p0 + 1] & (kHeadDim - 1))]);
          }
          uint32_t hi, lo;
          split_pair(x0, x1, hi, lo);
          *reinterpret_cast<uint32_t*>(bkh + tile_off(32, tau, p0)) = hi;
          *reinterpret_cast<uint32_t*>(bkl + tile_off(32, tau, p0)) = lo;
        }
      }
      proxy_fence();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
#pragma unroll 1
        for (int s = 0; s < kHeadDim / 16; ++s) {
          const uint64_t da = tile_desc(aq + s * 128 * 32);
          tc_mma(tmem, da, tile_desc(bkh + s * 32 * 32), kIdescK, s > 0);
          tc_mma(tmem, da, tile_desc(bkl + s * 32 * 32), kIdescK, true);
        }
        tc_commit(bar_k);
      }
      // ---- logits of this thread's row
      if (tid == 0) wait_bar(bar_k, nk & 1u, kDecodeWaitLimit);
      ++nk;
      __syncthreads();
      if (*fail) break;
      tc_fence_after();
      float lg[32];
      tmem_ld32(t_logit, lg);
      const int r = tid;
      const int lim = r < G ? vis_base + r / g.G : 0;   // tokens this row sees
      float mx = -INFINITY;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const bool vis = t < ntok && tok0 + t < lim;
        lg[t] = vis ? lg[t] * qscale : -INFINITY;
        mx = fmaxf(mx, lg[t]);
      }
      // ---- the previous group's value products are done with P, V and the outputs
      if (nv > 0) {
        if (tid == 0) wait_bar(bar_v, (nv - 1) & 1u, kDecodeWaitLimit);
        __syncthreads();
        if (*fail) break;
        tc_fence_after();
      }
      // lazy reference: raise it to max + 4 when a logit exceeds it, rescaling the row
      const bool raise = mx > m_row;
      float alpha = 1.f;
      if (raise) {
        const float mnew = mx + 4.f;
        alpha = m_row == -INFINITY ? 0.f : ex2(m_row - mnew);
        l_row *= alpha;
        m_row = mnew;
      }
      if (out_live && __any_sync(0xffffffffu, raise && alpha != 1.f)) {   // warp-collective TMEM traffic
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          float o[32];
          tmem_ld32(t_out + 32 * c4, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(t_out + 32 * c4, o);
        }
      }
      // P row (fp16) for the value product
#pragma unroll
      for (int t = 0; t < 32; t += 2) {
        const float p0 = lg[t] == -INFINITY ? 0.f : ex2(lg[t] - m_row);
        const float p1 = lg[t + 1] == -INFINITY ? 0.f : ex2(lg[t + 1] - m_row);
        l_row += p0 + p1;
        const uint32_t w = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(p0))) |
                           (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(p1))) << 16);
        *reinterpret_cast<uint32_t*>(ap + tile_off(128, r, t)) = w;
      }
      // ---- value tiles: v = code * s_v + z_v (or the bf16 residual value), split hi / lo
      if (!resid_item) {
        const uint8_t* vc = rec + KC + 512;
        const uint16_t* vs = reinterpret_cast<const uint16_t*>(rec + KC + 1536);
        const uint16_t* vz = reinterpret_cast<const uint16_t*>(rec + KC + 1792);
        for (int item = tid; item < 8 * 32; item += kTcThreads) {
          const int mw = item >> 5, L = item & 31, gq = L >> 2, tq = L & 3;
          const uint32_t word = *reinterpret_cast<const uint32_t*>(vc + vword_offset(mw, L));
#pragma unroll
          for (int rr = 0; rr < 2; ++rr)
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
              const int qq = rr * 4 + pp, ch = 16 * mw + gq + 8 * rr, jg = ch >> 5;
              const int t0 = 2 * tq + 8 * pp;
              const float c0 = static_cast<float>((word >> (2 * qq)) & 3u);
              const float c1 = static_cast<float>((word >> (16 + 2 * qq)) & 3u);
              const float x0 = fmaf(c0, __half2float(__ushort_as_half(vs[vscale_index(t0, jg)])),
                                    __half2float(__ushort_as_half(vz[vzero_index(t0, jg)])));
              const float x1 = fmaf(c1, __half2float(__ushort_as_half(vs[vscale_index(t0 + 1, jg)])),
                                    __half2float(__ushort_as_half(vz[vzero_index(t0 + 1, jg)])));
              uint32_t hi, lo;
              split_pair(x0, x1, hi, lo);
              *reinterpret_cast<uint32_t*>(bvh + tile_off(128, ch, t0)) = hi;
              *reinterpret_cast<uint32_t*>(bvl + tile_off(128, ch, t0)) = lo;
            }
        }
      } else {
        const uint16_t* rv = c.v_resid + static_cast<size_t>(unit) * kGroup * kHeadDim;
        for (int item = tid; item < kHeadDim * (kGroup / 2); item += kTcThreads) {
          const int ch = item >> 4, t0 = 2 * (item & 15);
          const float x0 = t0 < ntok ? bf16_bits_to_float(rv[t0 * kHeadDim + ch]) : 0.f;
          const float x1 = t0 + 1 < ntok ? bf16_bits_to_float(rv[(t0 + 1) * kHeadDim + ch]) : 0.f;
          uint32_t hi, lo;
          split_pair(x0, x1, hi, lo);
          *reinterpret_cast<uint32_t*>(bvh + tile_off(128, ch, t0)) = hi;
          *reinterpret_cast<uint32_t*>(bvl + tile_off(128, ch, t0)) = lo;
        }
      }
      proxy_fence();
      tc_fence_before();
      __syncthreads();   // the record's slot is free again; tiles and rescales are in place
      if (!resid_item) ++ncons;   // every thread: the ring position names the next record's slot
      if (tid == 0) {
        tc_fence_after();
        if (!resid_item) issue_next();
#pragma unroll 1
        for (int s = 0; s < kGroup / 16; ++s) {
          const uint64_t da = tile_desc(ap + s * 128 * 32);
          tc_mma(tmem + kTmemOut, da, tile_desc(bvh + s * 128 * 32), kIdescV, out_live || s > 0);
          tc_mma(tmem + kTmemOut, da, tile_desc(bvl + s * 128 * 32), kIdescV, true);
        }
        tc_commit(bar_v);
      }
      ++nv;
      out_live = true;
    }
    // ---- the segment's last value products (waited for even after a stop: TMEM and the
    // tiles must be idle before they are read or reused), then this row's partial
    if (nv > 0) {
      if (tid == 0)
        for (uint32_t spins = 0; spins < kDecodeWaitLimit && !mbar_try_wait(bar_v, (nv - 1) & 1u); ++spins) {
        }
      __syncthreads();
      tc_fence_after();
    }
    if (*fail && tid == 0) {   // let staged copies land before the shared memory is reused
      for (; ncons < nis; ++ncons) {
        const uint32_t slot = ncons % kTcSlots;
        for (uint32_t spins = 0; spins < g.wait_limit && !mbar_try_wait(full + slot, (ncons / kTcSlots) & 1u);
             ++spins) {
        }
      }
    }
    {
      float* o = partial_slot(ws, unit, G) + tid * kPartialStride;
      const bool live = tid < G && out_live && m_row != -INFINITY && !*fail;
#pragma unroll 1
      for (int c4 = 0; c4 < 4; ++c4) {
        float v[32];
        if (out_live) tmem_ld32(t_out + 32 * c4, v);   // warp-collective
        if (tid < G) {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[2 + 32 * c4 + i] = live ? v[i] : 0.f;
        }
      }
      if (tid < G) {
        o[0] = live ? m_row : -INFINITY;
        o[1] = live ? l_row : 0.f;
      }
    }
    tc_fence_before();
    combine_segment<kMaxRows>(ws, seg, G, out, g);
  });
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

constexpr int kMaxDevices = 64;

template <int BHI, int BLO, int NHS>
cudaError_t launch_tc_t(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax, float* out, DecodeWs ws,
                        cudaStream_t s) {
  static std::atomic<int> wave_cache[kMaxDevices];
  if (g.record_bytes != record_bytes_of<BHI, BLO, NHS>()) return cudaErrorInvalidValue;
  const TcSmem sm = tc_smem(g.record_bytes);
  auto kern = decode_tc_kernel<BHI, BLO, NHS>;
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
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kTcThreads, sm.total);
    if (e != cudaSuccess) return e;
    // TMEM: kTmemCols columns per CTA, 512 per SM
    if (occ > 512 / kTmemCols) occ = 512 / kTmemCols;
    wave = sms * (occ > 0 ? occ : 1);
    if (cacheable) wave_cache[dev].store(wave, std::memory_order_relaxed);
  }
  ws.N = wave < nmax ? wave : nmax;
  kern<<<ws.N, kTcThreads, sm.total, s>>>(g, q, c, out, ws);
  return cudaGetLastError();
}

template <int BHI, int BLO>
cudaError_t launch_tc_nhs(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax, float* out,
                          DecodeWs ws, cudaStream_t s) {
  switch (g.nhs) {
    case 0: return launch_tc_t<BHI, BLO, 0>(g, q, c, nmax, out, ws, s);
    case 2: return launch_tc_t<BHI, BLO, 2>(g, q, c, nmax, out, ws, s);
    case 4: return launch_tc_t<BHI, BLO, 4>(g, q, c, nmax, out, ws, s);
    case 8: return launch_tc_t<BHI, BLO, 8>(g, q, c, nmax, out, ws, s);
    default: break;
  }
  if constexpr (BLO == 2) {
    if (g.nhs == 1) return launch_tc_t<BHI, BLO, 1>(g, q, c, nmax, out, ws, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_tc(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax, float* out,
                             DecodeWs ws, cudaStream_t s) {
  if (g.bhi == 4 && g.blo == 2) return launch_tc_nhs<4, 2>(g, q, c, nmax, out, ws, s);
  if (g.bhi == 2 && g.blo == 1) return launch_tc_nhs<2, 1>(g, q, c, nmax, out, ws, s);
  return cudaErrorInvalidValue;
}

}  // namespace pnmix
