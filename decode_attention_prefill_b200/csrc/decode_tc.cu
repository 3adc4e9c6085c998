// decode_tc.cu -- decode attention on the 5th-generation tensor cores (tcgen05, TMEM) for
// many query rows per KV head: a multi-token step (speculative verify, chunked decode) with
// up to 64 rows = G * T.
//
// One CTA of 8 warps per slice of the work partition (decode_common.cuh), two CTAs per SM.
// Warps 0..3 run the softmax: query row r is TMEM lane r of every accumulator (rows >= G are
// zero).  Warps 4..7 build the operand tiles from the staged records.  A dequantised key
// is k = c * s + z (code c, fp16 scale s and zero z of its group and position), a value
// v = c * s_v + z_v.  Per 32-token group record:
//
//   logits  S = Q x K^T = Q x (C s)^T + Q x z:  A = the unit's query rows, fp16 (exact from
//           bf16), 128 rows x 128 positions, written once per segment.  c * s has at most
//           15 significant bits, so it is exactly the sum of two fp16 numbers, hi = fp16(c s)
//           (one half-precision multiply) and lo = c s - hi (one half-precision fma, whose
//           result is exact).  B is one tile of 80 rows x 128 positions: row 0 the zero
//           points z (the term Q z is the same for the group's 32 tokens), rows 1..15 zero,
//           rows 16..47 the hi and rows 48..79 the lo parts of the 32 tokens; 8 MMAs of
//           K = 16 (N = 80) accumulate the three sums of every row in TMEM, fp32, and the
//           logit of token t is D[16 + t] + D[48 + t] + D[0].
//   softmax the query rows are repeated in A rows 64..127, so TMEM lane r and r + 64 hold the
//           same row; lane r takes tokens 0..15 of every group and lane r + 64 tokens 16..31,
//           as two independent partials merged at the segment's end.  Each thread loads its
//           16 logits and the zero term (tcgen05.ld), applies the softmax scale and the causal
//           mask, and keeps a reference m (the first visible maximum, moved only when a logit
//           would give p = 2^(logit - m) above 2^14, which fp16 still holds; a move rescales
//           the lane's accumulators in TMEM).  The denominator is the product of P with a row
//           of ones in the value tile, so it sums the same fp16 p as the outputs.
//   values  O += P x (C_v s_v)^T + P x z_v:  A = P (fp16, 128 rows x 32 tokens), B = one
//           tile of 144 rows x 32 tokens: rows 0..3 the zero points of the four 32-channel
//           groups, row 4 all ones, rows 5..15 zero, rows 16..143 fp16(c s_v) of the 128
//           channels (one rounding, exact for codes 0 .. 2: the value side's precision in
//           every decode kernel); 2 MMAs (N = 144) accumulate the zero terms, the denominator
//           and the outputs in TMEM.  A row's result is O[ch] plus the zero term of ch's
//           channel group.
//
// Pipeline of one group: while its key products run, the builder warps write its value tile
// (two buffers); after the key commit (which also covers every earlier product, so TMEM, P
// and the value buffer two groups back are idle) the softmax warps write P and the builders
// the next group's key tile; after one barrier a single thread issues this group's value
// products and the next group's key products.  The bf16 residual window takes the same
// path as one more group (its keys split into hi / lo, its values rounded to fp16, zero
// tiles empty, the tokens past it masked).  The records arrive by TMA bulk copy (no
// multicast) into a ring of three.  Every wait is bounded.  At the end of a segment the
// softmax threads write each row's partial (m, l, O) for the fused combine.  Needs |c s|
// below 65504 (keys and values whose group range fits fp16).
#include <atomic>
#include <string.h>

#include "common.cuh"
#include "decode_common.cuh"
#include "decode_frag.cuh"

namespace pnmix {
namespace {

constexpr int kTcThreads = 256;   // warps 0..3: softmax (TMEM lanes 0..127); warps 4..7: tile building
constexpr int kTcHalf = 128;      // threads of one role
constexpr int kTcSlots = 3;       // record ring
constexpr int kTmemCols = 256;    // TMEM columns per CTA (two CTAs per SM)
// TMEM columns: key products 0 .. 79 (zero term in 0, hi in 16 .. 47, lo in 48 .. 79), value
// products 112 .. 255 (zero terms in 112 .. 115, outputs in 128 .. 255)
constexpr int kTmemKz = 0, kTmemKhi = 16, kTmemKlo = 48;
constexpr int kTmemV = 112, kTmemZv = 112, kTmemOut = 128;
constexpr int kKRows = 80;    // key B tile rows
constexpr float kRefSlack = 14.f;   // largest log2 of p before the row's reference moves
constexpr int kVRows = 144;   // value B tile rows

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
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane (warp-collective; no wait).
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld8_nowait(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld1_nowait(uint32_t taddr, uint32_t& r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld32_nowait(taddr, r);
  tmem_wait_ld();
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
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
               "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
               "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
               : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Named barrier ID of the 128 threads of one role (barrier 0 is __syncthreads).
template <int ID>
__device__ __forceinline__ void role_sync() {
  asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(128) : "memory");
}

__device__ __forceinline__ __half2 bits_h2(uint32_t x) {
  __half2 h;
  memcpy(&h, &x, 4);
  return h;
}
__device__ __forceinline__ uint32_t h2_bits(__half2 h) {
  uint32_t x;
  memcpy(&x, &h, 4);
  return x;
}
__device__ __forceinline__ uint32_t pack_f16(float lo_elem, float hi_elem) {
  return h2_bits(__floats2half2_rn(lo_elem, hi_elem));
}

// x split into two fp16 whose sum is x to 22 bits, packed (hi, lo) for two adjacent K.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
  const __half l0 = __float2half_rn(x0 - __half2float(h0)), l1 = __float2half_rn(x1 - __half2float(h1));
  hi = static_cast<uint32_t>(__half_as_ushort(h0)) | (static_cast<uint32_t>(__half_as_ushort(h1)) << 16);
  lo = static_cast<uint32_t>(__half_as_ushort(l0)) | (static_cast<uint32_t>(__half_as_ushort(l1)) << 16);
}

// Four code pairs of one 32-bit code word (both halves: two adjacent K of one tile row),
// the pair u at bit BITS * u of `w` in each half: the hi / lo parts of c * s for the scale
// pair `s2`, stored `step` bytes apart.  1024 + c is an fp16 with c in its low mantissa bits,
// so one subtraction gives c exactly; hi = fp16(c s) and lo = fma(c, s, -hi) are exact.
template <int BITS>
__device__ __forceinline__ void cs_pairs4(uint32_t w, uint32_t s2, uint8_t* dh, uint8_t* dl, int step) {
  constexpr uint32_t kMask = ((1u << BITS) - 1u) * 0x10001u;
  const __half2 s = bits_h2(s2);
  const __half2 k1024 = __float2half2_rn(1024.f);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const __half2 c = __hsub2(bits_h2(((w >> (BITS * u)) & kMask) | 0x64006400u), k1024);
    const __half2 hi = __hmul2(c, s);
    const __half2 lo = __hfma2(c, s, __hneg2(hi));
    *reinterpret_cast<uint32_t*>(dh + u * step) = h2_bits(hi);
    *reinterpret_cast<uint32_t*>(dl + u * step) = h2_bits(lo);
  }
}

struct TcSmem {
  int aq;      // fp16 [128 rows][128 positions]
  int bk;      // two buffers of fp16 [80 rows][128 positions] (zero row, hi, lo)
  int ap;      // fp16 [128 rows][32 tokens]
  int bv;      // two buffers of fp16 [144 rows][32 tokens] (zero rows, values)
  int qnat;    // fp32 [64 or 128 rows][128] (segment setup only): the key tiles, then P and the
               // value tiles
  int ring;    // [kTcSlots][R]
  int perm;    // 128 bytes
  int bars;    // uint64 full[kTcSlots], mma_k, mma_v, logits read; uint32 TMEM address
  int total;
};

constexpr int kStepK = kKRows * 32;     // bytes of one K = 16 step of the key tile
constexpr int kStepV = kVRows * 32;     // of the value tile
constexpr int kVBuf = 2 * kStepV;
constexpr int kBkBuf = 8 * kStepK;      // one key tile (8 K steps)

__host__ __device__ __forceinline__ TcSmem tc_smem(int R) {
  TcSmem m;
  m.aq = 0;
  m.bk = m.aq + 128 * 128 * 2;
  m.ap = m.bk + 2 * kBkBuf;
  m.bv = m.ap + 128 * 32 * 2;
  m.qnat = m.bk;   // 32 or 64 KB from the key tiles on (bk, ap, bv: 66 KB)
  m.ring = m.bv + 2 * kVBuf;
  m.perm = m.ring + kTcSlots * ((R + 127) / 128 * 128);
  m.bars = m.perm + 128;
  m.total = m.bars + 128;
  return m;
}

// DUP: up to 64 rows, each row in TMEM lanes r and r + 64 (two halves of every group's
// tokens); otherwise up to 128 rows, one per lane, each lane taking all 32 tokens.
template <int BHI, int BLO, int NHS, bool DUP>
__global__ void __launch_bounds__(kTcThreads, 2)
decode_tc_kernel(Geometry g, const uint16_t* __restrict__ q, pnmix_cache c, float* __restrict__ out, DecodeWs ws) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int R = record_bytes_of<BHI, BLO, NHS>();
  constexpr int WH = NHS * BHI / 2;                   // key-code words per lane, salient block
  constexpr int KC = key_code_bytes<BHI, BLO, NHS>();
  const TcSmem sm = tc_smem(R);
  const int G = g.rows;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tq = lane & 3;
  uint8_t* aq = smem + sm.aq;
  uint8_t* bk = smem + sm.bk;
  uint8_t* ap = smem + sm.ap;
  float* qnat = reinterpret_cast<float*>(smem + sm.qnat);
  uint8_t* perm = smem + sm.perm;
  constexpr int kSlotBytes = (R + 127) / 128 * 128;
  uint8_t* ring = smem + sm.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + sm.bars);
  uint64_t* bar_k = full + kTcSlots;
  uint64_t* bar_v = bar_k + 1;
  uint64_t* bar_l = bar_v + 1;   // every softmax thread has read this item's logits
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_l + 1);
  __shared__ int fail_sh;

  if (tid == 0) {
    fail_sh = 0;
    for (int k = 0; k < kTcSlots; ++k) mbar_init(full + k, 1);
    mbar_init(bar_k, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_l, kTcHalf);
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
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;   // this warp's TMEM lanes
  // roles: the softmax warps own the TMEM lanes (query rows); the builder warps turn each
  // record into the key and value tiles; bt / bw are a builder's thread / warp index
  const bool builder = warp >= 4;
  const int bt = tid & (kTcHalf - 1), bw = warp & 3;
  const uint32_t t_row = tmem + lane_base;
  volatile int* fail = &fail_sh;
  const float qscale = g.scale * kLog2e;
  constexpr uint32_t kIdescK = mma_idesc(kKRows), kIdescV = mma_idesc(kVRows);
  // operand descriptors of the first K step of each tile (a step further is a fixed offset)
  const uint64_t dq0 = tile_desc(aq), dk0 = tile_desc(bk), dp0 = tile_desc(ap), dv0 = tile_desc(smem + sm.bv);
  // softmax thread tid (TMEM lane tid) holds query row rr for the tokens [tb, tb + kTok) of
  // every group; with DUP rr = tid % 64, tb = 16 kc, and the two copies of a row are
  // independent partials, merged at the segment's end
  constexpr int kTok = DUP ? 16 : 32;
  const int kc = DUP ? (warp & 3) >> 1 : 0, rr = DUP ? tid & 63 : tid & 127;
  const int tb = kTok * kc;
  // records staged so far / taken so far (ring position); product commits and waits
  uint32_t nis = 0, ncons = 0, nk = 0, nv = 0, ck = 0, cv = 0, nl = 0;
  // bounded wait for phase `parity` of `bar`; gives up (error bit, CTA-wide stop) after
  // `limit` rounds: g.wait_limit for the staged records, kDecodeWaitLimit for the tensor
  // cores' commits (they always arrive; the bound only guards against a hang)
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

  // per-thread constants of the tile builds: word, scale and zero offsets inside a record,
  // destinations inside the tiles.  Key unit j = 4 bw + jj: code slots n = 4 j' .. 4 j' + 3
  // of its block (j' = j, or j - 2 NHS in the low block), i.e. slice j / 2, half j % 2,
  // tokens gq + 8 u.  Values: builder warp bw takes code words m = 2 bw, 2 bw + 1 (channels
  // 16 m + gq + 8 r) of channel group bw, tokens 8 p + 2 tq, + 1.
  int k_src[4], k_shift[4], k_s2[4], k_dst[4];
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int j = 4 * bw + jj, sigma = j >> 1, cc = j & 1;
    k_s2[jj] = (tq * 4 + (sigma >> 1)) * 4 + 2 * cc + (sigma & 1);
    k_dst[jj] = sigma * kStepK + 2 * 256 + cc * 128 + 4 * lane;   // row 16 + tau
    if (j < 2 * NHS) {
      constexpr int m = 16 / BHI;
      k_src[jj] = ((4 * j) / m) * 32 + lane;
      k_shift[jj] = BHI * ((4 * j) % m);
    } else {
      constexpr int m = 16 / BLO;
      const int jl = j - 2 * NHS;
      k_src[jj] = (WH + (4 * jl) / m) * 32 + lane;
      k_shift[jj] = BLO * ((4 * jl) % m);
    }
  }
  const int kz_src = bt >= 64 ? kscale_index(2 * (bt - 64)) >> 1 : 0;   // zero row: positions 2i, 2i + 1
  const int kz_dst = bt >= 64 ? tile_off(kKRows, 0, 2 * (bt - 64)) : 0;
  int v_s2[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) v_s2[p] = (4 * p + tq) * 4 + bw;
  const int v_src = vword_offset(2 * bw, lane);
  const int v_dst = (2 + 4 * bw) * 256 + 4 * lane;   // row 16 + channel of m = 2 bw, r = 0
  // value zero rows: channel group jg = bt / 16, tokens 2 tp, 2 tp + 1 (tp = bt % 16)
  const int vz_src = bt < 64 ? vzero_index(2 * (bt & 15), bt >> 4) >> 1 : 0;
  const int vz_dst = bt < 64 ? tile_off(kVRows, bt >> 4, 2 * (bt & 15)) : 0;
  const int row_query = rr < G ? rr / g.G : -1;   // the query of this lane's row

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
    // has been consumed: records are taken in order and a slot is refilled once the tiles of
    // its record were built)
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
    for (int i = tid; i < (DUP ? kMaxRows : kMaxTcRows) * (kHeadDim / 8); i += kTcThreads) {
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
    // A = Q (positions in order; bf16 -> fp16 is exact in fp16's normal range), one 16-byte
    // chunk of 8 positions per item; with DUP rows 64..127 repeat rows 0..63; rows >= G are
    // zero
    for (int item = tid; item < 128 * 16; item += kTcThreads) {
      const int r = item >> 4, c8 = item & 15, src = DUP ? r & 63 : r;
      uint32_t w[4] = {0u, 0u, 0u, 0u};
      if (src < G) {
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) {
          const int j = 8 * c8 + 2 * k2;
          w[k2] = pack_f16(qnat[src * kHeadDim + (perm[j] & (kHeadDim - 1))],
                           qnat[src * kHeadDim + (perm[j + 1] & (kHeadDim - 1))]);
        }
      }
      *reinterpret_cast<uint4*>(aq + tile_off(128, r, 8 * c8)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    __syncthreads();   // qnat is dead: the fixed rows of the tiles it overlapped
    // rows 0..15 of both key tiles' 8 steps and of both value buffers' 2 steps: zero, except
    // row 4 of the value tiles, all ones (its product is the row's softmax denominator)
    for (int i = tid; i < 20 * 32; i += kTcThreads) {
      const int step = i >> 5, j = i & 31;
      uint8_t* base = step < 16 ? bk + step * kStepK : smem + sm.bv + (step - 16) * kStepV;
      const uint32_t fill = (step >= 16 && (j == 4 || j == 12)) ? 0x3C003C00u : 0u;
      reinterpret_cast<uint4*>(base)[j] = make_uint4(fill, fill, fill, fill);
    }
    // this lane's P row outside its tokens stays zero
    if (DUP && !builder) {
#pragma unroll
      for (int c8 = 0; c8 < 2; ++c8)
        *reinterpret_cast<uint4*>(ap + tile_off(128, tid, 16 * (1 - kc) + 8 * c8)) = make_uint4(0u, 0u, 0u, 0u);
    }
    proxy_fence();
    if (tid == 0 && ngr > 0 && !*fail) wait_bar(full + (ncons % kTcSlots), (ncons / kTcSlots) & 1u, g.wait_limit);
    // the first record is in (or the CTA stops: a decision every thread takes alike, from a
    // barrier's reduction, since a wait that runs out sets the flag at any time)
    const bool stop0 = __syncthreads_or(*fail);

    float m_row = -INFINITY;
    bool out_live = false;   // the TMEM output rows hold a value product's result
    const int nitems = ngr + (seg_resid ? 1 : 0);
    // ---- key tile of item i (a record in `rec`, or the residual window): hi / lo of c * s
    // and the zero row
    auto build_keys = [&](int i, const uint8_t* rec) {
      uint8_t* bkb = bk + (i & 1) * kBkBuf;
      if (i < ngr) {
        const uint32_t* recw = reinterpret_cast<const uint32_t*>(rec);
        const uint32_t* ks2 = reinterpret_cast<const uint32_t*>(rec + KC);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const uint32_t s2 = ks2[k_s2[jj]];
          const uint32_t w = recw[k_src[jj]] >> k_shift[jj];
          uint8_t* dh = bkb + k_dst[jj];
          if (4 * bw + jj < 2 * NHS)
            cs_pairs4<BHI>(w, s2, dh, dh + 4 * 256, 256);   // hi in row 16 + tau, lo in 48 + tau
          else
            cs_pairs4<BLO>(w, s2, dh, dh + 4 * 256, 256);
        }
        if (bt >= 64)
          *reinterpret_cast<uint32_t*>(bkb + kz_dst) = reinterpret_cast<const uint32_t*>(rec + KC + 256)[kz_src];
      } else {
        const uint16_t* rk = c.k_resid + static_cast<size_t>(unit) * kGroup * kHeadDim;
        for (int item = bt; item < kGroup * (kHeadDim / 2); item += kTcHalf) {
          const int tau = item >> 6, p0 = 2 * (item & 63);
          float x0 = 0.f, x1 = 0.f;
          if (tau < seg.nr) {
            x0 = bf16_bits_to_float(rk[tau * kHeadDim + (perm[p0] & (kHeadDim - 1))]);
            x1 = bf16_bits_to_float(rk[tau * kHeadDim + (perm[p0 + 1] & (kHeadDim - 1))]);
          }
          uint32_t hi, lo;
          split_pair(x0, x1, hi, lo);
          *reinterpret_cast<uint32_t*>(bkb + tile_off(kKRows, 16 + tau, p0)) = hi;
          *reinterpret_cast<uint32_t*>(bkb + tile_off(kKRows, 48 + tau, p0)) = lo;
        }
        if (bt >= 64) *reinterpret_cast<uint32_t*>(bkb + kz_dst) = 0u;
      }
    };
    // ---- value tile of item i into buffer i % 2: fp16(c * s_v) and the zero rows
    auto build_values = [&](int i, const uint8_t* rec) {
      uint8_t* bv = smem + sm.bv + (i & 1) * kVBuf;
      if (i < ngr) {
        const uint32_t* vs2 = reinterpret_cast<const uint32_t*>(rec + KC + 1536);
        uint32_t s2[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) s2[p] = vs2[v_s2[p]];
        const uint2 wv = *reinterpret_cast<const uint2*>(rec + KC + 512 + v_src);   // m = 2w, 2w + 1
#pragma unroll
        for (int mm = 0; mm < 2; ++mm) {
          const uint32_t w = mm ? wv.y : wv.x;
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            uint8_t* dh = bv + v_dst + (2 * mm + r) * 256;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const __half2 cv = __hsub2(bits_h2(((w >> (2 * (4 * r + p))) & 0x00030003u) | 0x64006400u),
                                         __float2half2_rn(1024.f));
              *reinterpret_cast<uint32_t*>(dh + (p >> 1) * kStepV + (p & 1) * 128) =
                  h2_bits(__hmul2(cv, bits_h2(s2[p])));
            }
          }
        }
        if (bt < 64)
          *reinterpret_cast<uint32_t*>(bv + vz_dst) = reinterpret_cast<const uint32_t*>(rec + KC + 1792)[vz_src];
      } else {
        const uint16_t* rv = c.v_resid + static_cast<size_t>(unit) * kGroup * kHeadDim;
        for (int item = bt; item < kHeadDim * (kGroup / 2); item += kTcHalf) {
          const int ch = item >> 4, t0 = 2 * (item & 15);
          const float x0 = t0 < seg.nr ? bf16_bits_to_float(rv[t0 * kHeadDim + ch]) : 0.f;
          const float x1 = t0 + 1 < seg.nr ? bf16_bits_to_float(rv[(t0 + 1) * kHeadDim + ch]) : 0.f;
          *reinterpret_cast<uint32_t*>(bv + tile_off(kVRows, 16 + ch, t0)) = pack_f16(x0, x1);
        }
        if (bt < 64) *reinterpret_cast<uint32_t*>(bv + vz_dst) = 0u;
      }
    };
    auto issue_keys = [&](int i) {   // one thread: the key products of item i's tile
      const uint64_t dk = dk0 + (i & 1) * (kBkBuf >> 4);
#pragma unroll
      for (int s = 0; s < kHeadDim / 16; ++s)
        tc_mma(tmem + kTmemKz, dq0 + s * (128 * 32 >> 4), dk + s * (kStepK >> 4), kIdescK, s > 0);
      tc_commit(bar_k);
    };

    // Pipeline (item i): the builders write the key tile of item i + 1 (the other of two
    // buffers) while the key products of item i run; once every softmax thread has read
    // item i's logits (bar_l), one builder issues the key products of item i + 1 (they
    // overlap the rest of the softmax and the value tile of item i, which the builders write
    // next); the softmax warps wait for the value products of item i - 1 and write P of item
    // i; after one barrier thread 0 issues the value products of item i.  Every product is
    // committed to an mbarrier by the thread that issued it (keys: bar_k, values: bar_v);
    // ck / cv count the commits, nk / nv / nl the phases waited for (all threads count
    // alike).
    if (nitems > 0 && !stop0) {
      if (builder) build_keys(0, ring + (ncons % kTcSlots) * kSlotBytes);
      proxy_fence();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        issue_keys(0);
      }
      ++ck;
    }
    for (int it = 0; it < nitems && !stop0; ++it) {
      const bool resid_item = it == ngr;
      const int tok0 = resid_item ? seg.ng * kGroup : (seg.lo + it) * kGroup;
      const int ntok = resid_item ? seg.nr : kGroup;
      const bool next = it + 1 < nitems;
      if (builder) {
        if (next) {
          // the next record is in (one poller); its key tile goes to the other buffer, whose
          // last reader (the key products of item i - 1) completed before the last barrier
          if (bt == 0 && it + 1 < ngr)
            wait_bar(full + ((ncons + 1) % kTcSlots), ((ncons + 1) / kTcSlots) & 1u, g.wait_limit);
          role_sync<2>();
          build_keys(it + 1, ring + ((ncons + 1) % kTcSlots) * kSlotBytes);
          proxy_fence();
          role_sync<2>();   // the key tile is complete
          if (bt == 0) {   // item i's logits are read: the key accumulators may be overwritten
            wait_bar(bar_l, nl & 1u, kDecodeWaitLimit);
            tc_fence_after();
            issue_keys(it + 1);
          }
        }
        // this item's value tile (its buffer's last reader, the value products of item i - 2,
        // completed before the last barrier; the ring is not read for the residual)
        build_values(it, ring + (ncons % kTcSlots) * kSlotBytes);
      } else {
        // ---- the key products of this item are done: one poller, the role meets at its
        // barrier (waiting there issues nothing)
        if (bt == 0) wait_bar(bar_k, nk & 1u, kDecodeWaitLimit);
        role_sync<1>();
        tc_fence_after();
        // ---- logits of this lane's row and tokens: hi + lo products (fp32), the zero term
        float sv[kTok];
        float zk;
#pragma unroll
        for (int h16 = 0; h16 < kTok / 16; ++h16) {
          uint32_t rh[16], rl[16], zraw;
          tmem_ld16_nowait(t_row + kTmemKhi + tb + 16 * h16, rh);
          tmem_ld16_nowait(t_row + kTmemKlo + tb + 16 * h16, rl);
          tmem_ld1_nowait(t_row + kTmemKz, zraw);
          tmem_wait_ld();
          zk = __uint_as_float(zraw);
#pragma unroll
          for (int t = 0; t < 16; ++t) sv[16 * h16 + t] = __uint_as_float(rh[t]) + __uint_as_float(rl[t]);
        }
        tc_fence_before();
        if (next) mbar_arrive(bar_l);   // this thread's logits are read
        if (tid == 0 && it > 0) wait_bar(bar_v, nv & 1u, kDecodeWaitLimit);   // value products of item i - 1
        role_sync<1>();   // P and the value accumulators are free
        tc_fence_after();
        // tokens tb + t of the group this row sees: t < nvis
        const int lim = row_query >= 0 ? vis_base + row_query : 0;
        const int nvis = min(ntok, lim - tok0) - tb;
        if (nvis < kTok) {
#pragma unroll
          for (int t = 0; t < kTok; ++t)
            if (t >= nvis) sv[t] = -INFINITY;
        }
        float mxr = -INFINITY;
#pragma unroll
        for (int t = 0; t < kTok; ++t) mxr = fmaxf(mxr, sv[t]);
        const float mx = (mxr + zk) * qscale;   // -inf when no token is visible
        // reference m of the row: the first visible logit's group maximum, moved up only when a
        // logit would give p above 2^kRefSlack (fp16 holds p up to 65504; the accumulators are
        // fp32), so the accumulators in TMEM are rescaled almost never; a row that has seen no
        // token has zero accumulators and needs no rescale
        bool rescale = false;
        float alpha = 1.f;
        if (mx > m_row + kRefSlack) {
          rescale = m_row != -INFINITY;
          if (rescale) alpha = ex2(m_row - mx);
          m_row = mx;
        }
        if (out_live && __any_sync(0xffffffffu, rescale)) {   // warp-collective TMEM traffic
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            float o[32];
            tmem_ld32(t_row + kTmemOut + 32 * c4, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(t_row + kTmemOut + 32 * c4, o);
          }
          uint32_t zr[8];
          tmem_ld8_nowait(t_row + kTmemZv, zr);   // zero terms and the denominator
          tmem_wait_ld();
          float zf[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) zf[i] = __uint_as_float(zr[i]) * alpha;
          tmem_st8(t_row + kTmemZv, zf);
        }
        // P (fp16): p = 2^(logit * scale - m), 0 for a hidden token (and for all while the row
        // has seen none), 8 tokens per 16-byte store
        const float off = m_row == -INFINITY ? -INFINITY : zk * qscale - m_row;
#pragma unroll
        for (int c8 = 0; c8 < kTok / 8; ++c8) {
          uint32_t w[4];
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) {
            const int t = 8 * c8 + 2 * k2;
            w[k2] = pack_f16(ex2(fmaf(sv[t], qscale, off)), ex2(fmaf(sv[t + 1], qscale, off)));
          }
          *reinterpret_cast<uint4*>(ap + tile_off(128, tid, tb + 8 * c8)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      ++nk;
      if (next) {
        ++ck;
        ++nl;
      }
      if (it > 0) ++nv;
      proxy_fence();
      tc_fence_before();
      // P, the value tile, any rescale and the next key tile are in place; every thread is done
      // with this item's record
      if (__syncthreads_or(*fail)) break;
      if (!resid_item) ++ncons;   // the ring position names the next record's slot
      if (tid == 0) {
        tc_fence_after();
        if (!resid_item) issue_next();
        const uint64_t dv = dv0 + (it & 1) * (kVBuf >> 4);
#pragma unroll
        for (int s = 0; s < kGroup / 16; ++s)
          tc_mma(tmem + kTmemV, dp0 + s * (128 * 32 >> 4), dv + s * (kStepV >> 4), kIdescV, out_live || s > 0);
        tc_commit(bar_v);
      }
      ++cv;
      out_live = true;
    }
    // ---- every product of the segment completes (waited for even after a stop: TMEM and
    // the tiles must be idle before they are read or reused): the latest commit of each
    // barrier covers every earlier product
    if (tid == 0) {
      if (ck > 0)
        for (uint32_t spins = 0; spins < kDecodeWaitLimit && !mbar_try_wait(bar_k, (ck - 1) & 1u); ++spins) {
        }
      if (cv > 0)
        for (uint32_t spins = 0; spins < kDecodeWaitLimit && !mbar_try_wait(bar_v, (cv - 1) & 1u); ++spins) {
        }
    }
    __syncthreads();
    nk = ck;
    nv = cv;
    tc_fence_after();
    if (*fail && tid == 0) {   // let staged copies land before the shared memory is reused
      for (; ncons < nis; ++ncons) {
        const uint32_t slot = ncons % kTcSlots;
        for (uint32_t spins = 0; spins < g.wait_limit && !mbar_try_wait(full + slot, (ncons / kTcSlots) & 1u);
             ++spins) {
        }
      }
    }
    if constexpr (!DUP) {
      // one lane per row: its partial (m, l = the ones-row product, O = the outputs plus the
      // zero term of their channel group) goes to the slot directly
      if (!builder) {
        const bool live = out_live && !*fail;
        float* o = partial_slot(ws, unit, G) + rr * kPartialStride;
        float zv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) zv[i] = 0.f;
        if (out_live) {
          uint32_t zr[8];
          tmem_ld8_nowait(t_row + kTmemZv, zr);   // warp-collective
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i) zv[i] = __uint_as_float(zr[i]);
        }
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          float v[32];
          if (out_live) {
            tmem_ld32(t_row + kTmemOut + 32 * c4, v);   // warp-collective
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
          }
          if (rr < G) {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[2 + 32 * c4 + i] = live ? v[i] + zv[c4] : 0.f;
          }
        }
        if (rr < G) {
          o[0] = live ? m_row : -INFINITY;
          o[1] = live ? zv[4] : 0.f;
        }
      }
    } else
    // merge the two copies of each row (shared memory of the idle A and key tiles):
    // M = max(m0, m1), weights f = 2^(m - M), partial (M, f0 l0 + f1 l1, f0 O0 + f1 O1) with
    // O = the outputs plus the zero term of their channel group and l = the ones-row product
    {
      constexpr int kXRow = kHeadDim + 4;
      float* xch = reinterpret_cast<float*>(smem);          // [64][kXRow]: copy 1's weighted (l, O)
      float* msh = xch + 64 * kXRow;                         // [128]: every lane's m
      const bool live = out_live && !*fail;
      const float m_me = live ? m_row : -INFINITY;
      if (!builder) msh[tid] = m_me;
      __syncthreads();
      const float M = fmaxf(msh[rr], msh[rr + 64]);
      const float f = m_me == -INFINITY ? 0.f : ex2(m_me - M);
      float zv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) zv[i] = 0.f;
      if (!builder && out_live) {
        uint32_t zr[8];
        tmem_ld8_nowait(t_row + kTmemZv, zr);   // warp-collective
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; ++i) zv[i] = __uint_as_float(zr[i]);
      }
      float* mine = xch + rr * kXRow;
      if (!builder && kc == 1) mine[0] = f * zv[4];
#pragma unroll 1
      for (int c4 = 0; c4 < 4; ++c4) {
        float v[32];
        if (!builder && out_live) {
          tmem_ld32(t_row + kTmemOut + 32 * c4, v);   // warp-collective
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.f;
        }
        if (!builder && kc == 1) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(mine + 4 + 32 * c4 + i) =
                make_float4(f * (v[i] + zv[c4]), f * (v[i + 1] + zv[c4]), f * (v[i + 2] + zv[c4]),
                            f * (v[i + 3] + zv[c4]));
        }
        __syncthreads();
        if (!builder && kc == 0 && rr < G) {
          float* o = partial_slot(ws, unit, G) + rr * kPartialStride;
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 x = *reinterpret_cast<const float4*>(mine + 4 + 32 * c4 + i);
            o[2 + 32 * c4 + i] = f * (v[i] + zv[c4]) + x.x;
            o[3 + 32 * c4 + i] = f * (v[i + 1] + zv[c4]) + x.y;
            o[4 + 32 * c4 + i] = f * (v[i + 2] + zv[c4]) + x.z;
            o[5 + 32 * c4 + i] = f * (v[i + 3] + zv[c4]) + x.w;
          }
          if (c4 == 3) {
            o[0] = M;
            o[1] = f * zv[4] + mine[0];
          }
        }
      }
    }
    tc_fence_before();
    // the combine's scratch: the A tile, idle until the next segment's setup
    combine_segment<kMaxTcRows, true>(ws, seg, G, out, g, reinterpret_cast<CombineScratch<kMaxTcRows>*>(smem + sm.aq));
  });
  tc_fence_before();
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

constexpr int kMaxDevices = 64;

template <int BHI, int BLO, int NHS, bool DUP>
cudaError_t launch_tc_d(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax, float* out, DecodeWs ws,
                        cudaStream_t s) {
  static std::atomic<int> wave_cache[kMaxDevices];
  if (g.record_bytes != record_bytes_of<BHI, BLO, NHS>()) return cudaErrorInvalidValue;
  const TcSmem sm = tc_smem(g.record_bytes);
  auto kern = decode_tc_kernel<BHI, BLO, NHS, DUP>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cacheable = dev >= 0 && dev < kMaxDevices;
  int wave = cacheable ? wave_cache[dev].load(std::memory_order_relaxed) : 0;
  if (wave == 0) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sm.total);
    if (e != cudaSuccess) return e;
    // two CTAs per SM need the largest shared-memory carveout
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    // CTAs per SM: what TMEM (512 columns per SM), shared memory and registers allow.  (The
    // runtime's occupancy query answers one for this kernel; two are resident, measured.)
    int sms = 148, smem_sm = 0, reserved = 0;
    cudaFuncAttributes fa;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess ||
        (e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess)
      return e;
    const int per_block = sm.total + static_cast<int>(fa.sharedSizeBytes) + reserved;
    const int regs_warp = (fa.numRegs * 32 + 255) / 256 * 256;
    int occ = 512 / kTmemCols;
    occ = min(occ, smem_sm / per_block);
    occ = min(occ, 65536 / (regs_warp * (kTcThreads / 32)));
    wave = sms * (occ > 0 ? occ : 1);
    if (cacheable) wave_cache[dev].store(wave, std::memory_order_relaxed);
  }
  ws.N = wave < nmax ? wave : nmax;
  kern<<<ws.N, kTcThreads, sm.total, s>>>(g, q, c, out, ws);
  return cudaGetLastError();
}

template <int BHI, int BLO, int NHS>
cudaError_t launch_tc_t(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int nmax, float* out, DecodeWs ws,
                        cudaStream_t s) {
  if (g.rows > kMaxTcRows) return cudaErrorInvalidValue;
  return g.rows <= kMaxRows ? launch_tc_d<BHI, BLO, NHS, true>(g, q, c, nmax, out, ws, s)
                            : launch_tc_d<BHI, BLO, NHS, false>(g, q, c, nmax, out, ws, s);
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
