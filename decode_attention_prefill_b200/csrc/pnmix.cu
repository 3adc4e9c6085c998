// pnmix.cu -- the C ABI of include/pnmix.h: host-side validation, the cache layout and
// the launches.  No entry point allocates, frees or synchronises (except
// pnmix_read_error, which is a synchronous read by definition).
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "decode_common.cuh"

namespace pnmix {

static pnmix_status make_geometry(const pnmix_config* cfg, int batch, int capacity, Geometry* g) {
  if (!cfg || !g) return PNMIX_ERR_INVALID_ARG;
  if (cfg->n_q_heads <= 0 || cfg->n_kv_heads <= 0 || batch < 0 || capacity < 0)
    return PNMIX_ERR_INVALID_ARG;
  if (cfg->n_q_heads % cfg->n_kv_heads) return PNMIX_ERR_INVALID_ARG;
  if (cfg->head_dim != 128 || cfg->group_tokens != 32 || cfg->residual_tokens != 32 ||
      cfg->value_group != 32 || cfg->value_bits != 2)
    return PNMIX_ERR_UNSUPPORTED;
  const int G = cfg->n_q_heads / cfg->n_kv_heads;
  if (G < 1 || G > kMaxG) return PNMIX_ERR_UNSUPPORTED;
  const bool bits_ok = (cfg->key_bits_hi == 4 && cfg->key_bits_lo == 2) ||
                       (cfg->key_bits_hi == 2 && cfg->key_bits_lo == 1);
  if (!bits_ok) return PNMIX_ERR_UNSUPPORTED;
  const int k = cfg->n_salient_pairs;
  if (k != 0 && k != 8 && k != 16 && k != 32 && k != 64) return PNMIX_ERR_UNSUPPORTED;
  const int nhs = 2 * k / 16;
  if ((nhs * cfg->key_bits_hi) % 2 || ((8 - nhs) * cfg->key_bits_lo) % 2) return PNMIX_ERR_UNSUPPORTED;
  if (cfg->saliency_window < 1 || cfg->saliency_window > 1024) return PNMIX_ERR_UNSUPPORTED;
  if (cfg->saliency_score < PNMIX_SCORE_PNMIX || cfg->saliency_score > PNMIX_SCORE_RANGE_QUERY)
    return PNMIX_ERR_UNSUPPORTED;
  if (cfg->n_pruned_pairs < 0 || cfg->n_pruned_pairs > 63) return PNMIX_ERR_UNSUPPORTED;
  if (cfg->decode_kernel < PNMIX_DECODE_AUTO || cfg->decode_kernel > PNMIX_DECODE_TC)
    return PNMIX_ERR_UNSUPPORTED;
  if (cfg->n_pruned_slices < 0 || cfg->n_pruned_slices > 8) return PNMIX_ERR_UNSUPPORTED;
  if (cfg->n_pruned_pairs > 0 && cfg->n_pruned_slices > 0) return PNMIX_ERR_UNSUPPORTED;
  if (cfg->decode_kernel == PNMIX_DECODE_SIMT && (cfg->n_pruned_pairs > 0 || cfg->n_pruned_slices > 0))
    return PNMIX_ERR_UNSUPPORTED;
  g->B = batch;
  g->Hq = cfg->n_q_heads;
  g->Hkv = cfg->n_kv_heads;
  g->G = G;
  g->k = k;
  g->nhi = 2 * k;
  g->nhs = nhs;
  g->bhi = cfg->key_bits_hi;
  g->blo = cfg->key_bits_lo;
  g->bv = cfg->value_bits;
  g->wh = nhs * g->bhi / 2;
  g->wl = (8 - nhs) * g->blo / 2;
  g->kc_bytes = 128 * (g->wh + g->wl);
  g->record_bytes = g->kc_bytes + 2048;
  g->capacity = capacity;
  g->gcap = capacity / kGroup;
  g->scale = cfg->softmax_scale > 0.0f ? cfg->softmax_scale : 1.0f / sqrtf(128.0f);
  g->score = cfg->saliency_score;
  g->n_prune = cfg->n_pruned_pairs;
  g->n_prune_slices = cfg->n_pruned_slices;
  g->tq = 1;
  g->rows = G;
  g->kernel = cfg->decode_kernel;
  g->wait_limit = kDecodeWaitLimit;
  g->skip_unit = -1;
  g->append = 0;
  g->lead = 0;
  g->resid_w = 1;
  return PNMIX_OK;
}

struct Layout {
  size_t records, k_resid, v_resid, len, pair_idx, pair_mask, perm, pair_scores, scratch, error, total;
};

static Layout cache_layout(const Geometry& g) {
  Layout L;
  const size_t units = static_cast<size_t>(g.B) * g.Hkv;
  size_t off = 0;
  L.records = off;
  off = align256(off + units * g.gcap * static_cast<size_t>(g.record_bytes));
  L.k_resid = off;
  off = align256(off + units * kGroup * kHeadDim * 2);
  L.v_resid = off;
  off = align256(off + units * kGroup * kHeadDim * 2);
  L.len = off;
  off = align256(off + static_cast<size_t>(g.B) * 4);
  L.pair_idx = off;
  off = align256(off + units * 64);
  L.pair_mask = off;
  off = align256(off + units * 8);
  L.perm = off;
  off = align256(off + units * 128);
  L.pair_scores = off;
  off = align256(off + units * 64 * 4);
  L.scratch = off;
  off = align256(off + scratch_words(g.B, g.Hkv) * 4);
  L.error = off;
  off = align256(off + 4);
  L.total = off;
  return L;
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static pnmix_status cuda_status(cudaError_t e) { return e == cudaSuccess ? PNMIX_OK : PNMIX_ERR_CUDA; }

static pnmix_status check_cache(const Geometry& g, const pnmix_cache* c) {
  if (!c || !c->base || !c->records) return PNMIX_ERR_INVALID_ARG;
  if (c->batch != g.B || c->n_kv_heads != g.Hkv || c->record_bytes != g.record_bytes)
    return PNMIX_ERR_INVALID_ARG;
  return PNMIX_OK;
}

size_t decode_ticket_offset(const Geometry& g, int max_context) {
  const int nmax = decode_max_ctas(g, max_context);
  return decode_partial_bytes(nmax + g.B * g.Hkv, g.rows);
}

size_t decode_workspace_bytes(const Geometry& g, int max_context) {
  return decode_ticket_offset(g, max_context) + align256(sizeof(uint32_t) * g.B * g.Hkv);
}

pnmix_status check_decode_args(const pnmix_config* cfg, const uint16_t* q, const pnmix_cache* cache,
                               int max_context, const float* out, Geometry* g) {
  if (!cache) return PNMIX_ERR_INVALID_ARG;
  pnmix_status st = make_geometry(cfg, cache->batch, cache->capacity_tokens, g);
  if (st != PNMIX_OK) return st;
  if ((st = check_cache(*g, cache)) != PNMIX_OK) return st;
  if (!q || !out || max_context < 0) return PNMIX_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16)) return PNMIX_ERR_ALIGNMENT;
  return PNMIX_OK;
}

cudaError_t launch_decode(const Geometry& g, const uint16_t* q, const pnmix_cache& c, int max_context,
                          float* out, void* ws, cudaStream_t s, const DecodeMerge& merge) {
  const int nmax = decode_max_ctas(g, max_context);
  DecodeWs w;
  w.part = static_cast<float*>(ws);
  w.tickets = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + decode_ticket_offset(g, max_context));
  w.N = nmax;
  w.lse_out = merge.lse_out;
  w.prior_out = merge.prior_out;
  w.prior_lse = merge.prior_lse;
  w.k_new = merge.k_new;
  w.v_new = merge.v_new;
  // measured on B200 at 32K contexts: the tcgen05 kernel is ahead from 40 query rows per KV
  // head on (859 against 1110 us; its cost per group hardly depends on the rows), the
  // 8-row-warp kernel up to 32 rows (620 against 841 us)
  constexpr int kTcAutoRows = 33;
  if (g.kernel == PNMIX_DECODE_TC || (g.kernel == PNMIX_DECODE_AUTO && g.rows >= kTcAutoRows))
    return launch_decode_tc(g, q, c, nmax, out, w, s);
  if (g.rows > kMaxG) return launch_decode_rows(g, q, c, nmax, out, w, s);   // 9 .. 64 query rows
  switch (g.kernel) {
    case PNMIX_DECODE_SIMT: return launch_decode_simt(g, q, c, nmax, out, w, s);
    case PNMIX_DECODE_MMA: return launch_decode_mma(g, q, c, nmax, out, w, s);
    case PNMIX_DECODE_PAIRS: return launch_decode_ws(g, q, c, nmax, out, w, s);
    default:   // measured: single-role kernel for up to 4 rows per KV head, pairs above
      return g.rows <= 4 ? launch_decode_mma(g, q, c, nmax, out, w, s) : launch_decode_ws(g, q, c, nmax, out, w, s);
  }
}

// csrc/mix.cu: group scores, route and the split of K / V rows into two parts.
cudaError_t launch_split_groups(const Geometry& g, const uint16_t* q_window, int nw, const uint16_t* k,
                                const uint16_t* v, int L, int ld, int n_hi, float* scores, uint8_t* route,
                                int32_t* dest, uint16_t* k_hi, uint16_t* v_hi, uint16_t* k_lo, uint16_t* v_lo,
                                cudaStream_t s);

// csrc/shrink.cu: salient keys from b_hi to b_lo bits, src geometry gs -> dst geometry gd.
cudaError_t launch_shrink(const Geometry& gs, const Geometry& gd, const pnmix_cache& src,
                          const pnmix_cache& dst, cudaStream_t s);

}  // namespace pnmix

using namespace pnmix;

extern "C" {

size_t pnmix_record_bytes(const pnmix_config* cfg) {
  Geometry g;
  if (make_geometry(cfg, 1, 32, &g) != PNMIX_OK) return 0;
  return static_cast<size_t>(g.record_bytes);
}

pnmix_status pnmix_cache_bytes(const pnmix_config* cfg, int batch, int capacity_tokens,
                               size_t* total_bytes) {
  if (!total_bytes || batch <= 0 || capacity_tokens <= 0 || capacity_tokens % kGroup)
    return PNMIX_ERR_INVALID_ARG;
  Geometry g;
  pnmix_status st = make_geometry(cfg, batch, capacity_tokens, &g);
  if (st != PNMIX_OK) return st;
  *total_bytes = cache_layout(g).total;
  return PNMIX_OK;
}

pnmix_status pnmix_cache_init(const pnmix_config* cfg, int batch, int capacity_tokens,
                              void* device_base, size_t bytes, pnmix_cache* out) {
  if (!out || !device_base) return PNMIX_ERR_INVALID_ARG;
  if (!aligned(device_base, 256)) return PNMIX_ERR_ALIGNMENT;
  size_t need = 0;
  pnmix_status st = pnmix_cache_bytes(cfg, batch, capacity_tokens, &need);
  if (st != PNMIX_OK) return st;
  if (bytes < need) return PNMIX_ERR_CAPACITY;
  Geometry g;
  make_geometry(cfg, batch, capacity_tokens, &g);
  Layout L = cache_layout(g);
  char* base = static_cast<char*>(device_base);
  memset(out, 0, sizeof(*out));
  out->batch = batch;
  out->capacity_tokens = capacity_tokens;
  out->n_kv_heads = g.Hkv;
  out->record_bytes = g.record_bytes;
  out->records = reinterpret_cast<uint8_t*>(base + L.records);
  out->k_resid = reinterpret_cast<uint16_t*>(base + L.k_resid);
  out->v_resid = reinterpret_cast<uint16_t*>(base + L.v_resid);
  out->len = reinterpret_cast<int32_t*>(base + L.len);
  out->pair_idx = reinterpret_cast<uint8_t*>(base + L.pair_idx);
  out->pair_mask = reinterpret_cast<uint64_t*>(base + L.pair_mask);
  out->perm = reinterpret_cast<uint8_t*>(base + L.perm);
  out->pair_scores = reinterpret_cast<float*>(base + L.pair_scores);
  out->scratch = reinterpret_cast<uint32_t*>(base + L.scratch);
  out->error = reinterpret_cast<uint32_t*>(base + L.error);
  out->base = device_base;
  out->total_bytes = L.total;
  return PNMIX_OK;
}

pnmix_status pnmix_cache_reset(const pnmix_cache* cache, void* stream) {
  if (!cache || !cache->base) return PNMIX_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(cache->base, 0, cache->total_bytes, static_cast<cudaStream_t>(stream)));
}

pnmix_status pnmix_select_pairs(const pnmix_config* cfg, const uint16_t* q_window, int n_window,
                                const uint16_t* k, int L, int ld_tokens, pnmix_cache* cache,
                                void* stream) {
  if (!cache) return PNMIX_ERR_INVALID_ARG;
  Geometry g;
  pnmix_status st = make_geometry(cfg, cache->batch, cache->capacity_tokens, &g);
  if (st != PNMIX_OK) return st;
  if ((st = check_cache(g, cache)) != PNMIX_OK) return st;
  if (!q_window || !k || L < 1 || ld_tokens < L) return PNMIX_ERR_INVALID_ARG;
  const int want_w = L < cfg->saliency_window ? L : cfg->saliency_window;
  if (n_window != want_w) return PNMIX_ERR_INVALID_ARG;
  if (!aligned(q_window, 16) || !aligned(k, 16)) return PNMIX_ERR_ALIGNMENT;
  return cuda_status(launch_select_pairs(g, q_window, n_window, k, L, ld_tokens, *cache,
                                         static_cast<cudaStream_t>(stream)));
}

static pnmix_status check_prefill(const pnmix_config* cfg, const uint16_t* x, int L, int ld,
                                  const pnmix_cache* cache, Geometry* g) {
  if (!cache) return PNMIX_ERR_INVALID_ARG;
  pnmix_status st = make_geometry(cfg, cache->batch, cache->capacity_tokens, g);
  if (st != PNMIX_OK) return st;
  if ((st = check_cache(*g, cache)) != PNMIX_OK) return st;
  if (!x || L < 0 || ld < L || ld < 1) return PNMIX_ERR_INVALID_ARG;
  if (L > cache->capacity_tokens) return PNMIX_ERR_CAPACITY;
  if (!aligned(x, 16)) return PNMIX_ERR_ALIGNMENT;
  return PNMIX_OK;
}

pnmix_status pnmix_quantize_keys(const pnmix_config* cfg, const uint16_t* k, int L, int ld_tokens,
                                 pnmix_cache* cache, void* stream) {
  Geometry g;
  pnmix_status st = check_prefill(cfg, k, L, ld_tokens, cache, &g);
  if (st != PNMIX_OK) return st;
  return cuda_status(launch_quantize_keys(g, k, L, ld_tokens, *cache, static_cast<cudaStream_t>(stream)));
}

pnmix_status pnmix_quantize_values(const pnmix_config* cfg, const uint16_t* v, int L, int ld_tokens,
                                   pnmix_cache* cache, void* stream) {
  Geometry g;
  pnmix_status st = check_prefill(cfg, v, L, ld_tokens, cache, &g);
  if (st != PNMIX_OK) return st;
  return cuda_status(launch_quantize_values(g, v, L, ld_tokens, *cache, static_cast<cudaStream_t>(stream)));
}

pnmix_status pnmix_append(const pnmix_config* cfg, const uint16_t* k_new, const uint16_t* v_new,
                          pnmix_cache* cache, void* stream) {
  if (!cache) return PNMIX_ERR_INVALID_ARG;
  Geometry g;
  pnmix_status st = make_geometry(cfg, cache->batch, cache->capacity_tokens, &g);
  if (st != PNMIX_OK) return st;
  if ((st = check_cache(g, cache)) != PNMIX_OK) return st;
  if (!k_new || !v_new) return PNMIX_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16)) return PNMIX_ERR_ALIGNMENT;
  return cuda_status(launch_append(g, k_new, v_new, *cache, static_cast<cudaStream_t>(stream)));
}

size_t pnmix_workspace_bytes(const pnmix_config* cfg, int batch, int max_context) {
  Geometry g;
  if (batch <= 0 || make_geometry(cfg, batch, 32, &g) != PNMIX_OK) return 0;
  return decode_workspace_bytes(g, max_context);
}

pnmix_status pnmix_decode_attention(const pnmix_config* cfg, const uint16_t* q,
                                    const pnmix_cache* cache, int max_context, float* out,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  Geometry g;
  pnmix_status st = check_decode_args(cfg, q, cache, max_context, out, &g);
  if (st != PNMIX_OK) return st;
  if (!workspace) return PNMIX_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return PNMIX_ERR_ALIGNMENT;
  if (workspace_bytes < decode_workspace_bytes(g, max_context)) return PNMIX_ERR_CAPACITY;
  return cuda_status(launch_decode(g, q, *cache, max_context, out, workspace,
                                   static_cast<cudaStream_t>(stream)));
}

pnmix_status pnmix_append_decode(const pnmix_config* cfg, const uint16_t* k_new, const uint16_t* v_new,
                                 const uint16_t* q, pnmix_cache* cache, int max_context, float* out,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  Geometry g;
  pnmix_status st = check_decode_args(cfg, q, cache, max_context, out, &g);
  if (st != PNMIX_OK) return st;
  if (!k_new || !v_new || !workspace) return PNMIX_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(workspace, 256)) return PNMIX_ERR_ALIGNMENT;
  if (workspace_bytes < decode_workspace_bytes(g, max_context)) return PNMIX_ERR_CAPACITY;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the one-role tensor-core kernel appends inside the decode launch; the others take the
  // append kernel first
  const bool fused = g.kernel == PNMIX_DECODE_MMA || (g.kernel == PNMIX_DECODE_AUTO && g.rows <= 4);
  if (!fused) {
    const cudaError_t e = launch_append(g, k_new, v_new, *cache, s);
    if (e != cudaSuccess) return PNMIX_ERR_CUDA;
    return cuda_status(launch_decode(g, q, *cache, max_context, out, workspace, s));
  }
  g.append = 1;
  DecodeMerge rows;
  rows.k_new = k_new;
  rows.v_new = v_new;
  return cuda_status(launch_decode(g, q, *cache, max_context, out, workspace, s, rows));
}

size_t pnmix_workspace_bytes_two(const pnmix_config* cfg_a, const pnmix_config* cfg_b, int batch,
                                 int max_context_a, int max_context_b) {
  Geometry ga, gb;
  if (batch <= 0 || make_geometry(cfg_a, batch, 32, &ga) != PNMIX_OK || make_geometry(cfg_b, batch, 32, &gb) != PNMIX_OK)
    return 0;
  if (ga.Hq != gb.Hq || ga.Hkv != gb.Hkv || max_context_a < 0 || max_context_b < 0) return 0;
  const size_t wa = decode_workspace_bytes(ga, max_context_a), wb = decode_workspace_bytes(gb, max_context_b);
  const size_t rows = static_cast<size_t>(batch) * ga.Hq;
  return align256(wa > wb ? wa : wb) + align256(rows * kHeadDim * sizeof(float)) + align256(rows * sizeof(float));
}

pnmix_status pnmix_decode_attention_two(const pnmix_config* cfg_a, const pnmix_cache* cache_a, int max_context_a,
                                        const pnmix_config* cfg_b, const pnmix_cache* cache_b, int max_context_b,
                                        const uint16_t* q, float* out, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  Geometry ga, gb;
  pnmix_status st = check_decode_args(cfg_a, q, cache_a, max_context_a, out, &ga);
  if (st != PNMIX_OK) return st;
  if ((st = check_decode_args(cfg_b, q, cache_b, max_context_b, out, &gb)) != PNMIX_OK) return st;
  if (ga.B != gb.B || ga.Hq != gb.Hq || ga.Hkv != gb.Hkv) return PNMIX_ERR_INVALID_ARG;
  if (ga.n_prune_slices > 0 || gb.n_prune_slices > 0) return PNMIX_ERR_UNSUPPORTED;
  if (!workspace) return PNMIX_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return PNMIX_ERR_ALIGNMENT;
  const size_t wa = decode_workspace_bytes(ga, max_context_a), wb = decode_workspace_bytes(gb, max_context_b);
  const size_t rows = static_cast<size_t>(ga.B) * ga.Hq;
  const size_t split = align256(wa > wb ? wa : wb), tmp = align256(rows * kHeadDim * sizeof(float));
  if (workspace_bytes < split + tmp + align256(rows * sizeof(float))) return PNMIX_ERR_CAPACITY;
  char* w = static_cast<char*>(workspace);
  float* part_out = reinterpret_cast<float*>(w + split);
  float* part_lse = reinterpret_cast<float*>(w + split + tmp);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DecodeMerge first;
  first.lse_out = part_lse;
  cudaError_t e = launch_decode(ga, q, *cache_a, max_context_a, part_out, workspace, s, first);
  if (e != cudaSuccess) return PNMIX_ERR_CUDA;
  DecodeMerge second;
  second.prior_out = part_out;
  second.prior_lse = part_lse;
  return cuda_status(launch_decode(gb, q, *cache_b, max_context_b, out, workspace, s, second));
}

pnmix_status pnmix_debug_decode_stall(const pnmix_config* cfg, const uint16_t* q, const pnmix_cache* cache,
                                      int max_context, float* out, void* workspace, size_t workspace_bytes,
                                      int skip_unit, uint32_t wait_rounds, void* stream) {
  Geometry g;
  pnmix_status st = check_decode_args(cfg, q, cache, max_context, out, &g);
  if (st != PNMIX_OK) return st;
  if (!workspace || skip_unit < 0 || skip_unit >= g.B * g.Hkv || wait_rounds < 1) return PNMIX_ERR_INVALID_ARG;
  if (g.kernel == PNMIX_DECODE_SIMT) return PNMIX_ERR_UNSUPPORTED;
  if (!aligned(workspace, 256)) return PNMIX_ERR_ALIGNMENT;
  if (workspace_bytes < decode_workspace_bytes(g, max_context)) return PNMIX_ERR_CAPACITY;
  g.skip_unit = skip_unit;
  g.wait_limit = wait_rounds;
  return cuda_status(launch_decode(g, q, *cache, max_context, out, workspace, static_cast<cudaStream_t>(stream)));
}

// Query rows per KV head a multi-query call may have: up to 128 on the tcgen05 kernel (the
// automatic choice from 33 rows on, or forced), up to 64 on the others.
static int max_query_rows(const Geometry& g) {
  return g.kernel == PNMIX_DECODE_AUTO || g.kernel == PNMIX_DECODE_TC ? kMaxTcRows : kMaxRows;
}

size_t pnmix_workspace_bytes_multi(const pnmix_config* cfg, int batch, int max_context, int n_queries) {
  Geometry g;
  if (batch <= 0 || n_queries < 1 || make_geometry(cfg, batch, 32, &g) != PNMIX_OK) return 0;
  if (g.G * n_queries > max_query_rows(g)) return 0;
  g.tq = n_queries;
  g.rows = g.G * n_queries;
  return decode_workspace_bytes(g, max_context);
}

pnmix_status pnmix_decode_attention_multi(const pnmix_config* cfg, const uint16_t* q, int n_queries,
                                          const pnmix_cache* cache, int max_context, float* out,
                                          void* workspace, size_t workspace_bytes, void* stream) {
  if (!cache) return PNMIX_ERR_INVALID_ARG;
  Geometry g;
  pnmix_status st = make_geometry(cfg, cache->batch, cache->capacity_tokens, &g);
  if (st != PNMIX_OK) return st;
  if ((st = check_cache(g, cache)) != PNMIX_OK) return st;
  if (!q || !out || !workspace || max_context < 0 || n_queries < 1) return PNMIX_ERR_INVALID_ARG;
  if (g.G * n_queries > max_query_rows(g)) return PNMIX_ERR_UNSUPPORTED;
  if (g.kernel == PNMIX_DECODE_SIMT && n_queries > 1) return PNMIX_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(workspace, 256)) return PNMIX_ERR_ALIGNMENT;
  g.tq = n_queries;
  g.rows = g.G * n_queries;
  if (workspace_bytes < decode_workspace_bytes(g, max_context)) return PNMIX_ERR_CAPACITY;
  return cuda_status(launch_decode(g, q, *cache, max_context, out, workspace,
                                   static_cast<cudaStream_t>(stream)));
}

pnmix_status pnmix_shrink_keys(const pnmix_config* cfg, const pnmix_cache* src, pnmix_cache* dst,
                               void* stream) {
  if (!cfg || !src || !dst) return PNMIX_ERR_INVALID_ARG;
  Geometry gs, gd;
  pnmix_status st = make_geometry(cfg, src->batch, src->capacity_tokens, &gs);
  if (st != PNMIX_OK) return st;
  if ((st = check_cache(gs, src)) != PNMIX_OK) return st;
  if (gs.bhi != 2 * gs.blo || gs.k == 0) return PNMIX_ERR_UNSUPPORTED;
  pnmix_config small = *cfg;
  small.n_salient_pairs = 0;
  if ((st = make_geometry(&small, src->batch, src->capacity_tokens, &gd)) != PNMIX_OK) return st;
  if (dst->batch != src->batch || dst->capacity_tokens != src->capacity_tokens) return PNMIX_ERR_INVALID_ARG;
  if ((st = check_cache(gd, dst)) != PNMIX_OK) return st;
  const uintptr_t s0 = reinterpret_cast<uintptr_t>(src->base), d0 = reinterpret_cast<uintptr_t>(dst->base);
  if (s0 < d0 + dst->total_bytes && d0 < s0 + src->total_bytes) return PNMIX_ERR_INVALID_ARG;   // overlap
  return cuda_status(launch_shrink(gs, gd, *src, *dst, static_cast<cudaStream_t>(stream)));
}

pnmix_status pnmix_split_groups(const pnmix_config* cfg, int batch, const uint16_t* q_window, int n_window,
                                const uint16_t* k, const uint16_t* v, int L, int ld_tokens, int hi_percent,
                                float* scores, uint8_t* route, int32_t* dest, uint16_t* k_hi, uint16_t* v_hi,
                                uint16_t* k_lo, uint16_t* v_lo, void* stream) {
  if (!cfg || batch < 0 || L < 1 || ld_tokens < L) return PNMIX_ERR_INVALID_ARG;
  Geometry g;
  const pnmix_status st = make_geometry(cfg, batch, (L + kGroup - 1) / kGroup * kGroup, &g);
  if (st != PNMIX_OK) return st;
  if (!q_window || !k || !v) return PNMIX_ERR_INVALID_ARG;
  if (hi_percent < 0 || hi_percent > 100) return PNMIX_ERR_INVALID_ARG;
  const int want_w = L < cfg->saliency_window ? L : cfg->saliency_window;
  if (n_window != want_w) return PNMIX_ERR_INVALID_ARG;
  const int ng = L / kGroup;
  const int n_hi = static_cast<int>(static_cast<long long>(ng) * hi_percent / 100);
  const int L_hi = kGroup * n_hi, L_lo = L - L_hi;
  if (ng > 0 && (!scores || !route || !dest)) return PNMIX_ERR_INVALID_ARG;
  if (L_hi > 0 && (!k_hi || !v_hi)) return PNMIX_ERR_INVALID_ARG;
  if (L_lo > 0 && (!k_lo || !v_lo)) return PNMIX_ERR_INVALID_ARG;
  for (const void* p : {static_cast<const void*>(q_window), static_cast<const void*>(k),
                        static_cast<const void*>(v), static_cast<const void*>(k_hi), static_cast<const void*>(v_hi),
                        static_cast<const void*>(k_lo), static_cast<const void*>(v_lo)})
    if (p && !aligned(p, 16)) return PNMIX_ERR_ALIGNMENT;
  return cuda_status(launch_split_groups(g, q_window, n_window, k, v, L, ld_tokens, n_hi, scores, route, dest,
                                         k_hi, v_hi, k_lo, v_lo, static_cast<cudaStream_t>(stream)));
}

pnmix_status pnmix_read_error(const pnmix_cache* cache, int clear, uint32_t* host_error) {
  if (!cache || !cache->error || !host_error) return PNMIX_ERR_INVALID_ARG;
  cudaError_t e = cudaMemcpy(host_error, cache->error, sizeof(uint32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return PNMIX_ERR_CUDA;
  if (clear) {
    e = cudaMemset(cache->error, 0, sizeof(uint32_t));
    if (e != cudaSuccess) return PNMIX_ERR_CUDA;
  }
  return *host_error ? PNMIX_ERR_DEVICE : PNMIX_OK;
}

const char* pnmix_status_string(pnmix_status status) {
  switch (status) {
    case PNMIX_OK: return "ok";
    case PNMIX_ERR_INVALID_ARG: return "invalid argument";
    case PNMIX_ERR_UNSUPPORTED: return "unsupported configuration";
    case PNMIX_ERR_CAPACITY: return "capacity exceeded";
    case PNMIX_ERR_CUDA: return "CUDA runtime error";
    case PNMIX_ERR_ALIGNMENT: return "misaligned pointer";
    case PNMIX_ERR_DEVICE: return "device error word set";
  }
  return "unknown status";
}

const char* pnmix_version(void) { return "pnmix 0.1"; }

}  // extern "C"
