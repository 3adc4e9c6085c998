// decode_noalloc.cu -- decode attention that needs no caller-provided workspace.
//
// pnmix_decode_attention needs a split-K workspace from its caller.  Some callers
// have no way to get one: a plugin inside a host runtime that owns every byte of
// device memory and forbids allocations outside its own pool, or code whose
// interface has no slot for a workspace pointer and that may not call cudaMalloc
// itself (allocation can synchronise the device, fail under memory pressure, or
// break the host's memory plan).  For them this entry point takes its scratch from
// a fixed array that lives in the library image on every device that loads it.
//
// Limits and behaviour:
//  - the array holds kNoAllocScratchBytes (4 MiB); a call whose workspace
//    (pnmix_workspace_bytes for the same config, batch and max_context) is larger
//    is rejected with PNMIX_ERR_CAPACITY before anything is enqueued;
//  - every device that loads the library keeps those 4 MiB until the process exits;
//  - all calls on a device share the one array and it keeps what the last call left,
//    so each call first clears the part it uses (cudaMemsetAsync on `stream`);
//    calls whose work overlaps on the GPU (other streams, other threads) race on
//    the array and must be serialised by the caller;
//  - the first call on each device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current; make that first call before
//    any stream capture.
// Nothing here calls cudaMalloc, cudaFree or an allocating library routine.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
constexpr int kMaxDevices = 64;

// The scratch.  In host code this name is only a stand-in for the device
// variable; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices];

pnmix_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PNMIX_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) return PNMIX_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return PNMIX_OK;
}

bool is_aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" PNMIX_API pnmix_status pnmix_decode_attention_noalloc(const pnmix_config* cfg,
                                                                 const uint16_t* q,
                                                                 const pnmix_cache* cache,
                                                                 int max_context, float* out,
                                                                 void* stream) {
  // Everything pnmix_decode_attention would reject is rejected here first, so a
  // failing call enqueues nothing (not even the clearing memset).
  if (!cfg || !cache || !cache->base || !cache->records || !q || !out || max_context < 0)
    return PNMIX_ERR_INVALID_ARG;
  const size_t rb = pnmix_record_bytes(cfg);
  if (rb == 0) return PNMIX_ERR_UNSUPPORTED;
  if (cache->n_kv_heads != cfg->n_kv_heads || static_cast<size_t>(cache->record_bytes) != rb)
    return PNMIX_ERR_INVALID_ARG;
  if (!is_aligned(q, 16) || !is_aligned(out, 16)) return PNMIX_ERR_ALIGNMENT;
  const size_t need = pnmix_workspace_bytes(cfg, cache->batch, max_context);
  if (need == 0) return PNMIX_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return PNMIX_ERR_CAPACITY;
  void* ws = nullptr;
  pnmix_status st = scratch_address(&ws);
  if (st != PNMIX_OK) return st;
  if (cudaMemsetAsync(ws, 0, need, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PNMIX_ERR_CUDA;
  return pnmix_decode_attention(cfg, q, cache, max_context, out, ws, need, stream);
}
