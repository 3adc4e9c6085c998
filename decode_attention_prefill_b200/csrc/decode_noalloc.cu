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
//  - all calls on a device share the one array and it keeps what the last call left.
//    Only the split-K ticket words must start at zero (every partial slot is written
//    before it is read in the same launch), so each call clears just those words
//    (cudaMemsetAsync on `stream`) before its launch; calls whose work overlaps on the
//    GPU (other streams, other threads) race on the array and must be serialised by
//    the caller;
//  - the array's device address is looked up (cudaGetSymbolAddress) on every call,
//    with the caller's current device, so it stays right after a device reset or a new
//    primary context.  The first call on a device also loads the library's device code
//    there; make that first call before any stream capture.  `stream` must belong to
//    the current device.
// Nothing here calls cudaMalloc, cudaFree or an allocating library routine.
#include "common.cuh"
#include "decode_common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;

// The scratch.  In host code this name is only a stand-in for the device
// variable; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

pnmix_status scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess || p == nullptr) return PNMIX_ERR_CUDA;
  *out = p;
  return PNMIX_OK;
}

}  // namespace

extern "C" PNMIX_API pnmix_status pnmix_decode_attention_noalloc(const pnmix_config* cfg,
                                                                 const uint16_t* q,
                                                                 const pnmix_cache* cache,
                                                                 int max_context, float* out,
                                                                 void* stream) {
  // The same validation as pnmix_decode_attention, all before anything is enqueued: a
  // rejected call leaves the shared array alone.
  pnmix::Geometry g;
  pnmix_status st = pnmix::check_decode_args(cfg, q, cache, max_context, out, &g);
  if (st != PNMIX_OK) return st;
  const size_t need = pnmix::decode_workspace_bytes(g, max_context);
  if (need > kNoAllocScratchBytes) return PNMIX_ERR_CAPACITY;
  void* ws = nullptr;
  if ((st = scratch_address(&ws)) != PNMIX_OK) return st;
  const size_t tickets = pnmix::decode_ticket_offset(g, max_context);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(static_cast<char*>(ws) + tickets, 0, need - tickets, s) != cudaSuccess)
    return PNMIX_ERR_CUDA;
  return pnmix::launch_decode(g, q, *cache, max_context, out, ws, s) == cudaSuccess ? PNMIX_OK
                                                                                      : PNMIX_ERR_CUDA;
}
