// csa2_indexer_score_topk_noalloc: the indexer call for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand the library a workspace: code that runs
// while a framework holds every byte of device memory in its own pool and
// offers plugins no allocator, latency-critical serving loops that must never
// reach cudaMalloc (it can synchronise the whole device and take
// milliseconds), and hosts with a fixed memory budget decided up front.  For
// them the indexer's score buffer lives in one statically sized device array
// owned by this library.  The array exists on every GPU that loads the
// library, from load until process exit.
//
// Rules of use:
//  * the request must fit: csa2_workspace_bytes(CSA2_OP_INDEXER, ...) <=
//    CSA2_NOALLOC_SCRATCH_BYTES, else CSA2_ERR_WORKSPACE and nothing runs;
//  * every call shares the one array, so calls whose kernels overlap on the
//    GPU (other streams, other host threads) race; serialise them on one
//    stream;
//  * the array keeps whatever the previous call left; nothing in it has to
//    start at zero, because the scoring kernel writes every score entry the
//    selection kernel later reads;
//  * the first call on a device looks up the array's device address with that
//    device current (a one-time set-up); make that first call before any
//    stream capture.  The address is kept until the process exits: a
//    cudaDeviceReset() on that device invalidates it, and the call is not
//    supported after one.
// Nothing here allocates: no cudaMalloc, no cudaFree, no allocating library
// routine.
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/csa2.h"

namespace {

__device__ __align__(256) unsigned char g_indexer_scratch[CSA2_NOALLOC_SCRATCH_BYTES];

// Device address of g_indexer_scratch on the current device (looked up once
// per device; the host-side name is only a stand-in and is never passed to a
// kernel).
int scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return CSA2_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_indexer_scratch) != cudaSuccess || p == nullptr)
      return CSA2_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return CSA2_OK;
}

}  // namespace

extern "C" int csa2_indexer_score_topk_noalloc(const csa2_cache* cache, const uint16_t* idx_q,
                                               const float* head_w, const int32_t* q_seq,
                                               const int32_t* q_visible, int32_t nq,
                                               int64_t max_visible, int32_t mode,
                                               int32_t hierarchical, int32_t layer,
                                               csa2_indexset* set, csa2_stream_t stream) {
  if (nq < 0 || max_visible < 0) return CSA2_ERR_INVALID_ARG;
  const int32_t hier = mode == CSA2_REINDEX ? CSA2_HIER_MEAN : hierarchical;
  const size_t need = csa2_workspace_bytes(CSA2_OP_INDEXER, nq, 0, max_visible, hier);
  // an oversize request still gets the argument and mode-order checks first:
  // with no workspace the regular call reports those, else CSA2_ERR_WORKSPACE,
  // and launches nothing either way
  // (a size of 0 means csa2_workspace_bytes found the arguments invalid)
  if (need == 0 || need > (size_t)CSA2_NOALLOC_SCRATCH_BYTES)
    return csa2_indexer_score_topk(cache, idx_q, head_w, q_seq, q_visible, nq, max_visible, mode, hierarchical,
                                   layer, set, nullptr, 0, stream);
  void* scratch = nullptr;
  if (nq > 0) {
    const int st = scratch_address(&scratch);
    if (st != CSA2_OK) return st;
  }
  return csa2_indexer_score_topk(cache, idx_q, head_w, q_seq, q_visible, nq, max_visible, mode,
                                 hierarchical, layer, set, scratch,
                                 scratch ? (size_t)CSA2_NOALLOC_SCRATCH_BYTES : 0, stream);
}
