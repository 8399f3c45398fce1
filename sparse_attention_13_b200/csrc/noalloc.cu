// noalloc.cu -- dsa_indexer_topk_noalloc: the indexer + top-k entry point for
// callers that cannot hand the library a workspace buffer.
//
// Some callers have no way to obtain device memory on demand: an inference
// engine that reserves all of HBM up front for its own KV-cache pool and owns
// every byte through its own allocator, a C host program that links this
// library without any allocator of its own, or a latency-critical path where
// cudaMalloc/cudaFree are off limits because they can synchronise the device.
// For them the indexer's scratch (per-CTA candidate buffers and, for decode
// shapes, the per-split top-k lists) lives in one file-scope device array of
// fixed size that is part of the library image: every GPU that loads this
// library keeps kNoAllocScratchBytes reserved until the process exits.
//
// Host code must not pass the array's name to a kernel: on the host it is only
// a stand-in symbol, not a device address.  The device address is looked up
// once per device with cudaGetSymbolAddress (with that device current) and
// cached; the first call on a device does that lookup, so make the first call
// on each device before any stream capture begins.
//
// All calls share the one array.  Nothing in it has to start at zero (every
// word the kernels read is written earlier in the same call), but calls whose
// kernels overlap on the GPU -- on different streams, or from different host
// threads -- race on it; issue them one after another.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "dsa_internal.h"

namespace dsa {
namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(DSA_NOALLOC_SCRATCH_BYTES);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {nullptr};

// Device address of the scratch array on the current device (looked up once).
dsa_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error(DSA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return set_error(DSA_ERR_UNSUPPORTED, "device index beyond 63");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return set_error(DSA_ERR_CUDA, std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return DSA_OK;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" dsa_status dsa_indexer_topk_noalloc(const dsa_bf16* q_idx, const dsa_bf16* k_idx,
                                               const float* w, int B, int Lq, int Lk,
                                               int start_pos, int H_I, int d_I, int k,
                                               int32_t* idx, void* stream) {
  // Size check first: reject shapes whose scratch would not fit before
  // touching the device.
  if (B >= 1 && Lq >= 1 && k >= 1 && start_pos >= 0) {
    // the smaller of the decode-row layout (when it applies) and the
    // candidate-buffer layout; the launch picks whichever fits
    size_t need = indexer_plan(B, Lq, Lk, start_pos, std::min(k, 2048)).total_bytes;
    if (decode_indexer_applies(Lq, Lk, start_pos, H_I, d_I))
      need = std::min(need, decode_indexer_ws_bytes(B, Lk));
    if (need > kNoAllocScratchBytes)
      return set_error(DSA_ERR_WORKSPACE,
                       "dsa_indexer_topk_noalloc: this shape needs " + std::to_string(need) +
                           " bytes of scratch, more than the fixed " +
                           std::to_string(kNoAllocScratchBytes) +
                           " bytes; use dsa_indexer_topk with a workspace");
  }
  void* scratch = nullptr;
  dsa_status st = noalloc_scratch(&scratch);
  if (st != DSA_OK) return st;
  return dsa_indexer_topk(q_idx, k_idx, w, B, Lq, Lk, start_pos, H_I, d_I, k, idx, scratch,
                          kNoAllocScratchBytes, stream);
}
