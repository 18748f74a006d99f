// tq_logits_noalloc: the logit call for callers that cannot allocate device
// memory at the point of the call.
//
// tq_logits needs a device workspace for the per-query operands (R q and
// S R q).  Some callers cannot hand one over: code that runs while another
// component owns the whole device memory pool, plug-ins that are not allowed
// to call the CUDA allocator, or latency-critical paths that must not pay for
// an allocation (cudaMalloc may synchronize the device).  For them this entry
// point uses a fixed scratch area that lives in the library itself: a
// file-scope __device__ array of kNoAllocScratchBytes, which every GPU that
// loads the library keeps until the process exits.  Nothing is allocated on
// any call.
//
// The device address of that array is looked up once per device, on the
// first call made with that device current (cudaGetSymbolAddress), and cached.
// Make that first call before any stream capture begins.
//
// All calls share the one array, whatever their context or stream: calls that
// may overlap on the GPU (different streams, or different host threads) race
// on it and must be serialized by the caller.  The array keeps the previous
// call's contents; nothing in it needs to start at zero, because the query
// preparation kernel writes every byte the logit kernel reads.

#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "tq_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;    // 4 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" tq_status tq_logits_noalloc(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int64_t n_sets, int g,
                                       tq_packed keys, int64_t n_keys, float* out, void* stream) {
  if (!ctx) return tq::fail(TQ_ERR_INVALID_ARG, "ctx is NULL");
  if (n_sets < 0 || n_keys < 0) return tq::fail(TQ_ERR_INVALID_ARG, "n_sets and n_keys must be >= 0");
  if (g < 1 || g > 4096) return tq::fail(TQ_ERR_INVALID_ARG, "g must be in [1, 4096]");
  const size_t need = tq_logits_workspace_bytes(ctx, n_sets, g);
  if (need > kNoAllocScratchBytes)
    return tq::fail(TQ_ERR_UNSUPPORTED, "n_sets * g * (d + m) * 4 = " + std::to_string(need) +
                                            " bytes exceeds the 4 MiB static scratch of tq_logits_noalloc");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tq::fail(TQ_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return tq::fail(TQ_ERR_UNSUPPORTED, "device ordinal beyond 63");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || !p)
        return tq::fail(TQ_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }
  return tq_logits(ctx, q, q_dtype, n_sets, g, keys, n_keys, out, scratch, kNoAllocScratchBytes, stream);
}
