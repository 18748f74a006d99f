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
// Only the query operands go to the array.  On wide rows, where tq_logits
// would decode the keys into a binary16 operand for the tensor-core GEMM (a
// scratch of tens of megabytes), this call runs the general logit kernels
// instead, which read the packed keys directly; the results agree with
// tq_logits within the logit tolerance, not bit for bit.
//
// The device address of that array is looked up once per CUDA context, on
// the first call made with that context current (cudaGetSymbolAddress), and
// cached (up to kMaxContexts contexts per process).  Make that first call
// before any stream capture begins.
//
// All calls share the one array of a context, whatever their stream: calls
// that may overlap on the GPU (different streams, or different host threads)
// race on it and must be serialized by the caller.  The array keeps the
// previous call's contents; nothing in it needs to start at zero, because the
// query preparation kernel writes every byte the logit kernel reads.

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "tq_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;    // 4 MiB
constexpr int kMaxContexts = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

std::mutex g_mu;
CUcontext g_ctx_key[kMaxContexts] = {};
void* g_scratch_addr[kMaxContexts] = {};
int g_n_cached = 0;

// cuCtxGetCurrent through the runtime's driver entry point (no libcuda link)
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  return fn;
}

}  // namespace

extern "C" tq_status tq_logits_noalloc(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int64_t n_sets, int g,
                                       tq_packed keys, int64_t n_keys, float* out, void* stream) {
  bool empty = false;
  tq_status st = tq::logits_args(ctx, q, q_dtype, n_sets, g, keys, n_keys, out, &empty);
  if (st != TQ_OK || empty) return st;
  const size_t need = tq::qprep_bytes(ctx, n_sets * g);
  if (need > kNoAllocScratchBytes)
    return tq::fail(TQ_ERR_UNSUPPORTED, "n_sets * g * (d + m) * 4 = " + std::to_string(need) +
                                            " bytes exceeds the 4 MiB static scratch of tq_logits_noalloc");
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) return tq::fail(TQ_ERR_CUDA, "cuCtxGetCurrent is not available");
  CUcontext cu = nullptr;
  cudaError_t e = cudaSuccess;
  if (get(&cu) != CUDA_SUCCESS) return tq::fail(TQ_ERR_CUDA, "cuCtxGetCurrent failed");
  if (!cu) {
    // no context bound to this thread yet: the runtime binds the device's
    // primary context on its first call that needs one, as this lookup does
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return tq::fail(TQ_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    if (get(&cu) != CUDA_SUCCESS || !cu) return tq::fail(TQ_ERR_CUDA, "no current CUDA context");
  }
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_n_cached; ++i)
      if (g_ctx_key[i] == cu) scratch = g_scratch_addr[i];
    if (!scratch) {
      if (g_n_cached == kMaxContexts) return tq::fail(TQ_ERR_UNSUPPORTED, "more than 64 CUDA contexts");
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || !p)
        return tq::fail(TQ_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
      g_ctx_key[g_n_cached] = cu;
      g_scratch_addr[g_n_cached] = p;
      ++g_n_cached;
      scratch = p;
    }
  }
  return tq::logits_checked(ctx, q, q_dtype, n_sets, g, keys, n_keys, out, static_cast<float*>(scratch), nullptr,
                            stream);
}
