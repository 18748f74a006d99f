// C ABI of libtq: argument checks, context set-up and kernel dispatch.
// Every compute entry point validates its arguments on the host and launches
// nothing when a check fails; see include/tq.h for the contract.

#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>

#include "tq_internal.h"

namespace tq {

static thread_local std::string g_last_error;
static std::atomic<uint64_t> g_launches{0};

tq_status fail(tq_status s, const std::string& why) {
  g_last_error = why;
  return s;
}

void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

constexpr long long kDefaultWaitCycles = 2000000000ll;         // about one second at 2 GHz
static std::atomic<long long> g_wait_limit{kDefaultWaitCycles};
static std::atomic<int64_t> g_fail_alloc{0}, g_fail_launch{0}, g_fixup_cap{0};

long long wait_limit_cycles() { return g_wait_limit.load(std::memory_order_relaxed); }
int64_t fixup_cap_override() { return g_fixup_cap.load(std::memory_order_relaxed); }

static bool take_one(std::atomic<int64_t>& n) {
  int64_t v = n.load(std::memory_order_relaxed);
  while (v > 0)
    if (n.compare_exchange_weak(v, v - 1, std::memory_order_relaxed)) return true;
  return false;
}
bool take_injected_alloc_failure() { return take_one(g_fail_alloc); }
bool take_injected_launch_failure() { return take_one(g_fail_launch); }

int padded_dim(int d) {
  int p = 1;
  while (p < d) p <<= 1;
  return p;
}

tq_status check_dims(int d, int b, int m) {
  if (d < 32 || d > 4096) return fail(TQ_ERR_INVALID_ARG, "d must be in [32, 4096]");
  if (b < 2 || b > 5) return fail(TQ_ERR_INVALID_ARG, "b must be in [2, 5]");
  if (m < 32 || m > 4096 || (m % 32)) return fail(TQ_ERR_INVALID_ARG, "m must be a multiple of 32 in [32, 4096]");
  return TQ_OK;
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static tq_status cuda_fail(int err, const char* what) {
  return fail(TQ_ERR_CUDA, std::string(what) + ": " + cuda_error_string(err));
}

tq_status check_ctx(const tq_ctx* ctx) {
  if (!ctx) return fail(TQ_ERR_INVALID_ARG, "ctx is NULL");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(TQ_ERR_CUDA, "cudaGetDevice failed");
  if (dev != ctx->device) return fail(TQ_ERR_INVALID_ARG, "the current device is not the context's device");
  return TQ_OK;
}

static tq_status check_packed(const tq_ctx* ctx, const tq_packed& p) {
  if (!p.codes || !p.signs || !p.norm || !p.rnorm) return fail(TQ_ERR_INVALID_ARG, "a packed pointer is NULL");
  if (!aligned(p.codes, 16) || !aligned(p.signs, 16))
    return fail(TQ_ERR_INVALID_ARG, "packed codes/signs must be 16-byte aligned");
  if (!aligned(p.norm, 4) || !aligned(p.rnorm, 4))
    return fail(TQ_ERR_INVALID_ARG, "packed norm/rnorm must be 4-byte aligned");
  (void)ctx;
  return TQ_OK;
}

static Packed to_internal(const tq_packed& p) { return Packed{p.codes, p.signs, p.norm, p.rnorm}; }

// tq_quantize after its context, count and workspace checks: the remaining
// argument checks, then the launch (scratch null: no wide-row path)
tq_status quantize_checked(const tq_ctx* ctx, const void* x, tq_dtype x_dtype, int64_t n_rows, int64_t ld_x,
                           const tq_packed& out, void* scratch, void* stream) {
  if (!x) return fail(TQ_ERR_INVALID_ARG, "x is NULL");
  const size_t esz = x_dtype == TQ_BF16 ? 2 : 4;
  if (ld_x < ctx->d_in) return fail(TQ_ERR_INVALID_ARG, "ld_x < d");
  if (ctx->d_in == ctx->d) {
    if (!aligned(x, 16) || (static_cast<size_t>(ld_x) * esz) % 16)
      return fail(TQ_ERR_INVALID_ARG, "x and its row stride must be 16-byte aligned");
  } else if (!aligned(x, esz)) {        // padded rows are read element by element
    return fail(TQ_ERR_INVALID_ARG, "x must be aligned to its element size");
  }
  tq_status st = check_packed(ctx, out);
  if (st != TQ_OK) return st;
  int err = launch_quantize(*ctx, x, x_dtype == TQ_BF16, n_rows, ld_x, to_internal(out), scratch, stream);
  if (err) return cuda_fail(err, "tq_quantize launch");
  return TQ_OK;
}

size_t round16(size_t v) { return (v + 15) & ~static_cast<size_t>(15); }
size_t round256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// bytes of the query operands (R q | S R q per query) at the front of a
// logits workspace
size_t qprep_bytes(const tq_ctx* ctx, int64_t n_q) {
  return static_cast<size_t>(n_q) * (ctx->d + ctx->m) * sizeof(float);
}

// tq_logits after its argument checks: query prep into qp, then the logit
// kernels (scratch null: no wide-row path)
tq_status logits_checked(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int64_t n_sets, int g,
                         const tq_packed& keys, int64_t n_keys, float* out, float* qp, void* scratch, void* stream) {
  int err = launch_qprep(ctx->kp, q, q_dtype == TQ_BF16, n_sets * g, qp, stream);
  if (err) return cuda_fail(err, "tq_logits query-prep launch");
  err = launch_logits(*ctx, qp, n_sets, g, to_internal(keys), n_keys, out, scratch, stream);
  if (err) return cuda_fail(err, "tq_logits launch");
  return TQ_OK;
}

// the checks tq_logits makes before it looks at the workspace
tq_status logits_args(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int64_t n_sets, int g,
                      const tq_packed& keys, int64_t n_keys, const float* out, bool* empty) {
  *empty = false;
  tq_status st = check_ctx(ctx);
  if (st != TQ_OK) return st;
  if (n_sets < 0 || n_keys < 0) return fail(TQ_ERR_INVALID_ARG, "n_sets and n_keys must be >= 0");
  if (g < 1 || g > 4096) return fail(TQ_ERR_INVALID_ARG, "g must be in [1, 4096]");
  if (q_dtype != TQ_BF16 && q_dtype != TQ_F32) return fail(TQ_ERR_INVALID_ARG, "q_dtype must be TQ_BF16 or TQ_F32");
  if (n_sets == 0 || n_keys == 0) { *empty = true; return TQ_OK; }
  if (!q || !out) return fail(TQ_ERR_INVALID_ARG, "q or out is NULL");
  if (!aligned(q, 16) || !aligned(out, 4)) return fail(TQ_ERR_INVALID_ARG, "q must be 16-byte and out 4-byte aligned");
  return check_packed(ctx, keys);
}

double half_bits_to_double(uint16_t h) {
  const int sign = (h >> 15) & 1, e = (h >> 10) & 31, f = h & 1023;
  double v = e == 0 ? std::ldexp(static_cast<double>(f), -24) : std::ldexp(static_cast<double>(1024 + f), e - 25);
  return sign ? -v : v;
}

}  // namespace tq

using namespace tq;

extern "C" {

const char* tq_status_str(tq_status s) {
  switch (s) {
    case TQ_OK: return "TQ_OK";
    case TQ_ERR_INVALID_ARG: return "TQ_ERR_INVALID_ARG";
    case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED";
    case TQ_ERR_NOMEM: return "TQ_ERR_NOMEM";
    case TQ_ERR_CUDA: return "TQ_ERR_CUDA";
  }
  return "TQ_ERR_UNKNOWN";
}

const char* tq_last_error(void) { return g_last_error.c_str(); }

tq_status tq_sync_status(const tq_ctx* ctx, void* stream) {
  tq_status st = check_ctx(ctx);
  if (st != TQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int word = 0;
  e = cudaMemcpy(&word, ctx->kp.err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
  if (word) {
    const int zero = 0;
    cudaMemcpy(ctx->kp.err, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (word == 7) return fail(TQ_ERR_INVALID_ARG, "tq_quantize_scatter: a destination row index was out of range "
                                                   "(that row was not written)");
    if (word == 8) return fail(TQ_ERR_CUDA, "tq_quantize: more projections than expected fell inside the tensor-core "
                                            "error bound; some sign bits were not recomputed");
    return fail(TQ_ERR_CUDA, "a kernel wait ran out of time (code " + std::to_string(word) + "); outputs are invalid");
  }
  return TQ_OK;
}

uint64_t tq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

tq_status tq_init(int d, int b, int m, uint64_t seed, tq_ctx** out) {
  if (!out) return fail(TQ_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  tq_status st = check_dims(d, b, m);
  if (st != TQ_OK) return st;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0;
  e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  if (major != 10) return fail(TQ_ERR_UNSUPPORTED, "libtq is built for sm_100a (compute capability 10.x)");

  tq_ctx* ctx = new (std::nothrow) tq_ctx();
  if (!ctx) return fail(TQ_ERR_NOMEM, "host allocation failed");
  // a row length that is not a power of two is zero-padded to the next one
  // (0h-n0 "ICLR 2026論文解説: TurboQuant", "実装のポイント"): the rotation, the
  // codebook, D, S and the packed format are those of the padded dimension
  ctx->d_in = d;
  d = padded_dim(d);
  ctx->d = d; ctx->b = b; ctx->m = m; ctx->seed = seed; ctx->device = dev;
  const int B = b - 1, L = 1 << B;
  ctx->centroids.resize(L);
  ctx->thresholds.resize(L - 1);
  ctx->D.resize(d);
  ctx->S_bits.resize(static_cast<size_t>(m) * d);
  tq_host_params(d, b, m, seed, ctx->centroids.data(), ctx->thresholds.data(), ctx->D.data(), ctx->S_bits.data());

  // device block, 256-byte aligned parts: error word | Dmask (d/32 words) | S [m][d] | St [d][m] |
  // ||S_j||_2 [m]
  auto round256 = [](size_t v) { return (v + 255) / 256 * 256; };
  const size_t n_mask = static_cast<size_t>(d) / 32;
  const size_t sz_S = static_cast<size_t>(m) * d * sizeof(uint16_t);
  const size_t off_err = 0;
  const size_t off_mask = 256;
  const size_t off_S2 = off_mask + round256(n_mask * 4);
  const size_t off_St = off_S2 + round256(sz_S);
  const size_t off_sn = off_St + round256(sz_S);
  const size_t total = off_sn + round256(static_cast<size_t>(m) * 4);
  void* blk = nullptr;
  e = take_injected_alloc_failure() ? cudaErrorMemoryAllocation : cudaMalloc(&blk, total);
  if (e != cudaSuccess) { delete ctx; return fail(TQ_ERR_NOMEM, std::string("cudaMalloc: ") + cudaGetErrorString(e)); }
  ctx->dev_block = blk;

  std::vector<uint8_t> host(total, 0);
  uint32_t* mask = reinterpret_cast<uint32_t*>(host.data() + off_mask);
  for (int i = 0; i < d; ++i)
    if (ctx->D[i] < 0) mask[i / 32] |= (1u << (i % 32));
  std::memcpy(host.data() + off_S2, ctx->S_bits.data(), sz_S);
  uint16_t* St = reinterpret_cast<uint16_t*>(host.data() + off_St);
  for (int j = 0; j < m; ++j)
    for (int i = 0; i < d; ++i) St[static_cast<size_t>(i) * m + j] = ctx->S_bits[static_cast<size_t>(j) * d + i];
  float* snorm = reinterpret_cast<float*>(host.data() + off_sn);
  double smax = 0.0, s1max = 0.0;                      // max_j ||S_j||_2 and max_j ||S_j||_1
  for (int j = 0; j < m; ++j) {
    double acc = 0.0, acc1 = 0.0;
    for (int i = 0; i < d; ++i) {
      const double v = half_bits_to_double(ctx->S_bits[static_cast<size_t>(j) * d + i]);
      acc += v * v;
      acc1 += std::fabs(v);
    }
    snorm[j] = static_cast<float>(std::sqrt(acc) * (1.0 + 1e-6));   // rounded up
    smax = std::max(smax, std::sqrt(acc));
    s1max = std::max(s1max, acc1);
  }
  e = cudaMemcpy(blk, host.data(), total, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) { cudaFree(blk); delete ctx; return cuda_fail(e, "cudaMemcpy"); }

  KParams& kp = ctx->kp;
  std::memset(&kp, 0, sizeof(kp));
  kp.d = d; kp.m = m; kp.B = B; kp.L = L;
  kp.d_in = ctx->d_in;
  kp.ld_q = kp.ld_out = ctx->d_in;
  kp.codes_bytes = d * B / 8;
  kp.signs_bytes = m / 8;
  kp.inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
  kp.qjl_scale = static_cast<float>(std::sqrt(std::acos(-1.0) / 2.0) / m);
  for (int i = 0; i < L; ++i) kp.c[i] = ctx->centroids[i];
  for (int i = 0; i < L - 1; ++i) kp.t[i] = ctx->thresholds[i];
  kp.Dmask = reinterpret_cast<const uint32_t*>(static_cast<uint8_t*>(blk) + off_mask);
  kp.S = reinterpret_cast<const uint16_t*>(static_cast<uint8_t*>(blk) + off_S2);
  kp.St = reinterpret_cast<const uint16_t*>(static_cast<uint8_t*>(blk) + off_St);
  kp.err = reinterpret_cast<int*>(static_cast<uint8_t*>(blk) + off_err);

  int nsm = 0;
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  ctx->num_sms = nsm > 0 ? nsm : 148;
  const char* kern = std::getenv("TQ_KERNELS");
  ctx->use_tc = !(kern && std::strcmp(kern, "generic") == 0);
  // projection error bound coefficient 16 * 2^-22 * max_j ||S_j|| (the hi + lo
  // split leaves 2^-22 ||r||, 16 fp32 accumulation steps of the K = 256 chain
  // at most 2^-23 each, i.e. 9 * 2^-22 ||S_j|| ||r|| with truncating adds, and
  // a further margin; the tensor-core error measured over 10^6 projections
  // peaks at 1.7 * 2^-22 ||S_j|| ||r||), plus max_j ||S_j||_1 * 2^-25 / 64 for
  // binary16 underflow of the scaled residual
  ctx->s1max = s1max;
  ctx->snorm_dev = reinterpret_cast<const float*>(static_cast<uint8_t*>(blk) + off_sn);
  ctx->qjl_eps_scale = static_cast<float>(16.0 * std::ldexp(1.0, -22) * smax);
  ctx->qjl_eps_abs = static_cast<float>(2.0 * s1max * std::ldexp(1.0, -25) / 64.0);
  for (int i = 0; i < 128; ++i) ctx->colsum_d128[i] = 0.f;
  if (d == 128) {
    for (int i = 0; i < d; ++i) {
      double acc = 0.0;
      for (int j = 0; j < m; ++j) acc += half_bits_to_double(ctx->S_bits[static_cast<size_t>(j) * d + i]);
      ctx->colsum_d128[i] = static_cast<float>(acc);
    }
  }
  *out = ctx;
  return TQ_OK;
}

tq_status tq_destroy(tq_ctx* ctx) {
  if (!ctx) return TQ_OK;
  cudaError_t e = cudaSuccess;
  if (ctx->dev_block) e = cudaFree(ctx->dev_block);
  delete ctx;
  if (e != cudaSuccess) return cuda_fail(e, "cudaFree");
  return TQ_OK;
}

tq_status tq_packed_sizes(const tq_ctx* ctx, int64_t n_rows, size_t* codes_bytes, size_t* signs_bytes) {
  if (!ctx) return fail(TQ_ERR_INVALID_ARG, "ctx is NULL");
  if (n_rows < 0) return fail(TQ_ERR_INVALID_ARG, "n_rows < 0");
  if (codes_bytes) *codes_bytes = static_cast<size_t>(n_rows) * ctx->kp.codes_bytes;
  if (signs_bytes) *signs_bytes = static_cast<size_t>(n_rows) * ctx->kp.signs_bytes;
  return TQ_OK;
}

tq_status tq_get_params(const tq_ctx* ctx, float* centroids, float* thresholds, int8_t* D, uint16_t* S_bits) {
  if (!ctx) return fail(TQ_ERR_INVALID_ARG, "ctx is NULL");
  if (centroids) std::memcpy(centroids, ctx->centroids.data(), ctx->centroids.size() * sizeof(float));
  if (thresholds) std::memcpy(thresholds, ctx->thresholds.data(), ctx->thresholds.size() * sizeof(float));
  if (D) std::memcpy(D, ctx->D.data(), ctx->D.size());
  if (S_bits) std::memcpy(S_bits, ctx->S_bits.data(), ctx->S_bits.size() * sizeof(uint16_t));
  return TQ_OK;
}

size_t tq_quantize_workspace_bytes(const tq_ctx* ctx, int64_t n_rows) {
  if (!ctx || n_rows <= 0) return 0;
  return quantize_scratch_bytes(*ctx, n_rows);
}

tq_status tq_quantize(const tq_ctx* ctx, const void* x, tq_dtype x_dtype, int64_t n_rows, int64_t ld_x,
                      tq_packed out, void* workspace, size_t workspace_bytes, void* stream) {
  tq_status st = check_ctx(ctx);
  if (st != TQ_OK) return st;
  if (n_rows < 0) return fail(TQ_ERR_INVALID_ARG, "n_rows < 0");
  if (x_dtype != TQ_BF16 && x_dtype != TQ_F32) return fail(TQ_ERR_INVALID_ARG, "x_dtype must be TQ_BF16 or TQ_F32");
  if (n_rows == 0) return TQ_OK;
  const size_t need = quantize_scratch_bytes(*ctx, n_rows);
  if (need) {
    if (!workspace || workspace_bytes < need) return fail(TQ_ERR_INVALID_ARG, "workspace missing or too small");
    if (!aligned(workspace, 16)) return fail(TQ_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  }
  return quantize_checked(ctx, x, x_dtype, n_rows, ld_x, out, need ? workspace : nullptr, stream);
}

tq_status tq_quantize_scatter(const tq_ctx* ctx, const void* x, tq_dtype x_dtype, int64_t n_rows, int64_t ld_x,
                              const int64_t* dest_rows, int64_t n_cache_rows, tq_packed cache, void* stream) {
  tq_status st = check_ctx(ctx);
  if (st != TQ_OK) return st;
  if (n_rows < 0 || n_cache_rows < 0) return fail(TQ_ERR_INVALID_ARG, "n_rows and n_cache_rows must be >= 0");
  if (x_dtype != TQ_BF16 && x_dtype != TQ_F32) return fail(TQ_ERR_INVALID_ARG, "x_dtype must be TQ_BF16 or TQ_F32");
  if (n_rows == 0) return TQ_OK;
  if (!x || !dest_rows) return fail(TQ_ERR_INVALID_ARG, "x or dest_rows is NULL");
  const size_t esz = x_dtype == TQ_BF16 ? 2 : 4;
  if (ld_x < ctx->d_in) return fail(TQ_ERR_INVALID_ARG, "ld_x < d");
  if (!aligned(x, esz)) return fail(TQ_ERR_INVALID_ARG, "x must be aligned to its element size");
  if (!aligned(dest_rows, 8)) return fail(TQ_ERR_INVALID_ARG, "dest_rows must be 8-byte aligned");
  if ((st = check_packed(ctx, cache)) != TQ_OK) return st;
  int err = launch_quantize_scatter(ctx->kp, x, x_dtype == TQ_BF16, n_rows, ld_x, dest_rows, n_cache_rows,
                                    to_internal(cache), stream);
  if (err) return cuda_fail(err, "tq_quantize_scatter launch");
  return TQ_OK;
}

size_t tq_logits_workspace_bytes(const tq_ctx* ctx, int64_t n_sets, int g, int64_t n_keys) {
  if (!ctx || n_sets <= 0 || g <= 0 || n_keys <= 0) return 0;
  const size_t wide = logits_scratch_bytes(*ctx, n_sets, g, n_keys);
  return wide ? round256(qprep_bytes(ctx, n_sets * g)) + wide : qprep_bytes(ctx, n_sets * g);
}

tq_status tq_logits(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int64_t n_sets, int g, tq_packed keys,
                    int64_t n_keys, float* out, void* workspace, size_t workspace_bytes, void* stream) {
  bool empty = false;
  tq_status st = logits_args(ctx, q, q_dtype, n_sets, g, keys, n_keys, out, &empty);
  if (st != TQ_OK || empty) return st;
  const size_t need = tq_logits_workspace_bytes(ctx, n_sets, g, n_keys);
  if (!workspace || workspace_bytes < need) return fail(TQ_ERR_INVALID_ARG, "workspace missing or too small");
  if (!aligned(workspace, 16)) return fail(TQ_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  const bool wide = logits_scratch_bytes(*ctx, n_sets, g, n_keys) != 0;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  return logits_checked(ctx, q, q_dtype, n_sets, g, keys, n_keys, out, reinterpret_cast<float*>(w),
                        wide ? w + round256(qprep_bytes(ctx, n_sets * g)) : nullptr, stream);
}

size_t tq_search_workspace_bytes(const tq_ctx* ctx, int64_t n_q, int64_t n_keys, int k) {
  if (!ctx || n_q <= 0 || n_keys <= 0 || k <= 0) return 0;
  const size_t qp = round256(qprep_bytes(ctx, n_q));
  if (wide_search_applies(*ctx, n_q, n_keys, k)) return qp + wide_search_partial_bytes(*ctx, n_q, n_keys, k);
  return qp + round16(static_cast<size_t>(n_q) * n_keys * sizeof(float));
}

tq_status tq_search(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int64_t n_q, tq_packed keys, int64_t n_keys,
                    int k, int32_t* idx, float* val, void* workspace, size_t workspace_bytes, void* stream) {
  tq_status st = check_ctx(ctx);
  if (st != TQ_OK) return st;
  if (n_q < 0 || n_keys < 0) return fail(TQ_ERR_INVALID_ARG, "n_q and n_keys must be >= 0");
  if (n_q > 4096) return fail(TQ_ERR_INVALID_ARG, "n_q must be in [0, 4096]");
  if (k < 1 || k > 16) return fail(TQ_ERR_INVALID_ARG, "k must be in [1, 16]");
  if (q_dtype != TQ_BF16 && q_dtype != TQ_F32) return fail(TQ_ERR_INVALID_ARG, "q_dtype must be TQ_BF16 or TQ_F32");
  if (n_q == 0) return TQ_OK;
  if (k > n_keys) return fail(TQ_ERR_INVALID_ARG, "k > n_keys");
  if (n_keys > INT32_MAX) return fail(TQ_ERR_UNSUPPORTED, "n_keys must fit in int32");
  if (!q || !idx) return fail(TQ_ERR_INVALID_ARG, "q or idx is NULL");
  if (!aligned(q, 16) || !aligned(idx, 4) || (val && !aligned(val, 4)))
    return fail(TQ_ERR_INVALID_ARG, "q must be 16-byte and idx/val 4-byte aligned");
  if ((st = check_packed(ctx, keys)) != TQ_OK) return st;
  const size_t need = tq_search_workspace_bytes(ctx, n_q, n_keys, k);
  if (!workspace || workspace_bytes < need) return fail(TQ_ERR_INVALID_ARG, "workspace missing or too small");
  if (!aligned(workspace, 16)) return fail(TQ_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  uint8_t* w = static_cast<uint8_t*>(workspace);
  float* qp = reinterpret_cast<float*>(w);
  void* rest = w + round256(qprep_bytes(ctx, n_q));
  int err = launch_qprep(ctx->kp, q, q_dtype == TQ_BF16, n_q, qp, stream);
  if (err) return cuda_fail(err, "tq_search query-prep launch");
  if (wide_search_applies(*ctx, n_q, n_keys, k)) {
    err = launch_search_wide(*ctx, qp, n_q, to_internal(keys), n_keys, k, idx, val, rest, stream);
    if (err) return cuda_fail(err, "tq_search launch");
    return TQ_OK;
  }
  float* scores = static_cast<float*>(rest);         // [n_q, n_keys], then the top-k of each row
  err = launch_logits(*ctx, qp, 1, static_cast<int>(n_q), to_internal(keys), n_keys, scores, nullptr, stream);
  if (err) return cuda_fail(err, "tq_search logits launch");
  err = launch_topk(scores, n_q, n_keys, k, idx, val, stream);
  if (err) return cuda_fail(err, "tq_search top-k launch");
  return TQ_OK;
}

size_t tq_attention_workspace_bytes(const tq_ctx* ctx, int64_t n_sets, int g, int64_t n_keys) {
  if (!ctx || n_sets <= 0 || g <= 0 || n_keys <= 0) return 0;
  return round16(qprep_bytes(ctx, n_sets * g)) +
         round16(static_cast<size_t>(n_sets) * g * n_keys * sizeof(float)) +
         round16(attention_partial_bytes(ctx->kp, n_sets, g, n_keys));
}

tq_status tq_attention(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int64_t n_sets, int g, tq_packed keys,
                       tq_packed values, int64_t n_keys, float scale, tq_dequant_mode mode, float* out,
                       void* workspace, size_t workspace_bytes, void* stream) {
  tq_status st = check_ctx(ctx);
  if (st != TQ_OK) return st;
  if (n_sets < 0 || n_keys < 0) return fail(TQ_ERR_INVALID_ARG, "n_sets and n_keys must be >= 0");
  if (g < 1 || g > 8) return fail(TQ_ERR_INVALID_ARG, "g must be in [1, 8]");
  if (q_dtype != TQ_BF16 && q_dtype != TQ_F32) return fail(TQ_ERR_INVALID_ARG, "q_dtype must be TQ_BF16 or TQ_F32");
  if (mode != TQ_DEQUANT_PROD && mode != TQ_DEQUANT_MSE) return fail(TQ_ERR_INVALID_ARG, "bad dequant mode");
  if (!std::isfinite(scale)) return fail(TQ_ERR_INVALID_ARG, "scale must be finite");
  if (ctx->d + ctx->m > 2048) return fail(TQ_ERR_UNSUPPORTED, "tq_attention needs d + m <= 2048");
  if (n_sets == 0) return TQ_OK;
  if (n_keys == 0) return fail(TQ_ERR_INVALID_ARG, "n_keys must be >= 1 (softmax over no keys)");
  if (n_sets > 65535) return fail(TQ_ERR_UNSUPPORTED, "n_sets must be <= 65535");
  if (n_keys > (int64_t(1) << 31) - 4096) return fail(TQ_ERR_UNSUPPORTED, "n_keys too large");
  if (!q || !out) return fail(TQ_ERR_INVALID_ARG, "q or out is NULL");
  if (!aligned(q, 16) || !aligned(out, 4)) return fail(TQ_ERR_INVALID_ARG, "q must be 16-byte and out 4-byte aligned");
  if ((st = check_packed(ctx, keys)) != TQ_OK) return st;
  if ((st = check_packed(ctx, values)) != TQ_OK) return st;
  const size_t need = tq_attention_workspace_bytes(ctx, n_sets, g, n_keys);
  if (!workspace || workspace_bytes < need) return fail(TQ_ERR_INVALID_ARG, "workspace missing or too small");
  if (!aligned(workspace, 16)) return fail(TQ_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  uint8_t* w = static_cast<uint8_t*>(workspace);
  float* qp = reinterpret_cast<float*>(w);
  float* lg = reinterpret_cast<float*>(w + round16(qprep_bytes(ctx, n_sets * g)));
  float* part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(lg) +
                                         round16(static_cast<size_t>(n_sets) * g * n_keys * sizeof(float)));
  int err = launch_qprep(ctx->kp, q, q_dtype == TQ_BF16, n_sets * g, qp, stream);
  if (err) return cuda_fail(err, "tq_attention query-prep launch");
  err = launch_logits(*ctx, qp, n_sets, g, to_internal(keys), n_keys, lg, nullptr, stream);
  if (err) return cuda_fail(err, "tq_attention logits launch");
  err = launch_attention_tail(ctx->kp, lg, to_internal(values), n_sets, g, n_keys, scale,
                              mode == TQ_DEQUANT_PROD ? 1 : 0, part, out, stream);
  if (err) return cuda_fail(err, "tq_attention launch");
  return TQ_OK;
}

tq_status tq_dequant(const tq_ctx* ctx, tq_packed in, int64_t n_rows, void* out, tq_dtype out_dtype,
                     tq_dequant_mode mode, void* stream) {
  tq_status st = check_ctx(ctx);
  if (st != TQ_OK) return st;
  if (n_rows < 0) return fail(TQ_ERR_INVALID_ARG, "n_rows < 0");
  if (out_dtype != TQ_BF16 && out_dtype != TQ_F32) return fail(TQ_ERR_INVALID_ARG, "out_dtype must be TQ_BF16 or TQ_F32");
  if (mode != TQ_DEQUANT_PROD && mode != TQ_DEQUANT_MSE) return fail(TQ_ERR_INVALID_ARG, "bad dequant mode");
  if (n_rows == 0) return TQ_OK;
  if (!out) return fail(TQ_ERR_INVALID_ARG, "out is NULL");
  if (!aligned(out, 16)) return fail(TQ_ERR_INVALID_ARG, "out must be 16-byte aligned");
  if ((st = check_packed(ctx, in)) != TQ_OK) return st;
  int err = launch_dequant(*ctx, to_internal(in), n_rows, out, out_dtype == TQ_BF16, mode == TQ_DEQUANT_PROD, stream);
  if (err) return cuda_fail(err, "tq_dequant launch");
  return TQ_OK;
}

tq_status tq_topk(const float* scores, int64_t rows, int64_t cols, int k, int32_t* idx, float* val, void* stream) {
  if (rows < 0 || cols < 0) return fail(TQ_ERR_INVALID_ARG, "rows and cols must be >= 0");
  if (k < 1 || k > 64) return fail(TQ_ERR_INVALID_ARG, "k must be in [1, 64]");
  if (rows == 0) return TQ_OK;
  if (k > cols) return fail(TQ_ERR_INVALID_ARG, "k > cols");
  if (cols > INT32_MAX) return fail(TQ_ERR_UNSUPPORTED, "cols must fit in int32");
  if (!scores || !idx) return fail(TQ_ERR_INVALID_ARG, "scores or idx is NULL");
  if (!aligned(scores, 4) || !aligned(idx, 4) || (val && !aligned(val, 4)))
    return fail(TQ_ERR_INVALID_ARG, "scores/idx/val must be 4-byte aligned");
  int err = launch_topk(scores, rows, cols, k, idx, val, stream);
  if (err) return cuda_fail(err, "tq_topk launch");
  return TQ_OK;
}

tq_status tq_test_set(tq_test_knob knob, int64_t value) {
  if (value < 0) return fail(TQ_ERR_INVALID_ARG, "value must be >= 0");
  switch (knob) {
    case TQ_TEST_WAIT_LIMIT:
      g_wait_limit.store(value == 0 ? kDefaultWaitCycles : value, std::memory_order_relaxed);
      return TQ_OK;
    case TQ_TEST_FAIL_ALLOC: g_fail_alloc.store(value, std::memory_order_relaxed); return TQ_OK;
    case TQ_TEST_FAIL_LAUNCH: g_fail_launch.store(value, std::memory_order_relaxed); return TQ_OK;
    case TQ_TEST_FIXUP_CAP: g_fixup_cap.store(value, std::memory_order_relaxed); return TQ_OK;
  }
  return fail(TQ_ERR_INVALID_ARG, "unknown test setting");
}

tq_status tq_logits_bf16(const void* q, const void* keys, int64_t n_sets, int g, int64_t n_keys, int d, float* out,
                         void* stream) {
  if (n_sets < 0 || n_keys < 0) return fail(TQ_ERR_INVALID_ARG, "n_sets and n_keys must be >= 0");
  if (g < 1 || g > 8) return fail(TQ_ERR_INVALID_ARG, "g must be in [1, 8]");
  if (d != 64 && d != 128 && d != 256) return fail(TQ_ERR_INVALID_ARG, "d must be 64, 128 or 256");
  if (n_sets == 0 || n_keys == 0) return TQ_OK;
  if (n_sets > 65535) return fail(TQ_ERR_UNSUPPORTED, "n_sets must be <= 65535");
  if (!q || !keys || !out) return fail(TQ_ERR_INVALID_ARG, "a pointer is NULL");
  if (!aligned(q, 16) || !aligned(keys, 16) || !aligned(out, 4))
    return fail(TQ_ERR_INVALID_ARG, "q and keys must be 16-byte aligned, out 4-byte");
  int err = launch_logits_bf16(q, keys, n_sets, g, n_keys, d, out, stream);
  if (err) return cuda_fail(err, "tq_logits_bf16 launch");
  return TQ_OK;
}

}  // extern "C"
