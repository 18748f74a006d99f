// Internal declarations shared by the C-ABI layer (tq_api.cpp), the host
// parameter code and the CUDA kernels.  Not part of the public interface.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include "../../include/tq.h"

namespace tq {

constexpr int kMaxLevels = 16;      // 2^(b-1) for b <= 5
constexpr float kZeroNorm = 1e-10f; // rows with ||x|| below this are stored as zeros

// Everything a kernel needs about one parameter set, passed by value.
struct KParams {
  int d, m, B, L;                     // d: the rotation dimension (a power of two)
  int d_in;                           // the caller's row length (<= d; rows are zero-padded to d)
  int64_t ld_q, ld_out;               // row strides (elements) of the queries the query prep reads and of
                                      // the rows the general dequant writes: d_in, unless a caller's
                                      // view of wider rows (a channel split) says otherwise
  int codes_bytes, signs_bytes;       // per row
  float inv_sqrt_d;                   // 1/sqrt(d), fp32
  float qjl_scale;                    // sqrt(pi/2) / m, fp32
  float c[kMaxLevels];                // centroids, ascending
  float t[kMaxLevels];                // thresholds (L-1 used)
  const uint32_t* Dmask;              // d/32 words, bit i set iff D_i = -1
  const uint16_t* S;                  // [m][d] binary16
  const uint16_t* St;                 // [d][m] binary16 (transpose)
  int* err;                           // device error word (a bounded wait ran out)
};

struct Packed {
  uint8_t* codes;
  uint8_t* signs;
  float* norm;
  float* rnorm;
};

tq_status check_dims(int d, int b, int m);
size_t round16(size_t v);
size_t round256(size_t v);
int padded_dim(int d);                // the next power of two >= d
tq_status fail(tq_status s, const std::string& why);   // records tq_last_error()
void count_launch(int n = 1);
// test settings (tq_test_set): the bounded-wait limit the tensor-core
// quantize kernel's tile loop runs with, and injected host-side failures
long long wait_limit_cycles();
int64_t fixup_cap_override();          // 0: the default capacity of the quantize fix-up list
bool take_injected_alloc_failure();
bool take_injected_launch_failure();

// host_params.cpp
uint16_t double_to_half_bits(double v);
double half_bits_to_double(uint16_t h);         // (tq_api.cpp) finite values only
void rademacher(int d, uint64_t seed, int8_t* D);
void gaussian_projection_half(int m, int d, uint64_t seed, uint16_t* S_bits);
void lloyd_max(int d, int bits_mse, std::vector<double>& centroids, std::vector<double>& thresholds);

// kernels (return cudaError_t as int; 0 = success).  launch_* choose between
// the d = 128 hot-path kernels and the general ones (*_generic).
int launch_quantize_generic(const KParams& P, const void* x, int x_is_bf16, int64_t n_rows, int64_t ld_x,
                            const Packed& out, void* stream);
int launch_logits_generic(const KParams& P, const float* qp, int64_t n_sets, int g, const Packed& keys,
                          int64_t n_keys, float* out, void* stream);
int launch_dequant_generic(const KParams& P, const Packed& in, int64_t n_rows, void* out, int out_is_bf16, int prod,
                           void* stream);
// scratch: the wide-row path's part of the caller's workspace, or null (the
// wide-row path is then not taken)
size_t quantize_scratch_bytes(const tq_ctx& ctx, int64_t n_rows);
int launch_quantize(const tq_ctx& ctx, const void* x, int x_is_bf16, int64_t n_rows, int64_t ld_x,
                    const Packed& out, void* scratch, void* stream);
int launch_quantize_scatter(const KParams& P, const void* x, int bf16, int64_t n_rows, int64_t ld,
                            const int64_t* dest, int64_t n_dest, const Packed& out, void* stream);
int launch_qprep(const KParams& P, const void* q, int q_is_bf16, int64_t n_queries, float* qp, void* stream);
size_t logits_scratch_bytes(const tq_ctx& ctx, int64_t n_sets, int g, int64_t n_keys);
int launch_logits(const tq_ctx& ctx, const float* qp, int64_t n_sets, int g, const Packed& keys,
                  int64_t n_keys, float* out, void* scratch, void* stream);
int launch_dequant(const tq_ctx& ctx, const Packed& in, int64_t n_rows, void* out, int out_is_bf16, int prod,
                   void* stream);
// attention.cu: the softmax-weighted value sums after the logits are in place
size_t attention_partial_bytes(const KParams& P, int64_t n_sets, int g, int64_t n_keys);
int launch_attention_tail(const KParams& P, const float* logits, const Packed& values, int64_t n_sets, int g,
                          int64_t n_keys, float scale, int prod, float* partial, float* out, void* stream);
int launch_topk(const float* scores, int64_t rows, int64_t cols, int k, int32_t* idx, float* val, void* stream);
int launch_add(float* out, const float* in, int64_t n, void* stream);    // out += in, elementwise
int launch_logits_bf16(const void* q, const void* keys, int64_t n_sets, int g, int64_t n_keys, int d, float* out,
                       void* stream);
const char* cuda_error_string(int err);

}  // namespace tq

struct tq_ctx;

namespace tq {
// d = 128 hot-path kernels (quantize_d128.cu, ...)
bool quantize_d128_applies(const tq_ctx& ctx, int64_t n_rows, int x_is_bf16);   // x_is_bf16 < 0: either
size_t quantize_d128_scratch_bytes(const tq_ctx& ctx, int64_t n_rows);   // deferred sign fix-up list
int launch_quantize_d128(const tq_ctx& ctx, const void* x, int x_is_bf16, int64_t n_rows, int64_t ld,
                         const Packed& out, void* scratch, void* stream);
bool dequant_d128_applies(const tq_ctx& ctx, int64_t n_rows, int out_is_bf16);
bool logits_d128_applies(const tq_ctx& ctx, int64_t n_sets, int g, int64_t n_keys);
int launch_logits_d128(const tq_ctx& ctx, const float* qp, int64_t n_sets, int g, const Packed& keys, int64_t n_keys,
                       float* out, void* stream);
// out: rows of ld_out elements (ld_out >= d; the parts of a split row write
// into their columns of the full row)
int launch_dequant_d128(const tq_ctx& ctx, const Packed& in, int64_t n_rows, void* out, int64_t ld_out,
                        int out_is_bf16, int prod, void* stream);
// wide rows (d >= 256): tensor-core QJL projection and estimates (wide_tc.cu);
// their scratch is part of the caller's workspace
bool wide_quantize_applies(const tq_ctx& ctx, int64_t n_rows);
size_t wide_quantize_scratch_bytes(const tq_ctx& ctx, int64_t n_rows);
int launch_quantize_wide(const tq_ctx& ctx, const void* x, int x_is_bf16, int64_t n_rows, int64_t ld,
                         const Packed& out, void* scratch, void* stream);
bool wide_logits_applies(const tq_ctx& ctx, int64_t n_sets, int g, int64_t n_keys);
size_t wide_logits_scratch_bytes(const tq_ctx& ctx, int64_t n_sets, int g, int64_t n_keys);
int launch_logits_wide(const tq_ctx& ctx, const float* qp, int64_t n_sets, int g, const Packed& keys, int64_t n_keys,
                       float* out, void* scratch, void* stream);
// tq_api.cpp: the compute entry points' shared steps, for the other C-ABI files
tq_status check_ctx(const tq_ctx* ctx);      // non-null, and made on the current device
tq_status quantize_checked(const tq_ctx* ctx, const void* x, tq_dtype x_dtype, int64_t n_rows, int64_t ld_x,
                           const tq_packed& out, void* scratch, void* stream);
size_t qprep_bytes(const tq_ctx* ctx, int64_t n_q);
tq_status logits_args(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int64_t n_sets, int g,
                      const tq_packed& keys, int64_t n_keys, const float* out, bool* empty);
tq_status logits_checked(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int64_t n_sets, int g,
                         const tq_packed& keys, int64_t n_keys, float* out, float* qp, void* scratch, void* stream);
// vector search with the top-k fused into the estimates' epilogue
bool wide_search_applies(const tq_ctx& ctx, int64_t n_q, int64_t n_keys, int k);
size_t wide_search_partial_bytes(const tq_ctx& ctx, int64_t n_q, int64_t n_keys, int k);
int launch_search_wide(const tq_ctx& ctx, const float* qp, int64_t n_q, const Packed& keys, int64_t n_keys, int k,
                       int32_t* idx, float* val, void* part, void* stream);
}  // namespace tq

struct tq_ctx {
  int d, b, m;                        // d: padded (power-of-two) dimension
  int d_in;                           // the caller's row length
  uint64_t seed;
  int device;
  int num_sms;
  bool use_tc;                        // hot-path (tensor-core) kernels enabled
  float qjl_eps_scale;                // projection error bound coefficients (quantize_d128.cu)
  float qjl_eps_abs;
  float colsum_d128[128];             // sum_j S[j][i] (d = 128 only)
  std::vector<float> centroids, thresholds;
  std::vector<int8_t> D;
  std::vector<uint16_t> S_bits;
  double s1max;                       // max_j ||S_j||_1
  const float* snorm_dev;             // [m] ||S_j||_2 on the device (in dev_block)
  void* dev_block;                    // one allocation holding everything below
  tq::KParams kp;
};
