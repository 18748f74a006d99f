// Kernel selection: the d = 128 hot-path kernels where they apply, then the
// wide-row tensor-core paths (d >= 256, many rows; only when the caller's
// workspace holds their scratch), the general kernels everywhere else.
#include <cuda_runtime.h>

#include "tq_internal.h"

namespace tq {

size_t quantize_scratch_bytes(const tq_ctx& ctx, int64_t n_rows) {
  if (quantize_d128_applies(ctx, n_rows, -1)) return quantize_d128_scratch_bytes(ctx, n_rows);
  return wide_quantize_applies(ctx, n_rows) ? wide_quantize_scratch_bytes(ctx, n_rows) : 0;
}

int launch_quantize(const tq_ctx& ctx, const void* x, int x_is_bf16, int64_t n_rows, int64_t ld_x, const Packed& out,
                    void* scratch, void* stream) {
  if (take_injected_launch_failure()) return static_cast<int>(cudaErrorLaunchFailure);
  if (quantize_d128_applies(ctx, n_rows, x_is_bf16))
    return launch_quantize_d128(ctx, x, x_is_bf16, n_rows, ld_x, out, scratch, stream);
  if (scratch && wide_quantize_applies(ctx, n_rows))
    return launch_quantize_wide(ctx, x, x_is_bf16, n_rows, ld_x, out, scratch, stream);
  return launch_quantize_generic(ctx.kp, x, x_is_bf16, n_rows, ld_x, out, stream);
}

size_t logits_scratch_bytes(const tq_ctx& ctx, int64_t n_sets, int g, int64_t n_keys) {
  if (logits_d128_applies(ctx, n_sets, g, n_keys)) return 0;
  return wide_logits_applies(ctx, n_sets, g, n_keys) ? wide_logits_scratch_bytes(ctx, n_sets, g, n_keys) : 0;
}

int launch_logits(const tq_ctx& ctx, const float* qp, int64_t n_sets, int g, const Packed& keys, int64_t n_keys,
                  float* out, void* scratch, void* stream) {
  if (take_injected_launch_failure()) return static_cast<int>(cudaErrorLaunchFailure);
  if (logits_d128_applies(ctx, n_sets, g, n_keys))
    return launch_logits_d128(ctx, qp, n_sets, g, keys, n_keys, out, stream);
  if (scratch && wide_logits_applies(ctx, n_sets, g, n_keys))
    return launch_logits_wide(ctx, qp, n_sets, g, keys, n_keys, out, scratch, stream);
  return launch_logits_generic(ctx.kp, qp, n_sets, g, keys, n_keys, out, stream);
}

int launch_dequant(const tq_ctx& ctx, const Packed& in, int64_t n_rows, void* out, int out_is_bf16, int prod,
                   void* stream) {
  if (take_injected_launch_failure()) return static_cast<int>(cudaErrorLaunchFailure);
  if (dequant_d128_applies(ctx, n_rows, out_is_bf16))
    return launch_dequant_d128(ctx, in, n_rows, out, ctx.d, out_is_bf16, prod, stream);
  return launch_dequant_generic(ctx.kp, in, n_rows, out, out_is_bf16, prod, stream);
}

}  // namespace tq
