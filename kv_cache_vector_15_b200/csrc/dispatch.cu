// Kernel selection: the d = 128 hot-path kernels where they apply, then the
// wide-row tensor-core paths (d >= 256, many rows), the general kernels
// everywhere else.
#include "tq_internal.h"

namespace tq {

int launch_quantize(const tq_ctx& ctx, const void* x, int x_is_bf16, int64_t n_rows, int64_t ld_x, const Packed& out,
                    void* stream) {
  if (quantize_d128_applies(ctx, n_rows))
    return launch_quantize_d128(ctx, x, x_is_bf16, n_rows, ld_x, out, stream);
  if (wide_quantize_applies(ctx, n_rows)) return launch_quantize_wide(ctx, x, x_is_bf16, n_rows, ld_x, out, stream);
  return launch_quantize_generic(ctx.kp, x, x_is_bf16, n_rows, ld_x, out, stream);
}

int launch_logits(const tq_ctx& ctx, const float* qp, int64_t n_sets, int g, const Packed& keys, int64_t n_keys,
                  float* out, void* stream) {
  if (logits_d128_applies(ctx, n_sets, g, n_keys))
    return launch_logits_d128(ctx, qp, n_sets, g, keys, n_keys, out, stream);
  if (wide_logits_applies(ctx, n_sets, g, n_keys)) return launch_logits_wide(ctx, qp, n_sets, g, keys, n_keys, out, stream);
  return launch_logits_generic(ctx.kp, qp, n_sets, g, keys, n_keys, out, stream);
}

int launch_dequant(const tq_ctx& ctx, const Packed& in, int64_t n_rows, void* out, int out_is_bf16, int prod,
                   void* stream) {
  if (dequant_d128_applies(ctx, n_rows))
    return launch_dequant_d128(ctx, in, n_rows, out, out_is_bf16, prod, stream);
  return launch_dequant_generic(ctx.kp, in, n_rows, out, out_is_bf16, prod, stream);
}

}  // namespace tq
