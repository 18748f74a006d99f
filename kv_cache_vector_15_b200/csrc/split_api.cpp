// Fractional bit widths by a channel split: channels [0, d_hi) of every row
// form one TurboQuant instance with b_hi bits per coordinate, channels
// [d_hi, d) another with b_lo bits, so a row costs (d_hi b_hi + d_lo b_lo) / d
// bits per coordinate (2.5 bits at d = 128: 64 channels at 3 bits and 64 at 2;
// 3.5 bits: 64 at 4 and 64 at 3).  The pages report 2.5- and 3.5-bit results
// without the split rule (inlevel9 "TurboQuantのメモリ圧縮と半導体需要",
// section "TurboQuantが実際に行っていること": LongBench at 3.5 and 2.5 bits);
// this library's reading:
//   * two independent instances (own D, S and codebook for the part's
//     dimension, m = the part's dimension), seeds `seed` and `seed + 1`;
//   * inner products add over disjoint channel sets, so the estimate of
//     <q, k> is the sum of the two parts' estimates and stays unbiased;
//   * the caller chooses which channels get the higher width by ordering its
//     channels (for instance, channels with outliers first).
// Every step runs in the instances' own kernels; this file only aims them at
// the two column ranges (row strides) and adds the two logit halves.

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <new>
#include <string>

#include "tq_internal.h"

struct tq_split {
  tq_ctx* part[2];
  int d, d_hi;
};

namespace {

using namespace tq;

size_t r16(size_t v) { return (v + 15) & ~static_cast<size_t>(15); }

tq_status cuda_err(int err, const char* what) {
  return fail(TQ_ERR_CUDA, std::string(what) + ": " + cuda_error_string(err));
}

tq_status check_split(const tq_split* sp) {
  if (!sp || !sp->part[0] || !sp->part[1]) return fail(TQ_ERR_INVALID_ARG, "split context is NULL");
  return TQ_OK;
}

size_t esize(tq_dtype t) { return t == TQ_BF16 ? 2 : 4; }

}  // namespace

extern "C" {

tq_status tq_split_init(int d, int d_hi, int b_hi, int b_lo, uint64_t seed, tq_split** out) {
  if (!out) return fail(TQ_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  const int d_lo = d - d_hi;
  if (d_hi < 32 || d_lo < 32 || d_hi % 32 || d_lo % 32)
    return fail(TQ_ERR_INVALID_ARG, "d_hi and d - d_hi must be multiples of 32, each >= 32");
  tq_split* sp = new (std::nothrow) tq_split();
  if (!sp) return fail(TQ_ERR_NOMEM, "host allocation failed");
  sp->d = d;
  sp->d_hi = d_hi;
  tq_status st = tq_init(d_hi, b_hi, d_hi, seed, &sp->part[0]);
  if (st == TQ_OK) st = tq_init(d_lo, b_lo, d_lo, seed + 1, &sp->part[1]);
  if (st != TQ_OK) {
    tq_destroy(sp->part[0]);
    delete sp;
    return st;
  }
  *out = sp;
  return TQ_OK;
}

tq_status tq_split_destroy(tq_split* sp) {
  if (!sp) return TQ_OK;
  tq_status a = tq_destroy(sp->part[0]), b = tq_destroy(sp->part[1]);
  delete sp;
  return a != TQ_OK ? a : b;
}

tq_status tq_split_part(const tq_split* sp, int part, const tq_ctx** out) {
  tq_status st = check_split(sp);
  if (st != TQ_OK) return st;
  if (!out || part < 0 || part > 1) return fail(TQ_ERR_INVALID_ARG, "part must be 0 or 1 and out not NULL");
  *out = sp->part[part];
  return TQ_OK;
}

size_t tq_split_quantize_workspace_bytes(const tq_split* sp, int64_t n_rows) {
  if (!sp || n_rows <= 0) return 0;
  return std::max(tq_quantize_workspace_bytes(sp->part[0], n_rows), tq_quantize_workspace_bytes(sp->part[1], n_rows));
}

tq_status tq_split_quantize(const tq_split* sp, const void* x, tq_dtype x_dtype, int64_t n_rows, int64_t ld_x,
                            tq_packed out_hi, tq_packed out_lo, void* workspace, size_t workspace_bytes,
                            void* stream) {
  tq_status st = check_split(sp);
  if (st != TQ_OK) return st;
  if (x_dtype != TQ_BF16 && x_dtype != TQ_F32) return fail(TQ_ERR_INVALID_ARG, "x_dtype must be TQ_BF16 or TQ_F32");
  if (ld_x < sp->d) return fail(TQ_ERR_INVALID_ARG, "ld_x < d");
  if (n_rows < 0) return fail(TQ_ERR_INVALID_ARG, "n_rows < 0");
  for (int p = 0; p < 2; ++p)
    if ((st = check_ctx(sp->part[p])) != TQ_OK) return st;
  if (n_rows == 0) return TQ_OK;
  const size_t need = tq_split_quantize_workspace_bytes(sp, n_rows);
  if (need) {
    if (!workspace || workspace_bytes < need) return fail(TQ_ERR_INVALID_ARG, "workspace missing or too small");
    if (reinterpret_cast<uintptr_t>(workspace) & 15) return fail(TQ_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  }
  // the parts in turn on the caller's stream, each with the workspace its kernels need
  void* w[2];
  for (int p = 0; p < 2; ++p) w[p] = tq_quantize_workspace_bytes(sp->part[p], n_rows) ? workspace : nullptr;
  if ((st = quantize_checked(sp->part[0], x, x_dtype, n_rows, ld_x, out_hi, w[0], stream)) != TQ_OK) return st;
  const void* x_lo = x ? static_cast<const uint8_t*>(x) + static_cast<size_t>(sp->d_hi) * esize(x_dtype) : nullptr;
  return quantize_checked(sp->part[1], x_lo, x_dtype, n_rows, ld_x, out_lo, w[1], stream);
}

size_t tq_split_logits_workspace_bytes(const tq_split* sp, int64_t n_sets, int g, int64_t n_keys) {
  if (!sp || n_sets <= 0 || g <= 0 || n_keys <= 0) return 0;
  return r16(qprep_bytes(sp->part[0], n_sets * g)) + r16(qprep_bytes(sp->part[1], n_sets * g)) +
         r16(static_cast<size_t>(n_sets) * g * n_keys * sizeof(float));
}

tq_status tq_split_logits(const tq_split* sp, const void* q, tq_dtype q_dtype, int64_t n_sets, int g,
                          tq_packed keys_hi, tq_packed keys_lo, int64_t n_keys, float* out, void* workspace,
                          size_t workspace_bytes, void* stream) {
  tq_status st = check_split(sp);
  if (st != TQ_OK) return st;
  if (n_sets < 0 || n_keys < 0) return fail(TQ_ERR_INVALID_ARG, "n_sets and n_keys must be >= 0");
  if (g < 1 || g > 4096) return fail(TQ_ERR_INVALID_ARG, "g must be in [1, 4096]");
  if (q_dtype != TQ_BF16 && q_dtype != TQ_F32) return fail(TQ_ERR_INVALID_ARG, "q_dtype must be TQ_BF16 or TQ_F32");
  if (n_sets == 0 || n_keys == 0) return TQ_OK;
  if (!q || !out) return fail(TQ_ERR_INVALID_ARG, "q or out is NULL");
  if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(out) & 3))
    return fail(TQ_ERR_INVALID_ARG, "q must be 16-byte and out 4-byte aligned");
  for (const tq_packed* p : {&keys_hi, &keys_lo})
    if (!p->codes || !p->signs || !p->norm || !p->rnorm) return fail(TQ_ERR_INVALID_ARG, "a packed pointer is NULL");
  const size_t need = tq_split_logits_workspace_bytes(sp, n_sets, g, n_keys);
  if (!workspace || workspace_bytes < need) return fail(TQ_ERR_INVALID_ARG, "workspace missing or too small");
  if (reinterpret_cast<uintptr_t>(workspace) & 15) return fail(TQ_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  uint8_t* w = static_cast<uint8_t*>(workspace);
  float* qp[2];
  qp[0] = reinterpret_cast<float*>(w);
  qp[1] = reinterpret_cast<float*>(w + r16(qprep_bytes(sp->part[0], n_sets * g)));
  float* half = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(qp[1]) + r16(qprep_bytes(sp->part[1], n_sets * g)));
  const tq_packed* keys[2] = {&keys_hi, &keys_lo};
  const size_t off[2] = {0, static_cast<size_t>(sp->d_hi) * esize(q_dtype)};
  for (int p = 0; p < 2; ++p) {
    KParams P = sp->part[p]->kp;
    P.ld_q = sp->d;                                    // the part's columns of the caller's rows
    int err = launch_qprep(P, static_cast<const uint8_t*>(q) + off[p], q_dtype == TQ_BF16, n_sets * g, qp[p], stream);
    if (err) return cuda_err(err, "tq_split_logits query-prep launch");
    const Packed k{keys[p]->codes, keys[p]->signs, keys[p]->norm, keys[p]->rnorm};
    err = launch_logits(*sp->part[p], qp[p], n_sets, g, k, n_keys, p == 0 ? out : half, nullptr, stream);
    if (err) return cuda_err(err, "tq_split_logits launch");
  }
  int err = launch_add(out, half, n_sets * g * n_keys, stream);
  if (err) return cuda_err(err, "tq_split_logits sum launch");
  return TQ_OK;
}

tq_status tq_split_dequant(const tq_split* sp, tq_packed in_hi, tq_packed in_lo, int64_t n_rows, void* out,
                           tq_dtype out_dtype, tq_dequant_mode mode, void* stream) {
  tq_status st = check_split(sp);
  if (st != TQ_OK) return st;
  if (n_rows < 0) return fail(TQ_ERR_INVALID_ARG, "n_rows < 0");
  if (out_dtype != TQ_BF16 && out_dtype != TQ_F32) return fail(TQ_ERR_INVALID_ARG, "out_dtype must be TQ_BF16 or TQ_F32");
  if (mode != TQ_DEQUANT_PROD && mode != TQ_DEQUANT_MSE) return fail(TQ_ERR_INVALID_ARG, "unknown dequant mode");
  if (n_rows == 0) return TQ_OK;
  if (!out) return fail(TQ_ERR_INVALID_ARG, "out is NULL");
  if (reinterpret_cast<uintptr_t>(out) & (esize(out_dtype) - 1))
    return fail(TQ_ERR_INVALID_ARG, "out must be aligned to its element size");
  const tq_packed* in[2] = {&in_hi, &in_lo};
  for (int p = 0; p < 2; ++p) {
    if (!in[p]->codes || !in[p]->signs || !in[p]->norm || !in[p]->rnorm)
      return fail(TQ_ERR_INVALID_ARG, "a packed pointer is NULL");
    KParams P = sp->part[p]->kp;
    P.ld_out = sp->d;                                  // into the part's columns of [n_rows, d]
    const Packed pk{in[p]->codes, in[p]->signs, in[p]->norm, in[p]->rnorm};
    void* o = static_cast<uint8_t*>(out) + (p == 0 ? 0 : static_cast<size_t>(sp->d_hi) * esize(out_dtype));
    const bool bf16 = out_dtype == TQ_BF16, prod = mode == TQ_DEQUANT_PROD;
    // the tensor-core kernel stores through TMA: the part's columns start on a
    // 16-byte boundary and the row stride is a multiple of 16 bytes
    const size_t esz = esize(out_dtype);
    const bool tc = dequant_d128_applies(*sp->part[p], n_rows, bf16) &&
                    (reinterpret_cast<uintptr_t>(o) & 15) == 0 && (static_cast<size_t>(sp->d) * esz) % 16 == 0;
    const int err = tc ? launch_dequant_d128(*sp->part[p], pk, n_rows, o, sp->d, bf16, prod, stream)
                       : launch_dequant_generic(P, pk, n_rows, o, bf16, prod, stream);
    if (err) return cuda_err(err, "tq_split_dequant launch");
  }
  return TQ_OK;
}

}  // extern "C"
