// General CUDA-core kernels of libtq: every (d, b, m) the C ABI accepts.
//
// These are the reference-shaped kernels for all supported shapes:
//   k_quantize_warp  write half, one warp per row (norm, RHT, Lloyd-Max codes,
//                    residual, QJL projection and signs, packing)
//   k_qprep_warp     q_rot = R q and sq = S q_rot for each query
//   k_logits_rowkey  small query groups: one thread per key, all g queries
//   k_logits_tiled   large query groups: register-tiled (keys x queries) dot
//                    products over the combined d + m dimension
//   k_dequant_warp   PROD / MSE reconstruction, one warp per row
//   k_topk_row       per-row top-k, one CTA per row
//   k_logits_bf16    plain bf16-key logits (the comparison baseline)
// The d = 128 hot-path kernels live in kernels_d128.cu.
//
// Method references (page title, section):
//   rotation R = H_d D / sqrt(d): 0h-n0.github.io "ICLR 2026論文解説: TurboQuant",
//     "Step 1: PolarQuant"; butterfly FWHT: same page, "実装のポイント";
//   Lloyd-Max codes: Qiita TurboQuant explainer, "Stage 1: PolarQuant";
//   QJL signs and the logit estimator: Qiita explainer, "Stage 2: QJL";
//   (b-1)+1 bit split and unbiased dequantization: ai.spot.hk "Google
//     TurboQuant", "無偏內積估計".

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kWarps = 8;           // warps per CTA in the warp-per-row kernels
constexpr size_t kQprepStBytes = 64 * 1024;   // S^T staged in shared memory up to this size

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }

template <bool BF16>
__device__ __forceinline__ float load_elem(const void* base, int64_t idx) {
  if (BF16) {
    uint16_t u = __ldg(reinterpret_cast<const uint16_t*>(base) + idx);
    return __uint_as_float(static_cast<uint32_t>(u) << 16);
  } else {
    return __ldg(reinterpret_cast<const float*>(base) + idx);
  }
}

// Walsh-Hadamard butterflies over a warp-distributed vector: lane l holds
// elements l*E .. l*E+E-1.  Produces H_d v (Sylvester order), unnormalised.
template <int E>
__device__ __forceinline__ void warp_fwht(float (&v)[E], int lane, int d) {
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if ((e & h) == 0) {
        float a = v[e], b = v[e + h];
        v[e] = a + b;
        v[e + h] = a - b;
      }
    }
  }
  for (int h = E; h < d; h <<= 1) {
    const int lm = h / E;
    const bool upper = (lane & lm) != 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float p = __shfl_xor_sync(0xffffffffu, v[e], lm);
      v[e] = upper ? (p - v[e]) : (v[e] + p);
    }
  }
}

template <int E>
__device__ __forceinline__ void apply_D(float (&v)[E], const uint32_t* Dmask, int lane) {
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane * E + e;
    const uint32_t bit = (__ldg(Dmask + (i >> 5)) >> (i & 31)) & 1u;
    v[e] = bit ? -v[e] : v[e];
  }
}

// ---------------------------------------------------------------------------
// write half
// ---------------------------------------------------------------------------
// dest: when not null, input row i goes to packed row dest[i] (a paged cache);
// an index outside [0, n_dest) is not written and sets the error word (7).
// Each warp takes R rows at a time and projects them together, so that every
// S^T element read from L2 feeds R multiply-adds (R = 1 for a handful of rows,
// where latency matters more than L2 traffic).
template <int E, bool BF16, int R>
__global__ void __launch_bounds__(kWarps * 32)
k_quantize_warp(const KParams P, const void* __restrict__ x, int64_t n_rows, int64_t ld, const Packed out,
                const int64_t* __restrict__ dest, int64_t n_dest) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int d = P.d, m = P.m, B = P.B;
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  float* rs = reinterpret_cast<float*>(smem_raw) + static_cast<size_t>(wib) * R * d;        // [R][d] residuals
  uint8_t* cs = smem_raw + static_cast<size_t>(kWarps) * R * d * 4 + static_cast<size_t>(wib) * d;   // codes
  __shared__ float thr[kMaxLevels], lut[kMaxLevels];
  if (threadIdx.x < kMaxLevels) { thr[threadIdx.x] = P.t[threadIdx.x]; lut[threadIdx.x] = P.c[threadIdx.x]; }
  __syncthreads();

  const int nwords_codes = d * B / 32, nwords_signs = m / 32;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kWarps;
  for (int64_t row0 = static_cast<int64_t>(blockIdx.x) * kWarps + wib; row0 < n_rows; row0 += stride * R) {
    int64_t orows[R];
    bool live[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t row = row0 + r * stride;
      live[r] = false;
      orows[r] = row;
      if (row >= n_rows) continue;                             // warp-uniform
      int64_t orow = row;
      if (dest) {
        orow = __ldg(dest + row);
        if (orow < 0 || orow >= n_dest) {                      // warp-uniform: skip the row, flag it
          if (lane == 0 && P.err) atomicCAS(P.err, 0, 7);
          continue;
        }
      }
      orows[r] = orow;
      uint32_t* codes_out = reinterpret_cast<uint32_t*>(out.codes + orow * P.codes_bytes);
      uint32_t* signs_out = reinterpret_cast<uint32_t*>(out.signs + orow * P.signs_bytes);
      float v[E];
      if (P.d_in != d) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int col = lane * E + e;                        // zero padding beyond the caller's row
          v[e] = col < P.d_in ? load_elem<BF16>(x, row * ld + col) : 0.f;
        }
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = load_elem<BF16>(x, row * ld + lane * E + e);
      }
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) ss = fmaf(v[e], v[e], ss);
      ss = warp_sum(ss);
      const float n = sqrtf(ss);
      if (!(n >= kZeroNorm)) {                   // zero row (or a non-finite norm)
        for (int w = lane; w < nwords_codes; w += 32) codes_out[w] = 0u;
        for (int w = lane; w < nwords_signs; w += 32) signs_out[w] = 0u;
        if (lane == 0) { out.norm[orow] = 0.f; out.rnorm[orow] = 0.f; }
        continue;
      }
      apply_D<E>(v, P.Dmask, lane);
      warp_fwht<E>(v, lane, d);
      const float inv_n = 1.0f / n;
      float r2 = 0.f;
      float* rr = rs + r * d;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float y = (v[e] * inv_n) * P.inv_sqrt_d;
        int code = 0;
        for (int k = 0; k < P.L - 1; ++k) code += (y > thr[k]) ? 1 : 0;
        const float res = y - lut[code];
        rr[lane * E + e] = res;
        cs[lane * E + e] = static_cast<uint8_t>(code);
        r2 = fmaf(res, res, r2);
      }
      r2 = warp_sum(r2);
      __syncwarp();
      // codes: output word w holds stream bits [32w, 32w + 32)
      for (int w = lane; w < nwords_codes; w += 32) {
        uint32_t acc = 0;
        const int i0 = (32 * w) / B, i1 = (32 * w + 31) / B;
        for (int i = i0; i <= i1 && i < d; ++i) {
          const int sh = B * i - 32 * w;
          const uint32_t c = cs[i];
          acc |= sh >= 0 ? (c << sh) : (c >> (-sh));
        }
        codes_out[w] = acc;
      }
      if (lane == 0) { out.norm[orow] = n; out.rnorm[orow] = n * sqrtf(r2); }
      live[r] = true;
      __syncwarp();
    }
    // QJL: p_j = sum_i S[j][i] r_i, bit j = [p_j < 0]; lane handles j = 32 t + lane,
    // for the R rows at once (rows that are not live compute on stale data and
    // store nothing)
    for (int t = 0; t < nwords_signs; ++t) {
      const int j = 32 * t + lane;
      float p[R][2];
#pragma unroll
      for (int r = 0; r < R; ++r) p[r][0] = p[r][1] = 0.f;
#pragma unroll (R == 1 ? 16 : 4)
      for (int i = 0; i < d; i += 2) {
        const float s0 = half_bits_to_float(__ldg(P.St + static_cast<int64_t>(i) * m + j));
        const float s1 = half_bits_to_float(__ldg(P.St + static_cast<int64_t>(i + 1) * m + j));
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float2 rv = *reinterpret_cast<const float2*>(rs + r * d + i);
          p[r][0] = fmaf(s0, rv.x, p[r][0]);
          p[r][1] = fmaf(s1, rv.y, p[r][1]);
        }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint32_t bits = __ballot_sync(0xffffffffu, (p[r][0] + p[r][1]) < 0.f);
        if (live[r] && lane == 0)
          reinterpret_cast<uint32_t*>(out.signs + orows[r] * P.signs_bytes)[t] = bits;
      }
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// query prep: qp[row] = [R q (d floats) | S R q (m floats)]
// ---------------------------------------------------------------------------
template <int E, bool BF16>
__global__ void __launch_bounds__(kWarps * 32)
k_qprep_warp(const KParams P, const void* __restrict__ q, int64_t n_q, float* __restrict__ qp) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int d = P.d, m = P.m;
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  float* qs = reinterpret_cast<float*>(smem_raw) + wib * d;
  // S^T in shared memory when it is small (all warps of the CTA share it),
  // else read from L2
  const bool st_smem = static_cast<size_t>(d) * m * 2 <= kQprepStBytes;
  uint16_t* sst = reinterpret_cast<uint16_t*>(smem_raw + static_cast<size_t>(kWarps) * d * 4);
  if (st_smem) {
    const int n16 = d * m / 8;                                 // 16-byte pieces
    for (int e = threadIdx.x; e < n16; e += kWarps * 32)
      reinterpret_cast<uint4*>(sst)[e] = __ldg(reinterpret_cast<const uint4*>(P.St) + e);
    __syncthreads();
  }
  const uint16_t* st = st_smem ? sst : P.St;
  const bool padded = P.d_in != d;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * kWarps + wib; row < n_q;
       row += static_cast<int64_t>(gridDim.x) * kWarps) {
    float v[E];
    if (padded) {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int col = lane * E + e;                          // queries are zero-padded like keys
        v[e] = col < P.d_in ? load_elem<BF16>(q, row * P.ld_q + col) : 0.f;
      }
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = load_elem<BF16>(q, row * P.ld_q + lane * E + e);
    }
    apply_D<E>(v, P.Dmask, lane);
    warp_fwht<E>(v, lane, d);
    float* dst = qp + row * (d + m);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float y = v[e] * P.inv_sqrt_d;
      qs[lane * E + e] = y;
      dst[lane * E + e] = y;
    }
    __syncwarp();
    for (int j = lane; j < m; j += 32) {
      float a0 = 0.f, a1 = 0.f;
#pragma unroll 16
      for (int i = 0; i < d; i += 2) {
        a0 = fmaf(half_bits_to_float(st[static_cast<int64_t>(i) * m + j]), qs[i], a0);
        a1 = fmaf(half_bits_to_float(st[static_cast<int64_t>(i + 1) * m + j]), qs[i + 1], a1);
      }
      dst[d + j] = a0 + a1;
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// logits, small g: one thread per key, all g queries of its set
// ---------------------------------------------------------------------------
template <int B, int G>
__global__ void __launch_bounds__(256)
k_logits_rowkey(const KParams P, const float* __restrict__ qp, int64_t n_keys, const Packed keys,
                float* __restrict__ out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* qs = reinterpret_cast<float*>(smem_raw);        // [G][d + m]
  __shared__ float lut[kMaxLevels];
  const int d = P.d, m = P.m, dm = d + m;
  const int64_t set = blockIdx.y;
  for (int i = threadIdx.x; i < G * dm; i += blockDim.x) qs[i] = qp[(set * G) * dm + i];
  if (threadIdx.x < kMaxLevels) lut[threadIdx.x] = P.c[threadIdx.x];
  __syncthreads();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n_keys) return;
  const int64_t row = set * n_keys + t;
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(keys.codes + row * P.codes_bytes);
  const uint32_t* sw = reinterpret_cast<const uint32_t*>(keys.signs + row * P.signs_bytes);
  float am[G], aq[G];
#pragma unroll
  for (int g = 0; g < G; ++g) { am[g] = 0.f; aq[g] = 0.f; }
  constexpr uint32_t mask = (1u << B) - 1u;
  for (int c = 0; c < d / 32; ++c) {
    uint32_t w[B + 1];
#pragma unroll
    for (int b = 0; b < B; ++b) w[b] = __ldg(cw + c * B + b);
    w[B] = 0u;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int bit = B * i, wi = bit >> 5, sh = bit & 31;
      uint32_t code = w[wi] >> sh;
      if (sh + B > 32) code |= w[wi + 1] << (32 - sh);
      const float yv = lut[code & mask];
#pragma unroll
      for (int g = 0; g < G; ++g) am[g] = fmaf(qs[g * dm + c * 32 + i], yv, am[g]);
    }
  }
  for (int c = 0; c < m / 32; ++c) {
    const uint32_t s = __ldg(sw + c);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const bool neg = (s >> j) & 1u;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float v = qs[g * dm + d + c * 32 + j];
        aq[g] += neg ? -v : v;
      }
    }
  }
  const float nrm = keys.norm[row], rn = keys.rnorm[row] * P.qjl_scale;
#pragma unroll
  for (int g = 0; g < G; ++g) out[(set * G + g) * n_keys + t] = nrm * am[g] + rn * aq[g];
}

// ---------------------------------------------------------------------------
// logits, large g: 128 keys x 128 queries per CTA, 8 x 8 outputs per thread
// (register tiling: four shared-memory vector loads feed 64 FMAs).  The
// combined dimension d + m is walked in chunks of 16; each chunk of key
// values is decoded once per CTA into shared memory as norm*c[code] (MSE
// coordinates) or rnorm*sqrt(pi/2)/m*z (QJL coordinates).
// ---------------------------------------------------------------------------
constexpr int TK = 128, TQ = 128, KC = 16;

__global__ void __launch_bounds__(256)
k_logits_tiled(const KParams P, const float* __restrict__ qp, int g, int64_t n_keys, const Packed keys,
               float* __restrict__ out) {
  __shared__ __align__(16) float Ks[KC][TK];
  __shared__ __align__(16) float Qs[KC][TQ];
  __shared__ float lut[kMaxLevels];
  const int d = P.d, m = P.m, dm = d + m, B = P.B;
  const int64_t set = blockIdx.z;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * TK;
  const int q0 = blockIdx.y * TQ;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  if (tid < kMaxLevels) lut[tid] = P.c[tid];
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  // the key this thread decodes (8 coordinates of each chunk) and its scales
  const int dk = tid & (TK - 1), dc0 = (tid >> 7) * 8;
  const int64_t krow = set * n_keys + k0 + dk;
  const bool kvalid = (k0 + dk) < n_keys;
  float knorm = 0.f, krn = 0.f;
  if (kvalid) { knorm = keys.norm[krow]; krn = keys.rnorm[krow] * P.qjl_scale; }
  const uint8_t* cb = keys.codes + krow * P.codes_bytes;
  const uint8_t* sbp = keys.signs + krow * P.signs_bytes;
  // the query this thread stages (8 coordinates of each chunk)
  const int ql = tid & (TQ - 1);
  const bool qvalid = q0 + ql < g;
  const float* qrow = qp + (set * g + q0 + ql) * dm;
  __syncthreads();
  for (int kk = 0; kk < dm; kk += KC) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = kk + dc0 + u;
      float val = 0.f;
      if (kvalid) {
        if (c < d) {
          const int bit = B * c, by = bit >> 3, sh = bit & 7;
          uint32_t win = cb[by];
          if (sh + B > 8) win |= static_cast<uint32_t>(cb[by + 1]) << 8;
          val = knorm * lut[(win >> sh) & ((1u << B) - 1u)];
        } else {
          const int j = c - d;
          val = ((sbp[j >> 3] >> (j & 7)) & 1u) ? -krn : krn;
        }
      }
      Ks[dc0 + u][dk] = val;
    }
    if (qvalid) {
      const float4 a = *reinterpret_cast<const float4*>(qrow + kk + dc0);
      const float4 b = *reinterpret_cast<const float4*>(qrow + kk + dc0 + 4);
      Qs[dc0 + 0][ql] = a.x; Qs[dc0 + 1][ql] = a.y; Qs[dc0 + 2][ql] = a.z; Qs[dc0 + 3][ql] = a.w;
      Qs[dc0 + 4][ql] = b.x; Qs[dc0 + 5][ql] = b.y; Qs[dc0 + 6][ql] = b.z; Qs[dc0 + 7][ql] = b.w;
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) Qs[dc0 + u][ql] = 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < KC; ++c) {
      const float4 ka = *reinterpret_cast<const float4*>(&Ks[c][tx * 4]);
      const float4 kb = *reinterpret_cast<const float4*>(&Ks[c][64 + tx * 4]);
      const float4 qa = *reinterpret_cast<const float4*>(&Qs[c][ty * 4]);
      const float4 qb = *reinterpret_cast<const float4*>(&Qs[c][64 + ty * 4]);
      const float kv[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
      const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(kv[i], qv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int qi = q0 + (j < 4 ? ty * 4 + j : 64 + ty * 4 + (j - 4));
    if (qi >= g) continue;
    float* orow = out + (set * g + qi) * n_keys;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t kt = k0 + (i < 4 ? tx * 4 + i : 64 + tx * 4 + (i - 4));
      if (kt < n_keys) orow[kt] = acc[i][j];
    }
  }
}

// ---------------------------------------------------------------------------
// dequant: x~ = R^T (norm yhat [+ sqrt(pi/2)/m rnorm S^T z])
// ---------------------------------------------------------------------------
template <int E, bool BF16OUT>
__global__ void __launch_bounds__(kWarps * 32)
k_dequant_warp(const KParams P, const Packed in, int64_t n_rows, void* __restrict__ outv, int prod) {
  const int d = P.d, m = P.m, B = P.B;
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  __shared__ float lut[kMaxLevels];
  if (threadIdx.x < kMaxLevels) lut[threadIdx.x] = P.c[threadIdx.x];
  __syncthreads();
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * kWarps + wib; row < n_rows;
       row += static_cast<int64_t>(gridDim.x) * kWarps) {
    const uint8_t* cb = in.codes + row * P.codes_bytes;
    const uint32_t* sw = reinterpret_cast<const uint32_t*>(in.signs + row * P.signs_bytes);
    const float nrm = in.norm[row], rn = in.rnorm[row];
    float v[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int i = lane * E + e;
      const int bit = B * i, by = bit >> 3, sh = bit & 7;
      uint32_t win = cb[by];
      if (sh + B > 8) win |= static_cast<uint32_t>(cb[by + 1]) << 8;
      v[e] = nrm * lut[(win >> sh) & ((1u << B) - 1u)];
    }
    if (prod && rn != 0.f) {
      float acc[E];
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = 0.f;
      for (int c = 0; c < m / 32; ++c) {
        const uint32_t s = __ldg(sw + c);
        for (int jj = 0; jj < 32; ++jj) {
          const int j = c * 32 + jj;
          const bool neg = (s >> jj) & 1u;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float sv = half_bits_to_float(__ldg(P.S + static_cast<int64_t>(j) * d + lane * E + e));
            acc[e] += neg ? -sv : sv;
          }
        }
      }
      const float s = P.qjl_scale * rn;
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = fmaf(s, acc[e], v[e]);
    }
    warp_fwht<E>(v, lane, d);
    apply_D<E>(v, P.Dmask, lane);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float o = v[e] * P.inv_sqrt_d;
      const int col = lane * E + e;                          // the caller's coordinates only
      const int64_t idx = row * P.ld_out + col;
      if (col < P.d_in) {
        if (BF16OUT) reinterpret_cast<__nv_bfloat16*>(outv)[idx] = __float2bfloat16_rn(o);
        else reinterpret_cast<float*>(outv)[idx] = o;
      }
    }
  }
}

// out += in, elementwise (the two halves of a channel split's logits)
__global__ void __launch_bounds__(256) k_add_f32(float* __restrict__ out, const float* __restrict__ in, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] += in[i];
}

// ---------------------------------------------------------------------------
// top-k per row: larger first, equal values by lower index first
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

constexpr int kTopkThreads = 256;

__global__ void __launch_bounds__(kTopkThreads)
k_topk_row(const float* __restrict__ scores, int64_t cols, int k, int32_t* __restrict__ idx,
           float* __restrict__ val) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* cv = reinterpret_cast<float*>(smem_raw);                 // [threads][k]
  int* ci = reinterpret_cast<int*>(cv + kTopkThreads * k);        // [threads][k]
  __shared__ float wv[kTopkThreads / 32];
  __shared__ int wi[kTopkThreads / 32], wt[kTopkThreads / 32];
  __shared__ int win_thread;
  const int64_t row = blockIdx.x;
  const float* s = scores + row * cols;
  float* myv = cv + threadIdx.x * k;
  int* myi = ci + threadIdx.x * k;
  int cnt = 0;
  for (int64_t c = threadIdx.x; c < cols; c += kTopkThreads) {
    const float x = s[c];
    const int xi = static_cast<int>(c);
    if (cnt == k && !better(x, xi, myv[k - 1], myi[k - 1])) continue;
    int p = cnt < k ? cnt : k - 1;
    while (p > 0 && better(x, xi, myv[p - 1], myi[p - 1])) { myv[p] = myv[p - 1]; myi[p] = myi[p - 1]; --p; }
    myv[p] = x; myi[p] = xi;
    if (cnt < k) ++cnt;
  }
  int head = 0;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int r = 0; r < k; ++r) {
    float bv = head < cnt ? myv[head] : -INFINITY;
    int bi = head < cnt ? myi[head] : INT32_MAX;
    int bt = head < cnt ? static_cast<int>(threadIdx.x) : -1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      int ot = __shfl_xor_sync(0xffffffffu, bt, o);
      if (ot >= 0 && (bt < 0 || better(ov, oi, bv, bi))) { bv = ov; bi = oi; bt = ot; }
    }
    if (lane == 0) { wv[w] = bv; wi[w] = bi; wt[w] = bt; }
    __syncthreads();
    if (threadIdx.x == 0) {
      float xv = wv[0]; int xi = wi[0], xt = wt[0];
      for (int q = 1; q < kTopkThreads / 32; ++q)
        if (wt[q] >= 0 && (xt < 0 || better(wv[q], wi[q], xv, xi))) { xv = wv[q]; xi = wi[q]; xt = wt[q]; }
      idx[row * k + r] = xi;
      if (val) val[row * k + r] = xv;
      win_thread = xt;
    }
    __syncthreads();
    if (static_cast<int>(threadIdx.x) == win_thread) ++head;
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// bf16 unquantized-key logits (the comparison kernel).  L = d / 8 lanes share a
// key, each holding 8 of its coordinates; a warp covers 32 / L keys per step and
// kBfSteps steps per chunk.  Every lane prefetches its own 16-byte pieces of the
// next kBfStages - 1 chunks into shared memory with cp.async, so the bytes in
// flight cost no registers and no lane waits on another; the kBfSteps * G partial
// dot products of a chunk are then summed across the L lanes by transposing
// butterflies (each level halves the number of values a lane holds).
// ---------------------------------------------------------------------------
constexpr int kBfWarps = 8, kBfStages = 4, kBfSteps = 4;
constexpr int kBfSmem = kBfWarps * kBfStages * kBfSteps * 32 * 16;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// C values per lane, lane-mask level M.  Lanes with bit M set keep the upper half
// of their values and send the lower half, the others the reverse; once a lane holds
// one value the remaining levels are plain butterflies (recorded in plain).
template <int C, int M>
struct XposeSum {
  static __device__ __forceinline__ void run(float* a, int r, int& jbase, int& plain) {
    if constexpr (M > 0) {
      if constexpr (C > 1) {
        const bool hi = (r & M) != 0;
#pragma unroll
        for (int i = 0; i < C / 2; ++i) {
          const float keep = hi ? a[i + C / 2] : a[i];
          const float send = hi ? a[i] : a[i + C / 2];
          a[i] = keep + __shfl_xor_sync(0xffffffffu, send, M);
        }
        if (hi) jbase += C / 2;
        XposeSum<C / 2, M / 2>::run(a, r, jbase, plain);
      } else {
        a[0] += __shfl_xor_sync(0xffffffffu, a[0], M);
        plain |= M;
        XposeSum<1, M / 2>::run(a, r, jbase, plain);
      }
    }
  }
};

template <int L, int G>
__global__ void __launch_bounds__(kBfWarps * 32, 2)
k_logits_bf16(const uint16_t* __restrict__ q, const uint16_t* __restrict__ keys, int64_t n_sets, int64_t n_keys,
              int64_t per_warp, float* __restrict__ out) {
  constexpr int d = 8 * L, KPS = 32 / L, KW = kBfSteps * KPS;
  constexpr int V = kBfSteps * G, VP = V <= 4 ? 4 : V <= 8 ? 8 : V <= 16 ? 16 : 32;
  constexpr int kLeft = VP >= L ? VP / L : 1;       // values a lane holds after the sums
  extern __shared__ uint4 bf_sbuf[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, r = lane % L, ks = lane / L;
  // [warp][stage][step][lane]: each lane reads back only the pieces it copied itself
  const uint4* mine = bf_sbuf + warp * (kBfStages * kBfSteps * 32) + lane;
  const uint32_t mine_s = static_cast<uint32_t>(__cvta_generic_to_shared(mine));
  // the warp takes chunks [c0, c0 + n_mine) of the (set, key chunk) order; chunks do not
  // cross sets, the last chunk of a set may be ragged
  const int64_t cps = (n_keys + KW - 1) / KW, total = n_sets * cps;
  const int64_t c0 = (static_cast<int64_t>(blockIdx.x) * kBfWarps + warp) * per_warp;
  if (c0 >= total) return;                           // uniform over the warp
  const int n_mine = static_cast<int>(c0 + per_warp < total ? per_warp : total - c0);
  // copy cursor: key ikb of the current set, at row ip (set rows are contiguous, so the
  // row pointer runs on across a set boundary); compute cursor: key ckb of set cset
  const int64_t set0 = c0 / cps;
  int64_t ikb = (c0 - set0 * cps) * KW, ckb = ikb, cset = set0;
  const uint16_t* ip = keys + (set0 * n_keys + ikb) * d + r * 8;
  float* op = out + set0 * G * n_keys;

  auto issue = [&](int i, int stage) {
    if (i < n_mine) {
#pragma unroll
      for (int u = 0; u < kBfSteps; ++u) {
        const bool ok = ikb + u * KPS + ks < n_keys;   // else zero-fill, nothing read
        cp_async16(mine_s + (stage * kBfSteps + u) * 512, ip + (ok ? (u * KPS + ks) * d : 0), ok ? 16u : 0u);
      }
      if (ikb + KW >= n_keys) { ip += (n_keys - ikb) * d; ikb = 0; } else { ip += KW * d; ikb += KW; }
    }
    cp_async_commit();                               // one group per chunk slot, empty past the end
  };

#pragma unroll
  for (int i = 0; i < kBfStages - 1; ++i) issue(i, i);
  float2 q2[G][4];
  int64_t qset = -1;
  int stage = 0;
  for (int i = 0; i < n_mine; ++i) {
    issue(i + kBfStages - 1, stage == 0 ? kBfStages - 1 : stage - 1);
    cp_async_wait<kBfStages - 1>();                  // this lane's copies of chunk i have landed
    if (cset != qset) {
      qset = cset;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const uint4 qq = __ldg(reinterpret_cast<const uint4*>(q + (cset * G + g) * d + r * 8));
        const uint32_t w[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
        for (int h = 0; h < 4; ++h)
          q2[g][h] = make_float2(__uint_as_float(w[h] << 16), __uint_as_float(w[h] & 0xffff0000u));
      }
    }
    float a[VP];
#pragma unroll
    for (int u = 0; u < kBfSteps; ++u) {
      const uint4 kk = mine[(stage * kBfSteps + u) * 32];
      const uint32_t w[4] = {kk.x, kk.y, kk.z, kk.w};
      float2 kf[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) kf[h] = make_float2(__uint_as_float(w[h] << 16), __uint_as_float(w[h] & 0xffff0000u));
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float2 acc = __fmul2_rn(q2[g][0], kf[0]);
#pragma unroll
        for (int h = 1; h < 4; ++h) acc = __ffma2_rn(q2[g][h], kf[h], acc);
        a[u * G + g] = acc.x + acc.y;
      }
    }
#pragma unroll
    for (int j = V; j < VP; ++j) a[j] = 0.f;
    int jbase = 0, plain = 0;
    XposeSum<VP, L / 2>::run(a, r, jbase, plain);
    if ((r & plain) == 0) {
#pragma unroll
      for (int k = 0; k < kLeft; ++k) {
        const int j = jbase + k;                     // value j: step j / G, query j % G
        const int64_t t = ckb + (j / G) * KPS + ks;
        if (j < V && t < n_keys) op[(j % G) * n_keys + t] = a[k];
      }
    }
    if (ckb + KW >= n_keys) { ckb = 0; ++cset; op += G * n_keys; } else { ckb += KW; }
    stage = stage == kBfStages - 1 ? 0 : stage + 1;
  }
  cp_async_wait<0>();
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <typename F>
int set_smem(F* kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return 0;
  return static_cast<int>(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(bytes)));
}

int grid_rows(int64_t n_rows) {
  int64_t want = (n_rows + kWarps - 1) / kWarps;
  int64_t cap = static_cast<int64_t>(sm_count()) * 16;
  return static_cast<int>(want < cap ? want : cap);
}

template <int E, bool BF16, int R>
int launch_quantize_ER(const KParams& P, const void* x, int64_t n_rows, int64_t ld, const Packed& out,
                       cudaStream_t s, const int64_t* dest, int64_t n_dest) {
  const size_t smem = static_cast<size_t>(kWarps) * P.d * (4 * R + 1);
  const int g = grid_rows((n_rows + R - 1) / R);
  int err;
  if ((err = set_smem(k_quantize_warp<E, BF16, R>, smem))) return err;
  k_quantize_warp<E, BF16, R><<<g, kWarps * 32, smem, s>>>(P, x, n_rows, ld, out, dest, n_dest);
  return 0;
}

template <int E>
int launch_quantize_E(const KParams& P, const void* x, int bf16, int64_t n_rows, int64_t ld, const Packed& out,
                      cudaStream_t s, const int64_t* dest = nullptr, int64_t n_dest = 0) {
  // four rows per warp when there are many rows and their residuals fit
  const bool four = n_rows >= 65536 && P.d <= 1024;
  int err;
  if (bf16) err = four ? launch_quantize_ER<E, true, 4>(P, x, n_rows, ld, out, s, dest, n_dest)
                       : launch_quantize_ER<E, true, 1>(P, x, n_rows, ld, out, s, dest, n_dest);
  else err = four ? launch_quantize_ER<E, false, 4>(P, x, n_rows, ld, out, s, dest, n_dest)
                  : launch_quantize_ER<E, false, 1>(P, x, n_rows, ld, out, s, dest, n_dest);
  if (err) return err;
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

template <int E>
int launch_qprep_E(const KParams& P, const void* q, int bf16, int64_t n_q, float* qp, cudaStream_t s) {
  const size_t st_bytes = static_cast<size_t>(P.d) * P.m * 2;
  const size_t smem = static_cast<size_t>(kWarps) * P.d * 4 + (st_bytes <= kQprepStBytes ? st_bytes : 0);
  int g = grid_rows(n_q);
  int err;
  if (bf16) {
    if ((err = set_smem(k_qprep_warp<E, true>, smem))) return err;
    k_qprep_warp<E, true><<<g, kWarps * 32, smem, s>>>(P, q, n_q, qp);
  } else {
    if ((err = set_smem(k_qprep_warp<E, false>, smem))) return err;
    k_qprep_warp<E, false><<<g, kWarps * 32, smem, s>>>(P, q, n_q, qp);
  }
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

template <int E>
int launch_dequant_E(const KParams& P, const Packed& in, int64_t n_rows, void* out, int bf16, int prod,
                     cudaStream_t s) {
  int g = grid_rows(n_rows);
  if (bf16) k_dequant_warp<E, true><<<g, kWarps * 32, 0, s>>>(P, in, n_rows, out, prod);
  else k_dequant_warp<E, false><<<g, kWarps * 32, 0, s>>>(P, in, n_rows, out, prod);
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

template <int B, int G>
int launch_rowkey(const KParams& P, const float* qp, int64_t n_sets, int64_t n_keys, const Packed& keys, float* out,
                  cudaStream_t s) {
  const size_t smem = static_cast<size_t>(G) * (P.d + P.m) * 4;
  int err;
  if ((err = set_smem(k_logits_rowkey<B, G>, smem))) return err;
  for (int64_t s0 = 0; s0 < n_sets; s0 += 65535) {
    const int64_t ns = n_sets - s0 < 65535 ? n_sets - s0 : 65535;
    dim3 grid(static_cast<unsigned>((n_keys + 255) / 256), static_cast<unsigned>(ns));
    const Packed kk{keys.codes + s0 * n_keys * P.codes_bytes, keys.signs + s0 * n_keys * P.signs_bytes,
                    keys.norm + s0 * n_keys, keys.rnorm + s0 * n_keys};
    k_logits_rowkey<B, G><<<grid, 256, smem, s>>>(P, qp + s0 * G * (P.d + P.m), n_keys, kk, out + s0 * G * n_keys);
    count_launch();
  }
  return static_cast<int>(cudaGetLastError());
}

template <int B>
int launch_rowkey_B(const KParams& P, const float* qp, int64_t n_sets, int g, int64_t n_keys, const Packed& keys,
                    float* out, cudaStream_t s) {
  switch (g) {
    case 1: return launch_rowkey<B, 1>(P, qp, n_sets, n_keys, keys, out, s);
    case 2: return launch_rowkey<B, 2>(P, qp, n_sets, n_keys, keys, out, s);
    case 3: return launch_rowkey<B, 3>(P, qp, n_sets, n_keys, keys, out, s);
    case 4: return launch_rowkey<B, 4>(P, qp, n_sets, n_keys, keys, out, s);
    case 5: return launch_rowkey<B, 5>(P, qp, n_sets, n_keys, keys, out, s);
    case 6: return launch_rowkey<B, 6>(P, qp, n_sets, n_keys, keys, out, s);
    case 7: return launch_rowkey<B, 7>(P, qp, n_sets, n_keys, keys, out, s);
    default: return launch_rowkey<B, 8>(P, qp, n_sets, n_keys, keys, out, s);
  }
}

template <int L, int G>
int launch_bf16_LG(const void* q, const void* keys, int64_t n_sets, int64_t n_keys, float* out, cudaStream_t s) {
  constexpr int64_t KW = kBfSteps * (32 / L);
  const int64_t total = n_sets * ((n_keys + KW - 1) / KW);
  int64_t warps = static_cast<int64_t>(sm_count()) * 2 * kBfWarps;
  if (warps > total) warps = total;
  const int64_t per_warp = (total + warps - 1) / warps;
  const int64_t blocks = ((total + per_warp - 1) / per_warp + kBfWarps - 1) / kBfWarps;
  int err = set_smem(k_logits_bf16<L, G>, kBfSmem);
  if (err) return err;
  k_logits_bf16<L, G><<<static_cast<unsigned>(blocks), kBfWarps * 32, kBfSmem, s>>>(
      static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(keys), n_sets, n_keys, per_warp, out);
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

template <int L>
int launch_bf16_L(const void* q, const void* keys, int64_t n_sets, int g, int64_t n_keys, float* out,
                  cudaStream_t s) {
  switch (g) {
    case 1: return launch_bf16_LG<L, 1>(q, keys, n_sets, n_keys, out, s);
    case 2: return launch_bf16_LG<L, 2>(q, keys, n_sets, n_keys, out, s);
    case 3: return launch_bf16_LG<L, 3>(q, keys, n_sets, n_keys, out, s);
    case 4: return launch_bf16_LG<L, 4>(q, keys, n_sets, n_keys, out, s);
    case 5: return launch_bf16_LG<L, 5>(q, keys, n_sets, n_keys, out, s);
    case 6: return launch_bf16_LG<L, 6>(q, keys, n_sets, n_keys, out, s);
    case 7: return launch_bf16_LG<L, 7>(q, keys, n_sets, n_keys, out, s);
    default: return launch_bf16_LG<L, 8>(q, keys, n_sets, n_keys, out, s);
  }
}

}  // namespace

const char* cuda_error_string(int err) { return cudaGetErrorString(static_cast<cudaError_t>(err)); }

int launch_quantize_generic(const KParams& P, const void* x, int bf16, int64_t n_rows, int64_t ld,
                            const Packed& out, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
#define CALL(E) launch_quantize_E<E>(P, x, bf16, n_rows, ld, out, s)
  switch (P.d / 32) {
    case 1: return CALL(1);
    case 2: return CALL(2);
    case 4: return CALL(4);
    case 8: return CALL(8);
    case 16: return CALL(16);
    case 32: return CALL(32);
    case 64: return CALL(64);
    case 128: return CALL(128);
  }
#undef CALL
  return static_cast<int>(cudaErrorInvalidValue);
}

int launch_quantize_scatter(const KParams& P, const void* x, int bf16, int64_t n_rows, int64_t ld,
                            const int64_t* dest, int64_t n_dest, const Packed& out, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
#define CALL(E) launch_quantize_E<E>(P, x, bf16, n_rows, ld, out, s, dest, n_dest)
  switch (P.d / 32) {
    case 1: return CALL(1);
    case 2: return CALL(2);
    case 4: return CALL(4);
    case 8: return CALL(8);
    case 16: return CALL(16);
    case 32: return CALL(32);
    case 64: return CALL(64);
    case 128: return CALL(128);
  }
#undef CALL
  return static_cast<int>(cudaErrorInvalidValue);
}

int launch_qprep(const KParams& P, const void* q, int bf16, int64_t n_q, float* qp, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
#define CALL(E) launch_qprep_E<E>(P, q, bf16, n_q, qp, s)
  switch (P.d / 32) {
    case 1: return CALL(1);
    case 2: return CALL(2);
    case 4: return CALL(4);
    case 8: return CALL(8);
    case 16: return CALL(16);
    case 32: return CALL(32);
    case 64: return CALL(64);
    case 128: return CALL(128);
  }
#undef CALL
  return static_cast<int>(cudaErrorInvalidValue);
}

int launch_logits_generic(const KParams& P, const float* qp, int64_t n_sets, int g, const Packed& keys,
                          int64_t n_keys, float* out, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t rowkey_smem = static_cast<size_t>(g) * (P.d + P.m) * 4;
  if (g <= 8 && rowkey_smem <= 200 * 1024) {
    switch (P.B) {
      case 1: return launch_rowkey_B<1>(P, qp, n_sets, g, n_keys, keys, out, s);
      case 2: return launch_rowkey_B<2>(P, qp, n_sets, g, n_keys, keys, out, s);
      case 3: return launch_rowkey_B<3>(P, qp, n_sets, g, n_keys, keys, out, s);
      default: return launch_rowkey_B<4>(P, qp, n_sets, g, n_keys, keys, out, s);
    }
  }
  for (int64_t s0 = 0; s0 < n_sets; s0 += 65535) {
    const int64_t ns = n_sets - s0 < 65535 ? n_sets - s0 : 65535;
    dim3 grid(static_cast<unsigned>((n_keys + TK - 1) / TK), static_cast<unsigned>((g + TQ - 1) / TQ),
              static_cast<unsigned>(ns));
    const Packed kk{keys.codes + s0 * n_keys * P.codes_bytes, keys.signs + s0 * n_keys * P.signs_bytes,
                    keys.norm + s0 * n_keys, keys.rnorm + s0 * n_keys};
    k_logits_tiled<<<grid, 256, 0, s>>>(P, qp + s0 * g * (P.d + P.m), g, n_keys, kk, out + s0 * g * n_keys);
    count_launch();
  }
  return static_cast<int>(cudaGetLastError());
}

int launch_dequant_generic(const KParams& P, const Packed& in, int64_t n_rows, void* out, int bf16, int prod,
                           void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
#define CALL(E) launch_dequant_E<E>(P, in, n_rows, out, bf16, prod, s)
  switch (P.d / 32) {
    case 1: return CALL(1);
    case 2: return CALL(2);
    case 4: return CALL(4);
    case 8: return CALL(8);
    case 16: return CALL(16);
    case 32: return CALL(32);
    case 64: return CALL(64);
    case 128: return CALL(128);
  }
#undef CALL
  return static_cast<int>(cudaErrorInvalidValue);
}

int launch_topk(const float* scores, int64_t rows, int64_t cols, int k, int32_t* idx, float* val, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t smem = static_cast<size_t>(kTopkThreads) * k * 8;
  int err;
  if ((err = set_smem(k_topk_row, smem))) return err;
  for (int64_t r0 = 0; r0 < rows; r0 += 65535) {
    const int64_t nr = rows - r0 < 65535 ? rows - r0 : 65535;
    k_topk_row<<<static_cast<unsigned>(nr), kTopkThreads, smem, s>>>(scores + r0 * cols, cols, k, idx + r0 * k,
                                                                    val ? val + r0 * k : nullptr);
    count_launch();
  }
  return static_cast<int>(cudaGetLastError());
}

int launch_add(float* out, const float* in, int64_t n, void* stream) {
  if (n <= 0) return 0;
  const int64_t want = (n + 255) / 256, cap = static_cast<int64_t>(sm_count()) * 8;
  k_add_f32<<<static_cast<unsigned>(want < cap ? want : cap), 256, 0, static_cast<cudaStream_t>(stream)>>>(out, in, n);
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

int launch_logits_bf16(const void* q, const void* keys, int64_t n_sets, int g, int64_t n_keys, int d, float* out,
                       void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 64: return launch_bf16_L<8>(q, keys, n_sets, g, n_keys, out, s);
    case 128: return launch_bf16_L<16>(q, keys, n_sets, g, n_keys, out, s);
    case 256: return launch_bf16_L<32>(q, keys, n_sets, g, n_keys, out, s);
  }
  return static_cast<int>(cudaErrorInvalidValue);
}

}  // namespace tq
