// Decode attention straight from packed keys and values.
//
//   out[s][j] = sum_k softmax_k(scale * logit(q_sj, k_sk)) * dequant(v_sk)
//
// Attention scores come from the compressed keys (the logit estimator,
// tq_logits) and the values stay compressed: Qiita TurboQuant explainer,
// "APIの構成" (asymmetric_attention_scores on compressed keys, values kept by
// the MSE compressor).  Because dequantization is linear in what a packed row
// stores,
//   dequant(v) = R^T (norm yhat + sqrt(pi/2)/m rnorm S^T z)        (PROD)
// (ai.spot.hk "Google TurboQuant", "無偏內積估計"), the softmax-weighted sum of
// values is taken in the rotated domain and rotated back once per query:
//   out = R^T (a + sqrt(pi/2)/m S^T b),  a = sum_k w_k norm_k yhat_k,
//                                        b = sum_k w_k rnorm_k z_k,
// so no value row is ever reconstructed in memory.
//
// Kernels (after qprep + logits into the workspace):
//   k_attn_chunk128  d = m = 128, 2- and 3-bit codes: as below, with a pair of
//                    coordinates / projections per thread and packed FMAs;
//   k_attn_chunk     one CTA per (key chunk, set): the chunk's softmax maximum
//                    and normaliser per query, and its partial a, b (weights
//                    exp(scale (s - max_chunk))), one thread per coordinate /
//                    projection slot; the chunk's packed rows pass through
//                    shared memory 32 keys at a time
//   k_attn_finalize  one CTA per (set, query): combines the chunks (the usual
//                    rescaling by exp(max_chunk - max)), adds sqrt(pi/2)/m S^T b,
//                    rotates back (FWHT in shared memory, D, 1/sqrt(d))

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "tq_internal.h"

namespace tq {

namespace {

constexpr int kAttnThreads = 256;
constexpr int kAttnBatch = 32;            // keys staged in shared memory at a time
constexpr float kLog2e = 1.4426950408889634f;

// partial record per (set, query, chunk): [max (log2 units), normaliser, a (d), b (m)]
__host__ __device__ inline int64_t partial_floats(int d, int m) { return 2 + d + m; }

template <int G, int SLOTS>
__global__ void __launch_bounds__(kAttnThreads)
k_attn_chunk(const KParams P, const float* __restrict__ logits, const Packed values, int64_t n_keys, int chunk,
             float scale_log2, int prod, float* __restrict__ partial) {
  const int d = P.d, m = P.m, B = P.B;
  const int set = blockIdx.y, c = blockIdx.x, n_chunks = gridDim.x;
  const int64_t k0 = static_cast<int64_t>(c) * chunk;
  const int64_t k1 = k0 + chunk < n_keys ? k0 + chunk : n_keys;
  const int tid = threadIdx.x;
  const int cw32 = P.codes_bytes / 4, sw32 = P.signs_bytes / 4;   // words per packed row
  extern __shared__ __align__(16) uint32_t sm[];
  uint32_t* sCodes = sm;                                        // [batch][cw32 + 1]
  uint32_t* sSigns = sCodes + kAttnBatch * (cw32 + 1);          // [batch][sw32]
  constexpr int GP = (G + 3) / 4 * 4;                           // weights per key, padded for float4 loads
  float* sWn = reinterpret_cast<float*>(sSigns + kAttnBatch * sw32);     // [batch][GP] weight * norm
  float* sWr = sWn + kAttnBatch * GP;                           // [batch][GP] weight * rnorm
  float* sMax = sWr + kAttnBatch * GP;                          // [G]
  float* sRed = sMax + G;                                       // [kAttnThreads / 32][G]
  __shared__ float lut[kMaxLevels];
  if (tid < kMaxLevels) lut[tid] = P.c[tid];

  const float* lg = logits + static_cast<int64_t>(set) * G * n_keys;
  // ---- the chunk's maximum of scale * logit per query (log2 units) -------------
  float mx[G];
#pragma unroll
  for (int q = 0; q < G; ++q) mx[q] = -INFINITY;
  for (int64_t k = k0 + tid; k < k1; k += kAttnThreads)
#pragma unroll
    for (int q = 0; q < G; ++q) mx[q] = fmaxf(mx[q], lg[q * n_keys + k] * scale_log2);
#pragma unroll
  for (int q = 0; q < G; ++q) {
    float v = mx[q];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((tid & 31) == 0) sRed[(tid >> 5) * G + q] = v;
  }
  __syncthreads();
  if (tid < G) {
    float v = -INFINITY;
    for (int w = 0; w < kAttnThreads / 32; ++w) v = fmaxf(v, sRed[w * G + tid]);
    sMax[tid] = v;
  }
  __syncthreads();
  float cm[G];
#pragma unroll
  for (int q = 0; q < G; ++q) cm[q] = sMax[q];

  // ---- weighted sums: thread slot x = s * 256 + tid is coordinate x (x < d) or
  // projection x - d (PROD only) --------------------------------------------------
  float acc[SLOTS][G];
#pragma unroll
  for (int s = 0; s < SLOTS; ++s)
#pragma unroll
    for (int q = 0; q < G; ++q) acc[s][q] = 0.f;
  float lsum = 0.f;                                            // thread tid < batch*G: its (key, query)
  const int nx = d + (prod ? m : 0);
  const uint32_t mask = (1u << B) - 1u;
  for (int64_t kb = k0; kb < k1; kb += kAttnBatch) {
    const int nb = static_cast<int>(k1 - kb < kAttnBatch ? k1 - kb : kAttnBatch);
    __syncthreads();                                            // previous batch consumed
    const int64_t row0 = static_cast<int64_t>(set) * n_keys + kb;
    for (int e = tid; e < nb * cw32; e += kAttnThreads) {
      const int r = e / cw32, w = e - r * cw32;
      sCodes[r * (cw32 + 1) + w] = __ldg(reinterpret_cast<const uint32_t*>(values.codes) + (row0 + r) * cw32 + w);
    }
    for (int r = tid; r < nb; r += kAttnThreads) sCodes[r * (cw32 + 1) + cw32] = 0u;
    if (prod)
      for (int e = tid; e < nb * sw32; e += kAttnThreads) {
        const int r = e / sw32, w = e - r * sw32;
        sSigns[r * sw32 + w] = __ldg(reinterpret_cast<const uint32_t*>(values.signs) + (row0 + r) * sw32 + w);
      }
    for (int e = tid; e < nb * G; e += kAttnThreads) {        // (e == tid: one (key, query) per thread)
      const int r = e / G, q = e - r * G;
      const float w = exp2f(lg[q * n_keys + kb + r] * scale_log2 - cm[q]);
      sWn[r * GP + q] = w * __ldg(values.norm + row0 + r);
      sWr[r * GP + q] = w * __ldg(values.rnorm + row0 + r);
      lsum += w;
    }
    __syncthreads();
#pragma unroll
    for (int s = 0; s < SLOTS; ++s) {
      const int x = s * kAttnThreads + tid;
      if (x < d) {
        const int bit = B * x, wi = bit >> 5, sh = bit & 31;
        const bool one_word = (32 % B) == 0;                    // codes never straddle two words
#pragma unroll 8
        for (int r = 0; r < nb; ++r) {
          const uint32_t* cr = sCodes + r * (cw32 + 1);
          uint32_t code;
          if (one_word) code = (cr[wi] >> sh) & mask;
          else code = static_cast<uint32_t>(((static_cast<uint64_t>(cr[wi + 1]) << 32) | cr[wi]) >> sh) & mask;
          const float v = lut[code];
#pragma unroll
          for (int q4 = 0; q4 < GP; q4 += 4) {
            const float4 w = *reinterpret_cast<const float4*>(sWn + r * GP + q4);
            if (q4 + 0 < G) acc[s][q4 + 0] = fmaf(w.x, v, acc[s][q4 + 0]);
            if (q4 + 1 < G) acc[s][q4 + 1] = fmaf(w.y, v, acc[s][q4 + 1]);
            if (q4 + 2 < G) acc[s][q4 + 2] = fmaf(w.z, v, acc[s][q4 + 2]);
            if (q4 + 3 < G) acc[s][q4 + 3] = fmaf(w.w, v, acc[s][q4 + 3]);
          }
        }
      } else if (x < nx) {
        const int j = x - d;
#pragma unroll 8
        for (int r = 0; r < nb; ++r) {
          const uint32_t bitv = (sSigns[r * sw32 + (j >> 5)] >> (j & 31)) & 1u;
          const float z = bitv ? -1.f : 1.f;
#pragma unroll
          for (int q4 = 0; q4 < GP; q4 += 4) {
            const float4 w = *reinterpret_cast<const float4*>(sWr + r * GP + q4);
            if (q4 + 0 < G) acc[s][q4 + 0] = fmaf(w.x, z, acc[s][q4 + 0]);
            if (q4 + 1 < G) acc[s][q4 + 1] = fmaf(w.y, z, acc[s][q4 + 1]);
            if (q4 + 2 < G) acc[s][q4 + 2] = fmaf(w.z, z, acc[s][q4 + 2]);
            if (q4 + 3 < G) acc[s][q4 + 3] = fmaf(w.w, z, acc[s][q4 + 3]);
          }
        }
      }
    }
  }
  // ---- the chunk's normaliser per query and the partial record -----------------
  // thread tid accumulated (key tid / G, query tid % G) of every batch
  __syncthreads();
  float* sL = sRed;                                             // [kAttnThreads]
  sL[tid] = lsum;
  __syncthreads();
  float* rec = partial + ((static_cast<int64_t>(set) * G) * n_chunks + c) * partial_floats(d, m);
  const int64_t qstride = static_cast<int64_t>(n_chunks) * partial_floats(d, m);
  if (tid < G) {
    float l = 0.f;
    for (int t = tid; t < kAttnBatch * G && t < kAttnThreads; t += G) l += sL[t];
    rec[tid * qstride + 0] = cm[tid];
    rec[tid * qstride + 1] = l;
  }
#pragma unroll
  for (int s = 0; s < SLOTS; ++s) {
    const int x = s * kAttnThreads + tid;
    if (x < nx)
#pragma unroll
      for (int q = 0; q < G; ++q) rec[q * qstride + 2 + x] = acc[s][q];
  }
}

// The d = m = 128 form of the chunk kernel (code widths of 2 and 3 bits): a
// thread owns a pair of coordinates (threads 0..127) or of projections
// (128..255) for one half of each staged batch of keys, with every query's
// accumulators as packed fp32 pairs, so a key costs it one table lookup (both
// centroids of the pair from the pair's 2B code bits) or two sign bits, one
// weight load per four queries and G packed FMAs.  The two key halves are
// summed at the end; the record is that of the general kernel.
template <int B, int G>
__global__ void __launch_bounds__(kAttnThreads)
k_attn_chunk128(const KParams P, const float* __restrict__ logits, const Packed values, int64_t n_keys, int chunk,
                float scale_log2, int prod, float* __restrict__ partial) {
  constexpr int d = 128, m = 128;
  constexpr int cw32 = B * 4, sw32 = 4;                         // words per packed row
  constexpr int GP = (G + 3) / 4 * 4;
  constexpr int L = 1 << B;
  // keys per staged batch: 128 when the threads' (key, query) weight entries
  // keep one query per thread (G divides the thread count), else 32 G <= 256
  constexpr int KB = (kAttnThreads % G == 0 && G <= 4) ? 4 * kAttnBatch : kAttnBatch;
  constexpr int kCW = (KB * cw32 + kAttnThreads - 1) / kAttnThreads;   // code words staged per thread
  constexpr int kSP = (KB * sw32 + kAttnThreads - 1) / kAttnThreads;   // sign words staged per thread
  constexpr int kWP = (KB * G + kAttnThreads - 1) / kAttnThreads;      // weight entries per thread
  const int set = blockIdx.y, c = blockIdx.x, n_chunks = gridDim.x;
  const int64_t k0 = static_cast<int64_t>(c) * chunk;
  const int64_t k1 = k0 + chunk < n_keys ? k0 + chunk : n_keys;
  const int tid = threadIdx.x;
  __shared__ uint32_t sCodes[KB][cw32 + 1];                     // + a zero word for pairs that straddle words
  __shared__ uint32_t sSigns[KB][sw32];
  __shared__ __align__(16) float sWn[KB][GP];                   // weight * norm
  __shared__ __align__(16) float sWr[KB][GP];                   // weight * rnorm
  __shared__ float sMax[G];
  __shared__ float sRed[kAttnThreads];
  __shared__ float2 lut2[L * L];                                // (c[i mod L], c[i / L])
  __shared__ float2 sHalf[128][G];                              // the odd key half's sums
  for (int i = tid; i < L * L; i += kAttnThreads) lut2[i] = make_float2(P.c[i & (L - 1)], P.c[i >> B]);

  const float* lg = logits + static_cast<int64_t>(set) * G * n_keys;
  // ---- the chunk's maximum of scale * logit per query (log2 units) -------------
  float mx[G];
#pragma unroll
  for (int q = 0; q < G; ++q) mx[q] = -INFINITY;
  for (int64_t k = k0 + tid; k < k1; k += kAttnThreads)
#pragma unroll
    for (int q = 0; q < G; ++q) mx[q] = fmaxf(mx[q], lg[q * n_keys + k] * scale_log2);
#pragma unroll
  for (int q = 0; q < G; ++q) {
    float v = mx[q];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((tid & 31) == 0) sRed[(tid >> 5) * G + q] = v;
  }
  __syncthreads();
  if (tid < G) {
    float v = -INFINITY;
    for (int w = 0; w < kAttnThreads / 32; ++w) v = fmaxf(v, sRed[w * G + tid]);
    sMax[tid] = v;
  }
  __syncthreads();
  float cm[G];
#pragma unroll
  for (int q = 0; q < G; ++q) cm[q] = sMax[q];

  const int role = tid >> 7, pair = tid & 63, khalf = (tid >> 6) & 1;
  const bool active = role == 0 || prod;
  float2 acc[G];
#pragma unroll
  for (int q = 0; q < G; ++q) acc[q] = make_float2(0.f, 0.f);
  float lsum = 0.f;                                             // thread tid < batch*G: its (key, query)
  // my pair's bits: code bits 2 B pair .. + 2 B - 1, or sign bits 2 pair, 2 pair + 1
  const int cbit = 2 * B * pair, cw = cbit >> 5, csh = cbit & 31;
  const int sw = pair >> 4, ssh = (2 * pair) & 31;
  // staging of a batch: the next batch's words are loaded into registers while
  // the current one is summed, then stored once every thread is done with it
  struct Pref {
    uint32_t cw[kCW], sg[kSP];
    float lgv[kWP], nrm[kWP], rnm[kWP];
  };
  auto load_batch = [&](int64_t kb, int nb, Pref& p) {
    const int64_t row0 = static_cast<int64_t>(set) * n_keys + kb;
    const uint32_t* cwp = reinterpret_cast<const uint32_t*>(values.codes) + row0 * cw32;
#pragma unroll
    for (int i = 0; i < kCW; ++i) {
      const int e = tid + i * kAttnThreads;
      p.cw[i] = e < nb * cw32 ? __ldg(cwp + e) : 0u;
    }
#pragma unroll
    for (int i = 0; i < kSP; ++i) {
      const int e = tid + i * kAttnThreads;
      p.sg[i] = prod && e < nb * sw32 ? __ldg(reinterpret_cast<const uint32_t*>(values.signs) + row0 * sw32 + e) : 0u;
    }
#pragma unroll
    for (int i = 0; i < kWP; ++i) {                             // (key, query) entries e = tid + 256 i
      const int e = tid + i * kAttnThreads;
      if (e < nb * G) {
        const int r = e / G, q = e - r * G;
        p.lgv[i] = lg[q * n_keys + kb + r];
        p.nrm[i] = __ldg(values.norm + row0 + r);
        p.rnm[i] = __ldg(values.rnorm + row0 + r);
      }
    }
  };
  auto store_batch = [&](int nb, const Pref& p) {
#pragma unroll
    for (int i = 0; i < kCW; ++i) {
      const int e = tid + i * kAttnThreads;
      if (e < nb * cw32) sCodes[e / cw32][e % cw32] = p.cw[i];
    }
    if (tid < nb) sCodes[tid][cw32] = 0u;
#pragma unroll
    for (int i = 0; i < kSP; ++i) {
      const int e = tid + i * kAttnThreads;
      if (prod && e < nb * sw32) sSigns[e / sw32][e % sw32] = p.sg[i];
    }
    // every entry of a thread has the query tid % G (G divides 256 when kWP > 1)
    const int q = tid % G;
    float cq = cm[0];
#pragma unroll
    for (int qq = 1; qq < G; ++qq) cq = q == qq ? cm[qq] : cq;
#pragma unroll
    for (int i = 0; i < kWP; ++i) {
      const int e = tid + i * kAttnThreads;
      if (e < nb * G) {
        const int r = e / G;
        const float w = exp2f(p.lgv[i] * scale_log2 - cq);
        sWn[r][q] = w * p.nrm[i];
        sWr[r][q] = w * p.rnm[i];
        lsum += w;
      }
    }
  };
  Pref pf;
  int64_t kb = k0;
  int nb = static_cast<int>(k1 - kb < KB ? k1 - kb : KB);
  if (nb > 0) {
    load_batch(kb, nb, pf);
    store_batch(nb, pf);
  }
  for (; nb > 0;) {
    const int64_t kn = kb + KB;
    const int nbn = kn < k1 ? static_cast<int>(k1 - kn < KB ? k1 - kn : KB) : 0;
    if (nbn > 0) load_batch(kn, nbn, pf);
    __syncthreads();
    if (active) {
      if (role == 0) {
#pragma unroll 4
        for (int r = khalf; r < nb; r += 2) {
          uint32_t idx;
          if ((csh + 2 * B) <= 32) idx = sCodes[r][cw] >> csh;
          else idx = __funnelshift_r(sCodes[r][cw], sCodes[r][cw + 1], csh);
          const float2 c2 = lut2[idx & (L * L - 1)];
#pragma unroll
          for (int q4 = 0; q4 < GP; q4 += 4) {
            const float4 w = *reinterpret_cast<const float4*>(&sWn[r][q4]);
            if (q4 + 0 < G) acc[q4 + 0] = __ffma2_rn(make_float2(w.x, w.x), c2, acc[q4 + 0]);
            if (q4 + 1 < G) acc[q4 + 1] = __ffma2_rn(make_float2(w.y, w.y), c2, acc[q4 + 1]);
            if (q4 + 2 < G) acc[q4 + 2] = __ffma2_rn(make_float2(w.z, w.z), c2, acc[q4 + 2]);
            if (q4 + 3 < G) acc[q4 + 3] = __ffma2_rn(make_float2(w.w, w.w), c2, acc[q4 + 3]);
          }
        }
      } else {
#pragma unroll 4
        for (int r = khalf; r < nb; r += 2) {
          const uint32_t bits = sSigns[r][sw] >> ssh;           // z = 1 - 2 bit
          const float2 z2 = make_float2(__uint_as_float(0x3F800000u | (bits << 31)),
                                        __uint_as_float(0x3F800000u | ((bits & 2u) << 30)));
#pragma unroll
          for (int q4 = 0; q4 < GP; q4 += 4) {
            const float4 w = *reinterpret_cast<const float4*>(&sWr[r][q4]);
            if (q4 + 0 < G) acc[q4 + 0] = __ffma2_rn(make_float2(w.x, w.x), z2, acc[q4 + 0]);
            if (q4 + 1 < G) acc[q4 + 1] = __ffma2_rn(make_float2(w.y, w.y), z2, acc[q4 + 1]);
            if (q4 + 2 < G) acc[q4 + 2] = __ffma2_rn(make_float2(w.z, w.z), z2, acc[q4 + 2]);
            if (q4 + 3 < G) acc[q4 + 3] = __ffma2_rn(make_float2(w.w, w.w), z2, acc[q4 + 3]);
          }
        }
      }
    }
    __syncthreads();                                            // the batch is consumed
    if (nbn > 0) store_batch(nbn, pf);
    kb = kn;
    nb = nbn;
  }
  // ---- the two key halves, the chunk's normaliser per query, the partial record --------
  __syncthreads();
  if (khalf == 1) {
#pragma unroll
    for (int q = 0; q < G; ++q) sHalf[role * 64 + pair][q] = acc[q];
  }
  sRed[tid] = lsum;                                             // thread tid accumulated query tid % G
  __syncthreads();
  float* rec = partial + ((static_cast<int64_t>(set) * G) * n_chunks + c) * partial_floats(d, m);
  const int64_t qstride = static_cast<int64_t>(n_chunks) * partial_floats(d, m);
  if (tid < G) {
    float l = 0.f;
    for (int t = tid; t < kAttnThreads; t += G) l += sRed[t];
    rec[tid * qstride + 0] = cm[tid];
    rec[tid * qstride + 1] = l;
  }
  if (khalf == 0 && active) {
    const int x = role * d + 2 * pair;                          // coordinate, or d + projection
#pragma unroll
    for (int q = 0; q < G; ++q) {
      const float2 o = sHalf[role * 64 + pair][q];
      *reinterpret_cast<float2*>(rec + q * qstride + 2 + x) = make_float2(acc[q].x + o.x, acc[q].y + o.y);
    }
  }
}

__global__ void __launch_bounds__(kAttnThreads)
k_attn_finalize(const KParams P, const float* __restrict__ partial, int n_chunks, int prod, float* __restrict__ out) {
  const int d = P.d, m = P.m, tid = threadIdx.x;
  const int64_t rowq = blockIdx.x;                              // set * g + query
  const int64_t pf = partial_floats(d, m);
  const float* rec = partial + rowq * n_chunks * pf;
  extern __shared__ __align__(16) float fs[];
  float* sa = fs;                                               // [d]
  float* sb = fs + d;                                           // [m]
  __shared__ float sM, sLn;
  if (tid == 0) {
    float mx = -INFINITY;
    for (int c = 0; c < n_chunks; ++c) mx = fmaxf(mx, rec[c * pf]);
    float l = 0.f;
    for (int c = 0; c < n_chunks; ++c) l += rec[c * pf + 1] * exp2f(rec[c * pf] - mx);
    sM = mx;
    sLn = l;
  }
  __syncthreads();
  const float mx = sM, inv_l = 1.f / sLn;
  const int nx = d + (prod ? m : 0);
  for (int x = tid; x < nx; x += kAttnThreads) {
    float v = 0.f;
    for (int c = 0; c < n_chunks; ++c) v = fmaf(rec[c * pf + 2 + x], exp2f(rec[c * pf] - mx), v);
    v *= inv_l;
    if (x < d) sa[x] = v;
    else sb[x - d] = v;
  }
  __syncthreads();
  if (prod) {
    // a += sqrt(pi/2)/m S^T b   (S^T row i is contiguous in P.St)
    for (int i = tid; i < d; i += kAttnThreads) {
      const __half* st = reinterpret_cast<const __half*>(P.St) + static_cast<int64_t>(i) * m;
      float acc = 0.f;
      for (int j = 0; j < m; ++j) acc = fmaf(__half2float(st[j]), sb[j], acc);
      sa[i] = fmaf(P.qjl_scale, acc, sa[i]);
    }
    __syncthreads();
  }
  // R^T a = D (H a) / sqrt(d): Walsh-Hadamard butterflies in shared memory
  for (int h = 1; h < d; h <<= 1) {
    for (int p = tid; p < d / 2; p += kAttnThreads) {
      const int i = (p / h) * 2 * h + (p % h), j = i + h;
      const float u = sa[i], w = sa[j];
      sa[i] = u + w;
      sa[j] = u - w;
    }
    __syncthreads();
  }
  for (int i = tid; i < P.d_in; i += kAttnThreads) {         // the caller's coordinates only
    const bool neg = (P.Dmask[i >> 5] >> (i & 31)) & 1u;
    const float v = sa[i] * P.inv_sqrt_d;
    out[rowq * P.d_in + i] = neg ? -v : v;
  }
}

template <int G, int SLOTS>
int launch_chunk(const KParams& P, const float* logits, const Packed& values, int64_t n_sets, int64_t n_keys,
                 int chunk, int n_chunks, float scale_log2, int prod, float* partial, cudaStream_t s) {
  const int cw32 = P.codes_bytes / 4, sw32 = P.signs_bytes / 4;
  constexpr int GP = (G + 3) / 4 * 4;
  const size_t smem = (static_cast<size_t>(kAttnBatch) * (cw32 + 1) + kAttnBatch * sw32 + 2 * kAttnBatch * GP + G +
                       kAttnThreads) * 4;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_attn_chunk<G, SLOTS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return static_cast<int>(e);
  }
  dim3 grid(static_cast<unsigned>(n_chunks), static_cast<unsigned>(n_sets));
  k_attn_chunk<G, SLOTS><<<grid, kAttnThreads, smem, s>>>(P, logits, values, n_keys, chunk, scale_log2, prod, partial);
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

template <int G>
int launch_chunk_g(const KParams& P, const float* logits, const Packed& values, int64_t n_sets, int64_t n_keys,
                   int chunk, int n_chunks, float scale_log2, int prod, float* partial, cudaStream_t s) {
  if (P.d == 128 && P.m == 128 && (P.B == 2 || P.B == 3) && P.codes_bytes == P.B * 16 && P.signs_bytes == 16) {
    dim3 grid(static_cast<unsigned>(n_chunks), static_cast<unsigned>(n_sets));
    if (P.B == 2)
      k_attn_chunk128<2, G><<<grid, kAttnThreads, 0, s>>>(P, logits, values, n_keys, chunk, scale_log2, prod, partial);
    else
      k_attn_chunk128<3, G><<<grid, kAttnThreads, 0, s>>>(P, logits, values, n_keys, chunk, scale_log2, prod, partial);
    count_launch();
    return static_cast<int>(cudaGetLastError());
  }
  const int nx = P.d + (prod ? P.m : 0);
  const int slots = (nx + kAttnThreads - 1) / kAttnThreads;
  if (slots <= 1) return launch_chunk<G, 1>(P, logits, values, n_sets, n_keys, chunk, n_chunks, scale_log2, prod, partial, s);
  if (slots <= 2) return launch_chunk<G, 2>(P, logits, values, n_sets, n_keys, chunk, n_chunks, scale_log2, prod, partial, s);
  if (slots <= 4) return launch_chunk<G, 4>(P, logits, values, n_sets, n_keys, chunk, n_chunks, scale_log2, prod, partial, s);
  return launch_chunk<G, 8>(P, logits, values, n_sets, n_keys, chunk, n_chunks, scale_log2, prod, partial, s);
}

}  // namespace

int attention_chunk_keys() { return 2048; }

size_t attention_partial_bytes(const KParams& P, int64_t n_sets, int g, int64_t n_keys) {
  const int64_t n_chunks = (n_keys + attention_chunk_keys() - 1) / attention_chunk_keys();
  return static_cast<size_t>(n_sets) * g * n_chunks * partial_floats(P.d, P.m) * sizeof(float);
}

int launch_attention_tail(const KParams& P, const float* logits, const Packed& values, int64_t n_sets, int g,
                          int64_t n_keys, float scale, int prod, float* partial, float* out, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int chunk = attention_chunk_keys();
  const int n_chunks = static_cast<int>((n_keys + chunk - 1) / chunk);
  const float scale_log2 = scale * kLog2e;
  int err = 0;
  switch (g) {
    case 1: err = launch_chunk_g<1>(P, logits, values, n_sets, n_keys, chunk, n_chunks, scale_log2, prod, partial, s); break;
    case 2: err = launch_chunk_g<2>(P, logits, values, n_sets, n_keys, chunk, n_chunks, scale_log2, prod, partial, s); break;
    case 3: err = launch_chunk_g<3>(P, logits, values, n_sets, n_keys, chunk, n_chunks, scale_log2, prod, partial, s); break;
    case 4: err = launch_chunk_g<4>(P, logits, values, n_sets, n_keys, chunk, n_chunks, scale_log2, prod, partial, s); break;
    case 5: err = launch_chunk_g<5>(P, logits, values, n_sets, n_keys, chunk, n_chunks, scale_log2, prod, partial, s); break;
    case 6: err = launch_chunk_g<6>(P, logits, values, n_sets, n_keys, chunk, n_chunks, scale_log2, prod, partial, s); break;
    case 7: err = launch_chunk_g<7>(P, logits, values, n_sets, n_keys, chunk, n_chunks, scale_log2, prod, partial, s); break;
    default: err = launch_chunk_g<8>(P, logits, values, n_sets, n_keys, chunk, n_chunks, scale_log2, prod, partial, s); break;
  }
  if (err) return err;
  const size_t smem = static_cast<size_t>(P.d + P.m) * sizeof(float);
  k_attn_finalize<<<static_cast<unsigned>(n_sets * g), kAttnThreads, smem, s>>>(P, partial, n_chunks, prod, out);
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

}  // namespace tq
