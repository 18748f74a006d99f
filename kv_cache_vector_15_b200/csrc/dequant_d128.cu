// Read half, value reconstruction at d = 128, m = 128 on sm_100a.
//
//   PROD: x~ = R^T (norm yhat + sqrt(pi/2)/m rnorm S^T z)   ai.spot.hk "Google
//         TurboQuant", "無偏內積估計" (unbiased inverse of the quantizer)
//   MSE:  x~ = R^T (norm yhat)                              Qiita TurboQuant
//         explainer, "APIの構成" (values through the MSE stage alone)
//   R^T = D H_d / sqrt(d)                                   0h-n0.github.io "ICLR
//         2026論文解説: TurboQuant", "Step 1: PolarQuant"
//
// One thread per row (two warpgroups of 128 rows, persistent CTAs).  S^T z is
// a 128 x 128 x 128 tensor-core product per tile: with z_j = 1 - 2 b_j,
// S^T z = colsum(S) - 2 S^T b, and the sign bits b go into TMEM as binary16
// values {0, 2^-14} (two shifts and a mask per pair of bits; S b is exact
// in the MMA, the 2^14 comes back out as an exact scaling).  The centroid
// decode, the inverse Walsh-Hadamard transform, D, 1/sqrt(d) and the output
// rounding run in registers; the finished tile is written back by a TMA
// tensor store from a swizzled shared-memory stage.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>

#include "sm100.cuh"
#include "tq_internal.h"

namespace tq {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

namespace {

using namespace sm100;

constexpr int kD = 128, kM = 128, kTile = 128, kPairs = 2, kThreads = kPairs * 256;
constexpr long long kWaitCycles = 2000000000ll;
constexpr uint32_t kTmemCols = 512;     // per pair: 128 D columns + 64 A columns (in 256)

struct DequantD128Args {
  float Dscale[kD];                     // D_i / sqrt(d)
  float colsum[kD];                     // sum_j S[j][i]
  int* err;
};

template <bool BF16OUT>
struct OutStage {
  static constexpr int kColsPerBox = BF16OUT ? 64 : 32;
  static constexpr int kBoxes = kD / kColsPerBox;
  static constexpr int kBytes = kBoxes * kTile * 128;     // 32 KB or 64 KB
};

template <bool BF16OUT>
constexpr size_t dequant_smem_bytes() {
  return 1024 + 32768 /*St*/ + kPairs * OutStage<BF16OUT>::kBytes + 128;
}

__device__ __forceinline__ void tma_store_2d(const void* tmap, const void* smem_src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(tmap), "r"(smem_u32(smem_src)), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Two warpgroups ("halves") share every 128-row tile: thread t of warp w in
// half h owns output coordinates [64 h, 64 h + 64) of row 32 (w % 4) + t (the
// row's TMEM lane).  Two such pairs run per CTA (512 threads).  The inverse
// rotation starts with its stride-64 butterfly (the stages of H commute),
// exchanged through the row's TMEM lane, then runs six stages in registers.
template <int B, bool PROD, bool BF16OUT>
__global__ void __launch_bounds__(kThreads, 1)
k_dequant_d128_tc(const __grid_constant__ CUtensorMap tmap_out, const KParams P, const DequantD128Args X,
                  const Packed in, int64_t n_rows) {
  constexpr int L = 1 << B;
  constexpr int kStage = OutStage<BF16OUT>::kBytes;
  constexpr int kH = kD / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sSt = smem;                                   // B operand: St (N = i, K = j), swizzled
  uint8_t* sOut = smem + 32768;                          // [pair] output stages
  uint64_t* mdone = reinterpret_cast<uint64_t*>(sOut + kPairs * kStage);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + kPairs);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* lut = reinterpret_cast<float*>(tmem_slot + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_tiles = (n_rows + kTile - 1) / kTile;
  if (tid == 0) {
    for (int i = 0; i < kPairs; ++i) mbar_init(&mdone[i], 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (tid < L) lut[tid] = P.c[tid];
  if (PROD) {
    // B operand row i (output coordinate), K position kappa holds S[j(kappa)][i]
    // in the order the sign bits are laid out in TMEM (see the A construction):
    // column c = kappa / 2 holds bits (c % 16) and (c % 16) + 16 of sign word
    // c / 16, so j(kappa) = 32 (c / 16) + (c % 16) + 16 (kappa % 2).
    uint16_t* sSt16 = reinterpret_cast<uint16_t*>(sSt);
    for (int e = tid; e < kD * kM; e += kThreads) {
      const int i = e >> 7, kappa = e & 127;
      const int c = kappa >> 1, j = 32 * (c >> 4) + (c & 15) + 16 * (kappa & 1);
      const int kb = kappa >> 6, chunk = (kappa & 63) >> 3, within = kappa & 7;
      sSt16[(kb * 16384 + i * 128 + ((chunk ^ (i & 7)) << 4)) / 2 + within] = P.St[i * kM + j];
    }
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int wgi = warp >> 2, pair = wgi >> 1, half = wgi & 1, lb = warp & 3;
  const bool leader = (half == 0 && lb == 0 && lane == 0);
  const int trow = lb * 32 + lane;
  const uint32_t lane_base = static_cast<uint32_t>(lb * 32) << 16;
  const uint32_t t_acc = tmem + lane_base + pair * 256;   // S^T b (128 columns), then the exchange
  const uint32_t t_a = t_acc + 128;                       // sign bits as binary16 (64 columns)
  const uint32_t bar_id = 1 + pair;
  uint8_t* stage = sOut + pair * kStage;
  const float inv_sqrt_d = 0.08838834764831845f;
  const float qjl = P.qjl_scale;
  const int64_t t_first = blockIdx.x + static_cast<int64_t>(pair) * gridDim.x;
  const int64_t t_step = static_cast<int64_t>(kPairs) * gridDim.x;
  bool store_pending = false;
  int mine = 0;
  // my part of the packed row for the next tile, loaded one tile ahead: codes
  // of my 64 coordinates, the two sign words whose A columns I write, norms
  uint32_t ncw[B * 2], nsg0 = 0u, nsg1 = 0u;
  float nnrm = 0.f, nrn = 0.f;
  auto load_packed = [&](int64_t tile) {
    const int64_t row = tile * kTile + trow;
    if (tile < n_tiles && row < n_rows) {
      const uint8_t* cp = in.codes + row * (B * 16) + half * (B * 8);
      if constexpr (B == 1) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(cp));
        ncw[0] = u.x; ncw[1] = u.y;
      } else if constexpr (B == 2) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(cp));
        ncw[0] = u.x; ncw[1] = u.y; ncw[2] = u.z; ncw[3] = u.w;
      } else if constexpr (B == 3) {
        if (half == 0) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(cp));
          const uint2 w = __ldg(reinterpret_cast<const uint2*>(cp + 16));
          ncw[0] = u.x; ncw[1] = u.y; ncw[2] = u.z; ncw[3] = u.w; ncw[4] = w.x; ncw[5] = w.y;
        } else {
          const uint2 w = __ldg(reinterpret_cast<const uint2*>(cp));
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(cp + 8));
          ncw[0] = w.x; ncw[1] = w.y; ncw[2] = u.x; ncw[3] = u.y; ncw[4] = u.z; ncw[5] = u.w;
        }
      } else {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(cp));
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(cp + 16));
        ncw[0] = u.x; ncw[1] = u.y; ncw[2] = u.z; ncw[3] = u.w;
        ncw[4] = w.x; ncw[5] = w.y; ncw[6] = w.z; ncw[7] = w.w;
      }
      if (PROD) {
        const uint2 sg = __ldg(reinterpret_cast<const uint2*>(in.signs + row * 16 + half * 8));
        nsg0 = sg.x; nsg1 = sg.y;
      }
      nnrm = __ldg(in.norm + row);
      nrn = __ldg(in.rnorm + row);
    } else {
#pragma unroll
      for (int w = 0; w < B * 2; ++w) ncw[w] = 0u;
      nsg0 = nsg1 = 0u;
      nnrm = 0.f;
      nrn = 0.f;
    }
  };
  load_packed(t_first);
  for (int64_t t = t_first; t < n_tiles; t += t_step, ++mine) {
    uint32_t cw[B * 2];
#pragma unroll
    for (int w = 0; w < B * 2; ++w) cw[w] = ncw[w];
    const uint32_t sg0 = nsg0, sg1 = nsg1;
    const float nrm = nnrm, rn = nrn;
    load_packed(t + t_step);
    if (PROD) {
      // sign bits -> binary16 {0, 2^-14}: column k of sign word w holds bits
      // (k, k + 16) of the word, i.e. projections 32 w + k and 32 w + k + 16;
      // half h writes the columns of sign words 2h and 2h + 1
      uint32_t a[32];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const uint32_t sgw = q == 0 ? sg0 : sg1;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const uint32_t sh = (k <= 10) ? (sgw << (10 - k)) : (sgw >> (k - 10));
          a[q * 16 + k] = sh & 0x04000400u;
        }
      }
      tmem_st32(t_a + half * 32, a);
      tmem_wait_st();
      tc_fence_before();
      if (named_bar_sync_or(bar_id, 256, *reinterpret_cast<volatile int*>(abort_flag) != 0)) break;
      if (leader) {
        tc_fence_after();
        const uint32_t sbase = smem_u32(sSt);
        const uint32_t idesc = idesc_f16_f32(kTile, kD);
        const uint32_t d_tmem = tmem + pair * 256;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t bdesc = smem_desc_sw128(sbase + (k >> 2) * 16384 + (k & 3) * 32, 1024);
          mma_f16_ts(d_tmem, d_tmem + 128 + k * 8, bdesc, idesc, k > 0 ? 1u : 0u);
        }
        mma_commit(&mdone[pair]);
      }
    }
    // ---- norm * yhat of my coordinates while the MMA runs -------------------------
    float v[kH];
#pragma unroll
    for (int e = 0; e < kH; ++e) {
      const int bit = B * e, wi = bit >> 5, sh = bit & 31;
      uint32_t code = cw[wi] >> sh;
      if (sh + B > 32) code |= cw[wi + 1] << (32 - sh);
      code &= (1u << B) - 1u;
      v[e] = nrm * lut[code];
    }
    if (PROD) {
      if (!mbar_wait(&mdone[pair], mine & 1, kWaitCycles)) {
        if (X.err) atomicCAS(X.err, 0, 5);
        atomicExch(abort_flag, 1);
      }
      tc_fence_after();
      // sum_j z_j S[j][i] = colsum_i - 2 * 2^14 * acc_i
      const float w = qjl * rn;
      const float w2 = -2.0f * 16384.0f * w;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t acc[16];
        tmem_ld16(t_acc + half * 64 + c * 16, acc);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int e = c * 16 + k;
          v[e] = fmaf(w2, __uint_as_float(acc[k]), fmaf(w, X.colsum[half * kH + e], v[e]));
        }
      }
    }
    // ---- stride-64 butterfly across the halves through the TMEM lane ----------------
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t w16[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) w16[k] = __float_as_uint(v[c * 16 + k]);
      tmem_st16(t_acc + half * 64 + c * 16, w16);
    }
    tmem_wait_st();
    tc_fence_before();
    named_bar_sync(bar_id, 256);
    tc_fence_after();
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t w16[16];
      tmem_ld16(t_acc + (half ^ 1) * 64 + c * 16, w16);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float o = __uint_as_float(w16[k]);
        v[c * 16 + k] = half == 0 ? v[c * 16 + k] + o : o - v[c * 16 + k];
      }
    }
    tc_fence_before();
    // ---- six in-register stages --------------------------------------------------------
#pragma unroll
    for (int h = 2; h < kH; h <<= 1) {
#pragma unroll
      for (int e = 0; e < kH; e += 2) {
        if ((e & h) == 0) {
          const float2 a = make_float2(v[e], v[e + 1]), b = make_float2(v[e + h], v[e + h + 1]);
          const float2 sum = __fadd2_rn(a, b);
          const float2 dif = __ffma2_rn(b, make_float2(-1.f, -1.f), a);
          v[e] = sum.x; v[e + 1] = sum.y; v[e + h] = dif.x; v[e + h + 1] = dif.y;
        }
      }
    }
#pragma unroll
    for (int e = 0; e < kH; e += 2) {
      const float a = v[e], b = v[e + 1];
      v[e] = a + b;
      v[e + 1] = a - b;
    }
    // ---- stage my half row (swizzled for the TMA store) and write the tile -----------
    if (leader && store_pending) bulk_wait_read0();         // previous tile's store has read the stage
    named_bar_sync(bar_id, 256);
    if (BF16OUT) {
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {                      // box `half`: my 64 columns
        uint32_t wv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = cc * 8 + 2 * u;
          const __nv_bfloat162 p = __floats2bfloat162_rn(v[e] * X.Dscale[half * kH + e],
                                                         v[e + 1] * X.Dscale[half * kH + e + 1]);
          wv[u] = *reinterpret_cast<const uint32_t*>(&p);
        }
        *reinterpret_cast<uint4*>(stage + half * (kTile * 128) + trow * 128 + ((cc ^ (trow & 7)) << 4)) =
            make_uint4(wv[0], wv[1], wv[2], wv[3]);
      }
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c) {                        // boxes 2 half, 2 half + 1
        const int e = c * 4;
        float4 o;
        o.x = v[e + 0] * X.Dscale[half * kH + e + 0];
        o.y = v[e + 1] * X.Dscale[half * kH + e + 1];
        o.z = v[e + 2] * X.Dscale[half * kH + e + 2];
        o.w = v[e + 3] * X.Dscale[half * kH + e + 3];
        const int bx = 2 * half + (c >> 3), cc = c & 7;
        *reinterpret_cast<float4*>(stage + bx * (kTile * 128) + trow * 128 + ((cc ^ (trow & 7)) << 4)) = o;
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(bar_id, 256);
    if (leader) {
#pragma unroll
      for (int bx = 0; bx < OutStage<BF16OUT>::kBoxes; ++bx)
        tma_store_2d(&tmap_out, stage + bx * (kTile * 128), bx * OutStage<BF16OUT>::kColsPerBox,
                     static_cast<int>(t * kTile));
      bulk_commit();
      store_pending = true;
    }
  }
  if (leader && store_pending) bulk_wait0();               // all our stores have landed
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int B, bool PROD, bool BF16OUT>
int launch(const tq_ctx& ctx, const Packed& in, int64_t n_rows, void* out, cudaStream_t s) {
  const KParams& P = ctx.kp;
  auto encode = tensor_map_encoder();
  if (!encode) return static_cast<int>(cudaErrorNotSupported);
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(n_rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD) * (BF16OUT ? 2 : 4)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(OutStage<BF16OUT>::kColsPerBox), static_cast<cuuint32_t>(kTile)};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&tmap, BF16OUT ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, out, dims,
             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return static_cast<int>(cudaErrorInvalidValue);
  DequantD128Args X;
  for (int i = 0; i < kD; ++i) {
    X.Dscale[i] = static_cast<float>(ctx.D[i] / std::sqrt(128.0));
    X.colsum[i] = ctx.colsum_d128[i];
  }
  X.err = P.err;
  const size_t smem = dequant_smem_bytes<BF16OUT>();
  cudaError_t e = cudaFuncSetAttribute(k_dequant_d128_tc<B, PROD, BF16OUT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return static_cast<int>(e);
  const int64_t n_tiles = (n_rows + kTile - 1) / kTile;
  const int grid = static_cast<int>(n_tiles < ctx.num_sms ? n_tiles : ctx.num_sms);
  k_dequant_d128_tc<B, PROD, BF16OUT><<<grid, kThreads, smem, s>>>(tmap, P, X, in, n_rows);
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

template <int B>
int launch_B(const tq_ctx& ctx, const Packed& in, int64_t n_rows, void* out, int bf16, int prod, cudaStream_t s) {
  if (prod) return bf16 ? launch<B, true, true>(ctx, in, n_rows, out, s) : launch<B, true, false>(ctx, in, n_rows, out, s);
  return bf16 ? launch<B, false, true>(ctx, in, n_rows, out, s) : launch<B, false, false>(ctx, in, n_rows, out, s);
}

}  // namespace

bool dequant_d128_applies(const tq_ctx& ctx, int64_t n_rows) {
  const KParams& P = ctx.kp;
  return P.d == kD && P.m == kM && P.B >= 1 && P.B <= 4 && n_rows > 0 && n_rows < (int64_t(1) << 31) &&
         ctx.use_tc && tensor_map_encoder() != nullptr;
}

int launch_dequant_d128(const tq_ctx& ctx, const Packed& in, int64_t n_rows, void* out, int out_is_bf16, int prod,
                        void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (ctx.kp.B) {
    case 1: return launch_B<1>(ctx, in, n_rows, out, out_is_bf16, prod, s);
    case 2: return launch_B<2>(ctx, in, n_rows, out, out_is_bf16, prod, s);
    case 3: return launch_B<3>(ctx, in, n_rows, out, out_is_bf16, prod, s);
    default: return launch_B<4>(ctx, in, n_rows, out, out_is_bf16, prod, s);
  }
}

}  // namespace tq
