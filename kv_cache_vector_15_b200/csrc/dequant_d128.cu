// Read half, value reconstruction at d = 128, m = 128 on sm_100a.
//
//   PROD: x~ = R^T (norm yhat + sqrt(pi/2)/m rnorm S^T z)   ai.spot.hk "Google
//         TurboQuant", "無偏內積估計" (unbiased inverse of the quantizer)
//   MSE:  x~ = R^T (norm yhat)                              Qiita TurboQuant
//         explainer, "APIの構成" (values through the MSE stage alone)
//   R^T = D H_d / sqrt(d)                                   0h-n0.github.io "ICLR
//         2026論文解説: TurboQuant", "Step 1: PolarQuant"
//
// Both products run on the tcgen05 tensor cores, one 128-row tile at a time:
//   1. S^T z (PROD): the sign bits go into TMEM as binary16 z_j 2^-14 (one
//      shift and one mask per pair of bits), B = S^T (binary16, exact), so the
//      fp32 sums are S^T z scaled by an exact 2^-14.
//   2. the inverse rotation: each thread forms v = yhat + sqrt(pi/2)/m
//      (rnorm / norm) S^T z for its 64 coordinates (unit-norm domain, x64),
//      splits it into binary16 hi + lo in TMEM, and one MMA with
//      B = [D H; D H] (exact +-1 entries, K = 256) gives D H v in fp32;
//      norm / sqrt(d) / 64 scales the result.
// The CUDA cores are left with the centroid decode, one FMA per coordinate,
// the split and the output rounding; the finished tile leaves through a
// swizzled shared-memory stage and a TMA tensor store.

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
constexpr uint32_t kTmemCols = 512;     // per pair: 128 D columns + 128 A columns
constexpr float kUnit = 64.0f;          // scale of the unit-norm domain the rotation runs in

struct DequantD128Args {
  uint32_t Dneg[kD / 32];               // bit i of word i / 32: D_i = -1
  int* err;
  long long wait_cycles;                // limit of the bounded waits in the tile loop (SM clocks)
};

template <bool BF16OUT>
struct OutStage {
  static constexpr int kColsPerBox = BF16OUT ? 64 : 32;
  static constexpr int kBoxes = kD / kColsPerBox;
  static constexpr int kBytes = kBoxes * kTile * 128;     // 32 KB or 64 KB
};

template <bool BF16OUT>
constexpr size_t dequant_smem_bytes() {
  return 1024 + 32768 /*St*/ + 32768 /*D H*/ + kPairs * OutStage<BF16OUT>::kBytes + 512;
}
template <int KD>
constexpr size_t dequant_ovl_smem_bytes() {
  return 1024 + 2 * (KD * KD * 2) /*S^T, D H*/ + kPairs * (kTile * KD * 2) /*sign operands*/ +
         kPairs * (kTile * KD * 2) /*output stages*/ + 512;
}

__device__ __forceinline__ void tma_store_2d(const void* tmap, const void* smem_src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(tmap), "r"(smem_u32(smem_src)), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Two warpgroups ("halves") share every 128-row tile: thread t of warp w in
// half h owns coordinates [64 h, 64 h + 64) of row 32 (w % 4) + t (the row's
// TMEM lane), on the way in (code decode, S^T z) and on the way out (the
// rotated output columns).  Two such pairs run per CTA (512 threads).
template <int B, bool PROD, bool BF16OUT>
__global__ void __launch_bounds__(kThreads, 1)
k_dequant_d128_tc(const __grid_constant__ CUtensorMap tmap_out, const KParams P, const DequantD128Args X,
                  const Packed in, int64_t n_rows) {
  constexpr int L = 1 << B;
  constexpr int kStage = OutStage<BF16OUT>::kBytes;
  constexpr int kH = kD / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sSt = smem;                                   // B of the S^T z product (N = i, K = j), swizzled
  uint8_t* sDH = smem + 32768;                           // B of the rotation (N = n, K = k), swizzled
  uint8_t* sOut = smem + 65536;                          // [pair] output stages
  uint64_t* m1 = reinterpret_cast<uint64_t*>(sOut + kPairs * kStage);   // [pair] S^T z done
  uint64_t* m2 = m1 + kPairs;                                            // [pair] rotation done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(m2 + kPairs);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* lut = reinterpret_cast<float*>(tmem_slot + 2);                 // L centroids x kUnit
  float2* lut2 = reinterpret_cast<float2*>(lut + 16);                   // 2-bit codes: pairs (4 bits)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_tiles = (n_rows + kTile - 1) / kTile;
  if (tid == 0) {
    for (int i = 0; i < kPairs; ++i) { mbar_init(&m1[i], 1); mbar_init(&m2[i], 1); }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (tid < L) lut[tid] = P.c[tid] * kUnit;
  if (B == 2 && tid < 16) lut2[tid] = make_float2(P.c[tid & 3] * kUnit, P.c[tid >> 2] * kUnit);
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
  }
  {
    // (D H)[n][k] = D_n (-1)^popcount(n & k), binary16 +-1, same swizzled layout
    uint16_t* h16 = reinterpret_cast<uint16_t*>(sDH);
    for (int e = tid; e < kD * kD; e += kThreads) {
      const int n = e >> 7, k = e & 127;
      const bool neg = ((__popc(n & k) & 1) != 0) != (((X.Dneg[n >> 5] >> (n & 31)) & 1u) != 0);
      const int kb = k >> 6, chunk = (k & 63) >> 3, within = k & 7;
      h16[(kb * 16384 + n * 128 + ((chunk ^ (n & 7)) << 4)) / 2 + within] = neg ? 0xBC00u : 0x3C00u;
    }
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int wgi = warp >> 2, pair = wgi >> 1, half = wgi & 1, lb = warp & 3;
  const bool leader = (half == 0 && lb == 0 && lane == 0);        // issues the pair's MMAs
  const bool storer = (half == 1 && lb == 0 && lane == 0);        // issues the pair's TMA stores
  const int trow = lb * 32 + lane;
  const uint32_t lane_base = static_cast<uint32_t>(lb * 32) << 16;
  const uint32_t t_acc = tmem + lane_base + pair * 256;   // S^T z, then the rotated row (128 columns)
  const uint32_t t_a = t_acc + 128;                       // sign bits (64 columns), then v hi | lo (128)
  const uint32_t bar_id = 1 + pair;
  uint8_t* stage = sOut + pair * kStage;
  const float inv_sqrt_d = 0.08838834764831845f;
  const float qjl = P.qjl_scale * 16384.0f * kUnit;       // S^T z = 2^14 * acc, in unit-norm x kUnit
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
    // v in the unit-norm domain times kUnit (binary16 hi | lo stay clear of
    // underflow and overflow whatever the row's norm); norm / sqrt(d) / kUnit
    // is applied to the rotated output
    const float wq = nnrm > 0.f ? (nrn / nnrm) * qjl : 0.f;
    const float oscale = nnrm * (inv_sqrt_d / kUnit);
    load_packed(t + t_step);
    if (PROD) {
      // z_j 2^-14 as binary16: column k of sign word w holds bits (k, k + 16)
      // of the word, i.e. projections 32 w + k and 32 w + k + 16, moved to the
      // sign bits (15, 31) of the pair; half h writes sign words 2h and 2h + 1
      uint32_t a[32];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const uint32_t sgw = q == 0 ? sg0 : sg1;
#pragma unroll
        for (int k = 0; k < 16; ++k) a[q * 16 + k] = ((sgw << (15 - k)) & 0x80008000u) | 0x04000400u;
      }
      tmem_st32(t_a + half * 32, a);
      tmem_wait_st();
      tc_fence_before();
      // #1: the sign operand is complete, and the previous tile's outputs are read
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
        mma_commit(&m1[pair]);
      }
    }
    // ---- yhat of my coordinates while the MMA runs ----------------------------------
    float v[kH];
    if constexpr (B == 2) {
#pragma unroll
      for (int e = 0; e < kH; e += 2) {                    // two codes per lookup
        const float2 c2 = lut2[(cw[e >> 4] >> ((2 * e) & 31)) & 15u];
        v[e] = c2.x;
        v[e + 1] = c2.y;
      }
    } else {
#pragma unroll
      for (int e = 0; e < kH; ++e) {
        const int bit = B * e, wi = bit >> 5, sh = bit & 31;
        uint32_t code = cw[wi] >> sh;
        if (sh + B > 32) code |= cw[wi + 1] << (32 - sh);
        code &= (1u << B) - 1u;
        v[e] = lut[code];
      }
    }
    if (PROD) {
      if (!mbar_wait(&m1[pair], mine & 1, kWaitCycles)) {
        if (X.err) atomicCAS(X.err, 0, 5);
        atomicExch(abort_flag, 1);
      }
      tc_fence_after();
#pragma unroll
      for (int g2 = 0; g2 < 2; ++g2) {
        uint32_t acc[2][16];
        tmem_ld16(t_acc + half * 64 + g2 * 32, acc[0]);
        tmem_ld16(t_acc + half * 64 + g2 * 32 + 16, acc[1]);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) v[g2 * 32 + k] = fmaf(wq, __uint_as_float(acc[k >> 4][k & 15]), v[g2 * 32 + k]);
      }
    }
    // ---- v = hi + lo (binary16) into TMEM: the rotation's A operand ------------------
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      uint32_t hw[16], lw[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int e = ch * 32 + 2 * k;
        const __half2 h = __floats2half2_rn(v[e], v[e + 1]);
        const float2 hf = __half22float2(h);
        const __half2 l = __floats2half2_rn(v[e] - hf.x, v[e + 1] - hf.y);
        hw[k] = *reinterpret_cast<const uint32_t*>(&h);
        lw[k] = *reinterpret_cast<const uint32_t*>(&l);
      }
      tmem_st16(t_a + half * 32 + ch * 16, hw);
      tmem_st16(t_a + 64 + half * 32 + ch * 16, lw);
    }
    tmem_wait_st();
    tc_fence_before();
    // #2: v complete in TMEM and every S^T z read done (the rotation overwrites them)
    if (named_bar_sync_or(bar_id, 256, *reinterpret_cast<volatile int*>(abort_flag) != 0)) break;
    if (leader) {
      tc_fence_after();
      const uint32_t sbase = smem_u32(sDH);
      const uint32_t idesc = idesc_f16_f32(kTile, kD);
      const uint32_t d_tmem = tmem + pair * 256;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int kk = k & 7;
        const uint64_t bdesc = smem_desc_sw128(sbase + (kk >> 2) * 16384 + (kk & 3) * 32, 1024);
        mma_f16_ts(d_tmem, d_tmem + 128 + k * 8, bdesc, idesc, k > 0 ? 1u : 0u);
      }
      mma_commit(&m2[pair]);
    }
    if (!mbar_wait(&m2[pair], mine & 1, kWaitCycles)) {
      if (X.err) atomicCAS(X.err, 0, 8);
      atomicExch(abort_flag, 1);
    }
    tc_fence_after();
    // ---- my 64 output columns, staged (swizzled) for the TMA store --------------------
    uint32_t o[4][16];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld16(t_acc + half * 64 + c * 16, o[c]);
    tmem_wait_ld();
    tc_fence_before();
    if (storer && store_pending) bulk_wait_read0();         // previous tile's store has read the stage
    named_bar_sync(bar_id, 256);
    if (BF16OUT) {
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {                      // box `half`: my 64 columns
        uint32_t wv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = cc * 8 + 2 * u;
          const __nv_bfloat162 p2 = __floats2bfloat162_rn(__uint_as_float(o[e >> 4][e & 15]) * oscale,
                                                          __uint_as_float(o[(e + 1) >> 4][(e + 1) & 15]) * oscale);
          wv[u] = *reinterpret_cast<const uint32_t*>(&p2);
        }
        *reinterpret_cast<uint4*>(stage + half * (kTile * 128) + trow * 128 + ((cc ^ (trow & 7)) << 4)) =
            make_uint4(wv[0], wv[1], wv[2], wv[3]);
      }
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c) {                        // boxes 2 half, 2 half + 1
        const int e = c * 4;
        const float4 w4 = make_float4(__uint_as_float(o[e >> 4][e & 15]) * oscale,
                                      __uint_as_float(o[e >> 4][(e & 15) + 1]) * oscale,
                                      __uint_as_float(o[e >> 4][(e & 15) + 2]) * oscale,
                                      __uint_as_float(o[e >> 4][(e & 15) + 3]) * oscale);
        const int bx = 2 * half + (c >> 3), cc = c & 7;
        *reinterpret_cast<float4*>(stage + bx * (kTile * 128) + trow * 128 + ((cc ^ (trow & 7)) << 4)) = w4;
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(bar_id, 256);
    if (storer) {
#pragma unroll
      for (int bx = 0; bx < OutStage<BF16OUT>::kBoxes; ++bx)
        tma_store_2d(&tmap_out, stage + bx * (kTile * 128), bx * OutStage<BF16OUT>::kColsPerBox,
                     static_cast<int>(t * kTile));
      bulk_commit();
      store_pending = true;
    }
  }
  if (storer && store_pending) bulk_wait0();               // all our stores have landed
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// bf16 output, overlapped: the same two products per tile, arranged so that
// the tensor cores never wait for the CUDA cores of the same pair.
//   * The sign operand of S^T z lives in shared memory (A of an ss MMA, z_j
//     as binary16 +-1 in the K-major 128-byte-swizzled layout), written for
//     the NEXT tile while the current tile's rotation runs.
//   * Each pair has two 128-column TMEM regions with alternating roles: tile
//     k's S^T z and then its rotated output in region k mod 2, its v hi | lo
//     in the other; so the next tile's S^T z product can run into the region
//     of this tile's v as soon as the rotation has read it, under this tile's
//     output stores.
// Per tile (pair): wait S^T z -> v = yhat + w S^T z -> v hi | lo into TMEM,
// the next tile's signs into shared memory -> barrier -> rotation MMA; while
// it runs, decode the next tile's yhat -> wait -> the next tile's S^T z MMA
// -> read, scale, round and stage the output -> barrier -> TMA store.
template <int B, bool PROD, int KD>
__global__ void __launch_bounds__(kThreads, 1)
k_dequant_d128_ovl(const __grid_constant__ CUtensorMap tmap_out, const KParams P, const DequantD128Args X,
                   const Packed in, int64_t n_rows) {
  constexpr int L = 1 << B;
  constexpr int kStage = kTile * KD * 2;                  // bf16 output tile (KD / 64 boxes)
  constexpr int kH = KD / 2;                               // coordinates (and projections) per thread
  constexpr int kNW = B * kH / 32;                         // packed code words per thread
  constexpr int kOp = KD * KD * 2;                         // S^T or D H as a binary16 operand
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sSt = smem;                                   // B of S^T z: row i, K position j holds S[j][i]
  uint8_t* sDH = smem + kOp;                             // B of the rotation (N = n, K = k)
  uint8_t* sZ = sDH + kOp;                               // [pair] A of S^T z: row r, K position j holds z_j
  uint8_t* sOut = sZ + kPairs * kStage;                  // [pair] output stages
  uint64_t* m1 = reinterpret_cast<uint64_t*>(sOut + kPairs * kStage);   // [pair] S^T z done
  uint64_t* m2 = m1 + kPairs;                                            // [pair] rotation done
  uint64_t* fdone = m2 + kPairs;                                         // [2][pair] wind-down commits
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fdone + 2 * kPairs);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* lut = reinterpret_cast<float*>(tmem_slot + 2);                 // L centroids x kUnit
  float2* lut2 = reinterpret_cast<float2*>(lut + 16);                   // 2-bit codes: pairs (4 bits)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_tiles = (n_rows + kTile - 1) / kTile;
  const long long wait_cycles = X.wait_cycles;
  if (tid == 0) {
    for (int i = 0; i < kPairs; ++i) {
      mbar_init(&m1[i], 1);
      mbar_init(&m2[i], 1);
      mbar_init(&fdone[i], 1);
      mbar_init(&fdone[kPairs + i], 1);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (tid < L) lut[tid] = P.c[tid] * kUnit;
  if (B == 2 && tid < 16) lut2[tid] = make_float2(P.c[tid & 3] * kUnit, P.c[tid >> 2] * kUnit);
  if (PROD) {
    uint16_t* st16 = reinterpret_cast<uint16_t*>(sSt);
    for (int e = tid; e < KD * KD; e += kThreads) {
      const int i = e / KD, j = e % KD;
      const int kb = j >> 6, chunk = (j & 63) >> 3, within = j & 7;
      st16[(kb * (KD * 128) + i * 128 + ((chunk ^ (i & 7)) << 4)) / 2 + within] = P.St[i * KD + j];
    }
  }
  {
    // (D H)[n][k] = D_n (-1)^popcount(n & k), binary16 +-1, same swizzled layout
    uint16_t* h16 = reinterpret_cast<uint16_t*>(sDH);
    for (int e = tid; e < KD * KD; e += kThreads) {
      const int n = e / KD, k = e % KD;
      const bool neg = ((__popc(n & k) & 1) != 0) != (((X.Dneg[n >> 5] >> (n & 31)) & 1u) != 0);
      const int kb = k >> 6, chunk = (k & 63) >> 3, within = k & 7;
      h16[(kb * (KD * 128) + n * 128 + ((chunk ^ (n & 7)) << 4)) / 2 + within] = neg ? 0xBC00u : 0x3C00u;
    }
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(tmem_slot, 4 * KD);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int wgi = warp >> 2, pair = wgi >> 1, half = wgi & 1, lb = warp & 3;
  const bool leader = (half == 0 && lb == 0 && lane == 0);        // issues the pair's MMAs
  const bool storer = (half == 1 && lb == 0 && lane == 0);        // issues the pair's TMA stores
  // issues the pair's S^T z products: for 3-bit codes a second thread, so that
  // the leader's warp spends no issue time on them (one thread issues an MMA
  // only every few dozen cycles); 10 % faster there, while for the other code
  // widths the extra live state costs register spills and the leader keeps them
  constexpr bool kSplitIssue = B == 3;
  const bool zissuer = kSplitIssue ? (half == 1 && lb == 1 && lane == 0) : leader;
  const int trow = lb * 32 + lane;
  const uint32_t lane_base = static_cast<uint32_t>(lb * 32) << 16;
  const uint32_t t_reg0 = tmem + lane_base + pair * (2 * KD);   // region k mod 2: S^T z, then the output of tile k
  const uint32_t bar_id = 1 + pair;
  uint8_t* stage = sOut + pair * kStage;
  uint8_t* zbuf = sZ + pair * kStage;
  const float inv_sqrt_d = KD == 128 ? 0.08838834764831845f : 0.125f;
  const float qjl = P.qjl_scale * kUnit;                  // S^T z in unit-norm x kUnit
  const int64_t t_first = blockIdx.x + static_cast<int64_t>(pair) * gridDim.x;
  const int64_t t_step = static_cast<int64_t>(kPairs) * gridDim.x;
  bool store_pending = false, mma_issued = false, stz_issued = false;

  // my part of a packed row: codes of my 64 coordinates, my two sign words, norms
  struct Part {
    uint32_t cw[kNW];
    uint32_t sg0, sg1;
    float nrm, rn;
  };
  auto load_packed = [&](int64_t tile, Part& pt) {
    const int64_t row = tile * kTile + trow;
    if (tile < n_tiles && row < n_rows && KD == 64) {
      const uint8_t* cp = in.codes + row * (B * 8) + half * (B * 4);
      if constexpr (B == 1) {
        pt.cw[0] = __ldg(reinterpret_cast<const uint32_t*>(cp));
      } else if constexpr (B == 2) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(cp));
        pt.cw[0] = u.x; pt.cw[1] = u.y;
      } else if constexpr (B == 3) {
#pragma unroll
        for (int w = 0; w < 3; ++w) pt.cw[w] = __ldg(reinterpret_cast<const uint32_t*>(cp) + w);
      } else {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(cp));
        pt.cw[0] = u.x; pt.cw[1] = u.y; pt.cw[2] = u.z; pt.cw[3] = u.w;
      }
      pt.sg0 = PROD ? __ldg(reinterpret_cast<const uint32_t*>(in.signs + row * 8 + half * 4)) : 0u;
      pt.sg1 = 0u;
      pt.nrm = __ldg(in.norm + row);
      pt.rn = __ldg(in.rnorm + row);
    } else if (tile < n_tiles && row < n_rows) {
      const uint8_t* cp = in.codes + row * (B * 16) + half * (B * 8);
      if constexpr (B == 1) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(cp));
        pt.cw[0] = u.x; pt.cw[1] = u.y;
      } else if constexpr (B == 2) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(cp));
        pt.cw[0] = u.x; pt.cw[1] = u.y; pt.cw[2] = u.z; pt.cw[3] = u.w;
      } else if constexpr (B == 3) {
        if (half == 0) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(cp));
          const uint2 w = __ldg(reinterpret_cast<const uint2*>(cp + 16));
          pt.cw[0] = u.x; pt.cw[1] = u.y; pt.cw[2] = u.z; pt.cw[3] = u.w; pt.cw[4] = w.x; pt.cw[5] = w.y;
        } else {
          const uint2 w = __ldg(reinterpret_cast<const uint2*>(cp));
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(cp + 8));
          pt.cw[0] = w.x; pt.cw[1] = w.y; pt.cw[2] = u.x; pt.cw[3] = u.y; pt.cw[4] = u.z; pt.cw[5] = u.w;
        }
      } else {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(cp));
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(cp + 16));
        pt.cw[0] = u.x; pt.cw[1] = u.y; pt.cw[2] = u.z; pt.cw[3] = u.w;
        pt.cw[4] = w.x; pt.cw[5] = w.y; pt.cw[6] = w.z; pt.cw[7] = w.w;
      }
      if (PROD) {
        const uint2 sg = __ldg(reinterpret_cast<const uint2*>(in.signs + row * 16 + half * 8));
        pt.sg0 = sg.x; pt.sg1 = sg.y;
      } else {
        pt.sg0 = pt.sg1 = 0u;
      }
      pt.nrm = __ldg(in.norm + row);
      pt.rn = __ldg(in.rnorm + row);
    } else {
#pragma unroll
      for (int w = 0; w < kNW; ++w) pt.cw[w] = 0u;
      pt.sg0 = pt.sg1 = 0u;
      pt.nrm = 0.f;
      pt.rn = 0.f;
    }
  };
  // yhat x kUnit of my 64 coordinates
  auto decode = [&](const Part& pt, float (&v)[kH]) {
    if constexpr (B == 2) {
#pragma unroll
      for (int e = 0; e < kH; e += 2) {                    // two codes per lookup
        const float2 c2 = lut2[(pt.cw[e >> 4] >> ((2 * e) & 31)) & 15u];
        v[e] = c2.x;
        v[e + 1] = c2.y;
      }
    } else {
#pragma unroll
      for (int e = 0; e < kH; ++e) {
        const int bit = B * e, wi = bit >> 5, sh = bit & 31;
        uint32_t code = pt.cw[wi] >> sh;
        if (sh + B > 32) code |= pt.cw[wi + 1] << (32 - sh);
        code &= (1u << B) - 1u;
        v[e] = lut[code];
      }
    }
  };
  // my 64 sign bits as binary16 z_j = +-1 into row trow of the sign operand:
  // K block `half`, 16-byte chunk c (projections 64 half + 8 c ..) at chunk c ^ (trow & 7)
  auto write_signs = [&](const Part& pt) {
#pragma unroll
    for (int c = 0; c < kH / 8; ++c) {
      const uint32_t sgw = (c < 4 ? pt.sg0 : pt.sg1) >> ((c & 3) * 8);   // projections 8 c .. 8 c + 7 (of mine)
      uint32_t w4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t b2 = sgw >> (2 * u);                 // bits of projections 2u, 2u + 1
        w4[u] = 0x3C003C00u | ((b2 & 1u) << 15) | ((b2 & 2u) << 30);
      }
      // K atom and 16-byte chunk of projections half kH + 8 c .. + 7
      const int atom = KD == 128 ? half : 0, chunk = KD == 128 ? c : 4 * half + c;
      *reinterpret_cast<uint4*>(zbuf + atom * 16384 + trow * 128 + ((chunk ^ (trow & 7)) << 4)) =
          make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
  };
  auto issue_stz = [&](int k) {                            // S^T z of this pair's k-th tile
    tc_fence_after();
    const uint32_t zbase = smem_u32(zbuf), sbase = smem_u32(sSt);
    const uint32_t idesc = idesc_f16_f32(kTile, KD);
    const uint32_t d_tmem = tmem + pair * (2 * KD) + (k & 1) * KD;
#pragma unroll
    for (int kk = 0; kk < KD / 16; ++kk) {
      const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
      const uint32_t boff = (kk >> 2) * (KD * 128) + (kk & 3) * 32;
      mma_f16_ss(d_tmem, smem_desc_sw128(zbase + aoff, 1024), smem_desc_sw128(sbase + boff, 1024), idesc,
                 kk > 0 ? 1u : 0u);
    }
    mma_commit(&m1[pair]);
    (kSplitIssue ? stz_issued : mma_issued) = true;
  };

  Part cur, nxt;
  float v[kH];
  load_packed(t_first, cur);
  load_packed(t_first + t_step, nxt);
  if (PROD) write_signs(cur);
  decode(cur, v);
  fence_proxy_async_smem();
  named_bar_sync(bar_id, 256);                             // the first tile's sign operand is complete
  if (PROD && zissuer && t_first < n_tiles) issue_stz(0);

  int mine = 0;
  for (int64_t t = t_first; t < n_tiles; t += t_step, ++mine) {
    const uint32_t t_acc = t_reg0 + (mine & 1) * KD;       // S^T z, then the output
    const uint32_t t_a = t_reg0 + ((mine + 1) & 1) * KD;    // v hi | lo
    // v in the unit-norm domain times kUnit; norm / sqrt(d) / kUnit is applied to the output
    const float wq = cur.nrm > 0.f ? (cur.rn / cur.nrm) * qjl : 0.f;
    const float oscale = cur.nrm * (inv_sqrt_d / kUnit);
    if (PROD) {
      if (!mbar_wait(&m1[pair], mine & 1, wait_cycles)) {
        if (X.err) atomicCAS(X.err, 0, 5);
        atomicExch(abort_flag, 1);
      }
      tc_fence_after();
#pragma unroll
      for (int g2 = 0; g2 < kH / 32; ++g2) {
        uint32_t acc[32];
        tmem_ld32(t_acc + half * kH + g2 * 32, acc);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) v[g2 * 32 + k] = fmaf(wq, __uint_as_float(acc[k]), v[g2 * 32 + k]);
      }
      // S^T z of this tile has been read and its operand consumed: the next
      // tile's signs may take the operand's place
      write_signs(nxt);
    }
    // ---- v = hi + lo (binary16) into TMEM: the rotation's A operand ------------------
#pragma unroll
    for (int ch = 0; ch < kH / 32; ++ch) {
#pragma unroll
      for (int g8 = 0; g8 < 2; ++g8) {
        uint32_t hw[8], lw[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int e = ch * 32 + g8 * 16 + 2 * k;
          const __half2 h = __floats2half2_rn(v[e], v[e + 1]);
          const float2 hf = __half22float2(h);
          const float2 lf = __fadd2_rn(make_float2(v[e], v[e + 1]), make_float2(-hf.x, -hf.y));
          const __half2 l = __floats2half2_rn(lf.x, lf.y);
          hw[k] = *reinterpret_cast<const uint32_t*>(&h);
          lw[k] = *reinterpret_cast<const uint32_t*>(&l);
        }
        tmem_st8(t_a + half * (KD / 4) + ch * 16 + g8 * 8, hw);
        tmem_st8(t_a + KD / 2 + half * (KD / 4) + ch * 16 + g8 * 8, lw);
      }
    }
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    // #2: v complete in TMEM, every S^T z read done (the rotation overwrites
    // them), the next tile's sign operand written
    if (named_bar_sync_or(bar_id, 256, *reinterpret_cast<volatile int*>(abort_flag) != 0)) break;
    if (leader) {
      tc_fence_after();
      const uint32_t sbase = smem_u32(sDH);
      const uint32_t idesc = idesc_f16_f32(kTile, KD);
      const uint32_t d_tmem = tmem + pair * (2 * KD) + (mine & 1) * KD;
      const uint32_t a_tmem = tmem + pair * (2 * KD) + ((mine + 1) & 1) * KD;
#pragma unroll
      for (int k = 0; k < 2 * KD / 16; ++k) {
        const int kk = k % (KD / 16);
        const uint64_t bdesc = smem_desc_sw128(sbase + (kk >> 2) * (KD * 128) + (kk & 3) * 32, 1024);
        mma_f16_ts(d_tmem, a_tmem + k * 8, bdesc, idesc, k > 0 ? 1u : 0u);
      }
      mma_commit(&m2[pair]);
      mma_issued = true;
    }
    // ---- while the rotation runs: the next tile's yhat, and the packed row after it --
    cur = nxt;
    decode(cur, v);
    load_packed(t + 2 * t_step, nxt);
    if (!mbar_wait(&m2[pair], mine & 1, wait_cycles)) {
      if (X.err) atomicCAS(X.err, 0, 8);
      atomicExch(abort_flag, 1);
    }
    tc_fence_after();
    // the rotation has read v: the next tile's S^T z may run into its region
    if (PROD && zissuer && t + t_step < n_tiles && *reinterpret_cast<volatile int*>(abort_flag) == 0)
      issue_stz(mine + 1);
    // ---- my kH output columns, staged (swizzled) for the TMA store, 32 at a time -------
#pragma unroll
    for (int hh = 0; hh < kH / 32; ++hh) {
      uint32_t o[32];
      tmem_ld32(t_acc + half * kH + hh * 32, o);
      tmem_wait_ld();
      if (hh == 0) {
        if (storer && store_pending) bulk_wait_read0();     // previous tile's store has read the stage
        named_bar_sync(bar_id, 256);
      }
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {                      // 8 columns per 16-byte chunk
        const int cc = hh * 4 + c4;
        uint32_t wv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = c4 * 8 + 2 * u;
          const __nv_bfloat162 p2 =
              __floats2bfloat162_rn(__uint_as_float(o[e]) * oscale, __uint_as_float(o[e + 1]) * oscale);
          wv[u] = *reinterpret_cast<const uint32_t*>(&p2);
        }
        // box and 16-byte chunk of output columns half kH + 8 cc .. + 7
        const int box = KD == 128 ? half : 0, chunk = KD == 128 ? cc : 4 * half + cc;
        *reinterpret_cast<uint4*>(stage + box * (kTile * 128) + trow * 128 + ((chunk ^ (trow & 7)) << 4)) =
            make_uint4(wv[0], wv[1], wv[2], wv[3]);
      }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    // #3: the stage is complete, and every read of this tile's output region is
    // done (the next tile's v goes there)
    named_bar_sync(bar_id, 256);
    if (storer) {
#pragma unroll
      for (int bx = 0; bx < KD / 64; ++bx)
        tma_store_2d(&tmap_out, stage + bx * (kTile * 128), bx * 64, static_cast<int>(t * kTile));
      bulk_commit();
      store_pending = true;
    }
  }
  // wind-down (full wait limit): our MMAs and stores complete before the TMEM
  // and the shared memory are released
  if (leader && mma_issued) {
    mma_commit(&fdone[pair]);
    if (!mbar_wait(&fdone[pair], 0, kWaitCycles) && X.err) atomicCAS(X.err, 0, 4);
  }
  if (kSplitIssue && zissuer && stz_issued) {
    mma_commit(&fdone[kPairs + pair]);
    if (!mbar_wait(&fdone[kPairs + pair], 0, kWaitCycles) && X.err) atomicCAS(X.err, 0, 4);
  }
  if (storer && store_pending) bulk_wait0();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 4 * KD);
  }
}

template <int B, bool PROD, bool BF16OUT, int KD>
int launch(const tq_ctx& ctx, const Packed& in, int64_t n_rows, void* out, int64_t ld_out, cudaStream_t s) {
  static_assert(BF16OUT || KD == 128, "fp32 output: d = 128 only");
  const KParams& P = ctx.kp;
  auto encode = tensor_map_encoder();
  if (!encode) return static_cast<int>(cudaErrorNotSupported);
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(KD), static_cast<cuuint64_t>(n_rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_out) * (BF16OUT ? 2 : 4)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(OutStage<BF16OUT>::kColsPerBox), static_cast<cuuint32_t>(kTile)};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&tmap, BF16OUT ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, out, dims,
             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return static_cast<int>(cudaErrorInvalidValue);
  DequantD128Args X;
  for (int w = 0; w < kD / 32; ++w) X.Dneg[w] = 0u;
  for (int i = 0; i < KD; ++i)
    if (ctx.D[i] < 0) X.Dneg[i >> 5] |= 1u << (i & 31);
  X.err = P.err;
  X.wait_cycles = wait_limit_cycles();
  const int64_t n_tiles = (n_rows + kTile - 1) / kTile;
  const int grid = static_cast<int>(n_tiles < ctx.num_sms ? n_tiles : ctx.num_sms);
  if constexpr (BF16OUT) {                 // the overlapped kernel (bf16 output)
    const size_t smem = dequant_ovl_smem_bytes<KD>();
    cudaError_t e = cudaFuncSetAttribute(k_dequant_d128_ovl<B, PROD, KD>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return static_cast<int>(e);
    k_dequant_d128_ovl<B, PROD, KD><<<grid, kThreads, smem, s>>>(tmap, P, X, in, n_rows);
  } else {
    const size_t smem = dequant_smem_bytes<BF16OUT>();
    cudaError_t e = cudaFuncSetAttribute(k_dequant_d128_tc<B, PROD, BF16OUT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return static_cast<int>(e);
    k_dequant_d128_tc<B, PROD, BF16OUT><<<grid, kThreads, smem, s>>>(tmap, P, X, in, n_rows);
  }
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

template <int B>
int launch_B(const tq_ctx& ctx, const Packed& in, int64_t n_rows, void* out, int64_t ld_out, int bf16, int prod,
             cudaStream_t s) {
  if (ctx.kp.d == 64) {                    // bf16 output only (see dequant_d128_applies)
    return prod ? launch<B, true, true, 64>(ctx, in, n_rows, out, ld_out, s)
                : launch<B, false, true, 64>(ctx, in, n_rows, out, ld_out, s);
  }
  if (prod)
    return bf16 ? launch<B, true, true, 128>(ctx, in, n_rows, out, ld_out, s)
                : launch<B, true, false, 128>(ctx, in, n_rows, out, ld_out, s);
  return bf16 ? launch<B, false, true, 128>(ctx, in, n_rows, out, ld_out, s)
              : launch<B, false, false, 128>(ctx, in, n_rows, out, ld_out, s);
}

}  // namespace

bool dequant_d128_applies(const tq_ctx& ctx, int64_t n_rows, int out_is_bf16) {
  if (ctx.d_in != ctx.d) return false;                   // padded rows use the general kernel
  const KParams& P = ctx.kp;
  // d = m = 128 (bf16 or fp32 output), or d = m = 64 with bf16 output (the
  // 64-channel parts of a split row)
  const bool shape = (P.d == 128 && P.m == 128) || (P.d == 64 && P.m == 64 && out_is_bf16);
  return shape && P.B >= 1 && P.B <= 4 && n_rows > 0 && n_rows < (int64_t(1) << 31) && ctx.use_tc &&
         tensor_map_encoder() != nullptr;
}

int launch_dequant_d128(const tq_ctx& ctx, const Packed& in, int64_t n_rows, void* out, int64_t ld_out,
                        int out_is_bf16, int prod, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (ctx.kp.B) {
    case 1: return launch_B<1>(ctx, in, n_rows, out, ld_out, out_is_bf16, prod, s);
    case 2: return launch_B<2>(ctx, in, n_rows, out, ld_out, out_is_bf16, prod, s);
    case 3: return launch_B<3>(ctx, in, n_rows, out, ld_out, out_is_bf16, prod, s);
    default: return launch_B<4>(ctx, in, n_rows, out, ld_out, out_is_bf16, prod, s);
  }
}

}  // namespace tq
