// Write half at d = 128, m = 128 on sm_100a: TMA-staged rows, the
// randomized Hadamard rotation, Lloyd-Max bucketing, and the QJL projection
// S r on the tcgen05 tensor cores.
//
// Method (page title, section):
//   n = ||x||, y = H_d D x / (n sqrt(d))      0h-n0.github.io "ICLR 2026論文解説:
//                                             TurboQuant", "Step 1: PolarQuant"
//   code_i = #{k : t_k < y_i}, r = y - c[code]  Qiita TurboQuant explainer,
//                                             "Stage 1: PolarQuant" (Lloyd-Max)
//   bit_j = [ (S r)_j < 0 ], rnorm = n ||r||    Qiita explainer, "Stage 2: QJL"
//
// Two kernels, persistent (one CTA per SM), rows arriving by TMA:
//   k_quantize_d128_ws  bf16 rows, warp-specialized: sixteen compute warps
//                       share each 128-row tile (four threads per row, 32
//                       coordinates each, the row in its TMEM lane) and a
//                       seventeenth warp issues the TMA loads and the
//                       tensor-core work: the rotation itself as an MMA
//                       (A = the TMA stage, B = D H as bf16 +-1) and the
//                       projection MMA, into four rotating TMEM regions so
//                       both run under the CUDA-core work on the tile before;
//   k_quantize_d128_tc  fp32 rows: two pairs of warpgroups, the rotation in
//                       registers (five FWHT stages, the stride-64 stage
//                       through the TMEM lane), then the same codes and
//                       projection MMA.
//
// Projection precision: S is binary16 by definition (exact in the MMA).  The
// residual, scaled by 64, is split r = hi + lo into two binary16 parts
// (|r - hi - lo| <= 2^-22 |r| + 2^-25) and the MMA accumulates S hi + S lo
// (K = 256) in fp32.  A sign is taken from the tensor-core sum only where
// |p_j| exceeds a bound on that sum's error, eps = eps_scale ||r|| + eps_abs
// with eps_scale = 16 * 2^-22 * max_j ||S_j||_2 (the split's 2^-22 plus 16
// accumulation steps of at most 2^-23 each, with margin) and eps_abs =
// max_j ||S_j||_1 * 2^-25 / 64 (binary16 underflow); the rare projections
// below it are recomputed: by the fp32 kernel in fp32 on the CUDA cores from
// hi + lo, and for the bf16 kernel in fp64 from the input row by the fix-up
// kernel that runs after it.  The bf16 kernel decides each code bit from the sign of T^2 - y^2
// computed with one rounding (the threshold moves by at most about one ulp).
//
// Every mbarrier wait is bounded (about one second); a wait that runs out
// sets the context's error word, the CTA stops issuing work, waits for its
// own TMA loads, frees its TMEM and exits.

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "sm100.cuh"
#include "tq_internal.h"

namespace tq {

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

namespace {

using namespace sm100;

constexpr int kD = 128;              // row length
constexpr int kM = 128;              // projections
constexpr int kTile = 128;           // rows per tile = MMA M
constexpr int kPairs = 2;            // warpgroup pairs per CTA, one 128-row tile each in flight
constexpr int kThreads = kPairs * 256;
constexpr long long kWaitCycles = 2000000000ll;   // ~1 s at 2 GHz
constexpr uint32_t kTmemCols = 512;  // per pair: 128 accumulator + 128 A columns, x2

struct QuantD128Args {
  uint32_t Dsign[kD];                // Rademacher signs as fp32 sign-bit masks (0 or 0x80000000)
  float eps_scale;                   // see header comment
  float eps_abs;                     // binary16 underflow term of the bound (normalised units)
  int* err;                          // device error word
  long long wait_cycles;             // limit of the bounded waits in the tile loop (SM clocks)
  // bf16 kernel: projections inside the bound go to the exact fix-up kernel
  // that runs after it, as (row << 8) | j entries of fix_list (fix_count
  // claims slots, zeroed before the launch); a row whose entries do not fit
  // gets its bit in fix_rows instead (zeroed too), and all its signs are
  // recomputed
  unsigned long long* fix_list;
  unsigned int* fix_count;
  unsigned int fix_cap;
  unsigned int* fix_rows;
};

// The residual enters the MMA multiplied by 64 (exact), which keeps its
// binary16 parts clear of the subnormal range for all but tiny residuals.
constexpr float kResScale = 64.0f;

template <bool BF16IN>
struct XStage {
  static constexpr int kColsPerBox = BF16IN ? 64 : 32;    // 128 bytes of a row per box
  static constexpr int kBoxes = kD / kColsPerBox;
  static constexpr int kBytes = kBoxes * kTile * 128;     // 32 KB (bf16) or 64 KB (fp32)
  static constexpr int kStages = BF16IN ? 2 : 1;          // per warpgroup (shared memory budget)
};

constexpr int kSmemS = 32768;        // S as the MMA B operand (128 x 128 fp16, swizzled)

template <bool BF16IN>
constexpr size_t quant_smem_bytes() {
  return 1024 /*alignment slack*/ + kSmemS + XStage<BF16IN>::kStages * kPairs * XStage<BF16IN>::kBytes +
         2 * kPairs * 2 * kTile * 4 /*partial sums*/ + 256 /*barriers etc*/;
}

__device__ __forceinline__ void flag_error(int* err, int* abort_flag, int code) {
  if (err) atomicCAS(err, 0, code);
  atomicExch(abort_flag, 1);
}

// Two warpgroups ("halves") share every 128-row tile: thread t of warp w in
// half h owns coordinates [64 h, 64 h + 64) of row 32 (w % 4) + t, which is
// also the row's TMEM lane, so both halves of a row meet in the same lane.
// Two such pairs run per CTA (512 threads, 16 warps per SM).
template <int B, bool BF16IN>
__global__ void __launch_bounds__(kThreads, 1)
k_quantize_d128_tc(const __grid_constant__ CUtensorMap tmap, const KParams P, const QuantD128Args X,
                   int64_t n_rows, const Packed out) {
  constexpr int L = 1 << B;
  constexpr int kStage = XStage<BF16IN>::kBytes;
  constexpr int NS = XStage<BF16IN>::kStages;
  constexpr int kH = kD / 2;                                     // coordinates per thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sS = smem;
  uint8_t* sX = smem + kSmemS;                                   // [pair][NS] stages
  float* sPart = reinterpret_cast<float*>(sX + NS * kPairs * kStage);   // [2 sums][pair][half][row] partials
  uint64_t* full = reinterpret_cast<uint64_t*>(sPart + 2 * kPairs * 2 * kTile);   // [pair][2]
  uint64_t* mdone = full + 2 * kPairs;                           // [pair]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + kPairs);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* lut = reinterpret_cast<float*>(tmem_slot + 2);          // L centroids (scaled by 64)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_tiles = (n_rows + kTile - 1) / kTile;

  if (tid == 0) {
    for (int i = 0; i < 2 * kPairs; ++i) mbar_init(&full[i], 1);
    for (int i = 0; i < kPairs; ++i) mbar_init(&mdone[i], 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (tid < L) lut[tid] = P.c[tid] * kResScale;
  // S into the canonical K-major 128-byte-swizzled layout: K block kb (64
  // columns), row j at 128 B, 16-byte chunk c stored at chunk c ^ (j & 7).
  for (int e = tid; e < kM * 16; e += kThreads) {
    const int j = e >> 4, c = e & 15, kb = c >> 3, cc = c & 7;
    const uint4 v = *reinterpret_cast<const uint4*>(P.S + j * kD + c * 8);
    *reinterpret_cast<uint4*>(sS + kb * 16384 + j * 128 + ((cc ^ (j & 7)) << 4)) = v;
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
  const bool leader = (half == 0 && lb == 0 && lane == 0);       // issues this pair's TMA and MMAs
  const int trow = lb * 32 + lane;                               // row in tile == TMEM lane
  const uint32_t lane_base = static_cast<uint32_t>(lb * 32) << 16;
  const uint32_t t_acc = tmem + lane_base + pair * 256;          // projections, 128 columns
  const uint32_t t_a = t_acc + 128;                              // residual hi | lo, 128 columns
  const uint32_t bar_id = 1 + pair;                              // named barrier of the pair (256 threads)
  const float sqrt_d = 11.313708498984761f;                      // sqrt(128)
  uint8_t* stages = sX + pair * NS * kStage;
  uint64_t* pfull = full + 2 * pair;
  float* myN2 = sPart + (pair * 2 + half) * kTile;               // partial ||x||^2
  const float* otN2 = sPart + (pair * 2 + (half ^ 1)) * kTile;
  float* myR2 = sPart + kPairs * 2 * kTile + (pair * 2 + half) * kTile;   // partial ||r||^2
  const float* otR2 = sPart + kPairs * 2 * kTile + (pair * 2 + (half ^ 1)) * kTile;
  const int64_t t_first = blockIdx.x + static_cast<int64_t>(pair) * gridDim.x;
  const int64_t t_step = static_cast<int64_t>(kPairs) * gridDim.x;
  auto issue_load = [&](int64_t tile, int buf) {
    mbar_arrive_expect_tx(&pfull[buf], kStage);
#pragma unroll
    for (int bx = 0; bx < XStage<BF16IN>::kBoxes; ++bx)
      tma_load_2d(stages + buf * kStage + bx * (kTile * 128), &tmap, &pfull[buf],
                  bx * XStage<BF16IN>::kColsPerBox, static_cast<int>(tile * kTile));
  };
  int issued[2] = {0, 0}, waited[2] = {0, 0};                    // leader's TMA bookkeeping
  if (leader) {
    prefetch_tmap(&tmap);
    if (t_first < n_tiles) { issue_load(t_first, 0); ++issued[0]; }
    if (NS == 2 && t_first + t_step < n_tiles) { issue_load(t_first + t_step, 1); ++issued[1]; }
  }

  int mine = 0;
  for (int64_t t = t_first; t < n_tiles; t += t_step, ++mine) {
    const int buf = mine % NS;
    if (mbar_wait(&pfull[buf], (mine / NS) & 1, kWaitCycles)) {
      if (leader) ++waited[buf];
    } else {
      flag_error(X.err, abort_flag, 2);
    }
    const uint8_t* stage = stages + buf * kStage;

    // ---- my half row, D folded into the widening -------------------------------
    float v[kH];
    if (BF16IN) {
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {                           // box `half` holds my 64 columns
        const uint4 w = *reinterpret_cast<const uint4*>(stage + half * (kTile * 128) + trow * 128 +
                                                        ((cc ^ (trow & 7)) << 4));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = cc * 8 + 2 * u;
          v[e] = __uint_as_float((ws[u] << 16) ^ X.Dsign[half * kH + e]);
          v[e + 1] = __uint_as_float((ws[u] & 0xffff0000u) ^ X.Dsign[half * kH + e + 1]);
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c) {                             // boxes 2 half, 2 half + 1
        const int bx = 2 * half + (c >> 3), cc = c & 7;
        const uint4 w = *reinterpret_cast<const uint4*>(stage + bx * (kTile * 128) + trow * 128 +
                                                        ((cc ^ (trow & 7)) << 4));
        v[c * 4 + 0] = __uint_as_float(w.x ^ X.Dsign[half * kH + c * 4 + 0]);
        v[c * 4 + 1] = __uint_as_float(w.y ^ X.Dsign[half * kH + c * 4 + 1]);
        v[c * 4 + 2] = __uint_as_float(w.z ^ X.Dsign[half * kH + c * 4 + 2]);
        v[c * 4 + 3] = __uint_as_float(w.w ^ X.Dsign[half * kH + c * 4 + 3]);
      }
    }
    // partial norm (sign flips do not change it)
    {
      float2 a2 = make_float2(0.f, 0.f), b2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < kH; e += 4) {
        const float2 a = make_float2(v[e], v[e + 1]), b = make_float2(v[e + 2], v[e + 3]);
        a2 = __ffma2_rn(a, a, a2);
        b2 = __ffma2_rn(b, b, b2);
      }
      myN2[trow] = (a2.x + a2.y) + (b2.x + b2.y);
    }
    // Walsh-Hadamard within my 64 coordinates (strides 2..32 packed, then 1)
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
    // stride-64 stage across the halves, through this row's TMEM lane: my
    // values go to columns [64 half, 64 half + 64) of the (idle) accumulator
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t w[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) w[k] = __float_as_uint(v[c * 16 + k]);
      tmem_st16(t_acc + half * 64 + c * 16, w);
    }
    tmem_wait_st();
    tc_fence_before();
    named_bar_sync(bar_id, 256);                                  // #1: both halves in TMEM; stage read
    tc_fence_after();
    if (leader && t + NS * t_step < n_tiles) { issue_load(t + NS * t_step, buf); ++issued[buf]; }
    const float n = sqrtf(myN2[trow] + otN2[trow]);
    const bool zero_row = !(n >= kZeroNorm);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t w[16];
      tmem_ld16(t_acc + (half ^ 1) * 64 + c * 16, w);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float o = __uint_as_float(w[k]);
        v[c * 16 + k] = half == 0 ? v[c * 16 + k] + o : o - v[c * 16 + k];
      }
    }

    // ---- Lloyd-Max codes and the residual (x 64) ----------------------------------
    // v holds y' = n sqrt(d) y; compare against per-row scaled thresholds; the
    // residual in unit-normalised units times 64 is r64 = y' sc64 - 64 c[code].
    const float nsd = zero_row ? 1.f : n * sqrt_d;
    const float sc64 = zero_row ? 0.f : kResScale / nsd;
    float tq[L - 1];
#pragma unroll
    for (int k = 0; k < L - 1; ++k) tq[k] = P.t[k] * nsd;
    uint32_t cw[B * 2];                                          // codes of my 64 coordinates
#pragma unroll
    for (int w = 0; w < B * 2; ++w) cw[w] = 0u;
    float2 r2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {                             // 32 coordinates, then their hi | lo words
#pragma unroll
      for (int e = ch * 32; e < ch * 32 + 32; ++e) {
        const float y = v[e];
        uint32_t code;
        float r;
        {
          code = 0u;
#pragma unroll
          for (int lev = B - 1; lev >= 0; --lev) {
            const int base = (1 << lev) - 1;
            float thr = tq[base];
#pragma unroll
            for (int k = 1; k < (1 << (B - 1 - lev)); ++k)
              if (code == static_cast<uint32_t>(k << (lev + 1))) thr = tq[base + (k << (lev + 1))];
            if (y > thr) code |= (1u << lev);
          }
          r = fmaf(y, sc64, -lut[code]);
        }
        if (zero_row) r = 0.f;
        v[e] = r;
        if (e & 1) r2.y = fmaf(r, r, r2.y); else r2.x = fmaf(r, r, r2.x);
        const int bit = B * e, wi = bit >> 5, sh = bit & 31;   // my 64 codes start word aligned
        cw[wi] |= code << sh;
        if (sh + B > 32) cw[wi + 1] |= code >> (32 - sh);
      }
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
    if (zero_row) {
#pragma unroll
      for (int w = 0; w < B * 2; ++w) cw[w] = 0u;
    }
    myR2[trow] = r2.x + r2.y;
    tmem_wait_st();
    tc_fence_before();
    // #2: A complete, exchange reads done; ORs everyone's view of the abort
    // flag so every thread of the pair takes the same decision
    if (named_bar_sync_or(bar_id, 256, *reinterpret_cast<volatile int*>(abort_flag) != 0)) break;
    const float rho = zero_row ? 0.f : sqrtf(myR2[trow] + otR2[trow]) * (1.0f / kResScale);

    // ---- projection on the tensor cores: P = [hi | lo] [S ; S]^T ---------------------
    if (leader) {
      tc_fence_after();
      const uint32_t sbase = smem_u32(sS);
      const uint32_t idesc = idesc_f16_f32(kTile, kM);
      const uint32_t d_tmem = tmem + pair * 256;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int kk = k & 7;                                      // K step within S (16 columns each)
        const uint64_t bdesc = smem_desc_sw128(sbase + (kk >> 2) * 16384 + (kk & 3) * 32, 1024);
        mma_f16_ts(d_tmem, d_tmem + 128 + k * 8, bdesc, idesc, k > 0 ? 1u : 0u);
      }
      mma_commit(&mdone[pair]);
    }
    if (!mbar_wait(&mdone[pair], mine & 1, kWaitCycles)) flag_error(X.err, abort_flag, 3);
    tc_fence_after();

    // ---- my 64 signs, exact recomputation within the error bound of zero ------------
    const float eps = kResScale * fmaf(X.eps_scale, rho, X.eps_abs);   // in the MMA's (scaled) units
    uint32_t s0 = 0, s1 = 0, f0 = 0, f1 = 0;
    float pmin = INFINITY;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t p[16];
      tmem_ld16(t_acc + half * 64 + c * 16, p);
      tmem_wait_ld();
      uint32_t bits = 0u;
#pragma unroll
      for (int j = 15; j >= 0; --j) {
        bits = (bits << 1) | (p[j] >> 31);
        pmin = fminf(pmin, fabsf(__uint_as_float(p[j])));
      }
      if (c == 0) s0 = bits;
      if (c == 1) s0 |= bits << 16;
      if (c == 2) s1 = bits;
      if (c == 3) s1 |= bits << 16;
    }
    // rare: find which projections are within the bound.  The TMEM loads are
    // warp-collective, so the whole warp takes this branch when any lane needs it.
    if (__any_sync(0xffffffffu, pmin < eps)) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t p[16];
        tmem_ld16(t_acc + half * 64 + c * 16, p);
        tmem_wait_ld();
        uint32_t flags = 0u;
#pragma unroll
        for (int j = 15; j >= 0; --j) flags = (flags << 1) | (fabsf(__uint_as_float(p[j])) < eps ? 1u : 0u);
        if (c == 0) f0 = flags;
        if (c == 1) f0 |= flags << 16;
        if (c == 2) f1 = flags;
        if (c == 3) f1 |= flags << 16;
      }
    }
    const int nflag = __popc(f0) + __popc(f1);
    const int passes = __reduce_max_sync(0xffffffffu, static_cast<unsigned>(nflag));
    for (int q = 0; q < passes; ++q) {
      int j = -1;                                                  // local index in [0, 64)
      if (q < nflag) {
        if (f1) j = 32 + __ffs(f1) - 1;
        if (f0) j = __ffs(f0) - 1;
      }
      const int jg = half * 64 + (j < 0 ? 0 : j);                  // projection index
      float acc = 0.f;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {                                // 8 residual pairs (16 entries) at a time
        uint32_t ah[8], al[8];
        tmem_ld8(t_a + c * 8, ah);
        tmem_ld8(t_a + 64 + c * 8, al);
        tmem_wait_ld();
        if (j >= 0) {
#pragma unroll
          for (int qq = 0; qq < 2; ++qq) {                         // 16-byte chunks of S row jg: 8 entries
            const int chunk = c * 2 + qq, kb = chunk >> 3, cc = chunk & 7;
            const uint4 sv = *reinterpret_cast<const uint4*>(sS + kb * 16384 + jg * 128 + ((cc ^ (jg & 7)) << 4));
            const uint32_t sws[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int w = qq * 4 + u;
              const float2 sf = __half22float2(*reinterpret_cast<const __half2*>(&sws[u]));
              const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&ah[w]));
              const float2 lf = __half22float2(*reinterpret_cast<const __half2*>(&al[w]));
              acc = fmaf(sf.x, hf.x + lf.x, acc);
              acc = fmaf(sf.y, hf.y + lf.y, acc);
            }
          }
        }
      }
      if (j >= 0) {
        const uint32_t m = 1u << (j & 31), nb = acc < 0.f ? m : 0u;
        if (j < 32) { s0 = (s0 & ~m) | nb; f0 &= ~m; }
        else { s1 = (s1 & ~m) | nb; f1 &= ~m; }
      }
    }
    if (zero_row || rho == 0.f) s0 = s1 = 0u;
    tc_fence_before();

    // ---- stores: my half of the codes and signs; norms from half 0 ------------------
    const int64_t row = t * kTile + trow;
    if (row < n_rows) {
      uint32_t* co = reinterpret_cast<uint32_t*>(out.codes + row * (B * 16) + half * (B * 8));
      if constexpr (B == 1) {
        *reinterpret_cast<uint2*>(co) = make_uint2(cw[0], cw[1]);
      } else if constexpr (B == 2) {
        *reinterpret_cast<uint4*>(co) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      } else if constexpr (B == 3) {
        // 24 bytes per half: half 0 at row offset 0 (16 + 8), half 1 at 24 (8 + 16),
        // so that each 16-byte store stays 16-byte aligned
        if (half == 0) {
          *reinterpret_cast<uint4*>(co) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
          *reinterpret_cast<uint2*>(co + 4) = make_uint2(cw[4], cw[5]);
        } else {
          *reinterpret_cast<uint2*>(co) = make_uint2(cw[0], cw[1]);
          *reinterpret_cast<uint4*>(co + 2) = make_uint4(cw[2], cw[3], cw[4], cw[5]);
        }
      } else {
        *reinterpret_cast<uint4*>(co) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        *reinterpret_cast<uint4*>(co + 4) = make_uint4(cw[4], cw[5], cw[6], cw[7]);
      }
      *reinterpret_cast<uint2*>(out.signs + row * 16 + half * 8) = make_uint2(s0, s1);
      if (half == 0) {
        out.norm[row] = zero_row ? 0.f : n;
        out.rnorm[row] = zero_row ? 0.f : n * rho;
      }
    }
  }

  // ---- teardown: no TMA load of ours may still be in flight ----------------------
  if (leader) {
    for (int b2 = 0; b2 < 2; ++b2)
      while (waited[b2] < issued[b2]) {
        if (!mbar_wait(&pfull[b2], waited[b2] & 1, kWaitCycles)) { flag_error(X.err, abort_flag, 4); break; }
        ++waited[b2];
      }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// bf16 rows: the rotation itself on the tensor cores.  y' = H D x is a
// 128 x 128 x 128 product per tile with the x tile straight from its TMA stage
// (the 128-byte-swizzled layout the TMA writes is the MMA's K-major operand
// layout) and B = D H as bf16 +-1 values (exact products, fp32 accumulation),
// so no widening, no butterflies and no cross-thread exchange run on the CUDA
// cores.  Each thread reads its 64 rotated values from TMEM, the two halves of
// a row add their sums of squares through shared memory (||y'|| = sqrt(d) n),
// and the codes, residual and projection follow.
//
// Codes from the symmetric codebook (c[L-1-k] = -c[k], t[L/2-1] = 0, exact
// in fp32): with u = |y'|, the code's top bit is s = [y' > 0] and the rest is
// the magnitude index k = #{j : T_j < u} over the positive thresholds
// T_j = t[L/2 + j] n sqrt(d), complemented when s = 0 (code = L/2 + k or
// L/2 - 1 - k).  Each decision is the sign of an exact difference (T - u,
// 0 - y'), funnel-shifted into the packed words; the complement is applied
// to whole words afterwards.  The residual is r = +-(u 64 / (n sqrt(d)) -
// 64 c[L/2 + k]) with the centroid picked by bit masks from those signs.
// A value exactly equal (in fp32) to a negative scaled threshold lands in
// the upper of its two cells, every other value where the definition puts
// it; such ties lie inside the 1e-6 band in which a code may differ from the
// fp64 decision.
template <int B>
struct SymConsts {
  static constexpr int kMag = B - 1;                       // magnitude bits
  static constexpr int kNT = (1 << kMag) - 1;              // positive thresholds
  static constexpr int kNC = 1 << kMag;                    // centroid magnitudes
};

// one coordinate: pushes its B code bits (top bit s, then the magnitude bits
// from the highest, not yet complemented) into the running words and returns
// the residual x 64.  POS = B e, the position of the code's lowest bit (a
// constant once the caller's loops are unrolled, so cw stays in registers).
template <int B>
__device__ __forceinline__ float quant_coord(float y, const float* T, const uint32_t* nc, float sc,
                                             uint32_t* cw, const int POS) {
  const float sp = 0.f - y;                                  // negative iff y > 0 (0 - 0 = +0)
  const float u = fabsf(y);
  uint32_t negc;                                             // -64 c[L/2 + k] as fp32 bits
  cw[(POS + B - 1) >> 5] = __funnelshift_l(__float_as_uint(sp), cw[(POS + B - 1) >> 5], 1);
  if constexpr (B == 1) {
    negc = nc[0];
  } else if constexpr (B == 2) {
    const float d = T[0] - u;                                // negative iff u > T
    cw[POS >> 5] = __funnelshift_l(__float_as_uint(d), cw[POS >> 5], 1);
    const uint32_t m = static_cast<uint32_t>(static_cast<int>(__float_as_uint(d)) >> 31);
    negc = (m & (nc[0] ^ nc[1])) ^ nc[0];
  } else if constexpr (B == 3) {
    const float d2 = T[1] - u;
    cw[(POS + 1) >> 5] = __funnelshift_l(__float_as_uint(d2), cw[(POS + 1) >> 5], 1);
    const uint32_t m2 = static_cast<uint32_t>(static_cast<int>(__float_as_uint(d2)) >> 31);
    const uint32_t tb = (m2 & __float_as_uint(T[2])) | (~m2 & __float_as_uint(T[0]));
    const float d0 = __uint_as_float(tb) - u;
    cw[POS >> 5] = __funnelshift_l(__float_as_uint(d0), cw[POS >> 5], 1);
    const uint32_t m0 = static_cast<uint32_t>(static_cast<int>(__float_as_uint(d0)) >> 31);
    const uint32_t ca = (m2 & nc[2]) | (~m2 & nc[0]);
    const uint32_t cb = (m2 & nc[3]) | (~m2 & nc[1]);
    negc = (m0 & cb) | (~m0 & ca);
  } else {
    // three magnitude bits: binary search T[3], then T[1] / T[5], then T[0..6 even]
    const float d2 = T[3] - u;
    cw[(POS + 2) >> 5] = __funnelshift_l(__float_as_uint(d2), cw[(POS + 2) >> 5], 1);
    const uint32_t m2 = static_cast<uint32_t>(static_cast<int>(__float_as_uint(d2)) >> 31);
    const uint32_t t1 = (m2 & __float_as_uint(T[5])) | (~m2 & __float_as_uint(T[1]));
    const float d1 = __uint_as_float(t1) - u;
    cw[(POS + 1) >> 5] = __funnelshift_l(__float_as_uint(d1), cw[(POS + 1) >> 5], 1);
    const uint32_t m1 = static_cast<uint32_t>(static_cast<int>(__float_as_uint(d1)) >> 31);
    const uint32_t lo = (m2 & __float_as_uint(T[4])) | (~m2 & __float_as_uint(T[0]));
    const uint32_t hi = (m2 & __float_as_uint(T[6])) | (~m2 & __float_as_uint(T[2]));
    const float d0 = __uint_as_float((m1 & hi) | (~m1 & lo)) - u;
    cw[POS >> 5] = __funnelshift_l(__float_as_uint(d0), cw[POS >> 5], 1);
    const uint32_t m0 = static_cast<uint32_t>(static_cast<int>(__float_as_uint(d0)) >> 31);
    uint32_t c4[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) c4[q] = (m2 & nc[4 + q]) | (~m2 & nc[q]);
    const uint32_t c2a = (m1 & c4[2]) | (~m1 & c4[0]);
    const uint32_t c2b = (m1 & c4[3]) | (~m1 & c4[1]);
    negc = (m0 & c2b) | (~m0 & c2a);
  }
  const float rm = fmaf(u, sc, __uint_as_float(negc));
  return __uint_as_float(__float_as_uint(rm) ^ (~__float_as_uint(sp) & 0x80000000u));
}

// Two coordinates at once (e0 and e1 = e0 + 1, stream positions POS0 = B e0
// and POS0 + B) with packed fp32 arithmetic.  Decisions are the signs of
// T^2 - y^2 (one rounding, so a decision can differ from the exact one only
// for |y| within about one ulp of a threshold), the code bits are pushed
// from the highest stream position down, and the residual x 64 comes back
// as y sc - (+-64 c[L/2 + k]) in one packed FMA.  T2: squared magnitude
// thresholds; nc: -64 c[L/2 + k] as fp32 bits.
__device__ __forceinline__ uint32_t sel_neg(uint32_t m, uint32_t a, uint32_t b) {   // m all-ones: a, else b
  return (m & a) | (~m & b);
}
__device__ __forceinline__ uint32_t sign_mask(float v) {
  return static_cast<uint32_t>(static_cast<int>(__float_as_uint(v)) >> 31);
}
template <int B>
__device__ __forceinline__ float2 quant_pair(float y0, float y1, const float* T2, const uint32_t* nc, float sc,
                                             uint32_t* cw, const int POS0) {
  const float2 y = make_float2(y0, y1);
  const float2 sp = __ffma2_rn(y, make_float2(-1.f, -1.f), make_float2(0.f, 0.f));   // negative iff y > 0
  const int P1 = POS0 + B;
  auto push = [&](int pos, float v) { cw[pos >> 5] = __funnelshift_l(__float_as_uint(v), cw[pos >> 5], 1); };
  uint32_t n0, n1;                                         // -64 c[L/2 + k] of each coordinate
  if constexpr (B == 1) {
    push(P1, sp.y);
    push(POS0, sp.x);
    n0 = n1 = nc[0];
  } else if constexpr (B == 2) {
    const float2 d = __ffma2_rn(sp, y, make_float2(T2[0], T2[0]));
    push(P1 + 1, sp.y); push(P1, d.y);
    push(POS0 + 1, sp.x); push(POS0, d.x);
    // k = [d < 0] as 0.0 / 1.0 (|d| is 0 or far above 2^-126 for any row above
    // the zero-norm cut), then -64 c[L/2 + k] = k (-c1) + (1 - k) (-c0) with one
    // of the two terms exactly zero, so the centroid is exact
    const float2 kk = make_float2(__saturatef(d.x * -8.507059e37f), __saturatef(d.y * -8.507059e37f));
    const float c0 = __uint_as_float(nc[0]), c1 = __uint_as_float(nc[1]);
    const float2 lo = __ffma2_rn(kk, make_float2(-c0, -c0), make_float2(c0, c0));
    const float2 nv = __ffma2_rn(kk, make_float2(c1, c1), lo);
    n0 = __float_as_uint(nv.x);
    n1 = __float_as_uint(nv.y);
  } else if constexpr (B == 3) {
    const float2 d2 = __ffma2_rn(sp, y, make_float2(T2[1], T2[1]));
    const uint32_t m2a = sign_mask(d2.x), m2b = sign_mask(d2.y);
    const uint32_t t2 = __float_as_uint(T2[2]), t0 = __float_as_uint(T2[0]);
    const float2 d0 = __ffma2_rn(sp, y, make_float2(__uint_as_float(sel_neg(m2a, t2, t0)),
                                                    __uint_as_float(sel_neg(m2b, t2, t0))));
    push(P1 + 2, sp.y); push(P1 + 1, d2.y); push(P1, d0.y);
    push(POS0 + 2, sp.x); push(POS0 + 1, d2.x); push(POS0, d0.x);
    n0 = sel_neg(sign_mask(d0.x), sel_neg(m2a, nc[3], nc[1]), sel_neg(m2a, nc[2], nc[0]));
    n1 = sel_neg(sign_mask(d0.y), sel_neg(m2b, nc[3], nc[1]), sel_neg(m2b, nc[2], nc[0]));
  } else {
    // three magnitude bits: T[3], then T[1] / T[5], then T[0..6 even]
    const float2 d2 = __ffma2_rn(sp, y, make_float2(T2[3], T2[3]));
    const uint32_t m2a = sign_mask(d2.x), m2b = sign_mask(d2.y);
    const uint32_t t5 = __float_as_uint(T2[5]), t1 = __float_as_uint(T2[1]);
    const float2 d1 = __ffma2_rn(sp, y, make_float2(__uint_as_float(sel_neg(m2a, t5, t1)),
                                                    __uint_as_float(sel_neg(m2b, t5, t1))));
    const uint32_t m1a = sign_mask(d1.x), m1b = sign_mask(d1.y);
    const uint32_t t4 = __float_as_uint(T2[4]), t0 = __float_as_uint(T2[0]);
    const uint32_t t6 = __float_as_uint(T2[6]), t2 = __float_as_uint(T2[2]);
    const uint32_t ta = sel_neg(m1a, sel_neg(m2a, t6, t2), sel_neg(m2a, t4, t0));
    const uint32_t tb = sel_neg(m1b, sel_neg(m2b, t6, t2), sel_neg(m2b, t4, t0));
    const float2 d0 = __ffma2_rn(sp, y, make_float2(__uint_as_float(ta), __uint_as_float(tb)));
    push(P1 + 3, sp.y); push(P1 + 2, d2.y); push(P1 + 1, d1.y); push(P1, d0.y);
    push(POS0 + 3, sp.x); push(POS0 + 2, d2.x); push(POS0 + 1, d1.x); push(POS0, d0.x);
    auto pick = [&](uint32_t m2, uint32_t m1, uint32_t m0) {
      const uint32_t c0 = sel_neg(m2, nc[4], nc[0]), c1 = sel_neg(m2, nc[5], nc[1]);
      const uint32_t c2 = sel_neg(m2, nc[6], nc[2]), c3 = sel_neg(m2, nc[7], nc[3]);
      return sel_neg(m0, sel_neg(m1, c3, c1), sel_neg(m1, c2, c0));
    };
    n0 = pick(m2a, m1a, sign_mask(d0.x));
    n1 = pick(m2b, m1b, sign_mask(d0.y));
  }
  // +-64 c: the sign of the cell's centroid follows the code's top bit
  const uint32_t q0 = n0 ^ (~__float_as_uint(sp.x) & 0x80000000u);
  const uint32_t q1 = n1 ^ (~__float_as_uint(sp.y) & 0x80000000u);
  return __ffma2_rn(y, make_float2(sc, sc), make_float2(__uint_as_float(q0), __uint_as_float(q1)));
}

// Mask of the stream positions p in [32 w, 32 w + 32) with p mod B == j
// (B in 2..4).
__device__ __forceinline__ uint32_t residue_mask(int B, int w, int j) {
  if (B == 3) {
    const int r = ((j - 2 * w) % 3 + 3) % 3;                  // 32 = 2 (mod 3)
    return r == 0 ? 0x49249249u : (r == 1 ? 0x92492492u : 0x24924924u);
  }
  return (B == 2 ? 0x55555555u : 0x11111111u) << j;
}

// Complement the magnitude bits of every code whose top bit (s) is 0: bit j
// of code i (position B i + j, j < B - 1) ^= !s_i (position B i + B - 1).
template <int B>
__device__ __forceinline__ void complement_negative_codes(uint32_t (&cw)[2 * B]) {
  if constexpr (B > 1) {
    uint32_t fix[2 * B];
#pragma unroll
    for (int w = 0; w < 2 * B; ++w) fix[w] = 0u;
#pragma unroll
    for (int j = 0; j < B - 1; ++j) {
      const int o = B - 1 - j;
#pragma unroll
      for (int w = 0; w < 2 * B; ++w) {
        const uint32_t above = w + 1 < 2 * B ? ~cw[w + 1] : 0u;
        fix[w] |= __funnelshift_r(~cw[w], above, o) & residue_mask(B, w, j);
      }
    }
#pragma unroll
    for (int w = 0; w < 2 * B; ++w) cw[w] ^= fix[w];
  }
}

// Complement the magnitude bits of every negative code (as above) in a run
// of NW words that starts on a word boundary of the code stream where no code
// straddles the run's ends (NW = B: 32 coordinates).
template <int B, int NW>
__device__ __forceinline__ void complement_negative_codes_run(uint32_t (&cw)[NW]) {
  if constexpr (B > 1) {
    uint32_t fix[NW];
#pragma unroll
    for (int w = 0; w < NW; ++w) fix[w] = 0u;
#pragma unroll
    for (int j = 0; j < B - 1; ++j) {
      const int o = B - 1 - j;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const uint32_t above = w + 1 < NW ? ~cw[w + 1] : 0u;
        fix[w] |= __funnelshift_r(~cw[w], above, o) & residue_mask(B, w, j);
      }
    }
#pragma unroll
    for (int w = 0; w < NW; ++w) cw[w] ^= fix[w];
  }
}

// mbarrier phase test that may suspend the thread until the phase completes
// (or about 20 us pass)
__device__ __forceinline__ bool try_wait_suspend(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 20000;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// min(|a|, |b|, c) in one three-input minimum
__device__ __forceinline__ float min3_abs(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(fabsf(a)), "f"(fabsf(b)), "f"(c));
  return d;
}

// bf16 rows, warp-specialized.  Sixteen compute warps share every 128-row
// tile: warp w owns coordinates (and projections) [32 g, 32 g + 32), g = w / 4,
// of rows 32 (w % 4) .. + 31, each row in the TMEM lane of its index, so the
// four threads of a row sit in the four warps of one lane quadrant.  A
// seventeenth warp issues everything asynchronous: the TMA loads of the row
// tiles (a ring of four stages), the rotation y' = x (D H)^T (A = the TMA
// stage, B = D H as bf16 +-1, exact products, fp32 sums) and the projection
// p = (64 r) S^T from the residual's binary16 hi | lo parts (K = 256).
//
// TMEM holds four 128-column regions.  Tile k reads y' from region Y(k),
// writes its residual to Z(k), and gets p back in Y(k); the next tile of the
// same parity uses the regions the other way round (Y(k + 2) = Z(k)), so the
// rotation of tile k + 2 runs as soon as the projection of tile k has read
// its residual, and two tiles are always in flight: the compute warps turn
// tile k into codes while the tensor cores finish the projection of tile
// k - 1, whose signs are taken next.  A thread reads and writes the same
// 32 columns of every region: y' and p of its coordinates / projections and,
// in Z, the hi parts (16 columns) then the lo parts of its 32 residuals, so
// no thread ever overwrites a column another thread still has to read.  The
// projection's K order is hi(0..31) lo(0..31) hi(32..63) ..., and its B
// operand (S) is addressed to match.
//
// Codes, residual and the tensor-core error bound are those of the kernel
// above; projections inside the bound go to the exact fix-up kernel.
// Shape of the kernel for rows of KD coordinates (m = KD projections): KD / 32
// threads per row, 32 coordinates each, so KD / 8 compute warps; TMEM regions
// of KD columns (four of them); the row-tile stages hold KD / 64 boxes of 64
// bf16 columns.  At KD = 64 two CTAs share an SM (256 TMEM columns each).
template <int KD>
struct WsShape {
  static constexpr int kG = KD / 32;                 // threads per row
  static constexpr int kCompute = KD / 8;            // compute warps
  static constexpr int kThreads = (kCompute + 1) * 32;
  static constexpr int kStages = 4;                  // row tiles in shared memory
  static constexpr int kStage = (KD / 64) * kTile * 128;
  static constexpr int kOpBytes = KD * KD * 2;       // S or D H as a 16-bit MMA operand
  static constexpr uint32_t kTmemCols = 4 * KD;
  static constexpr int kCtasPerSm = KD == 64 ? 2 : 1;
};

template <int KD>
constexpr size_t quant_ws_smem_bytes() {
  using W = WsShape<KD>;
  return 1024 + 2 * W::kOpBytes + W::kStages * W::kStage + 2 * W::kG * kTile * 4 /*norm partials*/ +
         2 * W::kG * kTile * 4 /*residual partials*/ + 2 * W::kCompute * 32 * 4 /*norms*/ + 256;
}

template <int B, int KD>
__global__ void __launch_bounds__(WsShape<KD>::kThreads, WsShape<KD>::kCtasPerSm)
k_quantize_d128_ws(const __grid_constant__ CUtensorMap tmap, const KParams P, const QuantD128Args X,
                   int64_t n_rows, const Packed out) {
  using W = WsShape<KD>;
  constexpr int L = 1 << B;
  constexpr int kStage = W::kStage;
  constexpr int kWsStages = W::kStages;
  constexpr int kWsCompute = W::kCompute;
  constexpr int kWsThreads = W::kThreads;
  constexpr int kG = W::kG;
  constexpr int kNT = SymConsts<B>::kNT > 0 ? SymConsts<B>::kNT : 1;
  constexpr int kNC = SymConsts<B>::kNC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sS = smem;                                            // projection B operand (S, fp16)
  uint8_t* sHD = smem + W::kOpBytes;                             // rotation B operand (D H, bf16 +-1)
  uint8_t* stages = sHD + W::kOpBytes;                           // [kWsStages] row tiles
  float* sN2 = reinterpret_cast<float*>(stages + kWsStages * kStage);   // [2][kG][row] partial ||y'||^2
  float* sR2 = sN2 + 2 * kG * kTile;                             // [2][kG][row] partial ||64 r||^2
  float* sNrm = sR2 + 2 * kG * kTile;                            // [2][compute thread] norms awaiting signs
  uint64_t* full = reinterpret_cast<uint64_t*>(sNrm + 2 * kWsCompute * 32);   // [kWsStages]
  uint64_t* yrdy = full + kWsStages;                             // [2] rotation done
  uint64_t* prdy = yrdy + 2;                                     // [2] projection done
  uint64_t* rrdy = prdy + 2;                                     // [2] residual written (one arrival per compute warp)
  uint64_t* nrdy = rrdy + 2;                                     // [2] norm partials written (likewise)
  uint64_t* fdone = nrdy + 2;                                    // wind-down commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fdone + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_tiles = (n_rows + kTile - 1) / kTile;
  const int64_t n_mine = n_tiles > blockIdx.x ? (n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  const long long wait_cycles = X.wait_cycles;
  if (tid == 0) {
    for (int i = 0; i < kWsStages; ++i) mbar_init(&full[i], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&yrdy[i], 1);
      mbar_init(&prdy[i], 1);
      mbar_init(&rrdy[i], kWsCompute);
      mbar_init(&nrdy[i], kWsCompute);
    }
    mbar_init(fdone, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  // S (m = KD rows of KD coordinates) and D H, K-major, 64-coordinate atoms of KD rows
  for (int e = tid; e < KD * (KD / 8); e += kWsThreads) {
    const int j = e / (KD / 8), c = e % (KD / 8), kb = c >> 3, cc = c & 7;
    const uint4 v = *reinterpret_cast<const uint4*>(P.S + j * KD + c * 8);
    *reinterpret_cast<uint4*>(sS + kb * (KD * 128) + j * 128 + ((cc ^ (j & 7)) << 4)) = v;
  }
  // (D H)[n][k] = H[n][k] D_k = (-1)^popcount(n & k) D_k, as bf16 +-1.0, same swizzled layout
  uint16_t* hd16 = reinterpret_cast<uint16_t*>(sHD);
  for (int e = tid; e < KD * KD; e += kWsThreads) {
    const int n = e / KD, k = e % KD;
    const bool neg = ((__popc(n & k) & 1) != 0) != (X.Dsign[k] != 0u);
    const int kb = k >> 6, chunk = (k & 63) >> 3, within = k & 7;
    hd16[(kb * (KD * 128) + n * 128 + ((chunk ^ (n & 7)) << 4)) / 2 + within] = neg ? 0xBF80u : 0x3F80u;
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(tmem_slot, W::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // regions of local tile k: Y (y', then p) and Z (residual hi | lo)
  auto region_y = [](int64_t k) { return static_cast<uint32_t>(2 * (k & 1) + ((k >> 1) & 1)) * KD; };
  auto region_z = [](int64_t k) { return static_cast<uint32_t>(2 * (k & 1) + 1 - ((k >> 1) & 1)) * KD; };
  // a bounded wait that also gives up once another thread has flagged an
  // abort; with a limit of a second or so a waiting thread is suspended
  // between polls (so the waiting warps leave the issue slots to the others),
  // with a short limit it polls and keeps to the cycle count
  const bool suspend = wait_cycles >= (1ll << 24);
  auto wait_or_abort = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!(suspend ? try_wait_suspend(bar, parity) : mbar_try_wait(bar, parity))) {
      if (*reinterpret_cast<volatile int*>(abort_flag) != 0) return false;
      if (clock64() - t0 > wait_cycles) return false;
    }
    return true;
  };

  if (warp == kWsCompute) {
    // ================================ control warp ================================
    if (lane == 0) {
      prefetch_tmap(&tmap);
      int64_t loads = 0, landed = 0;                             // stage loads issued / waited for
      bool mma_issued = false;
      auto tile_of = [&](int64_t k) { return static_cast<int64_t>(blockIdx.x) + k * gridDim.x; };
      auto issue_load = [&](int64_t k) {
        const int st = static_cast<int>(k % kWsStages);
        mbar_arrive_expect_tx(&full[st], kStage);
#pragma unroll
        for (int bx = 0; bx < KD / 64; ++bx)
          tma_load_2d(stages + st * kStage + bx * (kTile * 128), &tmap, &full[st], bx * 64,
                      static_cast<int>(tile_of(k) * kTile));
        ++loads;
      };
      // rotation of local tile k into Y(k); false if its stage never arrived
      auto rotate = [&](int64_t k) -> bool {
        const int st = static_cast<int>(k % kWsStages);
        if (!wait_or_abort(&full[st], static_cast<uint32_t>((k / kWsStages) & 1))) return false;
        ++landed;
        tc_fence_after();
        const uint32_t xbase = smem_u32(stages + st * kStage), hbase = smem_u32(sHD);
        const uint32_t idesc = idesc_bf16_f32(kTile, KD);
        const uint32_t d_tmem = tmem + region_y(k);
#pragma unroll
        for (int kk = 0; kk < KD / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * (kTile * 128) + (kk & 3) * 32;
          const uint32_t boff = (kk >> 2) * (KD * 128) + (kk & 3) * 32;
          mma_f16_ss(d_tmem, smem_desc_sw128(xbase + aoff, 1024), smem_desc_sw128(hbase + boff, 1024), idesc,
                     kk > 0 ? 1u : 0u);
        }
        mma_commit(&yrdy[k & 1]);
        mma_issued = true;
        return true;
      };
      bool ok = true;
      for (int64_t k = 0; k < kWsStages && k < n_mine; ++k) issue_load(k);
      for (int64_t k = 0; k < 2 && k < n_mine && ok; ++k) ok = rotate(k);
      for (int64_t k = 0; k < n_mine && ok; ++k) {
        const uint32_t ph = static_cast<uint32_t>((k >> 1) & 1);
        if (!wait_or_abort(&rrdy[k & 1], ph)) { ok = false; break; }
        tc_fence_after();
        // tile k's stage was read by its rotation (the compute warps waited for it)
        if (k + kWsStages < n_mine) issue_load(k + kWsStages);
        {
          const uint32_t sbase = smem_u32(sS);
          const uint32_t idesc = idesc_f16_f32(kTile, KD);
          const uint32_t d_tmem = tmem + region_y(k), a_tmem = tmem + region_z(k);
#pragma unroll
          for (int kk = 0; kk < 2 * KD / 16; ++kk) {
            // A step kk: hi (kk & 2 == 0) or lo parts of coordinates 32 (kk >> 2) + 16 (kk & 1) .. + 15
            const int sk = 2 * (kk >> 2) + (kk & 1);
            const uint64_t bdesc = smem_desc_sw128(sbase + (sk >> 2) * (KD * 128) + (sk & 3) * 32, 1024);
            mma_f16_ts(d_tmem, a_tmem + kk * 8, bdesc, idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(&prdy[k & 1]);
        }
        if (k + 2 < n_mine) {
          // Y(k + 2) = Z(k): free once this projection has read it
          if (!wait_or_abort(&prdy[k & 1], ph)) { ok = false; break; }
          ok = rotate(k + 2);
        }
      }
      if (!ok) {
        if (X.err) atomicCAS(X.err, 0, 2);
        atomicExch(abort_flag, 1);
      }
      // wind-down with the full limit: no MMA of ours still running, no stage load still landing
      if (mma_issued) {
        mma_commit(fdone);
        if (!mbar_wait(fdone, 0, kWaitCycles)) flag_error(X.err, abort_flag, 4);
      }
      for (; landed < loads; ++landed)
        if (!mbar_wait(&full[landed % kWsStages], static_cast<uint32_t>((landed / kWsStages) & 1), kWaitCycles)) {
          flag_error(X.err, abort_flag, 4);
          break;
        }
    }
  } else {
    // ================================ compute warps ================================
    const int quad = warp & 3, g = warp >> 2;                    // g < kG
    const int trow = quad * 32 + lane;
    const uint32_t tbase = tmem + (static_cast<uint32_t>(quad * 32) << 16) + 32 * g;   // my lane, my columns
    const int n_k = static_cast<int>(n_mine);
    // this thread's row of local tile k is row0 + k * row_step (below 2^31:
    // the kernel takes fewer than 2^31 - 256 rows)
    const int row0 = static_cast<int>(blockIdx.x) * kTile + trow;
    const int row_step = static_cast<int>(gridDim.x) * kTile;
    const int nr = static_cast<int>(n_rows);
    // each tile's norm (0 for a zero row) waits in shared memory for its signs
    float* my_norm = sNrm + tid;                                 // [2][compute threads]
    // region offsets of local tile k: Y = 2 KD (k & 1) + KD ((k >> 1) & 1), Z = Y ^ KD
    constexpr int kLog = KD == 128 ? 7 : 6;
    auto off_y = [](int k) { return static_cast<uint32_t>(((k & 1) << (kLog + 1)) | ((k & 2) << (kLog - 1))); };
    // the sum of the kG partial ||64 r||^2 of tile k (written before rrdy(k))
    auto resid2 = [&](int k) {
      const float* r2 = sR2 + (k & 1) * kG * kTile + trow;
      return kG == 4 ? (r2[0] + r2[kTile]) + (r2[2 * kTile] + r2[3 * kTile]) : r2[0] + r2[kTile];
    };
    // signs of local tile k (its projection), exact recomputation listed within the error bound
    auto signs = [&](int k, float rr) {
      if (!wait_or_abort(&prdy[k & 1], static_cast<uint32_t>((k >> 1) & 1))) {
        flag_error(X.err, abort_flag, 3);
        return;
      }
      tc_fence_after();
      const float nk = my_norm[(k & 1) * (kWsCompute * 32)];
      const bool zero = nk == 0.f;
      const float rho = zero ? 0.f : sqrtf(rr) * (1.0f / kResScale);
      const float eps = kResScale * fmaf(X.eps_scale, rho, X.eps_abs);
      uint32_t p[32];
      tmem_ld32(tbase + off_y(k), p);
      tmem_wait_ld();
      uint32_t sw = 0u;
#pragma unroll
      for (int j = 31; j >= 0; --j) sw = __funnelshift_l(p[j], sw, 1);
      float pmin = INFINITY;
#pragma unroll
      for (int j = 0; j < 32; j += 2) pmin = min3_abs(__uint_as_float(p[j]), __uint_as_float(p[j + 1]), pmin);
      const int row = row0 + k * row_step;
      const bool live = row < nr;
      if (pmin < eps && !zero && rho != 0.f && live) {
        // rare: list each projection inside the bound for the fix-up kernel;
        // a row whose entries do not all fit is marked for a full recomputation
        uint32_t f = 0u;
#pragma unroll
        for (int j = 31; j >= 0; --j) f = (f << 1) | (fabsf(__uint_as_float(p[j])) < eps ? 1u : 0u);
        unsigned int slot = atomicAdd(X.fix_count, static_cast<unsigned int>(__popc(f)));
        while (f) {
          const int j = 32 * g + __ffs(f) - 1;
          if (slot < X.fix_cap)
            X.fix_list[slot] = (static_cast<unsigned long long>(row) << 8) | static_cast<unsigned>(j);
          ++slot;
          f &= f - 1;
        }
        if (slot > X.fix_cap) atomicOr(X.fix_rows + (row >> 5), 1u << (row & 31));
      }
      if (zero || rho == 0.f) sw = 0u;
      if (live) {
        reinterpret_cast<uint32_t*>(out.signs + static_cast<size_t>(row) * (KD / 8))[g] = sw;
        if (g == 0) out.rnorm[row] = zero ? 0.f : nk * rho;
      }
    };

    // Per tile k: y' -> partial ||y'||^2 -> arrive -> the signs of tile k - 2
    // (its projection finished long ago) while the other warps' partial sums
    // come in -> wait -> codes and residual -> arrive for the projection.
    int k = 0;
    for (; k < n_k; ++k) {
      const int row = row0 + k * row_step;
      const uint32_t oy = off_y(k);
      const uint32_t ph = static_cast<uint32_t>((k >> 1) & 1);
      if (!wait_or_abort(&yrdy[k & 1], ph)) { flag_error(X.err, abort_flag, 5); break; }
      tc_fence_after();
      uint32_t u[32];
      tmem_ld32(tbase + oy, u);
      tmem_wait_ld();
      {
        float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float2 a = make_float2(__uint_as_float(u[j]), __uint_as_float(u[j + 1]));
          const float2 b2 = make_float2(__uint_as_float(u[j + 2]), __uint_as_float(u[j + 3]));
          s0 = __ffma2_rn(a, a, s0);
          s1 = __ffma2_rn(b2, b2, s1);
        }
        sN2[(k & 1) * kG * kTile + g * kTile + trow] = (s0.x + s0.y) + (s1.x + s1.y);
      }
      // tile k - 2's residual partials share a buffer with this tile's: read
      // them before this warp's arrival lets the others write this tile's
      const float rr_old = k >= 2 ? resid2(k) : 0.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(&nrdy[k & 1]);
      if (k >= 2) signs(k - 2, rr_old);
      if (!wait_or_abort(&nrdy[k & 1], ph)) { flag_error(X.err, abort_flag, 5); break; }
      const float* n2 = sN2 + (k & 1) * kG * kTile + trow;
      const float ss = kG == 4 ? (n2[0] + n2[kTile]) + (n2[2 * kTile] + n2[3 * kTile]) : n2[0] + n2[kTile];
      const float nsd = sqrtf(ss);                               // ||H D x|| = sqrt(d) ||x||
      const float n = nsd * (KD == 128 ? 0.08838834764831845f : 0.125f);   // / sqrt(KD)
      const bool zero_row = !(n >= kZeroNorm);
      const float nsd_t = zero_row ? 1.f : nsd;
      const float sc = zero_row ? 0.f : kResScale * __frcp_rn(nsd_t);   // = RN(64 / nsd)
      // squared thresholds and the centroids (x 64, as negated fp32 bit
      // patterns) straight from the parameter space
      float T2[kNT];
      uint32_t nc[kNC];
#pragma unroll
      for (int j = 0; j < kNT; ++j) {
        const float tj = (B > 1 ? P.t[L / 2 + j] : 0.f) * nsd_t;
        T2[j] = tj * tj;
      }
#pragma unroll
      for (int c = 0; c < kNC; ++c) nc[c] = zero_row ? 0u : __float_as_uint(-kResScale * P.c[L / 2 + c]);

      // ---- codes and the residual (x 64): hi parts to Z + 32 g, lo parts to Z + 32 g + 16 ----
      uint32_t cw[B];
#pragma unroll
      for (int w = 0; w < B; ++w) cw[w] = 0u;
      float2 r2a = make_float2(0.f, 0.f), r2b = make_float2(0.f, 0.f);
      const uint32_t zb = tbase + (oy ^ static_cast<uint32_t>(KD));
#pragma unroll
      for (int g8 = 1; g8 >= 0; --g8) {                         // 16 coordinates -> 8 hi and 8 lo columns
        uint32_t hw[8], lw[8];
#pragma unroll
        for (int q = 7; q >= 0; --q) {
          const int e0 = g8 * 16 + 2 * q;
          const float2 rv = quant_pair<B>(__uint_as_float(u[e0]), __uint_as_float(u[e0 + 1]), T2, nc, sc, cw, B * e0);
          if (q & 1) r2a = __ffma2_rn(rv, rv, r2a); else r2b = __ffma2_rn(rv, rv, r2b);
          // hi = r rounded to binary16, lo = r - hi (exact in fp32), then rounded to binary16
          const __half2 h = __floats2half2_rn(rv.x, rv.y);
          const float2 lf = __ffma2_rn(__half22float2(h), make_float2(-1.f, -1.f), rv);
          const __half2 l = __floats2half2_rn(lf.x, lf.y);
          hw[q] = *reinterpret_cast<const uint32_t*>(&h);
          lw[q] = *reinterpret_cast<const uint32_t*>(&l);
        }
        tmem_st8(zb + g8 * 8, hw);
        tmem_st8(zb + 16 + g8 * 8, lw);
      }
      complement_negative_codes_run<B, B>(cw);
      if (zero_row) {
#pragma unroll
        for (int w = 0; w < B; ++w) cw[w] = 0u;
      }
      sR2[(k & 1) * kG * kTile + g * kTile + trow] = (r2a.x + r2a.y) + (r2b.x + r2b.y);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&rrdy[k & 1]);
      if (row < nr) {
        uint32_t* co = reinterpret_cast<uint32_t*>(out.codes + static_cast<size_t>(row) * (B * KD / 8)) + B * g;
        if constexpr (B == 1) {
          co[0] = cw[0];
        } else if constexpr (B == 2) {
          *reinterpret_cast<uint2*>(co) = make_uint2(cw[0], cw[1]);
        } else if constexpr (B == 3) {
          co[0] = cw[0]; co[1] = cw[1]; co[2] = cw[2];
        } else {
          *reinterpret_cast<uint4*>(co) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        }
        if (g == 0) out.norm[row] = zero_row ? 0.f : n;
      }
      my_norm[(k & 1) * (kWsCompute * 32)] = zero_row ? 0.f : n;
    }
    if (k == n_k) {
      // the last two tiles' signs, once every warp has written its residual partials
      for (int j = n_k >= 2 ? n_k - 2 : 0; j < n_k; ++j) {
        if (!wait_or_abort(&rrdy[j & 1], static_cast<uint32_t>((j >> 1) & 1))) {
          flag_error(X.err, abort_flag, 3);
          break;
        }
        signs(j, resid2(j));
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, W::kTmemCols);
  }
}

// Exact signs of the projections the tensor-core kernel left inside its
// error bound, in fp64 from the input row and the codes the kernel stored for
// it: norm, D, the Walsh-Hadamard butterflies, r = y - c[code], p_j = S_j . r,
// and the sign bit set or cleared in place (1 = negative; p_j = 0 counts as
// positive).  Listed (row, j) entries first, one warp each; then the rows
// marked in the overflow bitmap, all of whose m = KD signs are recomputed.
// Lane l holds coordinates V l .. V l + V - 1, V = KD / 32.
template <int B, bool BF16IN, int KD>
__device__ __forceinline__ void fixup_residual(const KParams& P, const void* __restrict__ x, int64_t ld, int64_t row,
                                               const Packed& out, int lane, double (&r)[KD / 32]) {
  constexpr int V = KD / 32;
  double v[V];
  if constexpr (BF16IN) {
    const uint16_t* xr = static_cast<const uint16_t*>(x) + row * ld + V * lane;
    if constexpr (V == 4) {
      const uint2 xw = *reinterpret_cast<const uint2*>(xr);
      v[0] = __uint_as_float(xw.x << 16); v[1] = __uint_as_float(xw.x & 0xffff0000u);
      v[2] = __uint_as_float(xw.y << 16); v[3] = __uint_as_float(xw.y & 0xffff0000u);
    } else {
      const uint32_t xw = *reinterpret_cast<const uint32_t*>(xr);
      v[0] = __uint_as_float(xw << 16); v[1] = __uint_as_float(xw & 0xffff0000u);
    }
  } else {
    const float* xr = static_cast<const float*>(x) + row * ld + V * lane;
#pragma unroll
    for (int q = 0; q < V; ++q) v[q] = xr[q];
  }
  // codes of coordinates V lane .. V lane + V - 1: bits [V B lane, V B lane + V B) of the row
  const uint8_t* cb = out.codes + row * (B * KD / 8);
  const int bit0 = V * B * lane;
  uint32_t win = 0;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int byte = (bit0 >> 3) + k;
    if (byte < B * KD / 8) win |= static_cast<uint32_t>(cb[byte]) << (8 * k);
  }
  win >>= (bit0 & 7);
  const uint32_t dm = P.Dmask[(V * lane) >> 5] >> ((V * lane) & 31);
  double ss = 0.0;
#pragma unroll
  for (int q = 0; q < V; ++q) {
    if ((dm >> q) & 1u) v[q] = -v[q];
    ss = fma(v[q], v[q], ss);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  // butterflies over the coordinate bits inside the lane, then across lanes
#pragma unroll
  for (int h = 1; h < V; h <<= 1)
#pragma unroll
    for (int q = 0; q < V; ++q)
      if ((q & h) == 0) {
        const double a = v[q], c2 = v[q + h];
        v[q] = a + c2;
        v[q + h] = a - c2;
      }
#pragma unroll
  for (int lh = 1; lh < 32; lh <<= 1)
#pragma unroll
    for (int q = 0; q < V; ++q) {
      const double o = __shfl_xor_sync(0xffffffffu, v[q], lh);
      v[q] = (lane & lh) ? o - v[q] : v[q] + o;
    }
  const double inv = 1.0 / (sqrt(ss) * sqrt(static_cast<double>(KD)));
#pragma unroll
  for (int q = 0; q < V; ++q) {
    const uint32_t code = (win >> (B * q)) & ((1u << B) - 1u);
    r[q] = v[q] * inv - static_cast<double>(P.c[code]);
  }
}

// S_j . r over the warp (lane l: coordinates V l .. V l + V - 1), all lanes get it
template <int KD>
__device__ __forceinline__ double fixup_project(const KParams& P, int j, int lane, const double (&r)[KD / 32]) {
  constexpr int V = KD / 32;
  double p = 0.0;
  if constexpr (V == 4) {
    const uint2 sw = __ldg(reinterpret_cast<const uint2*>(P.S + j * KD + 4 * lane));
    const float2 s01 = __half22float2(*reinterpret_cast<const __half2*>(&sw.x));
    const float2 s23 = __half22float2(*reinterpret_cast<const __half2*>(&sw.y));
    p = static_cast<double>(s01.x) * r[0];
    p = fma(static_cast<double>(s01.y), r[1], p);
    p = fma(static_cast<double>(s23.x), r[2], p);
    p = fma(static_cast<double>(s23.y), r[3], p);
  } else {
    const uint32_t sw = __ldg(reinterpret_cast<const uint32_t*>(P.S + j * KD + 2 * lane));
    const float2 s01 = __half22float2(*reinterpret_cast<const __half2*>(&sw));
    p = static_cast<double>(s01.x) * r[0];
    p = fma(static_cast<double>(s01.y), r[1], p);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
  return p;
}

template <int B, bool BF16IN, int KD>
__global__ void __launch_bounds__(256)
k_qjl_fixup_d128(const KParams P, const void* __restrict__ x, int64_t ld, int64_t n_rows, const Packed out,
                 const unsigned long long* __restrict__ fix_list, const unsigned int* __restrict__ fix_count,
                 unsigned int fix_cap, const unsigned int* __restrict__ fix_rows) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const unsigned int claimed = *fix_count;
  const int64_t n_list = claimed < fix_cap ? claimed : fix_cap;
  for (int64_t e = warp; e < n_list; e += nwarps) {
    const unsigned long long ent = fix_list[e];
    const int64_t row = static_cast<int64_t>(ent >> 8);
    const int j = static_cast<int>(ent & 0xffu);
    if (row >= n_rows || j >= KD) continue;                      // never listed; kept in bounds regardless
    double r[KD / 32];
    fixup_residual<B, BF16IN, KD>(P, x, ld, row, out, lane, r);
    const double p = fixup_project<KD>(P, j, lane, r);
    if (lane == 0) {
      unsigned int* word = reinterpret_cast<unsigned int*>(out.signs + row * (KD / 8)) + (j >> 5);
      const unsigned int m = 1u << (j & 31);
      if (p < 0.0) atomicOr(word, m); else atomicAnd(word, ~m);
    }
  }
  if (claimed <= fix_cap) return;                                // no overflow: the bitmap is empty
  const int64_t n_words = (n_rows + 31) >> 5;
  for (int64_t w = warp; w < n_words; w += nwarps) {
    uint32_t bits = fix_rows[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      const int64_t row = w * 32 + b;
      double r[KD / 32];
      fixup_residual<B, BF16IN, KD>(P, x, ld, row, out, lane, r);
      uint32_t word = 0u;                                        // lane l builds sign word l
#pragma unroll 1
      for (int j = 0; j < KD; ++j) {
        const double p = fixup_project<KD>(P, j, lane, r);
        if (lane == (j >> 5) && p < 0.0) word |= 1u << (j & 31);
      }
      if (lane < KD / 32) reinterpret_cast<uint32_t*>(out.signs + row * (KD / 8))[lane] = word;
    }
  }
}

// -------------------------------------------------------------------------- host
PFN_cuTensorMapEncodeTiled_v12000 get_encode() { return tensor_map_encoder(); }

// The bf16 kernel's fix-up scratch in the caller's workspace: the overflow
// bitmap (one bit per row), the list counter (both zeroed before each
// launch), then the list.  Two entries per tile is about three times what the
// error bound flags on Gaussian-like rows.
size_t fix_bitmap_bytes(int64_t n_rows) { return (static_cast<size_t>((n_rows + 31) / 32) * 4 + 255) / 256 * 256; }
int64_t fix_cap_for(int64_t n_rows) { return 2 * ((n_rows + kTile - 1) / kTile) + 4096; }
size_t fix_scratch_bytes(int64_t n_rows) {
  return fix_bitmap_bytes(n_rows) + 256 + static_cast<size_t>(fix_cap_for(n_rows)) * sizeof(unsigned long long);
}

template <int B, bool BF16IN, int KD>
int launch_tc(const tq_ctx& ctx, const void* x, int64_t n_rows, int64_t ld, const Packed& out, void* scratch,
              cudaStream_t s) {
  static_assert(BF16IN || KD == 128, "fp32 rows: d = 128 only");
  const KParams& P = ctx.kp;
  auto encode = get_encode();
  if (!encode) return static_cast<int>(cudaErrorNotSupported);
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(KD), static_cast<cuuint64_t>(n_rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * (BF16IN ? 2 : 4)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(XStage<BF16IN>::kColsPerBox), static_cast<cuuint32_t>(kTile)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(&tmap, BF16IN ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                      const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return static_cast<int>(cudaErrorInvalidValue);
  QuantD128Args X;
  for (int i = 0; i < kD; ++i) X.Dsign[i] = (i < KD && ctx.D[i] < 0) ? 0x80000000u : 0u;
  X.eps_scale = ctx.qjl_eps_scale;
  X.eps_abs = ctx.qjl_eps_abs;
  X.err = P.err;
  X.wait_cycles = wait_limit_cycles();
  X.fix_rows = nullptr;
  X.fix_list = nullptr;
  X.fix_count = nullptr;
  X.fix_cap = 0;
  const int64_t n_tiles = (n_rows + kTile - 1) / kTile;
  if constexpr (BF16IN) {                // bf16 rows: the rotation on the tensor cores
    if (!scratch) return static_cast<int>(cudaErrorInvalidValue);   // the fix-up scratch lives there
    uint8_t* sc = static_cast<uint8_t*>(scratch);
    X.fix_rows = reinterpret_cast<unsigned int*>(sc);
    X.fix_count = reinterpret_cast<unsigned int*>(sc + fix_bitmap_bytes(n_rows));
    X.fix_list = reinterpret_cast<unsigned long long*>(sc + fix_bitmap_bytes(n_rows) + 256);
    const int64_t cap = fix_cap_for(n_rows), forced = fixup_cap_override();
    X.fix_cap = static_cast<unsigned int>(forced > 0 && forced < cap ? forced : cap);
    cudaError_t e = cudaMemsetAsync(sc, 0, fix_bitmap_bytes(n_rows) + 256, s);
    if (e != cudaSuccess) return static_cast<int>(e);
    const size_t smem = quant_ws_smem_bytes<KD>();
    e = cudaFuncSetAttribute(k_quantize_d128_ws<B, KD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return static_cast<int>(e);
    const int64_t slots = static_cast<int64_t>(ctx.num_sms) * WsShape<KD>::kCtasPerSm;
    const int grid = static_cast<int>(n_tiles < slots ? n_tiles : slots);
    k_quantize_d128_ws<B, KD><<<grid, WsShape<KD>::kThreads, smem, s>>>(tmap, P, X, n_rows, out);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return static_cast<int>(e);
    k_qjl_fixup_d128<B, true, KD><<<ctx.num_sms * 8, 256, 0, s>>>(P, x, ld, n_rows, out, X.fix_list, X.fix_count,
                                                                     X.fix_cap, X.fix_rows);
  } else {                                // fp32 rows: the rotation in registers
    const int grid = static_cast<int>(n_tiles < ctx.num_sms ? n_tiles : ctx.num_sms);
    const size_t smem = quant_smem_bytes<false>();
    cudaError_t e = cudaFuncSetAttribute(k_quantize_d128_tc<B, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return static_cast<int>(e);
    k_quantize_d128_tc<B, false><<<grid, kThreads, smem, s>>>(tmap, P, X, n_rows, out);
  }
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

size_t quantize_d128_scratch_bytes(const tq_ctx& ctx, int64_t n_rows) {
  (void)ctx;
  return fix_scratch_bytes(n_rows);
}

bool quantize_d128_applies(const tq_ctx& ctx, int64_t n_rows, int x_is_bf16) {
  if (ctx.d_in != ctx.d) return false;                   // padded rows use the general kernel
  const KParams& P = ctx.kp;
  // d = m = 128 (bf16 or fp32 rows), or d = m = 64 for bf16 rows (the
  // 64-channel parts of a split row); x_is_bf16 < 0: either input type
  const bool shape = (P.d == 128 && P.m == 128) || (P.d == 64 && P.m == 64 && x_is_bf16 != 0);
  return shape && P.B >= 1 && P.B <= 4 && n_rows > 0 && n_rows < (int64_t(1) << 31) - 256 && ctx.use_tc &&
         get_encode() != nullptr;
}

int launch_quantize_d128(const tq_ctx& ctx, const void* x, int x_is_bf16, int64_t n_rows, int64_t ld,
                         const Packed& out, void* scratch, void* stream) {
  const KParams& P = ctx.kp;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (P.d == 64) {
    switch (P.B) {
      case 1: return launch_tc<1, true, 64>(ctx, x, n_rows, ld, out, scratch, s);
      case 2: return launch_tc<2, true, 64>(ctx, x, n_rows, ld, out, scratch, s);
      case 3: return launch_tc<3, true, 64>(ctx, x, n_rows, ld, out, scratch, s);
      default: return launch_tc<4, true, 64>(ctx, x, n_rows, ld, out, scratch, s);
    }
  }
  if (x_is_bf16) {
    switch (P.B) {
      case 1: return launch_tc<1, true, 128>(ctx, x, n_rows, ld, out, scratch, s);
      case 2: return launch_tc<2, true, 128>(ctx, x, n_rows, ld, out, scratch, s);
      case 3: return launch_tc<3, true, 128>(ctx, x, n_rows, ld, out, scratch, s);
      default: return launch_tc<4, true, 128>(ctx, x, n_rows, ld, out, scratch, s);
    }
  }
  switch (P.B) {
    case 1: return launch_tc<1, false, 128>(ctx, x, n_rows, ld, out, scratch, s);
    case 2: return launch_tc<2, false, 128>(ctx, x, n_rows, ld, out, scratch, s);
    case 3: return launch_tc<3, false, 128>(ctx, x, n_rows, ld, out, scratch, s);
    default: return launch_tc<4, false, 128>(ctx, x, n_rows, ld, out, scratch, s);
  }
}

}  // namespace tq
