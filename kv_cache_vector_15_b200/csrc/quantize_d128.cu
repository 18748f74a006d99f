// Write half at d = 128, m = 128 on sm_100a: TMA-staged rows, the
// randomized Hadamard rotation and Lloyd-Max bucketing in registers (one
// thread per row), and the QJL projection S r on the tcgen05 tensor cores.
//
// Method (page title, section):
//   n = ||x||, y = H_d D x / (n sqrt(d))      0h-n0.github.io "ICLR 2026論文解説:
//                                             TurboQuant", "Step 1: PolarQuant"
//   code_i = #{k : t_k < y_i}, r = y - c[code]  Qiita TurboQuant explainer,
//                                             "Stage 1: PolarQuant" (Lloyd-Max)
//   bit_j = [ (S r)_j < 0 ], rnorm = n ||r||    Qiita explainer, "Stage 2: QJL"
//
// CTA layout (persistent, one CTA per SM): two warpgroups, each with its own
// stage buffer.  Warpgroup w handles every other 128-row tile; thread t of the
// warpgroup owns row t of the tile, which is also TMEM lane t, so the
// projection result comes back to the thread that owns the row.  As soon as
// all its threads have read a tile into registers, the warpgroup's first
// thread issues the TMA load of its next tile into the same stage, so the
// load overlaps the rest of the tile's work.
//
// Projection precision: S is binary16 by definition (exact in the MMA).  The
// residual, scaled by 64, is split r = hi + lo into two binary16 parts
// (|r - hi - lo| <= 2^-22 |r| + 2^-25) and the MMA accumulates S hi + S lo
// (K = 256) in fp32.  A sign is taken from the tensor-core sum only where
// |p_j| exceeds a bound on that sum's error, eps = eps_scale ||r|| + eps_abs
// with eps_scale = 4 * 18 * 2^-22 * max_j ||S_j||_2 (18 = 16 accumulation
// steps + the split + slack, times 4 for margin) and eps_abs =
// max_j ||S_j||_1 * 2^-25 / 64 (binary16 underflow); the rare projections
// below it are recomputed in fp32 on the CUDA cores from hi + lo.
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
constexpr int kWG = 2;               // compute warpgroups
constexpr int kThreads = kWG * 128;
constexpr long long kWaitCycles = 2000000000ll;   // ~1 s at 2 GHz
constexpr uint32_t kTmemCols = 512;  // per warpgroup: 128 accumulator + 128 A columns, x2

struct QuantD128Args {
  uint32_t Dsign[kD];                // Rademacher signs as fp32 sign-bit masks (0 or 0x80000000)
  float eps_scale;                   // see header comment
  float eps_abs;                     // binary16 underflow term of the bound (normalised units)
  int* err;                          // device error word
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
  return 1024 /*alignment slack*/ + kSmemS + XStage<BF16IN>::kStages * kWG * XStage<BF16IN>::kBytes +
         256 /*barriers etc*/;
}

__device__ __forceinline__ void flag_error(int* err, int* abort_flag, int code) {
  if (err) atomicCAS(err, 0, code);
  atomicExch(abort_flag, 1);
}

// bf16 pair in one 32-bit word -> two floats (exact)
__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xffff0000u);
}

// State a warpgroup thread carries from a tile's first half (rotation, codes,
// residual into TMEM) to its second half (signs from the MMA, stores).
template <int B>
struct RowState {
  uint32_t cw[B * 4];                // packed codes
  float n, rho;
  int64_t row;
  bool zero, valid;
};

template <int B, bool BF16IN>
__global__ void __launch_bounds__(kThreads, 1)
k_quantize_d128_tc(const __grid_constant__ CUtensorMap tmap, const KParams P, const QuantD128Args X,
                   int64_t n_rows, const Packed out) {
  constexpr int L = 1 << B;
  constexpr int kStage = XStage<BF16IN>::kBytes;
  constexpr int NS = XStage<BF16IN>::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sS = smem;
  uint8_t* sX = smem + kSmemS;                                   // [warpgroup][NS buffers] stages
  uint64_t* full = reinterpret_cast<uint64_t*>(sX + NS * kWG * kStage);  // [warpgroup][2]
  uint64_t* mdone = full + 2 * kWG;                              // [warpgroup]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + kWG);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* lut = reinterpret_cast<float*>(tmem_slot + 2);          // L centroids (scaled by 64)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_tiles = (n_rows + kTile - 1) / kTile;

  if (tid == 0) {
    for (int i = 0; i < 2 * kWG; ++i) mbar_init(&full[i], 1);
    for (int i = 0; i < kWG; ++i) mbar_init(&mdone[i], 1);
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

  const int wg = warp >> 2, wl = warp & 3;
  const bool leader = (wl == 0 && lane == 0);                    // issues this warpgroup's TMA and MMAs
  const int trow = wl * 32 + lane;                               // row in tile == TMEM lane
  const uint32_t lane_base = static_cast<uint32_t>(wl * 32) << 16;
  const uint32_t t_acc = tmem + lane_base + wg * 256;            // projections, 128 columns
  const uint32_t t_a = t_acc + 128;                              // residual hi | lo, 128 columns
  const float sqrt_d = 11.313708498984761f;                      // sqrt(128)
  uint8_t* stages = sX + wg * NS * kStage;
  uint64_t* wfull = full + 2 * wg;
  const int64_t t_first = blockIdx.x + static_cast<int64_t>(wg) * gridDim.x;
  const int64_t t_step = static_cast<int64_t>(kWG) * gridDim.x;
  auto issue_load = [&](int64_t tile, int buf) {
    mbar_arrive_expect_tx(&wfull[buf], kStage);
#pragma unroll
    for (int bx = 0; bx < XStage<BF16IN>::kBoxes; ++bx)
      tma_load_2d(stages + buf * kStage + bx * (kTile * 128), &tmap, &wfull[buf],
                  bx * XStage<BF16IN>::kColsPerBox, static_cast<int>(tile * kTile));
  };
  // loads in flight (leader only): fill count per buffer issued vs waited
  int issued[2] = {0, 0}, waited[2] = {0, 0};
  if (leader) {
    prefetch_tmap(&tmap);
    if (t_first < n_tiles) { issue_load(t_first, 0); ++issued[0]; }
    if (NS == 2 && t_first + t_step < n_tiles) { issue_load(t_first + t_step, 1); ++issued[1]; }
  }

  RowState<B> prev;
  bool have_prev = false;
  int mine = 0;
  bool aborted = false;

  // second half of a tile: signs from the accumulator (exact recomputation of
  // the projections within the error bound of zero), then the stores
  auto finish = [&](const RowState<B>& st, int tile_no) {
    if (!mbar_wait(&mdone[wg], tile_no & 1, kWaitCycles)) flag_error(X.err, abort_flag, 3);
    tc_fence_after();
    const float eps = kResScale * fmaf(X.eps_scale, st.rho, X.eps_abs);   // in the MMA's (scaled) units
    uint32_t s0 = 0, s1 = 0, s2 = 0, s3 = 0, f0 = 0, f1 = 0, f2 = 0, f3 = 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {                  // 16 projections at a time
      uint32_t p[16];
      tmem_ld16(t_acc + c * 16, p);
      tmem_wait_ld();
      uint32_t bits = 0u, flags = 0u;
#pragma unroll
      for (int j = 15; j >= 0; --j) {
        bits = (bits << 1) | (p[j] >> 31);
        flags = (flags << 1) | (fabsf(__uint_as_float(p[j])) < eps ? 1u : 0u);
      }
      const int sh = (c & 1) * 16;
      if ((c >> 1) == 0) { s0 |= bits << sh; f0 |= flags << sh; }
      if ((c >> 1) == 1) { s1 |= bits << sh; f1 |= flags << sh; }
      if ((c >> 1) == 2) { s2 |= bits << sh; f2 |= flags << sh; }
      if ((c >> 1) == 3) { s3 |= bits << sh; f3 |= flags << sh; }
    }
    // Recompute flagged projections in fp32 from hi + lo, one flagged j per
    // lane per pass; the TMEM reads are warp-collective, so every lane runs
    // max-over-lanes passes.
    const int nflag = __popc(f0) + __popc(f1) + __popc(f2) + __popc(f3);
    const int passes = __reduce_max_sync(0xffffffffu, static_cast<unsigned>(nflag));
    for (int q = 0; q < passes; ++q) {
      int j = -1;
      if (q < nflag) {                           // the lowest remaining flagged projection
        if (f3) j = 96 + __ffs(f3) - 1;
        if (f2) j = 64 + __ffs(f2) - 1;
        if (f1) j = 32 + __ffs(f1) - 1;
        if (f0) j = __ffs(f0) - 1;
      }
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {              // 16 residual pairs (32 entries) at a time
        uint32_t ah[16], al[16];
        tmem_ld16(t_a + c * 16, ah);
        tmem_ld16(t_a + 64 + c * 16, al);
        tmem_wait_ld();
        if (j >= 0) {
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {                      // 16-byte chunks of S row j: 8 entries
            const int chunk = c * 4 + qq, kb = chunk >> 3, cc = chunk & 7;
            const uint4 sv = *reinterpret_cast<const uint4*>(sS + kb * 16384 + j * 128 + ((cc ^ (j & 7)) << 4));
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
        const int c = j >> 5;
        if (c == 0) { s0 = (s0 & ~m) | nb; f0 &= ~m; }
        if (c == 1) { s1 = (s1 & ~m) | nb; f1 &= ~m; }
        if (c == 2) { s2 = (s2 & ~m) | nb; f2 &= ~m; }
        if (c == 3) { s3 = (s3 & ~m) | nb; f3 &= ~m; }
      }
    }
    if (st.zero || st.rho == 0.f) s0 = s1 = s2 = s3 = 0u;
    tc_fence_before();
    if (st.valid) {
      uint4* co = reinterpret_cast<uint4*>(out.codes + st.row * (B * 16));
#pragma unroll
      for (int q = 0; q < B; ++q)
        co[q] = make_uint4(st.cw[4 * q], st.cw[4 * q + 1], st.cw[4 * q + 2], st.cw[4 * q + 3]);
      *reinterpret_cast<uint4*>(out.signs + st.row * 16) = make_uint4(s0, s1, s2, s3);
      out.norm[st.row] = st.zero ? 0.f : st.n;
      out.rnorm[st.row] = st.zero ? 0.f : st.n * st.rho;
    }
  };

  for (int64_t t = t_first; t < n_tiles; t += t_step, ++mine) {
    const int buf = mine % NS;
    if (mbar_wait(&wfull[buf], (mine / NS) & 1, kWaitCycles)) {
      if (leader) ++waited[buf];
    } else {
      flag_error(X.err, abort_flag, 2);
    }
    const uint8_t* stage = stages + buf * kStage;
    RowState<B> cur;
    cur.row = t * kTile + trow;
    cur.valid = cur.row < n_rows;

    // ---- this thread's row, D folded into the bf16 -> fp32 widening ----------
    float v[kD];
    if (BF16IN) {
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int bx = c >> 3, cc = c & 7;
        const uint4 w = *reinterpret_cast<const uint4*>(stage + bx * (kTile * 128) + trow * 128 +
                                                        ((cc ^ (trow & 7)) << 4));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = c * 8 + 2 * u;
          v[e] = __uint_as_float((ws[u] << 16) ^ X.Dsign[e]);
          v[e + 1] = __uint_as_float((ws[u] & 0xffff0000u) ^ X.Dsign[e + 1]);
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int bx = c >> 3, cc = c & 7;
        const uint4 w = *reinterpret_cast<const uint4*>(stage + bx * (kTile * 128) + trow * 128 +
                                                        ((cc ^ (trow & 7)) << 4));
        v[c * 4 + 0] = __uint_as_float(w.x ^ X.Dsign[c * 4 + 0]);
        v[c * 4 + 1] = __uint_as_float(w.y ^ X.Dsign[c * 4 + 1]);
        v[c * 4 + 2] = __uint_as_float(w.z ^ X.Dsign[c * 4 + 2]);
        v[c * 4 + 3] = __uint_as_float(w.w ^ X.Dsign[c * 4 + 3]);
      }
    }

    // ---- norm (sign flips do not change it), Walsh-Hadamard (unnormalised) ----
    float2 ssa = make_float2(0.f, 0.f), ssb = make_float2(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < kD; e += 4) {
      const float2 a = make_float2(v[e], v[e + 1]), b = make_float2(v[e + 2], v[e + 3]);
      ssa = __ffma2_rn(a, a, ssa);
      ssb = __ffma2_rn(b, b, ssb);
    }
    cur.n = sqrtf((ssa.x + ssa.y) + (ssb.x + ssb.y));
    cur.zero = !(cur.n >= kZeroNorm);
#pragma unroll
    for (int h = 2; h < kD; h <<= 1) {
#pragma unroll
      for (int e = 0; e < kD; e += 2) {
        if ((e & h) == 0) {
          const float2 a = make_float2(v[e], v[e + 1]), b = make_float2(v[e + h], v[e + h + 1]);
          const float2 sum = __fadd2_rn(a, b);
          const float2 dif = __ffma2_rn(b, make_float2(-1.f, -1.f), a);
          v[e] = sum.x; v[e + 1] = sum.y; v[e + h] = dif.x; v[e + h + 1] = dif.y;
        }
      }
    }
#pragma unroll
    for (int e = 0; e < kD; e += 2) {
      const float a = v[e], b = v[e + 1];
      v[e] = a + b;
      v[e + 1] = a - b;
    }

    // ---- Lloyd-Max codes and the residual (x 64) ----------------------------------
    // v holds y' = n sqrt(d) y; compare against per-row scaled thresholds; the
    // residual in unit-normalised units times 64 is r64 = y' sc64 - 64 c[code].
    const float nsd = cur.zero ? 1.f : cur.n * sqrt_d;
    const float sc64 = cur.zero ? 0.f : kResScale / nsd;
    float tq[L - 1];
#pragma unroll
    for (int k = 0; k < L - 1; ++k) tq[k] = P.t[k] * nsd;
#pragma unroll
    for (int w = 0; w < B * 4; ++w) cur.cw[w] = 0u;
    float2 r2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int e = 0; e < kD; ++e) {
      const float y = v[e];
      uint32_t code;
      float cval;
      if constexpr (B == 1) {
        const bool up = y > 0.f;
        code = up ? 1u : 0u;
        cval = up ? lut[1] : -lut[1];
      } else if constexpr (B == 2) {
        // symmetric 4-level codebook: t = (-tau, 0, tau), c = (-c3, -c2, c2, c3).
        // Outer cell by |y| > tau (y exactly equal to -tau, a boundary tie, would
        // take the inner cell; such a coordinate lies in the tie band).
        const bool up = y > 0.f, outer = fabsf(y) > tq[2];
        code = (up ? 2u : 0u) | ((up == outer) ? 1u : 0u);
        const float mag = outer ? lut[3] : lut[2];
        cval = up ? mag : -mag;
      } else {
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
        cval = lut[code];
      }
      const float r = fmaf(y, sc64, -cval);
      v[e] = r;
      if (e & 1) r2.y = fmaf(r, r, r2.y); else r2.x = fmaf(r, r, r2.x);
      const int bit = B * e, wi = bit >> 5, sh = bit & 31;
      cur.cw[wi] |= code << sh;
      if (sh + B > 32) cur.cw[wi + 1] |= code >> (32 - sh);
    }
    cur.rho = sqrtf(r2.x + r2.y) * (1.0f / kResScale);
    if (cur.zero) {
      cur.rho = 0.f;
#pragma unroll
      for (int w = 0; w < B * 4; ++w) cur.cw[w] = 0u;
#pragma unroll
      for (int e = 0; e < kD; ++e) v[e] = 0.f;
    }

    // ---- previous tile's signs and stores, now that its MMA has had time ---------
    if (have_prev) finish(prev, mine - 1);

    // ---- residual -> TMEM as binary16 hi | lo (A operand) --------------------------
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
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
      tmem_st16(t_a + ch * 16, hw);
      tmem_st16(t_a + 64 + ch * 16, lw);
    }
    tmem_wait_st();
    tc_fence_before();
    // barrier over the warpgroup that also ORs everyone's view of the abort
    // flag, so the decision to stop is the same in every thread
    if (named_bar_sync_or(1 + wg, 128, *reinterpret_cast<volatile int*>(abort_flag) != 0)) { aborted = true; break; }

    // ---- projection on the tensor cores: P = [hi | lo] [S ; S]^T; refill the stage --
    if (leader) {
      tc_fence_after();
      const uint32_t sbase = smem_u32(sS);
      const uint32_t idesc = idesc_f16_f32(kTile, kM);
      const uint32_t d_tmem = tmem + wg * 256;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const int kk = k & 7;                                      // K step within S (16 columns each)
        const uint64_t bdesc = smem_desc_sw128(sbase + (kk >> 2) * 16384 + (kk & 3) * 32, 1024);
        mma_f16_ts(d_tmem, d_tmem + 128 + k * 8, bdesc, idesc, k > 0 ? 1u : 0u);
      }
      mma_commit(&mdone[wg]);
      if (t + NS * t_step < n_tiles) { issue_load(t + NS * t_step, buf); ++issued[buf]; }
    }
    prev = cur;
    have_prev = true;
  }
  if (have_prev && !aborted) finish(prev, mine - 1);

  // ---- teardown: no TMA load of ours may still be in flight ----------------------
  if (leader) {
    for (int b2 = 0; b2 < 2; ++b2)
      while (waited[b2] < issued[b2]) {
        if (!mbar_wait(&wfull[b2], waited[b2] & 1, kWaitCycles)) { flag_error(X.err, abort_flag, 4); break; }
        ++waited[b2];
      }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// -------------------------------------------------------------------------- host
PFN_cuTensorMapEncodeTiled_v12000 get_encode() { return tensor_map_encoder(); }

template <int B, bool BF16IN>
int launch_tc(const tq_ctx& ctx, const void* x, int64_t n_rows, int64_t ld, const Packed& out, cudaStream_t s) {
  const KParams& P = ctx.kp;
  auto encode = get_encode();
  if (!encode) return static_cast<int>(cudaErrorNotSupported);
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(n_rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * (BF16IN ? 2 : 4)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(XStage<BF16IN>::kColsPerBox), static_cast<cuuint32_t>(kTile)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(&tmap, BF16IN ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                      const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return static_cast<int>(cudaErrorInvalidValue);
  QuantD128Args X;
  for (int i = 0; i < kD; ++i) X.Dsign[i] = ctx.D[i] < 0 ? 0x80000000u : 0u;
  X.eps_scale = ctx.qjl_eps_scale;
  X.eps_abs = ctx.qjl_eps_abs;
  X.err = P.err;
  const size_t smem = quant_smem_bytes<BF16IN>();
  cudaError_t e = cudaFuncSetAttribute(k_quantize_d128_tc<B, BF16IN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return static_cast<int>(e);
  const int64_t n_tiles = (n_rows + kTile - 1) / kTile;
  const int grid = static_cast<int>(n_tiles < ctx.num_sms ? n_tiles : ctx.num_sms);
  k_quantize_d128_tc<B, BF16IN><<<grid, kThreads, smem, s>>>(tmap, P, X, n_rows, out);
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

bool quantize_d128_applies(const tq_ctx& ctx, int64_t n_rows) {
  const KParams& P = ctx.kp;
  return P.d == kD && P.m == kM && P.B >= 1 && P.B <= 4 && n_rows > 0 && n_rows < (int64_t(1) << 31) &&
         ctx.use_tc && get_encode() != nullptr;
}

int launch_quantize_d128(const tq_ctx& ctx, const void* x, int x_is_bf16, int64_t n_rows, int64_t ld,
                         const Packed& out, void* stream) {
  const KParams& P = ctx.kp;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (x_is_bf16) {
    switch (P.B) {
      case 1: return launch_tc<1, true>(ctx, x, n_rows, ld, out, s);
      case 2: return launch_tc<2, true>(ctx, x, n_rows, ld, out, s);
      case 3: return launch_tc<3, true>(ctx, x, n_rows, ld, out, s);
      default: return launch_tc<4, true>(ctx, x, n_rows, ld, out, s);
    }
  }
  switch (P.B) {
    case 1: return launch_tc<1, false>(ctx, x, n_rows, ld, out, s);
    case 2: return launch_tc<2, false>(ctx, x, n_rows, ld, out, s);
    case 3: return launch_tc<3, false>(ctx, x, n_rows, ld, out, s);
    default: return launch_tc<4, false>(ctx, x, n_rows, ld, out, s);
  }
}

}  // namespace tq
