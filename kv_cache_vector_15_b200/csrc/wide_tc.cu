// Tensor-core paths for wide rows (d >= 256): the QJL projection of the write
// half and the all-pairs inner-product estimates of the read half, both as
// fp16 GEMMs on tcgen05 with fp32 accumulation in TMEM.
//
// Method references (page title, section):
//   QJL signs of S r and the estimator <q, x~> = norm <R q, c[code]> +
//     sqrt(pi/2)/m * rnorm <S R q, z>: Qiita TurboQuant explainer, "Stage 2:
//     QJL"; ai.spot.hk "Google TurboQuant", "無偏內積估計";
//   the vector-search use (quantize a database, estimate every query-row inner
//     product, keep the best): 0h-n0.github.io "ICLR 2026論文解説: TurboQuant",
//     "実験結果 — ベクトル検索（Recall評価）"; Qiita TurboQuant explainer,
//     "ベクトル検索への応用".
//
// Scratch (residual halves, decoded keys, split queries, candidate lists)
// lives in the workspace the caller passes; no call allocates device memory.
//
// Both products have an operand that is only exact in fp32, so it enters as
// two binary16 halves (hi = rn(v), lo = rn(v - hi), |v - hi - lo| <= 2^-22 |v|)
// whose products with the other operand's binary16 values are exact in fp32.
// The GEMM kernel walks a list of K segments, each pairing 64-column blocks
// of A with blocks of B and naming one of (up to) two accumulators:
//
//   write half   A = [r_hi | r_lo] (scaled residual rows), B = S:
//                P = r_hi S^T + r_lo S^T; the sign of P is the QJL bit
//   read half    A = [c_hi | c_lo | z] (decoded key rows), B = [q_hi | q_lo |
//                sq_hi | sq_lo] (rotated and projected queries):
//                acc0 = c_hi q_hi + c_lo q_hi + c_hi q_lo, acc1 = z sq_hi + z sq_lo
//                (c_lo q_lo is below 2^-22 of the sum and left out)
//
// Tiles are 128 rows x 256 columns (M = 128, N = 256, K = 16 per MMA), four
// 48 KB TMA stages; one thread issues the loads, one the MMAs, and the four
// warps read the accumulators back (warp w owns TMEM lanes 32w..32w+31).
//
// The vector search (tq_search) runs the read-half product with the roles
// swapped -- A = the split queries, B = the decoded keys -- in a persistent
// kernel (k_search_tc) whose epilogue threads each own one query and keep its
// running top-k in registers across key tiles, so no score is written.
//
// A projection is given its sign by the tensor cores only where |p_j|
// exceeds a bound on the product's error: the split's 2^-22 plus d/8 fp32
// accumulation steps of at most 2^-22 of sum |S_ji r_i| <= ||S_j|| ||r||
// each, plus binary16 underflow of the halves (2^-24 ||S_j||_1).  The rare
// projections inside the bound are listed and recomputed in fp64 from the
// halves by a fix-up kernel.
//
// Every mbarrier wait is bounded (about one second); a wait that runs out sets
// the context's error word and the CTA winds down (its MMAs and TMA loads are
// waited for, its TMEM freed) without writing results.

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "sm100.cuh"
#include "tq_internal.h"

namespace tq {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

namespace {

using namespace sm100;

constexpr int kTM = 128;                 // rows per tile (MMA M)
constexpr int kTN = 256;                 // columns per tile (MMA N)
constexpr int kKB = 64;                  // K elements per stage (one 128-byte swizzle row)
constexpr int kStages = 4;
constexpr uint32_t kABytes = kTM * 128;  // 16 KB
constexpr uint32_t kBBytes = kTN * 128;  // 32 KB
constexpr int kThreads = 128;
constexpr long long kWaitCycles = 2000000000ll;   // ~1 s at 2 GHz
constexpr int kChunkTiles = 148;         // key tiles per chunk of the estimates (one wave per column tile at 1 CTA / SM)
constexpr int kQuantChunkTiles = 296;    // row tiles per chunk of the write half (two waves per column tile)
constexpr int kMaxSeg = 6;
constexpr int kLocalFix = 512;           // ambiguous projections a tile lists in shared memory

struct GemmSeg {
  int a_kb, b_kb, nkb, acc;              // first K-block of A and of B, K-blocks, accumulator
};
struct GemmPlan {
  GemmSeg seg[kMaxSeg];
  int nseg;
  int b_row0;                            // first row of B that column 0 maps to
};

// epilogue of the write half: QJL sign words of a chunk of rows
struct SignEpi {
  uint32_t* signs;                       // sign words of the chunk's first row, m/32 words per row
  int words_per_row;
  const float* rn;                       // per chunk row: s ||r|| (0 for rows stored as zeros)
  const float* snorm;                    // [m] ||S_j||_2
  float eps_rel;                         // (d/8 + 2) 2^-22
  float eps_abs;                         // 2^-24 max_j ||S_j||_1, scaled units
  uint32_t* fix;                         // ambiguous projections: (chunk row << 12) | j
  uint32_t* nfix;
  uint32_t fix_cap;
};

// epilogue of the read half: estimates of one (set, chunk of keys)
struct LogitEpi {
  float* out;                            // out[q * ld_out + key0 + key] for this set
  int64_t ld_out, key0;
  const float* norm;                     // the chunk's first key
  const float* rnorm;
  const float* qscale;                   // [n_q][2] for this set's queries
};

enum { kSigns = 0, kScores = 1 };
constexpr int kMaxSearchK = 16;

__device__ __forceinline__ void set_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

template <int NACC, int MODE, class Epi>
__global__ void __launch_bounds__(kThreads, 1)
k_gemm_wide_tc(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb, const GemmPlan plan,
               int64_t n_rows, int n_cols, const Epi E, int* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + kStages * kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStages * kBBytes);
  uint64_t* empty = full + kStages;
  uint64_t* done = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_col = reinterpret_cast<float*>(tmem_slot + 4);          // per column: ||S_j|| or 2 query scales
  uint32_t* s_nfix = reinterpret_cast<uint32_t*>(s_col + 2 * kTN);   // this tile's ambiguous projections
  uint32_t* s_fix = s_nfix + 4;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col0 = blockIdx.x * kTN;
  const int64_t row0 = static_cast<int64_t>(blockIdx.y) * kTM;
  constexpr uint32_t kCols = NACC * 256;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(done, 1);
    *abort_flag = 0;
    *s_nfix = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kCols);
    tmem_relinquish();
  }
  for (int c = threadIdx.x; c < kTN; c += kThreads) {
    if constexpr (MODE != kSigns) {
      const int q = col0 + c;
      s_col[2 * c] = q < n_cols ? E.qscale[2 * q] : 0.f;
      s_col[2 * c + 1] = q < n_cols ? E.qscale[2 * q + 1] : 0.f;
    } else {
      const int j = col0 + c;
      s_col[c] = j < n_cols ? E.snorm[j] : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int issued = 0;                        // loads issued (producer thread)
  bool my_fail = false;

  if (warp == 0 && lane == 0) {
    // ---- producer: TMA loads of A and B blocks into the stage ring
    prefetch_tmap(&ta);
    prefetch_tmap(&tb);
    int kb = 0;
    for (int sg = 0; sg < plan.nseg && !my_fail; ++sg) {
      const GemmSeg S = plan.seg[sg];
      for (int i = 0; i < S.nkb; ++i, ++kb) {
        const int st = kb % kStages;
        if (kb >= kStages && !mbar_wait(&empty[st], ((kb / kStages) - 1) & 1, kWaitCycles)) {
          set_error(err, 2);
          *abort_flag = 1;
          my_fail = true;
          break;
        }
        if (*abort_flag) { my_fail = true; break; }
        mbar_arrive_expect_tx(&full[st], kABytes + kBBytes);
        tma_load_2d(sA + st * kABytes, &ta, &full[st], (S.a_kb + i) * kKB, static_cast<int>(row0));
        tma_load_2d(sB + st * kBBytes, &tb, &full[st], (S.b_kb + i) * kKB, plan.b_row0 + col0);
        ++issued;
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer
    constexpr uint32_t idesc = idesc_f16_f32(kTM, kTN);
    bool started[2] = {false, false};
    int kb = 0;
    for (int sg = 0; sg < plan.nseg && !my_fail; ++sg) {
      const GemmSeg S = plan.seg[sg];
      for (int i = 0; i < S.nkb; ++i, ++kb) {
        const int st = kb % kStages;
        if (!mbar_wait(&full[st], (kb / kStages) & 1, kWaitCycles)) {
          set_error(err, 2);
          *abort_flag = 1;
          my_fail = true;
          break;
        }
        tc_fence_after();
        const uint32_t a = smem_u32(sA + st * kABytes), b = smem_u32(sB + st * kBBytes);
        const uint32_t d_t = tmem + static_cast<uint32_t>(S.acc) * 256u;
#pragma unroll
        for (int k = 0; k < kKB / 16; ++k) {
          mma_f16_ss(d_t, smem_desc_sw128(a + k * 32, 1024), smem_desc_sw128(b + k * 32, 1024), idesc,
                     (started[S.acc] || k > 0) ? 1u : 0u);
        }
        started[S.acc] = true;
        mma_commit(&empty[st]);
      }
    }
    mma_commit(done);                    // after every MMA issued above
  }
  __syncwarp();

  // ---- accumulators ready
  if (!mbar_wait(done, 0, kWaitCycles)) { set_error(err, 2); my_fail = true; }
  tc_fence_after();
  const bool bad = __syncthreads_or(my_fail || *abort_flag);

  if (!bad) {
    const int rl = warp * 32 + lane;
    const int64_t row = row0 + rl;
    const bool valid = row < n_rows;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    if constexpr (MODE != kSigns) {
      const float nrm = valid ? E.norm[row] : 0.f, rn = valid ? E.rnorm[row] : 0.f;
      float* orow = E.out + E.key0 + row;
      for (int c = 0; c < kTN / 32; ++c) {
        const int q0 = col0 + c * 32;
        if (q0 >= n_cols) break;                     // uniform over the CTA
        uint32_t a0[32], a1[32];
        tmem_ld32(taddr + c * 32, a0);
        tmem_ld32(taddr + 256 + c * 32, a1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int q = q0 + i;
          const float v = nrm * (__uint_as_float(a0[i]) * s_col[2 * (c * 32 + i)]) +
                          rn * (__uint_as_float(a1[i]) * s_col[2 * (c * 32 + i) + 1]);
          if (valid && q < n_cols) orow[static_cast<int64_t>(q) * E.ld_out] = v;
        }
      }
    } else {
      const float rn = valid ? E.rn[row] : 0.f;
      for (int c = 0; c < kTN / 32; ++c) {
        const int j0 = col0 + c * 32;
        if (j0 >= n_cols) break;
        uint32_t a0[32];
        tmem_ld32(taddr + c * 32, a0);
        tmem_wait_ld();
        uint32_t bits = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p = __uint_as_float(a0[i]);
          bits |= (p < 0.f ? 1u : 0u) << i;
          const float eps = rn * E.eps_rel * s_col[c * 32 + i] + E.eps_abs;
          if (valid && rn > 0.f && fabsf(p) <= eps) {
            const uint32_t ent = (static_cast<uint32_t>(row) << 12) | static_cast<uint32_t>(j0 + i);
            const uint32_t slot = atomicAdd(s_nfix, 1u);
            if (slot < kLocalFix) {
              s_fix[slot] = ent;
            } else {                                 // a crowded tile: straight to the global list
              const uint32_t g = atomicAdd(E.nfix, 1u);
              if (g < E.fix_cap) E.fix[g] = ent;
            }
          }
        }
        if (valid) E.signs[row * E.words_per_row + (j0 >> 5)] = bits;
      }
    }
  }

  if constexpr (MODE == kSigns) {               // the tile's list joins the global one (one reservation)
    __syncthreads();
    __shared__ uint32_t s_base;
    const uint32_t nloc = min(*s_nfix, static_cast<uint32_t>(kLocalFix));
    if (threadIdx.x == 0) s_base = nloc ? atomicAdd(E.nfix, nloc) : 0u;
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < nloc; i += kThreads)
      if (s_base + i < E.fix_cap) E.fix[s_base + i] = s_fix[i];
  }

  // ---- wind down: the producer waits for its own loads, the MMA thread (if
  // the wait above gave up) for its MMAs; TMEM is freed
  if (bad && warp == 1 && lane == 0) {
    if (!mbar_wait(done, 0, kWaitCycles)) set_error(err, 2);
  }
  if (warp == 0 && lane == 0) {
    for (int st = 0; st < kStages; ++st) {
      if (st >= issued) break;
      const int last = st + ((issued - 1 - st) / kStages) * kStages;     // last load issued into this stage
      if (!mbar_wait(&full[st], (last / kStages) & 1, kWaitCycles)) set_error(err, 2);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

// ---------------------------------------------------------------------------
// write half, CUDA-core part: one warp per row, lane l holding coordinates
// 32 e + l (every load and store of the warp is one contiguous run).  Norm,
// rotation (D, FWHT with the butterflies in order of increasing distance,
// 1/sqrt(d)), Lloyd-Max codes (binary search over the thresholds), packed
// codes, norm and rnorm, and the residual r = y - c[code] (unit-norm domain)
// scaled by s and split into binary16 halves: res[row] = [hi (d) | lo (d)].
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <bool BF16>
__device__ __forceinline__ float load_elem(const void* base, int64_t idx) {
  if (BF16) {
    const uint16_t u = __ldg(reinterpret_cast<const uint16_t*>(base) + idx);
    return __uint_as_float(static_cast<uint32_t>(u) << 16);
  }
  return __ldg(reinterpret_cast<const float*>(base) + idx);
}

struct PrepArgs {
  __half* res;                           // [rows][2d]
  float* rn;                             // [rows]: s ||r||, 0 for zero rows
  float s;                               // residual scale (a power of two)
  uint32_t* nfix;                        // the chunk's fix-up list counter, reset here
};

template <int E, bool BF16>
__global__ void __launch_bounds__(256)
k_quantize_residual_warp(const KParams P, const void* __restrict__ x, int64_t n_rows, int64_t ld, const Packed out,
                         const PrepArgs A) {
  __shared__ float thr[kMaxLevels], lut[kMaxLevels];
  __shared__ uint8_t cs_all[8][E * 32];
  if (threadIdx.x < kMaxLevels) { thr[threadIdx.x] = P.t[threadIdx.x]; lut[threadIdx.x] = P.c[threadIdx.x]; }
  // the previous chunk's fix-up has run (stream order); this chunk's GEMM appends after this kernel
  if (blockIdx.x == 0 && threadIdx.x == 0 && A.nfix) *A.nfix = 0u;
  __syncthreads();
  const int d = E * 32, B = P.B, half_levels = P.L >> 1;
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  uint8_t* cs = cs_all[wib];
  const int nwords_codes = d * B / 32;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + wib; row < n_rows;
       row += static_cast<int64_t>(gridDim.x) * 8) {
    uint32_t* codes_out = reinterpret_cast<uint32_t*>(out.codes + row * P.codes_bytes);
    __half* rrow = A.res + row * 2 * d;
    float v[E];
    if (P.d_in != d) {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int col = 32 * e + lane;                 // zero padding beyond the caller's row
        v[e] = col < P.d_in ? load_elem<BF16>(x, row * ld + col) : 0.f;
      }
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) v[e] = load_elem<BF16>(x, row * ld + 32 * e + lane);
    }
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) ss = fmaf(v[e], v[e], ss);
    ss = warp_sum(ss);
    const float n = sqrtf(ss);
    if (!(n >= kZeroNorm)) {                           // stored as zeros; its projections are all 0
      for (int w = lane; w < nwords_codes; w += 32) codes_out[w] = 0u;
      const __half z = __ushort_as_half(0);
#pragma unroll
      for (int e = 0; e < E; ++e) { rrow[32 * e + lane] = z; rrow[d + 32 * e + lane] = z; }
      if (lane == 0) { out.norm[row] = 0.f; out.rnorm[row] = 0.f; A.rn[row] = 0.f; }
      continue;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {                      // D: bit (32 e + lane) of the mask
      const uint32_t bit = (__ldg(P.Dmask + e) >> lane) & 1u;
      v[e] = bit ? -v[e] : v[e];
    }
    // butterflies at distance 1 .. 16 across lanes, then 32 .. d/2 within a lane
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
      const float sgn = (lane & h) ? -1.f : 1.f;       // upper lane: partner - own; lower: own + partner
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float p = __shfl_xor_sync(0xffffffffu, v[e], h);
        v[e] = fmaf(sgn, v[e], p);                     // exact sign flip, one rounding: as p -/+ v
      }
    }
#pragma unroll
    for (int h = 1; h < E; h <<= 1) {
#pragma unroll
      for (int e = 0; e < E; ++e) {
        if ((e & h) == 0) {
          const float a = v[e], b = v[e + h];
          v[e] = a + b;
          v[e + h] = a - b;
        }
      }
    }
    const float inv_n = 1.0f / n;
    float r2 = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float y = (v[e] * inv_n) * P.inv_sqrt_d;
      int code = 0;                                    // #{k : t_k < y} over the ascending thresholds
      for (int step = half_levels; step > 0; step >>= 1) code += (y > thr[code + step - 1]) ? step : 0;
      const float r = y - lut[code];
      cs[32 * e + lane] = static_cast<uint8_t>(code);
      r2 = fmaf(r, r, r2);
      const float rs = r * A.s;
      const __half h = __float2half_rn(rs);
      rrow[32 * e + lane] = h;
      rrow[d + 32 * e + lane] = __float2half_rn(rs - __half2float(h));
    }
    r2 = warp_sum(r2);
    __syncwarp();
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
    if (lane == 0) {
      const float rr = sqrtf(r2);
      out.norm[row] = n;
      out.rnorm[row] = n * rr;
      A.rn[row] = A.s * rr;
    }
    __syncwarp();
  }
}

// Projections the tensor cores could not sign: p = sum_i S[j][i] (hi_i + lo_i)
// in fp64, one warp per listed (row, j), eight coordinates per lane and load;
// the bit is set or cleared atomically.
__global__ void __launch_bounds__(256)
k_qjl_fixup(const KParams P, const __half* __restrict__ res, const uint32_t* __restrict__ fix,
            const uint32_t* __restrict__ nfix, uint32_t cap, uint32_t* __restrict__ signs, int words_per_row) {
  const uint32_t n = *nfix;
  if (n > cap) {
    if (blockIdx.x == 0 && threadIdx.x == 0 && P.err) atomicCAS(P.err, 0, 8);
  }
  const uint32_t cnt = n < cap ? n : cap;
  const int d = P.d;
  const int lane = threadIdx.x & 31;
  for (uint32_t e = blockIdx.x * 8 + (threadIdx.x >> 5); e < cnt; e += gridDim.x * 8) {
    const uint32_t ent = fix[e];
    const int64_t row = ent >> 12;
    const int j = static_cast<int>(ent & 4095u);
    const uint4* hr = reinterpret_cast<const uint4*>(res + row * 2 * d);
    const uint4* lr = reinterpret_cast<const uint4*>(res + row * 2 * d + d);
    const uint4* sj = reinterpret_cast<const uint4*>(P.S + static_cast<int64_t>(j) * d);
    double acc = 0.0;
#pragma unroll 4
    for (int i = lane; i < d / 8; i += 32) {
      const uint4 h4 = __ldg(hr + i), l4 = __ldg(lr + i), s4 = __ldg(sj + i);
      const uint32_t hw[4] = {h4.x, h4.y, h4.z, h4.w}, lw[4] = {l4.x, l4.y, l4.z, l4.w},
                     sw[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint16_t hb = static_cast<uint16_t>(hw[u] >> (16 * hh)), lb = static_cast<uint16_t>(lw[u] >> (16 * hh)),
                         sb = static_cast<uint16_t>(sw[u] >> (16 * hh));
          const double r = static_cast<double>(__half2float(__ushort_as_half(hb))) +
                           static_cast<double>(__half2float(__ushort_as_half(lb)));
          acc += r * static_cast<double>(__half2float(__ushort_as_half(sb)));
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      uint32_t* w = signs + row * words_per_row + (j >> 5);
      const uint32_t bit = 1u << (j & 31);
      if (acc < 0.0) atomicOr(w, bit);
      else atomicAnd(w, ~bit);
    }
  }
}

// ---------------------------------------------------------------------------
// read half, CUDA-core parts
// ---------------------------------------------------------------------------
struct KeyOpArgs {
  uint16_t c_hi[kMaxLevels], c_lo[kMaxLevels];   // binary16 halves of s_c c[code]
};

// keys -> A rows [c_hi (d) | c_lo (d) | z (m)], one warp per key
__global__ void __launch_bounds__(256)
k_key_operand(const KParams P, const Packed keys, int64_t n_keys, const KeyOpArgs K, __half* __restrict__ a) {
  __shared__ uint16_t lh[kMaxLevels], ll[kMaxLevels];
  if (threadIdx.x < kMaxLevels) { lh[threadIdx.x] = K.c_hi[threadIdx.x]; ll[threadIdx.x] = K.c_lo[threadIdx.x]; }
  __syncthreads();
  const int d = P.d, m = P.m, B = P.B;
  const int lane = threadIdx.x & 31;
  const uint32_t mask = (1u << B) - 1u;
  const int64_t ld = 2 * d + m;
  for (int64_t key = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); key < n_keys;
       key += static_cast<int64_t>(gridDim.x) * 8) {
    const uint8_t* cb = keys.codes + key * P.codes_bytes;
    const uint8_t* sb = keys.signs + key * P.signs_bytes;
    __half* arow = a + key * ld;
    for (int g = lane; g < d / 8; g += 32) {          // coordinates 8g .. 8g + 7: bytes gB .. gB + B - 1
      uint32_t w = 0;
      for (int k = 0; k < B; ++k) w |= static_cast<uint32_t>(__ldg(cb + g * B + k)) << (8 * k);
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int u = 0; u < 8; u += 2) {
        const uint32_t c0 = (w >> (B * u)) & mask, c1 = (w >> (B * (u + 1))) & mask;
        hi[u >> 1] = static_cast<uint32_t>(lh[c0]) | (static_cast<uint32_t>(lh[c1]) << 16);
        lo[u >> 1] = static_cast<uint32_t>(ll[c0]) | (static_cast<uint32_t>(ll[c1]) << 16);
      }
      *reinterpret_cast<uint4*>(arow + 8 * g) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(arow + d + 8 * g) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    for (int g = lane; g < m / 8; g += 32) {          // z = 1 - 2 bit: +1 = 0x3C00, -1 = 0xBC00
      const uint32_t s = __ldg(sb + g);
      uint32_t z[4];
#pragma unroll
      for (int u = 0; u < 8; u += 2) {
        const uint32_t z0 = ((s >> u) & 1u) ? 0xBC00u : 0x3C00u;
        const uint32_t z1 = ((s >> (u + 1)) & 1u) ? 0xBC00u : 0x3C00u;
        z[u >> 1] = z0 | (z1 << 16);
      }
      *reinterpret_cast<uint4*>(arow + 2 * d + 8 * g) = make_uint4(z[0], z[1], z[2], z[3]);
    }
  }
}

// prepared queries [R q (d) | S R q (m)] -> B rows [q_hi | q_lo | sq_hi | sq_lo],
// each part scaled by a power of two that brings its largest magnitude into
// [1, 2); qscale[q] = {1 / (s_c s_q), qjl_scale / s_sq}
__global__ void __launch_bounds__(256)
k_query_operand(const KParams P, const float* __restrict__ qp, int64_t n_q, float inv_sc, __half* __restrict__ b,
                float* __restrict__ qscale) {
  const int d = P.d, m = P.m;
  const int lane = threadIdx.x & 31;
  for (int64_t q = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); q < n_q;
       q += static_cast<int64_t>(gridDim.x) * 8) {
    const float* src = qp + q * (d + m);
    __half* brow = b + q * 2 * (d + m);
    float mx[2] = {0.f, 0.f};
    for (int i = lane; i < d + m; i += 32) {
      const float a = fabsf(src[i]);
      const int part = i < d ? 0 : 1;
      mx[part] = fmaxf(mx[part], a);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], o));
      mx[1] = fmaxf(mx[1], __shfl_xor_sync(0xffffffffu, mx[1], o));
    }
    float sc[2];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      int e = 0;
      frexpf(mx[p], &e);                               // mx in [2^(e-1), 2^e)
      sc[p] = mx[p] > 0.f ? ldexpf(1.f, 1 - e) : 1.f;
    }
    for (int i = lane; i < d + m; i += 32) {
      const bool first = i < d;
      const float v = src[i] * sc[first ? 0 : 1];
      const __half h = __float2half_rn(v);
      const __half l = __float2half_rn(v - __half2float(h));
      if (first) { brow[i] = h; brow[d + i] = l; }
      else { brow[d + i] = h; brow[d + m + i] = l; }  // sq_hi at 2d + j, sq_lo at 2d + m + j
    }
    if (lane == 0) {
      qscale[2 * q] = inv_sc / sc[0];
      qscale[2 * q + 1] = P.qjl_scale / sc[1];
    }
  }
}

// ---------------------------------------------------------------------------
// vector search: the roles of the estimates GEMM swapped -- A = the split
// queries (128 per CTA, query = TMEM lane), B = decoded keys (256 per tile) --
// and the CTA persistent over its share of a chunk's key tiles, so that each
// epilogue thread owns one query and keeps that query's running top-k in
// registers from tile to tile (and, through sv / si, from chunk to chunk).
// Warps 0-3 read TMEM (lanes 32w .. 32w + 31), warp 4 issues TMA, warp 5 the
// MMAs; the single 512-column accumulator pair is handed back by an mbarrier
// once the four warps have read it.
// ---------------------------------------------------------------------------
constexpr int kSearchThreads = 192;
constexpr int kSearchTiles = 296;        // key tiles of 256 per chunk at most (75776 keys, 450 MB decoded at d = m = 1024)

struct SearchArgs {
  const float* norm;                     // the chunk's first key
  const float* rnorm;
  const float* qscale;                   // [n_q][2]
  float* sv;                             // running lists [n_q][S][k], larger first
  int32_t* si;
  int k, S, n_q;
  int64_t key0, nk;                      // index of the chunk's first key, keys in the chunk
  int tiles_per_split;
  int first;                             // the chunk that starts the lists
};

__global__ void __launch_bounds__(kSearchThreads, 1)
k_search_tc(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb, const GemmPlan plan,
            const SearchArgs X, int* err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + kStages * kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStages * kBBytes);
  uint64_t* empty = full + kStages;
  uint64_t* done = empty + kStages;      // a tile's MMAs completed
  uint64_t* tfree = done + 1;            // the four epilogue warps have read the accumulators
  uint64_t* fin = tfree + 1;             // every MMA of the CTA completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_nrm = reinterpret_cast<float*>(tmem_slot + 4);
  float* s_rn = s_nrm + kTN;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, split = blockIdx.y;
  const int n_tiles = static_cast<int>((X.nk + kTN - 1) / kTN);
  const int t_begin = split * X.tiles_per_split;
  const int t_end = min(t_begin + X.tiles_per_split, n_tiles);
  const int my_tiles = max(0, t_end - t_begin);

  if (threadIdx.x == 0) {
    for (int st = 0; st < kStages; ++st) { mbar_init(&full[st], 1); mbar_init(&empty[st], 1); }
    mbar_init(done, 1);
    mbar_init(tfree, 128);
    mbar_init(fin, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int issued = 0;

  if (warp == 4) {
    if (lane == 0) {                     // ---- TMA producer
      prefetch_tmap(&ta);
      prefetch_tmap(&tb);
      int g = 0;
      bool stop = false;
      for (int i = 0; i < my_tiles && !stop; ++i) {
        const int tile = t_begin + i;
        for (int sg = 0; sg < plan.nseg && !stop; ++sg) {
          const GemmSeg S = plan.seg[sg];
          for (int j = 0; j < S.nkb; ++j, ++g) {
            const int st = g % kStages;
            if (g >= kStages && !mbar_wait(&empty[st], ((g / kStages) - 1) & 1, kWaitCycles)) {
              set_error(err, 2);
              *abort_flag = 1;
            }
            if (*abort_flag) { stop = true; break; }
            mbar_arrive_expect_tx(&full[st], kABytes + kBBytes);
            tma_load_2d(sA + st * kABytes, &ta, &full[st], (S.a_kb + j) * kKB, qt * kTM);
            tma_load_2d(sB + st * kBBytes, &tb, &full[st], (S.b_kb + j) * kKB, tile * kTN);
            issued = g + 1;
          }
        }
      }
      for (int st = 0; st < kStages && st < issued; ++st) {     // wait for this thread's own loads
        const int last = st + ((issued - 1 - st) / kStages) * kStages;
        if (!mbar_wait(&full[st], (last / kStages) & 1, kWaitCycles)) set_error(err, 2);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {                     // ---- MMA issuer
      constexpr uint32_t idesc = idesc_f16_f32(kTM, kTN);
      int g = 0;
      bool stop = false;
      for (int i = 0; i < my_tiles && !stop; ++i) {
        if (i > 0 && !mbar_wait(tfree, (i - 1) & 1, kWaitCycles)) {
          set_error(err, 2);
          *abort_flag = 1;
        }
        if (*abort_flag) break;
        tc_fence_after();
        bool started[2] = {false, false};
        for (int sg = 0; sg < plan.nseg && !stop; ++sg) {
          const GemmSeg S = plan.seg[sg];
          for (int j = 0; j < S.nkb; ++j, ++g) {
            const int st = g % kStages;
            if (!mbar_wait(&full[st], (g / kStages) & 1, kWaitCycles)) {
              set_error(err, 2);
              *abort_flag = 1;
              stop = true;
              break;
            }
            tc_fence_after();
            const uint32_t a = smem_u32(sA + st * kABytes), b = smem_u32(sB + st * kBBytes);
            const uint32_t d_t = tmem + static_cast<uint32_t>(S.acc) * 256u;
#pragma unroll
            for (int kk = 0; kk < kKB / 16; ++kk)
              mma_f16_ss(d_t, smem_desc_sw128(a + kk * 32, 1024), smem_desc_sw128(b + kk * 32, 1024), idesc,
                         (started[S.acc] || kk > 0) ? 1u : 0u);
            started[S.acc] = true;
            mma_commit(&empty[st]);
          }
        }
        if (!stop) mma_commit(done);
      }
      mma_commit(fin);                   // after every MMA issued above
      if (!mbar_wait(fin, 0, kWaitCycles)) set_error(err, 2);
    }
  } else {
    // ---- epilogue: thread = query
    const int q = qt * kTM + warp * 32 + lane;
    const bool qv = q < X.n_q;
    const int K = X.k;
    const float qs0 = qv ? X.qscale[2 * q] : 0.f, qs1 = qv ? X.qscale[2 * q + 1] : 0.f;
    float tv[kMaxSearchK];
    int32_t ti[kMaxSearchK];
#pragma unroll
    for (int u = 0; u < kMaxSearchK; ++u) { tv[u] = -INFINITY; ti[u] = INT32_MAX; }
    float* lv = X.sv + (static_cast<int64_t>(q) * X.S + split) * K;
    int32_t* li = X.si + (static_cast<int64_t>(q) * X.S + split) * K;
    if (qv && !X.first) {
#pragma unroll
      for (int u = 0; u < kMaxSearchK; ++u)
        if (u < K) { tv[u] = lv[u]; ti[u] = li[u]; }
    }
    float kth = -INFINITY;
#pragma unroll
    for (int u = 0; u < kMaxSearchK; ++u)
      if (u == K - 1) kth = tv[u];
    const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    for (int i = 0; i < my_tiles; ++i) {
      const bool ok = mbar_wait(done, i & 1, kWaitCycles);
      if (named_bar_sync_or(1, 128, !ok || *abort_flag)) {      // every epilogue thread leaves together
        if (!ok) set_error(err, 2);
        *abort_flag = 1;
        break;
      }
      const int64_t kb = static_cast<int64_t>(t_begin + i) * kTN;
      for (int c = threadIdx.x; c < kTN; c += 128) {
        const int64_t key = kb + c;
        s_nrm[c] = key < X.nk ? X.norm[key] : 0.f;
        s_rn[c] = key < X.nk ? X.rnorm[key] : 0.f;
      }
      named_bar_sync(1, 128);
      tc_fence_after();
      for (int c = 0; c < kTN / 32; ++c) {
        uint32_t a0[32], a1[32];
        tmem_ld32(taddr + c * 32, a0);
        tmem_ld32(taddr + 256 + c * 32, a1);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int col = c * 32 + j;
          float x = s_nrm[col] * (__uint_as_float(a0[j]) * qs0) + s_rn[col] * (__uint_as_float(a1[j]) * qs1);
          if (qv && kb + col < X.nk && x > kth) {
            // insertion network: keys reach a list in increasing order, so a
            // strictly larger value is the only one that moves in
            int32_t xi = static_cast<int32_t>(X.key0 + kb + col);
#pragma unroll
            for (int u = 0; u < kMaxSearchK; ++u) {
              const bool take = x > tv[u];
              const float pv = tv[u];
              const int32_t pi = ti[u];
              tv[u] = take ? x : pv;
              ti[u] = take ? xi : pi;
              x = take ? pv : x;
              xi = take ? pi : xi;
            }
#pragma unroll
            for (int u = 0; u < kMaxSearchK; ++u)
              if (u == K - 1) kth = tv[u];
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tfree);
    }
    if (qv && !*abort_flag) {
#pragma unroll
      for (int u = 0; u < kMaxSearchK; ++u)
        if (u < K) { lv[u] = tv[u]; li[u] = ti[u]; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The k best of each query's S lists (value larger first, equal values by
// lower key index), one warp per query: every lane keeps the best k of its
// share of the S k candidates, then k rounds of a warp-wide best.
__device__ __forceinline__ bool better_vi(float va, int32_t ia, float vb, int32_t ib) {
  return va > vb || (va == vb && ia < ib);
}

__global__ void __launch_bounds__(256)
k_merge_lists(const float* __restrict__ sv, const int32_t* __restrict__ si, int n_cand, int k, int n_q,
              int32_t* __restrict__ idx, float* __restrict__ val) {
  const int q = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (q >= n_q) return;                                  // warp-uniform
  float tv[kMaxSearchK];
  int32_t ti[kMaxSearchK];
#pragma unroll
  for (int u = 0; u < kMaxSearchK; ++u) { tv[u] = -INFINITY; ti[u] = INT32_MAX; }
  for (int c = lane; c < n_cand; c += 32) {
    float x = sv[static_cast<int64_t>(q) * n_cand + c];
    int32_t xi = si[static_cast<int64_t>(q) * n_cand + c];
#pragma unroll
    for (int u = 0; u < kMaxSearchK; ++u) {
      const bool take = better_vi(x, xi, tv[u], ti[u]);
      const float pv = tv[u];
      const int32_t pi = ti[u];
      tv[u] = take ? x : pv;
      ti[u] = take ? xi : pi;
      x = take ? pv : x;
      xi = take ? pi : xi;
    }
  }
  for (int r = 0; r < k; ++r) {
    float bv = tv[0];
    int32_t bi = ti[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int32_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (better_vi(ov, oi, bv, bi)) { bv = ov; bi = oi; }
    }
    if (lane == 0) {
      idx[static_cast<int64_t>(q) * k + r] = bi;
      if (val) val[static_cast<int64_t>(q) * k + r] = bv;
    }
    if (ti[0] == bi && tv[0] == bv) {                    // the winner's lane moves to its next candidate
#pragma unroll
      for (int u = 0; u + 1 < kMaxSearchK; ++u) { tv[u] = tv[u + 1]; ti[u] = ti[u + 1]; }
      tv[kMaxSearchK - 1] = -INFINITY;
      ti[kMaxSearchK - 1] = INT32_MAX;
    }
  }
}

// ---------------------------------------------------------------------------
// host
// ---------------------------------------------------------------------------
// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per device (bit d of
// `done`); devices beyond 63 set it on every call
int set_smem_once(const void* fn, size_t bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return static_cast<int>(e);
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return 0;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e != cudaSuccess) return static_cast<int>(e);
  if (bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return 0;
}

constexpr size_t gemm_smem_bytes() { return 1024 + kStages * (kABytes + kBBytes) + 256 + kTN * 8 + 16 + kLocalFix * 4; }

int make_map(CUtensorMap* map, const void* ptr, int64_t cols, int64_t rows, int box_rows) {
  auto encode = tensor_map_encoder();
  if (!encode) return static_cast<int>(cudaErrorNotSupported);
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kKB), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : static_cast<int>(cudaErrorInvalidValue);
}

template <int NACC, int MODE, class Epi>
int launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmPlan& plan, int64_t n_rows, int n_cols,
                const Epi& E, int* err, cudaStream_t s) {
  const size_t smem = gemm_smem_bytes();
  static std::atomic<uint64_t> attr_set{0};          // per device, once (a host-side cost per launch otherwise)
  const int e = set_smem_once(reinterpret_cast<const void*>(k_gemm_wide_tc<NACC, MODE, Epi>), smem, attr_set);
  if (e) return e;
  const dim3 grid(static_cast<unsigned>((n_cols + kTN - 1) / kTN), static_cast<unsigned>((n_rows + kTM - 1) / kTM));
  k_gemm_wide_tc<NACC, MODE, Epi><<<grid, kThreads, smem, s>>>(ta, tb, plan, n_rows, n_cols, E, err);
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

int pow2_at_least_sqrt(int d) {          // 2^ceil(log2 sqrt(d))
  int k = 0;
  while ((1 << (2 * k)) < d) ++k;
  return 1 << k;
}

int grid_warps(int64_t n, int nsm) {     // 8 warps per CTA, at most 16 CTAs per SM
  const int64_t want = (n + 7) / 8, cap = static_cast<int64_t>(nsm) * 16;
  return static_cast<int>(want < cap ? want : cap);
}

template <int E, bool BF16>
int launch_prep(const KParams& P, const void* x, int64_t n_rows, int64_t ld, const Packed& out, const PrepArgs& A,
                int nsm, cudaStream_t s) {
  k_quantize_residual_warp<E, BF16><<<grid_warps(n_rows, nsm), 256, 0, s>>>(P, x, n_rows, ld, out, A);
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

template <int E>
int launch_prep_E(const KParams& P, const void* x, int bf16, int64_t n_rows, int64_t ld, const Packed& out,
                  const PrepArgs& A, int nsm, cudaStream_t s) {
  return bf16 ? launch_prep<E, true>(P, x, n_rows, ld, out, A, nsm, s)
              : launch_prep<E, false>(P, x, n_rows, ld, out, A, nsm, s);
}

}  // namespace

bool wide_applies(const tq_ctx& ctx) {
  const KParams& P = ctx.kp;
  return ctx.use_tc && P.d >= 256 && P.d <= 4096 && P.m <= 4096 &&
         tensor_map_encoder() != nullptr;
}

bool wide_quantize_applies(const tq_ctx& ctx, int64_t n_rows) {
  return wide_applies(ctx) && n_rows >= 4096;            // any m (a multiple of 32): B rows past m read as zeros
}

bool wide_logits_applies(const tq_ctx& ctx, int64_t n_sets, int g, int64_t n_keys) {
  // the z segment is whole 64-column blocks; queries fill 256-column tiles
  return wide_applies(ctx) && ctx.kp.m % 64 == 0 && g >= 64 && n_keys >= 4096 && n_sets >= 1;
}

int64_t wide_chunk_rows() { return static_cast<int64_t>(kChunkTiles) * kTM; }


namespace {
// Write-half scratch of one call, carved from the caller's workspace:
// residual halves [rows, 2d] binary16 | s ||r|| [rows] f32 | fix-up list
// [rows m / 8] u32 | its counter, for one chunk of at most kQuantChunkTiles
// row tiles.
struct QuantScratch {
  int64_t rows_cap;
  uint32_t fix_cap;
  size_t rn_off, fix_off, cnt_off, total;
};
QuantScratch quant_scratch(const KParams& P, int64_t n_rows) {
  QuantScratch q{};
  const int64_t chunk = static_cast<int64_t>(kQuantChunkTiles) * kTM;
  q.rows_cap = n_rows < chunk ? n_rows : chunk;
  q.fix_cap = static_cast<uint32_t>(q.rows_cap * P.m / 8);
  const size_t res_bytes = static_cast<size_t>(q.rows_cap) * 2 * P.d * 2;
  q.rn_off = (res_bytes + 255) / 256 * 256;
  q.fix_off = q.rn_off + (static_cast<size_t>(q.rows_cap) * 4 + 255) / 256 * 256;
  q.cnt_off = q.fix_off + (static_cast<size_t>(q.fix_cap) * 4 + 255) / 256 * 256;
  q.total = q.cnt_off + 256;
  return q;
}
}  // namespace

size_t wide_quantize_scratch_bytes(const tq_ctx& ctx, int64_t n_rows) {
  return quant_scratch(ctx.kp, n_rows).total;
}

int launch_quantize_wide(const tq_ctx& ctx, const void* x, int x_is_bf16, int64_t n_rows, int64_t ld,
                         const Packed& out, void* scratch, void* stream) {
  const KParams& P = ctx.kp;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int d = P.d, m = P.m;
  const int64_t chunk = static_cast<int64_t>(kQuantChunkTiles) * kTM;
  const QuantScratch Q = quant_scratch(P, n_rows);
  const int64_t rows_cap = Q.rows_cap;
  const uint32_t fix_cap = Q.fix_cap;
  const size_t rn_off = Q.rn_off, fix_off = Q.fix_off, cnt_off = Q.cnt_off;
  cudaError_t e = cudaSuccess;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  PrepArgs A;
  A.res = reinterpret_cast<__half*>(base);
  A.rn = reinterpret_cast<float*>(base + rn_off);
  A.s = static_cast<float>(8 * pow2_at_least_sqrt(d));
  uint32_t* fix = reinterpret_cast<uint32_t*>(base + fix_off);
  uint32_t* nfix = reinterpret_cast<uint32_t*>(base + cnt_off);
  A.nfix = nfix;

  CUtensorMap ta, tb;
  int err;
  if ((err = make_map(&ta, A.res, 2 * d, rows_cap, kTM))) return err;
  if ((err = make_map(&tb, P.S, d, m, kTN))) return err;
  GemmPlan plan{};
  plan.nseg = 2;
  plan.seg[0] = {0, 0, d / kKB, 0};                   // r_hi S^T
  plan.seg[1] = {d / kKB, 0, d / kKB, 0};             // r_lo S^T
  plan.b_row0 = 0;
  SignEpi Ep;
  Ep.words_per_row = m / 32;
  Ep.rn = A.rn;
  Ep.snorm = ctx.snorm_dev;
  Ep.eps_rel = static_cast<float>((d / 8 + 2) * std::ldexp(1.0, -22));
  Ep.eps_abs = static_cast<float>(std::ldexp(1.0, -24) * ctx.s1max);
  Ep.fix = fix;
  Ep.nfix = nfix;
  Ep.fix_cap = fix_cap;

  for (int64_t r0 = 0; r0 < n_rows; r0 += chunk) {
    const int64_t nr = n_rows - r0 < chunk ? n_rows - r0 : chunk;
    const Packed po{out.codes + r0 * P.codes_bytes, out.signs + r0 * P.signs_bytes, out.norm + r0, out.rnorm + r0};
    const void* xr = static_cast<const uint8_t*>(x) + r0 * ld * (x_is_bf16 ? 2 : 4);
    switch (d / 32) {
      case 8: err = launch_prep_E<8>(P, xr, x_is_bf16, nr, ld, po, A, ctx.num_sms, s); break;
      case 16: err = launch_prep_E<16>(P, xr, x_is_bf16, nr, ld, po, A, ctx.num_sms, s); break;
      case 32: err = launch_prep_E<32>(P, xr, x_is_bf16, nr, ld, po, A, ctx.num_sms, s); break;
      case 64: err = launch_prep_E<64>(P, xr, x_is_bf16, nr, ld, po, A, ctx.num_sms, s); break;
      case 128: err = launch_prep_E<128>(P, xr, x_is_bf16, nr, ld, po, A, ctx.num_sms, s); break;
      default: err = static_cast<int>(cudaErrorInvalidValue);
    }
    if (err) return err;
    Ep.signs = reinterpret_cast<uint32_t*>(po.signs);
    if ((err = launch_gemm<1, kSigns>(ta, tb, plan, nr, m, Ep, P.err, s))) return err;
    k_qjl_fixup<<<ctx.num_sms * 8, 256, 0, s>>>(P, A.res, fix, nfix, fix_cap, Ep.signs, m / 32);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return static_cast<int>(e);
  }
  return 0;
}

namespace {

// estimates of every query of a set against every key of that set, per
// 18944-key chunk: key operand, then the GEMM with the MODE epilogue
// Estimates scratch, carved from the caller's workspace: decoded keys
// [keys per chunk, 2d + m] binary16 | split queries [n_q, 2(d + m)] binary16 |
// query scales [n_q, 2] f32.
struct EstScratch {
  int64_t keys_cap;
  size_t b_off, qs_off, total;
};
EstScratch est_scratch(const KParams& P, int64_t n_q, int64_t n_keys) {
  EstScratch q{};
  const int64_t chunk = wide_chunk_rows();
  q.keys_cap = n_keys < chunk ? n_keys : chunk;
  const size_t a_bytes = static_cast<size_t>(q.keys_cap) * (2 * P.d + P.m) * 2;
  q.b_off = (a_bytes + 255) / 256 * 256;
  q.qs_off = q.b_off + (static_cast<size_t>(n_q) * 2 * (P.d + P.m) * 2 + 255) / 256 * 256;
  q.total = q.qs_off + (static_cast<size_t>(n_q) * 8 + 255) / 256 * 256;
  return q;
}

template <int MODE>
int run_estimates(const tq_ctx& ctx, const float* qp, int64_t n_sets, int g, const Packed& keys, int64_t n_keys,
                  const LogitEpi& tmpl, void* scratch, cudaStream_t s) {
  const KParams& P = ctx.kp;
  const int d = P.d, m = P.m;
  const int64_t n_q = n_sets * g;
  const int64_t chunk = wide_chunk_rows();
  const EstScratch Q = est_scratch(P, n_q, n_keys);
  const int64_t keys_cap = Q.keys_cap;
  const int64_t lda = 2 * d + m, ldb = 2 * (d + m);
  const size_t b_off = Q.b_off, qs_off = Q.qs_off;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  __half* a = reinterpret_cast<__half*>(base);
  __half* b = reinterpret_cast<__half*>(base + b_off);
  float* qscale = reinterpret_cast<float*>(base + qs_off);

  const int sc = pow2_at_least_sqrt(d);
  k_query_operand<<<grid_warps(n_q, ctx.num_sms), 256, 0, s>>>(P, qp, n_q, 1.0f / static_cast<float>(sc), b,
                                                               qscale);
  count_launch();
  KeyOpArgs K{};
  for (int i = 0; i < P.L; ++i) {
    const double v = static_cast<double>(P.c[i]) * sc;
    const uint16_t h = double_to_half_bits(v);
    K.c_hi[i] = h;
    K.c_lo[i] = double_to_half_bits(v - half_bits_to_double(h));
  }
  CUtensorMap ta, tb;
  int err;
  if ((err = make_map(&ta, a, lda, keys_cap, kTM))) return err;
  if ((err = make_map(&tb, b, ldb, n_q, kTN))) return err;
  GemmPlan plan{};
  plan.nseg = 5;
  const int nd = d / kKB, nm = m / kKB;
  plan.seg[0] = {0, 0, nd, 0};                        // c_hi q_hi
  plan.seg[1] = {nd, 0, nd, 0};                       // c_lo q_hi
  plan.seg[2] = {0, nd, nd, 0};                       // c_hi q_lo
  plan.seg[3] = {2 * nd, 2 * nd, nm, 1};              // z sq_hi
  plan.seg[4] = {2 * nd, 2 * nd + nm, nm, 1};         // z sq_lo
  for (int64_t set = 0; set < n_sets; ++set) {
    plan.b_row0 = static_cast<int>(set * g);
    for (int64_t k0 = 0; k0 < n_keys; k0 += chunk) {
      const int64_t nk = n_keys - k0 < chunk ? n_keys - k0 : chunk;
      const int64_t row = set * n_keys + k0;
      const Packed kk{keys.codes + row * P.codes_bytes, keys.signs + row * P.signs_bytes, keys.norm + row,
                      keys.rnorm + row};
      k_key_operand<<<grid_warps(nk, ctx.num_sms), 256, 0, s>>>(P, kk, nk, K, a);
      count_launch();
      LogitEpi Ep = tmpl;
      if (MODE == kScores) Ep.out = tmpl.out + set * g * n_keys;
      Ep.ld_out = n_keys;
      Ep.key0 = k0;
      Ep.norm = kk.norm;
      Ep.rnorm = kk.rnorm;
      Ep.qscale = qscale + 2 * set * g;
      if ((err = launch_gemm<2, MODE>(ta, tb, plan, nk, g, Ep, P.err, s))) return err;
    }
  }
  return 0;
}


}  // namespace

size_t wide_logits_scratch_bytes(const tq_ctx& ctx, int64_t n_sets, int g, int64_t n_keys) {
  return est_scratch(ctx.kp, n_sets * g, n_keys).total;
}

int launch_logits_wide(const tq_ctx& ctx, const float* qp, int64_t n_sets, int g, const Packed& keys,
                       int64_t n_keys, float* out, void* scratch, void* stream) {
  LogitEpi t{};
  t.out = out;
  return run_estimates<kScores>(ctx, qp, n_sets, g, keys, n_keys, t, scratch, static_cast<cudaStream_t>(stream));
}

bool wide_search_applies(const tq_ctx& ctx, int64_t n_q, int64_t n_keys, int k) {
  return wide_applies(ctx) && ctx.kp.m % 64 == 0 && n_q >= 64 && n_keys >= 4096 && k >= 1 && k <= kMaxSearchK;
}

namespace {
int search_splits(const tq_ctx& ctx, int64_t n_q) {     // CTAs per query tile
  const int64_t qtiles = (n_q + kTM - 1) / kTM;
  const int64_t s = ctx.num_sms / qtiles;
  return static_cast<int>(s < 1 ? 1 : s);
}
}  // namespace

namespace {
// Search scratch, carved from the caller's workspace: per-CTA candidate
// values and rows [n_q, splits, k] | decoded keys [keys per chunk, 2d + m]
// binary16 | split queries [n_q, 2(d + m)] binary16 | query scales [n_q, 2] f32.
struct SearchScratch {
  int S, tps;
  int64_t chunk, keys_cap;
  size_t si_off, kop_off, a_off, qs_off, total;
};
SearchScratch search_scratch(const tq_ctx& ctx, int64_t n_q, int64_t n_keys, int k) {
  const KParams& P = ctx.kp;
  SearchScratch q{};
  q.S = search_splits(ctx, n_q);
  q.tps = kSearchTiles / q.S > 0 ? kSearchTiles / q.S : 1;       // key tiles per CTA and chunk
  q.chunk = static_cast<int64_t>(q.S) * q.tps * kTN;
  q.keys_cap = n_keys < q.chunk ? n_keys : q.chunk;
  const size_t lists = round256(static_cast<size_t>(n_q) * q.S * k * 4);
  q.si_off = lists;
  q.kop_off = 2 * lists;
  q.a_off = q.kop_off + round256(static_cast<size_t>(q.keys_cap) * (2 * P.d + P.m) * 2);
  q.qs_off = q.a_off + round256(static_cast<size_t>(n_q) * 2 * (P.d + P.m) * 2);
  q.total = q.qs_off + round256(static_cast<size_t>(n_q) * 8);
  return q;
}
}  // namespace

size_t wide_search_partial_bytes(const tq_ctx& ctx, int64_t n_q, int64_t n_keys, int k) {
  return search_scratch(ctx, n_q, n_keys, k).total;
}

int launch_search_wide(const tq_ctx& ctx, const float* qp, int64_t n_q, const Packed& keys, int64_t n_keys, int k,
                       int32_t* idx, float* val, void* part, void* stream) {
  const KParams& P = ctx.kp;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int d = P.d, m = P.m;
  const SearchScratch Q = search_scratch(ctx, n_q, n_keys, k);
  const int S = Q.S;
  const int qtiles = static_cast<int>((n_q + kTM - 1) / kTM);
  const int tps = Q.tps;
  const int64_t chunk = Q.chunk;
  const int64_t keys_cap = Q.keys_cap;
  const int64_t lda = 2 * (d + m), ldb = 2 * d + m;              // A: split queries, B: decoded keys
  cudaError_t e = cudaSuccess;
  uint8_t* base = static_cast<uint8_t*>(part);
  float* sv = reinterpret_cast<float*>(base);
  int32_t* si = reinterpret_cast<int32_t*>(base + Q.si_off);
  __half* kop = reinterpret_cast<__half*>(base + Q.kop_off);
  __half* qop = reinterpret_cast<__half*>(base + Q.a_off);
  float* qscale = reinterpret_cast<float*>(base + Q.qs_off);

  const int sc = pow2_at_least_sqrt(d);
  k_query_operand<<<grid_warps(n_q, ctx.num_sms), 256, 0, s>>>(P, qp, n_q, 1.0f / static_cast<float>(sc), qop,
                                                               qscale);
  count_launch();
  KeyOpArgs K{};
  for (int i = 0; i < P.L; ++i) {
    const double v = static_cast<double>(P.c[i]) * sc;
    const uint16_t h = double_to_half_bits(v);
    K.c_hi[i] = h;
    K.c_lo[i] = double_to_half_bits(v - half_bits_to_double(h));
  }
  CUtensorMap ta, tb;
  int err;
  if ((err = make_map(&ta, qop, lda, n_q, kTM))) return err;
  if ((err = make_map(&tb, kop, ldb, keys_cap, kTN))) return err;
  GemmPlan plan{};
  plan.nseg = 5;
  const int nd = d / kKB, nm = m / kKB;
  plan.seg[0] = {0, 0, nd, 0};                        // q_hi c_hi
  plan.seg[1] = {0, nd, nd, 0};                       // q_hi c_lo
  plan.seg[2] = {nd, 0, nd, 0};                       // q_lo c_hi
  plan.seg[3] = {2 * nd, 2 * nd, nm, 1};              // sq_hi z
  plan.seg[4] = {2 * nd + nm, 2 * nd, nm, 1};         // sq_lo z
  const size_t smem = 1024 + kStages * (kABytes + kBBytes) + 256 + 2 * kTN * 4;
  static std::atomic<uint64_t> attr_set{0};
  if ((err = set_smem_once(reinterpret_cast<const void*>(k_search_tc), smem, attr_set))) return err;
  for (int64_t k0 = 0; k0 < n_keys; k0 += chunk) {
    const int64_t nk = n_keys - k0 < chunk ? n_keys - k0 : chunk;
    const Packed kk{keys.codes + k0 * P.codes_bytes, keys.signs + k0 * P.signs_bytes, keys.norm + k0,
                    keys.rnorm + k0};
    k_key_operand<<<grid_warps(nk, ctx.num_sms), 256, 0, s>>>(P, kk, nk, K, kop);
    count_launch();
    SearchArgs X{};
    X.norm = kk.norm;
    X.rnorm = kk.rnorm;
    X.qscale = qscale;
    X.sv = sv;
    X.si = si;
    X.k = k;
    X.S = S;
    X.n_q = static_cast<int>(n_q);
    X.key0 = k0;
    X.nk = nk;
    X.tiles_per_split = tps;
    X.first = k0 == 0;
    k_search_tc<<<dim3(qtiles, S), kSearchThreads, smem, s>>>(ta, tb, plan, X, P.err);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return static_cast<int>(e);
  }
  k_merge_lists<<<static_cast<unsigned>((n_q + 7) / 8), 256, 0, s>>>(sv, si, S * k, k, static_cast<int>(n_q), idx,
                                                                      val);
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

}  // namespace tq
