// Read half, estimated attention logits from packed keys at d = 128, m = 128,
// b = 2 or 3 (1- or 2-bit codes), on the tcgen05 tensor cores.
//
//   logit(q, k) = norm <R q, yhat> + rnorm sqrt(pi/2)/m <S R q, z>
//   -- Qiita TurboQuant explainer, "Stage 2: QJL" (the estimator), with
//      q_rot = R q and sq = S q_rot prepared once per query.
//
// Both inner products are linear in the stored bits.  For 1- and 2-bit
// symmetric Lloyd-Max codebooks the centroid is affine in the code bits,
//   B = 2: c[code] = -c3 + (c3 - c2) b0 + (c3 + c2) b1,   B = 1: c = -c1 + 2 c1 b0.
// A symmetric 3-bit codebook is an odd function of x_i = 2 b_i - 1 (the
// mirror code complements every bit), so it is a0 x0 + a1 x1 + a2 x2 +
// a3 x0 x1 x2 exactly, and x0 x1 x2 = 2 p - 1 with p = b0 ^ b1 ^ b2:
//   B = 3: c[code] = sum_i 2 a_i b_i + 2 a3 p - (a0 + a1 + a2 + a3),
// one more bit plane (the per-code parity) next to the three code planes.
// z_j = 1 - 2 bit_j, so for each key
//   <q_rot, yhat> = const_q + sum_(bits) weight(bit) q_rot[coord(bit)] * bit
//   <sq, z>       = sum_j sq_j - 2 sum_j sq_j bit_j.
// Each key's bits become an unsigned 8-bit row of 0/1 values in TMEM (two
// integer ops per four bits, taken straight from the packed words), and one
// integer MMA (kind::i8, exact int32 accumulation) per 128-key tile multiplies
// them with the set's queries, which sit in shared memory as three signed
// 8-bit limbs of a fixed-point value per (bit, query).  The epilogue recombines
// the limbs, adds the constants and applies norm and rnorm.
//
// Work split, two forms.  Warp-specialized (k_logits_d128_ws, used whenever
// every CTA's contiguous range of 128-key tiles spans at most two sets):
// decode, MMA-issue and epilogue warps pass tiles through four (two for 3-bit
// codes) TMEM slots.  General (k_logits_d128_i8): persistent CTAs of four
// warpgroups (two for 3-bit codes, whose wider operand takes 160 of a
// warpgroup's TMEM columns); each warpgroup walks a contiguous range of tiles
// (so the set, and with it the query operand it builds in its own
// shared-memory slot, changes rarely), one thread per key, decode, MMAs and
// epilogue in turn.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "sm100.cuh"
#include "tq_internal.h"

namespace tq {

namespace {

using namespace sm100;

constexpr int kD = 128, kM = 128, kTile = 128;
constexpr uint32_t kTmemCols = 512;          // split evenly between the warpgroups (A columns, then D)

__host__ __device__ constexpr uint32_t idesc_i8(uint32_t M, uint32_t N) {
  return (2u << 4)              // D format: S32
         | (0u << 7)            // A: unsigned 8-bit
         | (1u << 10)           // B: signed 8-bit
         | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// the same with a signed 8-bit A
__host__ __device__ constexpr uint32_t idesc_s8(uint32_t M, uint32_t N) { return idesc_i8(M, N) | (1u << 7); }

__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// K-steps [K0, K1) of a 128-key tile into one accumulator: A (0/1 bytes) from the
// tile's TMEM columns, B from rows of the query operand (N rows per 128-byte K atom)
// (ACC: the first step accumulates onto what the accumulator holds)
template <int K0, int K1, int N, bool ACC = false>
__device__ __forceinline__ void mma_chain(uint32_t d_tmem, uint32_t a_tmem, uint32_t sbase, uint32_t idesc) {
#pragma unroll
  for (int k = K0; k < K1; ++k) {
    const uint64_t bdesc = smem_desc_sw128(sbase + (k >> 2) * (N * 128) + (k & 3) * 32, 1024);
    mma_i8_ts(d_tmem, a_tmem + k * 8, bdesc, idesc, (ACC || k > K0) ? 1u : 0u);
  }
}

template <int B>
struct Shape {
  static constexpr int kCodeWords = B * 4;                  // 32-bit words of codes per key
  static constexpr int kParWords = B == 3 ? 4 : 0;          // per-code parity bits (3-bit codes)
  static constexpr int kCodeBytes = B * 16;
  static constexpr int kWG = B == 3 ? 2 : 4;                // warpgroups per CTA
  static constexpr int kThreads = kWG * 128;
  static constexpr uint32_t kColsPerWG = kTmemCols / kWG;
  static constexpr int kAWords = 8 * (kCodeWords + kParWords + 4);   // 0/1 bytes, four per TMEM column
  static constexpr int kK = 4 * kAWords;                    // K of the MMA (bytes)
  static constexpr int kKBlocks = kK / 128;                 // 128-byte swizzle atoms along K
  static constexpr int kKSteps = kK / 32;
  static constexpr int kStageBytes = kTile * (kCodeBytes + 16);   // one tile's codes | signs
  // K-steps of the code (and parity) planes, then 4 of the sign plane.  They run as
  // separate MMA chains issued by different warps (one thread issues an MMA only every
  // few dozen cycles): the code steps against the N / 2 code-limb rows of the query
  // operand, the sign steps against the sign-limb rows, and for 3-bit codes the code
  // steps split once more into a second accumulator of their own.
  static constexpr int kMseSteps = kCodeWords + kParWords;
  static constexpr int kChains = B == 3 ? 3 : 2;
};

constexpr int kStages = 4;                   // packed tiles in flight per warpgroup
constexpr int kScalFloats = 160;             // per-warpgroup partial maxima / sums, constants, scales

// Four signed 8-bit limbs of v (|v| < 2^31): v = l0 + 2^8 l1 + 2^16 l2 + 2^24 l3.
__device__ __forceinline__ void split_limbs(int v, int8_t* l) {
  const int l0 = static_cast<int8_t>(v & 0xff);
  const int r1 = (v - l0) >> 8;
  const int l1 = static_cast<int8_t>(r1 & 0xff);
  const int r2 = (r1 - l1) >> 8;
  const int l2 = static_cast<int8_t>(r2 & 0xff);
  l[0] = static_cast<int8_t>(l0);
  l[1] = static_cast<int8_t>(l1);
  l[2] = static_cast<int8_t>(l2);
  l[3] = static_cast<int8_t>((r2 - l2) >> 8);
}

// Recombined limb sums.  Each accumulator is at most 128 * (255 / 8) * K < 2^22 in
// magnitude (K <= 640 operand bytes), so the two
// low limbs join exactly in 32-bit integers; the rest is two fp32 FMAs.
__device__ __forceinline__ float join_limbs(const uint32_t* a) {
  const int lo = static_cast<int>(a[0]) + static_cast<int>(a[1] << 8);
  return fmaf(static_cast<float>(static_cast<int>(a[3])), 16777216.f,
              fmaf(static_cast<float>(static_cast<int>(a[2])), 65536.f, static_cast<float>(lo)));
}

// The same for accumulators up to 2^23 in magnitude (centroid byte planes):
// the two low limbs join in 64-bit integers.
__device__ __forceinline__ float join_limbs_wide(const uint32_t* a) {
  const long long lo = static_cast<long long>(static_cast<int>(a[0])) +
                       static_cast<long long>(static_cast<int>(a[1])) * 256ll;
  return fmaf(static_cast<float>(static_cast<int>(a[3])), 16777216.f,
              fmaf(static_cast<float>(static_cast<int>(a[2])), 65536.f, static_cast<float>(lo)));
}

struct LogitsArgs {
  float wbit[3];                  // weight of code bit 0 / 1 / 2 in the centroid
  float wpar;                     // weight of the code's parity bit (3-bit codes)
  float cconst;                   // centroid constant term
  // 3-bit codes in the warp-specialized kernel: each centroid as a 16-bit fixed
  // point value round(c s), s = 32767 / max |c|, split into a signed high byte
  // and an unsigned low byte (lut8: high bytes of codes 0..3, 4..7, low bytes
  // likewise, for byte permutes), and 1 / s
  uint32_t lut8[4];
  float cinv;
  long long wait_cycles;          // bound of every wait
  int* err;
};

// Every third bit of x (bits 0, 3, ..., 30) packed into bits 0..10.
__device__ __forceinline__ uint32_t every_third_bit(uint32_t x) {
  x &= 0x49249249u;
  x = (x | (x >> 2)) & 0xC30C30C3u;
  x = (x | (x >> 4)) & 0x0F00F00Fu;
  x = (x | (x >> 8)) & 0xFF0000FFu;
  x = (x | (x >> 16)) & 0x0000FFFFu;
  return x;
}

// Parity of each of the 32 3-bit codes held in three consecutive stream words
// (code i in bits 3i .. 3i + 2 of w0 | w1 << 32 | w2 << 64), bit i of the result.
__device__ __forceinline__ uint32_t code_parities(uint32_t w0, uint32_t w1, uint32_t w2) {
  const uint32_t x0 = w0 ^ __funnelshift_r(w0, w1, 1) ^ __funnelshift_r(w0, w1, 2);
  const uint32_t x1 = w1 ^ __funnelshift_r(w1, w2, 1) ^ __funnelshift_r(w1, w2, 2);
  const uint32_t x2 = w2 ^ (w2 >> 1) ^ (w2 >> 2);
  return every_third_bit(x0) | (every_third_bit(x1 >> 1) << 11) | ((every_third_bit(x2 >> 2) & 0x3FFu) << 22);
}

// The query operand of one set in shared memory, built by the 128 threads of
// a warpgroup (thread trow = 32 wl + lane owns coordinate / projection trow):
// per (K position, query) the fixed-point value as four signed 8-bit limbs in
// the MMA's B layout (N rows of 128-byte K atoms, swizzled), plus the per-query
// constants and inverse scales in sScal (partial maxima at 0, partial sums at
// 64, constants at 128, inverse scales at 144).  Ends with the operand visible
// to the tensor cores and a barrier of the 128 threads.
//
// BYTES: the byte-plane operand of 3-bit codes (warp-specialized kernel): K
// positions 0..127 the centroids' high bytes of coordinates 0..127, 128..255
// their low bytes, 256..383 the sign bits as in the bit-plane form; the query
// value of a coordinate, at 2^fe, times 256 against the high byte; no constant
// term, and the inverse scale carries 1 / s instead of 2^-7.
template <int B, int G, int NG, bool BYTES = false>
__device__ __forceinline__ void build_query_operand(const LogitsArgs& X, const float* __restrict__ qs, int trow,
                                                    int wl, int lane, float* sScal, uint8_t* sB, uint32_t bar_id) {
  using S = Shape<B>;
  constexpr int N = 2 * NG;
  constexpr int kK = BYTES ? 384 : S::kK;
  constexpr int kSignCol = BYTES ? 64 : 8 * (S::kCodeWords + S::kParWords);   // first column of the sign plane
  // per-warp maxima and sums of every query's two halves, combined below in a
  // fixed order (thread trow owns coordinate / projection trow)
  float* sPM = sScal;                               // [warp][2G] partial maxima
  float* sPS = sScal + 64;                          // [warp][2G] partial sums
  float* sC = sScal + 128;                          // [2G] constant terms
  float* sInv = sScal + 144;                        // [2G] inverse fixed-point scales
#pragma unroll
  for (int q = 0; q < G; ++q) {
    const float va = qs[q * (kD + kM) + trow], vb = qs[q * (kD + kM) + kD + trow];
    float a = fabsf(va), b = fabsf(vb), sa = va, sb = vb;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      b = fmaxf(b, __shfl_xor_sync(0xffffffffu, b, o));
      sa += __shfl_xor_sync(0xffffffffu, sa, o);
      sb += __shfl_xor_sync(0xffffffffu, sb, o);
    }
    if (lane == 0) {
      sPM[wl * 16 + q] = a;
      sPM[wl * 16 + G + q] = b;
      sPS[wl * 16 + q] = sa;
      sPS[wl * 16 + G + q] = sb;
    }
  }
  named_bar_sync(bar_id, 128);
  float wmax = fabsf(X.wbit[0]);
  if (B >= 2) wmax = fmaxf(wmax, fabsf(X.wbit[1]));
  if (B == 3) wmax = fmaxf(wmax, fmaxf(fabsf(X.wbit[2]), fabsf(X.wpar)));
  if (BYTES) wmax = 1.f;
  // fixed-point exponent of half h of query q: |value| * 2^F <= 2^22
  auto fp_exp = [&](int h, int q) {
    const int i = h * G + q;
    const float m = fmaxf(fmaxf(sPM[i], sPM[16 + i]), fmaxf(sPM[32 + i], sPM[48 + i]));
    const float v = h == 0 ? m * wmax : m * 2.f;
    int e = 0;
    frexpf(v > 0.f ? v : 1.f, &e);
    return 22 - e;
  };
  int fe[2 * G];
#pragma unroll
  for (int q = 0; q < G; ++q) {
    fe[q] = fp_exp(0, q);
    fe[G + q] = fp_exp(1, q);
  }
  // operand bytes: K position kappa (byte t of A column o) of this thread.  Column
  // o holds bit t * 8 + (o & 7) of a packed word at bit (o & 7) of each byte, so
  // the byte is bit * 2^(o & 7); the query value is scaled by 2^(7 - (o & 7)) and
  // every product carries the common factor 2^7.
#pragma unroll
  for (int r = 0; r < kK / 128; ++r) {
    const int kappa = trow + 128 * r;
    const int o = kappa >> 2, tb = kappa & 3;
    const int up = 7 - (o & 7);
    int8_t limb[N];
#pragma unroll
    for (int n = 0; n < N; ++n) limb[n] = 0;
    if (BYTES && r < 2) {
      // centroid byte plane r of coordinate trow
#pragma unroll
      for (int q = 0; q < G; ++q) {
        const int v = __float2int_rn(ldexpf(qs[q * (kD + kM) + trow], fe[q])) * (r == 0 ? 256 : 1);
        split_limbs(v, &limb[4 * q]);
      }
    } else if (!BYTES && o < kSignCol) {
      int coord;
      float w;
      if (o < 8 * S::kCodeWords) {
        const int c = o >> 3, k = o & 7;
        const int s = 32 * c + k + 8 * tb;        // bit position in the code stream
        coord = s / B;
        w = X.wbit[s % B];
      } else {
        const int c = (o - 8 * S::kCodeWords) >> 3, k = o & 7;
        coord = 32 * c + k + 8 * tb;              // parity bit of this code
        w = X.wpar;
      }
#pragma unroll
      for (int q = 0; q < G; ++q) {
        const int v = __float2int_rn(ldexpf(w * qs[q * (kD + kM) + coord], fe[q])) * (1 << up);
        split_limbs(v, &limb[4 * q]);
      }
    } else {
      const int c = (o - kSignCol) >> 3, k = o & 7;
      const int j = 32 * c + k + 8 * tb;           // projection
#pragma unroll
      for (int q = 0; q < G; ++q) {
        const int v = __float2int_rn(ldexpf(-2.f * qs[q * (kD + kM) + kD + j], fe[G + q])) * (1 << up);
        split_limbs(v, &limb[NG + 4 * q]);
      }
    }
    const int kb = kappa >> 7, chunk = (kappa & 127) >> 4, within = kappa & 15;
#pragma unroll
    for (int n = 0; n < N; ++n)
      sB[kb * (N * 128) + n * 128 + ((chunk ^ (n & 7)) << 4) + within] = static_cast<uint8_t>(limb[n]);
  }
  // per-query constants (c_const * sum q_rot, sum sq) and the inverse scales
  // with the 2^-7 of the shifted bits
  if (trow < 2 * G) {
    const float sum = (sPS[trow] + sPS[16 + trow]) + (sPS[32 + trow] + sPS[48 + trow]);
    const int h = trow >= G ? 1 : 0;
    sC[trow] = h ? sum : (BYTES ? 0.f : X.cconst * sum);
    sInv[trow] = (BYTES && h == 0) ? ldexpf(X.cinv, -fp_exp(h, trow)) : ldexpf(1.f, -fp_exp(h, trow - h * G) - 7);
  }
  fence_proxy_async_smem();
  named_bar_sync(bar_id, 128);
}

template <int B, int G, int NG>
__global__ void __launch_bounds__(Shape<B>::kThreads, 1)
k_logits_d128_i8(const KParams P, const LogitsArgs X, const float* __restrict__ qp, int64_t n_sets,
                 int64_t n_keys, const Packed keys, float* __restrict__ out) {
  using S = Shape<B>;
  constexpr int kWG = S::kWG;
  constexpr int N = 2 * NG;
  constexpr int kBBytes = S::kKBlocks * N * 128;            // query operand per warpgroup
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wg = warp >> 2, wl = warp & 3;
  uint8_t* sB = smem + wg * kBBytes;
  uint8_t* stages = smem + kWG * kBBytes + wg * kStages * S::kStageBytes;
  float* sScal = reinterpret_cast<float*>(smem + kWG * (kBBytes + kStages * S::kStageBytes)) + wg * kScalFloats;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWG * (kBBytes + kStages * S::kStageBytes) + kWG * kScalFloats * 4);
  uint64_t* full = bars + wg * kStages;                     // [wg][stage]
  uint64_t* mdone = bars + kWG * kStages;                   // [wg]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + kWG);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  if (tid == 0) {
    for (int i = 0; i < kWG * kStages; ++i) mbar_init(&bars[i], 1);
    for (int i = 0; i < kWG; ++i) mbar_init(&mdone[i], S::kChains);   // one commit per chain
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool leader = (wl == 0 && lane == 0);
  const int trow = wl * 32 + lane;
  const uint32_t t_base = tmem + (static_cast<uint32_t>(wl * 32) << 16) + wg * S::kColsPerWG;   // my lane
  // A columns, then the accumulator: N columns (code limbs | sign limbs), and for
  // 3-bit codes NG more for the second half of the code steps
  const uint32_t t_a = t_base, t_d = t_base + S::kAWords;

  // contiguous tile range of this warpgroup; (set, key tile) advance incrementally
  const int64_t tiles_per_set = (n_keys + kTile - 1) / kTile;
  const int64_t n_tiles = tiles_per_set * n_sets;
  const int64_t n_wg = static_cast<int64_t>(gridDim.x) * kWG;
  const int64_t wid = static_cast<int64_t>(blockIdx.x) * kWG + wg;
  const int64_t t0 = n_tiles * wid / n_wg, t1 = n_tiles * (wid + 1) / n_wg;
  const int64_t n_mine = t1 - t0;
  int64_t set = t0 / tiles_per_set, kt = t0 - (t0 / tiles_per_set) * tiles_per_set;

  // producer (the warpgroup's leader): bulk copies of a tile's codes and signs
  int64_t p_set = set, p_kt = kt, issued = 0, consumed = 0;
  auto issue = [&](int stage) {
    const int64_t row0 = p_set * n_keys + p_kt * kTile;
    const int64_t left = n_keys - p_kt * kTile;
    const uint32_t valid = static_cast<uint32_t>(left < kTile ? left : kTile);
    uint8_t* st = stages + stage * S::kStageBytes;
    mbar_arrive_expect_tx(&full[stage], valid * (S::kCodeBytes + 16));
    bulk_load(st, keys.codes + row0 * S::kCodeBytes, valid * S::kCodeBytes, &full[stage]);
    bulk_load(st + kTile * S::kCodeBytes, keys.signs + row0 * 16, valid * 16, &full[stage]);
    if (++p_kt == tiles_per_set) { p_kt = 0; ++p_set; }
    ++issued;
  };
  if (leader)
    for (int i = 0; i < kStages && i < n_mine; ++i) issue(i);

  // norms of this thread's key, loaded one tile ahead
  float nnrm = 0.f, nrn = 0.f;
  auto load_norms = [&](int64_t s_, int64_t kt_) {
    const int64_t key = kt_ * kTile + trow;
    nnrm = nrn = 0.f;
    if (key < n_keys) {
      nnrm = __ldg(keys.norm + s_ * n_keys + key);
      nrn = __ldg(keys.rnorm + s_ * n_keys + key);
    }
  };
  if (n_mine > 0) load_norms(set, kt);

  int64_t cur_set = -1;
  for (int64_t i = 0; i < n_mine; ++i) {
    const int stage = static_cast<int>(i % kStages);
    const uint32_t parity = static_cast<uint32_t>((i / kStages) & 1);
    const int64_t key = kt * kTile + trow;
    const bool valid = key < n_keys;
    const float nrm = nnrm, rn = nrn * P.qjl_scale;
    int64_t nset = set, nkt = kt + 1;
    if (nkt == tiles_per_set) { nkt = 0; ++nset; }
    if (i + 1 < n_mine) load_norms(nset, nkt);
    if (set != cur_set) {
      // ---- build the query operand of this set --------------------------------
      cur_set = set;
      named_bar_sync(1 + wg, 128);                      // previous tile's MMA inputs no longer in use
      build_query_operand<B, G, NG>(X, qp + set * G * (kD + kM), trow, wl, lane, sScal, sB, 1 + wg);
    }
    // ---- this thread's key from the stage, decoded into TMEM -----------------------
    if (mbar_wait(&full[stage], parity, X.wait_cycles)) {
      if (leader) ++consumed;
    } else {
      if (X.err) atomicCAS(X.err, 0, 7);
      atomicExch(abort_flag, 1);
    }
    {
      uint32_t cw[S::kCodeWords + S::kParWords + 4];
      const uint8_t* st = stages + stage * S::kStageBytes;
      if (valid) {
#pragma unroll
        for (int q = 0; q < B; ++q) {
          const uint4 u = *reinterpret_cast<const uint4*>(st + trow * S::kCodeBytes + 16 * q);
          cw[4 * q] = u.x; cw[4 * q + 1] = u.y; cw[4 * q + 2] = u.z; cw[4 * q + 3] = u.w;
        }
        const uint4 u = *reinterpret_cast<const uint4*>(st + kTile * S::kCodeBytes + trow * 16);
        constexpr int so = S::kCodeWords + S::kParWords;
        cw[so] = u.x; cw[so + 1] = u.y; cw[so + 2] = u.z; cw[so + 3] = u.w;
        if constexpr (B == 3) {
#pragma unroll
          for (int g2 = 0; g2 < 4; ++g2)
            cw[S::kCodeWords + g2] = code_parities(cw[3 * g2], cw[3 * g2 + 1], cw[3 * g2 + 2]);
        }
      } else {
#pragma unroll
        for (int w = 0; w < S::kCodeWords + S::kParWords + 4; ++w) cw[w] = 0u;
      }
      uint32_t a[32];
      int n = 0, col = 0;
#pragma unroll
      for (int c = 0; c < S::kCodeWords + S::kParWords + 4; ++c) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          a[n++] = cw[c] & (0x01010101u << k);
          if (n == 32) {
            tmem_st32(t_a + col, a);
            col += 32;
            n = 0;
          }
        }
      }
    }
    tmem_wait_st();
    tc_fence_before();
    // every thread has read its key from the stage and written its TMEM row
    if (named_bar_sync_or(1 + wg, 128, *reinterpret_cast<volatile int*>(abort_flag) != 0)) break;
    if (leader && issued < n_mine) issue(stage);
    if (lane == 0 && wl < S::kChains) {
      // chain wl: 0 = code steps [0, h), 1 = sign steps, 2 = code steps [h, kMseSteps)
      constexpr int h = S::kChains == 3 ? S::kMseSteps / 2 : S::kMseSteps;
      tc_fence_after();
      const uint32_t a_tmem = tmem + wg * S::kColsPerWG, d_tmem = a_tmem + S::kAWords;
      const uint32_t sbase = smem_u32(sB), idesc = idesc_i8(kTile, NG);
      if (wl == 0) mma_chain<0, h, N>(d_tmem, a_tmem, sbase, idesc);
      else if (wl == 1) mma_chain<S::kMseSteps, S::kKSteps, N>(d_tmem + NG, a_tmem, sbase + NG * 128, idesc);
      else mma_chain<h, S::kMseSteps, N>(d_tmem + N, a_tmem, sbase, idesc);
      mma_commit(&mdone[wg]);
    }
    if (!mbar_wait(&mdone[wg], static_cast<uint32_t>(i & 1), X.wait_cycles)) {
      if (X.err) atomicCAS(X.err, 0, 6);
      atomicExch(abort_flag, 1);
    }
    tc_fence_after();
    // ---- epilogue: recombine limbs, constants, norms ----------------------------------
    uint32_t acc[N];
    {
      uint32_t part[32];
#pragma unroll
      for (int c = 0; c < N / 32; ++c) {
        tmem_ld32(t_d + 32 * c, part);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) acc[32 * c + k] = part[k];
      }
      if constexpr (S::kChains == 3) {
        // the second code accumulator joins the first exactly (integer limbs)
        if constexpr (NG == 16) {
          uint32_t p16[16];
          tmem_ld16(t_d + N, p16);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 16; ++k) acc[k] += p16[k];
        } else {
          tmem_ld32(t_d + N, part);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) acc[k] += part[k];
        }
      }
    }
    tc_fence_before();
    if (valid) {
      float* o = out + set * G * n_keys + key;
      const float* sC = sScal + 128;
      const float* sInv = sScal + 144;
#pragma unroll
      for (int q = 0; q < G; ++q) {
        const float mse_f = join_limbs(&acc[4 * q]);
        const float qjl_f = join_limbs(&acc[NG + 4 * q]);
        const float mse = fmaf(mse_f, sInv[q], sC[q]);
        const float qjl = fmaf(qjl_f, sInv[G + q], sC[G + q]);
        o[q * n_keys] = fmaf(nrm, mse, rn * qjl);
      }
    }
    set = nset;
    kt = nkt;
  }
  if (leader) {
    // copies still in flight (only after an abort): let them land before exit
    for (; consumed < issued; ++consumed) {
      const int64_t j = consumed;
      if (!mbar_wait(&full[j % kStages], static_cast<uint32_t>((j / kStages) & 1), X.wait_cycles)) break;
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Warp-specialized form: one CTA per SM walks a contiguous range of 128-key
// tiles, spanning at most two sets, through kSlots TMEM slots (A columns, then
// the accumulators), so the decode of later tiles runs while the tensor cores
// and the epilogue work on earlier ones.  Warps, in pairs of groups that take
// the tiles of even / odd local index:
//   0 .. 7    two epilogue groups: accumulators -> limbs joined, constants,
//             norms, stores; first, group e builds the query operand of the
//             range's set e (one buffer each);
//   8 .. 15   two decode groups: the group's leader keeps bulk copies of the
//             group's next tiles (codes and signs) in flight in its own stages;
//             the packed words go from the stage into TMEM 0/1 bytes;
//   16 .. 19  MMA issuers, one thread each (a thread issues an MMA only every
//             60 to 100 cycles, so the four issue side by side), one or two
//             per slot: the code steps against the code-limb rows of the query
//             operand, the sign steps against the sign-limb rows.
// 3-bit codes take their centroids as two byte planes here, the high and low
// byte of round(c s) with s = 32767 / max |c| (a byte permute per four
// coordinates from an eight-entry table; the high bytes signed), so a slot
// has the 96 operand columns of b = 3 and the TMEM holds four: the centroid
// error is at most max |c| / 65534 per coordinate, a logit error of at most
// 3.3e-5 |q| |k| at d = 128 (the bit-plane form of the general kernel is exact).
// Barriers per slot: a_ready (decode -> issuers), mma_done (issuers ->
// epilogue), slot_free (epilogue -> decode); per stage: full, stage_free; per
// query buffer: q_ready.  Every wait is bounded and gives up once another
// thread has flagged an abort.
// ---------------------------------------------------------------------------
template <int B, int NG>
struct WsLog {
  using S = Shape<B>;
  static constexpr int N = 2 * NG;                                  // code limbs | sign limbs
  // 3-bit codes as two centroid byte planes (high, low) instead of four bit
  // planes (three code bits and the parity): 96 operand columns, as at b = 3
  static constexpr bool kBytes = B == 3;
  static constexpr int kAWords = kBytes ? 96 : S::kAWords;
  static constexpr int kKSteps = kBytes ? 12 : S::kKSteps;
  static constexpr int kMseSteps = kBytes ? 8 : S::kMseSteps;
  static constexpr int kKBlocks = kBytes ? 3 : S::kKBlocks;
  // a slot: A, then the code | sign accumulators; four slots of 128 columns
  // (one issuer each) or two of 256, each with two issuers, the code steps split
  // between them into a second code accumulator
  static constexpr int kSlots = kAWords + N <= 128 ? 4 : 2;
  static constexpr int kSlotCols = 512 / kSlots;
  static constexpr int kIssuersPerSlot = 4 / kSlots;
  static constexpr int kChains = kSlots == 2 ? 3 : 2;
  static constexpr int kStages = 6;                                 // three per decode group
  static constexpr int kBBytes = kKBlocks * N * 128;
  static constexpr int kThreads = 20 * 32;
};

template <int B, int NG>
constexpr size_t logits_ws_smem_bytes() {
  using W = WsLog<B, NG>;
  return 1024 + 2 * W::kBBytes + W::kStages * Shape<B>::kStageBytes + 2 * kScalFloats * 4 +
         (3 * W::kSlots + 2 * W::kStages + 2 + 4) * 8 + 16;
}

// bounded wait that also gives up once the abort flag is set; a long limit lets
// the waiting thread be suspended between polls (leaving the issue slots to the
// other warps), a short one polls and keeps to the cycle count
__device__ __forceinline__ bool ws_wait(uint64_t* bar, uint32_t parity, long long limit, const int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const bool suspend = limit >= (1ll << 24);
  const long long t0 = clock64();
  for (;;) {
    bool ok;
    if (suspend) {
      uint32_t r;
      asm volatile(
          "{\n\t.reg .pred p;\n\t"
          "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 20000;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(r)
          : "r"(smem_u32(bar)), "r"(parity)
          : "memory");
      ok = r != 0;
    } else {
      ok = mbar_try_wait(bar, parity);
    }
    if (ok) return true;
    if (*reinterpret_cast<volatile const int*>(abort_flag) != 0) return false;
    if (clock64() - t0 > limit) return false;
  }
}

// (set, key tile) of local tile i, stepped forward by a few tiles at a time
struct TileCursor {
  int64_t set, kt, tps;
  __device__ __forceinline__ void step(int by) {
    kt += by;
    while (kt >= tps) {
      kt -= tps;
      ++set;
    }
  }
};

template <int B, int G, int NG>
__global__ void __launch_bounds__(WsLog<B, NG>::kThreads, 1)
k_logits_d128_ws(const KParams P, const LogitsArgs X, const float* __restrict__ qp, int64_t n_sets, int64_t n_keys,
                 const Packed keys, float* __restrict__ out) {
  using S = Shape<B>;
  using W = WsLog<B, NG>;
  constexpr int N = W::N, kSlots = W::kSlots, kSt = W::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sBq = smem;                                                // [2] query operands
  uint8_t* stages = smem + 2 * W::kBBytes;                            // [kSt] codes | signs of a tile
  float* sScal = reinterpret_cast<float*>(stages + kSt * S::kStageBytes);   // [2][kScalFloats]
  uint64_t* a_ready = reinterpret_cast<uint64_t*>(sScal + 2 * kScalFloats);
  uint64_t* mma_done = a_ready + kSlots;
  uint64_t* slot_free = mma_done + kSlots;
  uint64_t* full = slot_free + kSlots;
  uint64_t* stage_free = full + kSt;
  uint64_t* q_ready = stage_free + kSt;                               // [2]
  uint64_t* fdone = q_ready + 2;                                      // [4] issuers' wind-down
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fdone + 4);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long lim = X.wait_cycles;
  if (tid == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&a_ready[s], 4);
      mbar_init(&mma_done[s], W::kIssuersPerSlot);
      mbar_init(&slot_free[s], 4);
    }
    for (int i = 0; i < kSt; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&stage_free[i], 4);
    }
    mbar_init(&q_ready[0], 1);
    mbar_init(&q_ready[1], 1);
    for (int i = 0; i < 4; ++i) mbar_init(&fdone[i], 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto fail = [&](int code) {
    if (X.err) atomicCAS(X.err, 0, code);
    atomicExch(abort_flag, 1);
  };

  // this CTA's contiguous tile range
  const int64_t tps = (n_keys + kTile - 1) / kTile;
  const int64_t n_tiles = tps * n_sets;
  const int64_t t0 = n_tiles * blockIdx.x / gridDim.x, t1 = n_tiles * (blockIdx.x + 1) / gridDim.x;
  const int64_t set0 = t0 / tps;
  const int64_t kt0 = t0 - set0 * tps;
  const int64_t last_set = t1 > t0 ? (t1 - 1) / tps : set0;
  // the launch keeps every range within two sets (one query buffer each)
  const bool span_ok = last_set <= set0 + 1;
  if (!span_ok && tid == 0) fail(9);
  const int n_mine = span_ok ? static_cast<int>(t1 - t0) : 0;

  if (warp < 8) {
    // ================================ epilogue groups ================================
    const int eg = warp >> 2, wl = warp & 3;
    const int trow = wl * 32 + lane;
    const uint32_t bar = 1 + eg;                                      // this group's named barrier
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wl * 32) << 16);
    if (n_mine > 0 && set0 + eg <= last_set) {
      build_query_operand<B, G, NG, W::kBytes>(X, qp + (set0 + eg) * G * (kD + kM), trow, wl, lane,
                                               sScal + eg * kScalFloats, sBq + eg * W::kBBytes, bar);
      if (wl == 0 && lane == 0) mbar_arrive(&q_ready[eg]);
    }
    TileCursor c{set0, kt0, tps};
    c.step(eg);
    float nnrm = 0.f, nrn = 0.f;
    auto load_norms = [&](const TileCursor& cc) {
      const int64_t key = cc.kt * kTile + trow;
      nnrm = nrn = 0.f;
      if (key < n_keys) {
        nnrm = __ldg(keys.norm + cc.set * n_keys + key);
        nrn = __ldg(keys.rnorm + cc.set * n_keys + key);
      }
    };
    if (eg < n_mine) load_norms(c);
    for (int i = eg; i < n_mine; i += 2) {
      const int s = i % kSlots;
      const float nrm = nnrm, rn = nrn * P.qjl_scale;
      TileCursor nx = c;
      nx.step(2);
      if (i + 2 < n_mine) load_norms(nx);
      // (the group's warps meet in no barrier after the operand build: each
      // waits for the accumulators on its own)
      if (!ws_wait(&mma_done[s], static_cast<uint32_t>((i / kSlots) & 1), lim, abort_flag)) { fail(9); break; }
      tc_fence_after();
      const uint32_t t_d = t_lane + s * W::kSlotCols + W::kAWords;
      uint32_t acc[N];
      {
        uint32_t part[32];
#pragma unroll
        for (int cc = 0; cc < N / 32; ++cc) {
          tmem_ld32(t_d + 32 * cc, part);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) acc[32 * cc + k] = part[k];
        }
        if constexpr (W::kChains == 3) {
          // the second code accumulator joins the first exactly (integer limbs)
#pragma unroll
          for (int h = 0; h < NG / 16; ++h) {
            uint32_t p16[16];
            tmem_ld16(t_d + N + 16 * h, p16);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k) acc[16 * h + k] += p16[k];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&slot_free[s]);
      const int64_t key = c.kt * kTile + trow;
      if (key < n_keys) {
        const float* sc = sScal + static_cast<int>(c.set - set0) * kScalFloats;
        float* o = out + c.set * G * n_keys + key;
#pragma unroll
        for (int q = 0; q < G; ++q) {
          const float mse = fmaf(W::kBytes ? join_limbs_wide(&acc[4 * q]) : join_limbs(&acc[4 * q]), sc[144 + q],
                                 sc[128 + q]);
          const float qjl = fmaf(join_limbs(&acc[NG + 4 * q]), sc[144 + G + q], sc[128 + G + q]);
          o[q * n_keys] = fmaf(nrm, mse, rn * qjl);
        }
      }
      c = nx;
    }
  } else if (warp < 16) {
    // ================================ decode groups ================================
    const int grp = (warp - 8) >> 2, wl = warp & 3;
    const int trow = wl * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(wl * 32) << 16);
    const bool leader = wl == 0 && lane == 0;
    constexpr int kGS = kSt / 2;                                      // stages of this group
    // the leader's bulk copies of local tile m (global local index grp + 2 m) into stage grp kGS + m % kGS
    TileCursor cl{set0, kt0, tps};
    cl.step(grp);
    int loads = 0;
    auto issue_load = [&]() {
      const int st = grp * kGS + loads % kGS;
      const int64_t row0 = cl.set * n_keys + cl.kt * kTile;
      const int64_t left = n_keys - cl.kt * kTile;
      const uint32_t valid = static_cast<uint32_t>(left < kTile ? left : kTile);
      uint8_t* sg = stages + st * S::kStageBytes;
      mbar_arrive_expect_tx(&full[st], valid * (S::kCodeBytes + 16));
      bulk_load(sg, keys.codes + row0 * S::kCodeBytes, valid * S::kCodeBytes, &full[st]);
      bulk_load(sg + kTile * S::kCodeBytes, keys.signs + row0 * 16, valid * 16, &full[st]);
      ++loads;
      cl.step(2);
    };
    const int n_grp = n_mine > grp ? (n_mine - grp + 1) / 2 : 0;       // tiles of this group
    if (leader)
      while (loads < kGS && loads < n_grp) issue_load();
    TileCursor c{set0, kt0, tps};
    c.step(grp);
    int m = 0;
    for (int i = grp; i < n_mine; i += 2, c.step(2), ++m) {
      const int s = i % kSlots, n = i / kSlots, st = grp * kGS + m % kGS;
      const uint32_t sph = static_cast<uint32_t>((m / kGS) & 1);
      if (n >= 1 && !ws_wait(&slot_free[s], static_cast<uint32_t>((n - 1) & 1), lim, abort_flag)) { fail(9); break; }
      if (!ws_wait(&full[st], sph, lim, abort_flag)) { fail(9); break; }
      const bool valid = c.kt * kTile + trow < n_keys;
      uint32_t cw[S::kCodeWords + S::kParWords + 4];
      const uint8_t* sg = stages + st * S::kStageBytes;
      if (valid) {
#pragma unroll
        for (int q = 0; q < B; ++q) {
          const uint4 u = *reinterpret_cast<const uint4*>(sg + trow * S::kCodeBytes + 16 * q);
          cw[4 * q] = u.x; cw[4 * q + 1] = u.y; cw[4 * q + 2] = u.z; cw[4 * q + 3] = u.w;
        }
        const uint4 u = *reinterpret_cast<const uint4*>(sg + kTile * S::kCodeBytes + trow * 16);
        constexpr int so = S::kCodeWords + S::kParWords;
        cw[so] = u.x; cw[so + 1] = u.y; cw[so + 2] = u.z; cw[so + 3] = u.w;
      } else {
#pragma unroll
        for (int w = 0; w < S::kCodeWords + S::kParWords + 4; ++w) cw[w] = 0u;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&stage_free[st]);
      const uint32_t t_a = t_lane + s * W::kSlotCols;
      if constexpr (W::kBytes) {
        // the centroid bytes of four coordinates per byte permute: the eight
        // 3-bit codes of a 24-bit group spread to the nibbles of two selectors
        // (three shift-and-merge steps)
#pragma unroll
        for (int j8 = 0; j8 < 4; ++j8) {
          uint32_t hw[8], lw[8];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            const int j = 4 * j8 + jj, bit = 24 * j, w = bit >> 5, sh = bit & 31;
            uint32_t x = sh + 24 <= 32 ? cw[w] >> sh : __funnelshift_r(cw[w], cw[w + 1], sh);
            x = (x & 0xFFFu) | ((x << 4) & 0x0FFF0000u);               // codes 4..7 to bits 16..
            x = (x & 0x003F003Fu) | ((x << 2) & 0x3F003F00u);          // codes 2, 3 (and 6, 7) up by 2
            x = (x & 0x07070707u) | ((x << 1) & 0x70707070u);          // codes 1, 3, 5, 7 up by 1
            hw[2 * jj] = __byte_perm(X.lut8[0], X.lut8[1], x);
            lw[2 * jj] = __byte_perm(X.lut8[2], X.lut8[3], x);
            hw[2 * jj + 1] = __byte_perm(X.lut8[0], X.lut8[1], x >> 16);
            lw[2 * jj + 1] = __byte_perm(X.lut8[2], X.lut8[3], x >> 16);
          }
          tmem_st8(t_a + 8 * j8, hw);
          tmem_st8(t_a + 32 + 8 * j8, lw);
        }
        uint32_t a[32];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int k = 0; k < 8; ++k) a[8 * cc + k] = cw[S::kCodeWords + S::kParWords + cc] & (0x01010101u << k);
        tmem_st32(t_a + 64, a);
      } else {
        if constexpr (B == 3) {
#pragma unroll
          for (int g2 = 0; g2 < 4; ++g2)
            cw[S::kCodeWords + g2] = code_parities(cw[3 * g2], cw[3 * g2 + 1], cw[3 * g2 + 2]);
        }
        uint32_t a[32];
        int na = 0, col = 0;
#pragma unroll
        for (int cc = 0; cc < S::kCodeWords + S::kParWords + 4; ++cc) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            a[na++] = cw[cc] & (0x01010101u << k);
            if (na == 32) {
              tmem_st32(t_a + col, a);
              col += 32;
              na = 0;
            }
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_ready[s]);
      if (leader && loads < n_grp) {
        // refill the stage (the group's four warps read it long before their
        // TMEM rows were written)
        if (!ws_wait(&stage_free[st], sph, lim, abort_flag)) { fail(9); break; }
        issue_load();
      }
    }
    if (leader) {
      // copies still in flight (only after an abort): let them land before exit
      for (int k = loads > kGS ? loads - kGS : 0; k < loads; ++k)
        if (!mbar_wait(&full[grp * kGS + k % kGS], static_cast<uint32_t>((k / kGS) & 1), 2000000000ll)) break;
    }
  } else {
    // ================================ MMA issuers ================================
    const int j = warp - 16, slot = j / W::kIssuersPerSlot, part = j % W::kIssuersPerSlot;
    if (lane == 0) {
      bool issued = false;
      int64_t q_set = -1;
      TileCursor c{set0, kt0, tps};
      c.step(slot);
      const uint32_t idesc = idesc_i8(kTile, NG);
      const uint32_t a_tmem = tmem + slot * W::kSlotCols, d_tmem = a_tmem + W::kAWords;
      // every use of the slot, in order (the slot's barriers complete once per use)
      for (int i = slot; i < n_mine; i += kSlots, c.step(kSlots)) {
        if (c.set != q_set) {
          q_set = c.set;
          if (!ws_wait(&q_ready[c.set - set0], 0u, lim, abort_flag)) { fail(9); break; }
        }
        if (!ws_wait(&a_ready[slot], static_cast<uint32_t>((i / kSlots) & 1), lim, abort_flag)) { fail(9); break; }
        tc_fence_after();
        const uint32_t sbase = smem_u32(sBq + static_cast<int>(c.set - set0) * W::kBBytes);
        // code steps [0, h) and [h, kMseSteps): with centroid byte planes the high
        // bytes (steps 0..3) are signed, the low bytes (4..7) unsigned
        constexpr int h = W::kBytes ? 4 : W::kMseSteps / 2;
        const uint32_t idesc_a = W::kBytes ? idesc_s8(kTile, NG) : idesc;
        if constexpr (W::kIssuersPerSlot == 1) {
          mma_chain<0, h, N>(d_tmem, a_tmem, sbase, idesc_a);
          mma_chain<h, W::kMseSteps, N, true>(d_tmem, a_tmem, sbase, idesc);
          mma_chain<W::kMseSteps, W::kKSteps, N>(d_tmem + NG, a_tmem, sbase + NG * 128, idesc);
        } else {
          if (part == 0) {
            mma_chain<0, h, N>(d_tmem, a_tmem, sbase, idesc_a);
          } else {
            mma_chain<h, W::kMseSteps, N>(d_tmem + N, a_tmem, sbase, idesc);
            mma_chain<W::kMseSteps, W::kKSteps, N>(d_tmem + NG, a_tmem, sbase + NG * 128, idesc);
          }
        }
        mma_commit(&mma_done[slot]);
        issued = true;
      }
      // wind-down with the full limit: no MMA of ours still running
      if (issued) {
        mma_commit(&fdone[j]);
        if (!mbar_wait(&fdone[j], 0, 2000000000ll)) fail(9);
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// The 3-bit codebook as an odd function of x_i = 2 b_i - 1: coefficients of
// x0, x1, x2 and x0 x1 x2 (a Walsh transform of the eight centroids), and the
// largest deviation of that fit from the centroids (zero for a symmetric book).
double odd_fit3(const float* c, double a[4]) {
  for (int i = 0; i < 4; ++i) a[i] = 0.0;
  for (int k = 0; k < 8; ++k) {
    const double x0 = 2.0 * (k & 1) - 1.0, x1 = 2.0 * ((k >> 1) & 1) - 1.0, x2 = 2.0 * ((k >> 2) & 1) - 1.0;
    a[0] += c[k] * x0 / 8.0;
    a[1] += c[k] * x1 / 8.0;
    a[2] += c[k] * x2 / 8.0;
    a[3] += c[k] * x0 * x1 * x2 / 8.0;
  }
  double worst = 0.0, cmax = 0.0;
  for (int k = 0; k < 8; ++k) {
    const double x0 = 2.0 * (k & 1) - 1.0, x1 = 2.0 * ((k >> 1) & 1) - 1.0, x2 = 2.0 * ((k >> 2) & 1) - 1.0;
    const double f = a[0] * x0 + a[1] * x1 + a[2] * x2 + a[3] * x0 * x1 * x2;
    worst = std::max(worst, std::fabs(f - c[k]));
    cmax = std::max(cmax, std::fabs(static_cast<double>(c[k])));
  }
  return cmax > 0.0 ? worst / cmax : worst;
}

template <int B, int G>
int launch_G(const tq_ctx& ctx, const float* qp, int64_t n_sets, int64_t n_keys, const Packed& keys, float* out,
             cudaStream_t s) {
  constexpr int NG = (4 * G <= 16) ? 16 : 32;
  using Sh = Shape<B>;
  constexpr int kWG = Sh::kWG;
  const KParams& P = ctx.kp;
  LogitsArgs X;
  X.wbit[2] = 0.f;
  X.wpar = 0.f;
  if (B == 3) {
    double a[4];
    odd_fit3(P.c, a);
    X.wbit[0] = static_cast<float>(2.0 * a[0]);
    X.wbit[1] = static_cast<float>(2.0 * a[1]);
    X.wbit[2] = static_cast<float>(2.0 * a[2]);
    X.wpar = static_cast<float>(2.0 * a[3]);
    X.cconst = static_cast<float>(-(a[0] + a[1] + a[2] + a[3]));
  } else if (B == 2) {
    X.wbit[0] = P.c[3] - P.c[2];
    X.wbit[1] = P.c[3] + P.c[2];
    X.cconst = -P.c[3];
  } else {
    X.wbit[0] = 2.f * P.c[1];
    X.wbit[1] = 0.f;
    X.cconst = -P.c[1];
  }
  // centroid byte planes (warp-specialized kernel, 3-bit codes): round(c s) as a
  // signed high byte and an unsigned low byte, |error| <= max |c| / 65534
  for (int i = 0; i < 4; ++i) X.lut8[i] = 0u;
  X.cinv = 1.f;
  if (B == 3) {
    float cmax = 0.f;
    for (int k = 0; k < 8; ++k) cmax = std::max(cmax, std::fabs(P.c[k]));
    const double sc = cmax > 0.f ? 32767.0 / cmax : 1.0;
    for (int k = 0; k < 8; ++k) {
      long v = std::lrint(static_cast<double>(P.c[k]) * sc);
      v = std::min(32767l, std::max(-32767l, v));
      const uint32_t hi = static_cast<uint32_t>((v >> 8) & 0xFF), lo = static_cast<uint32_t>(v & 0xFF);
      X.lut8[k >> 2] |= hi << (8 * (k & 3));
      X.lut8[2 + (k >> 2)] |= lo << (8 * (k & 3));
    }
    X.cinv = static_cast<float>(1.0 / sc);
  }
  X.err = P.err;
  X.wait_cycles = wait_limit_cycles();
  const int64_t tps = (n_keys + kTile - 1) / kTile, n_tiles = tps * n_sets;
  // warp-specialized form when every CTA's contiguous tile range spans at most
  // two sets: ranges of at most tps + 1 tiles
  const int64_t ws_grid = n_tiles < ctx.num_sms ? n_tiles : ctx.num_sms;
  if ((n_tiles + ws_grid - 1) / ws_grid <= tps + 1) {
    const size_t smem = logits_ws_smem_bytes<B, NG>();
    cudaError_t e = cudaFuncSetAttribute(k_logits_d128_ws<B, G, NG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return static_cast<int>(e);
    k_logits_d128_ws<B, G, NG><<<static_cast<int>(ws_grid), WsLog<B, NG>::kThreads, smem, s>>>(P, X, qp, n_sets,
                                                                                              n_keys, keys, out);
  } else {
    const size_t smem = 1024 + static_cast<size_t>(kWG) * (Sh::kKBlocks * (2 * NG) * 128 + kStages * Sh::kStageBytes) +
                        kWG * kScalFloats * 4 + (kWG * kStages + kWG) * 8 + 16;
    cudaError_t e = cudaFuncSetAttribute(k_logits_d128_i8<B, G, NG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return static_cast<int>(e);
    int64_t grid = (n_tiles + kWG - 1) / kWG;
    if (grid > ctx.num_sms) grid = ctx.num_sms;
    k_logits_d128_i8<B, G, NG><<<static_cast<int>(grid), Sh::kThreads, smem, s>>>(P, X, qp, n_sets, n_keys, keys, out);
  }
  count_launch();
  return static_cast<int>(cudaGetLastError());
}

template <int B>
int launch_B(const tq_ctx& ctx, const float* qp, int64_t n_sets, int g, int64_t n_keys, const Packed& keys, float* out,
             cudaStream_t s) {
  switch (g) {
    case 1: return launch_G<B, 1>(ctx, qp, n_sets, n_keys, keys, out, s);
    case 2: return launch_G<B, 2>(ctx, qp, n_sets, n_keys, keys, out, s);
    case 3: return launch_G<B, 3>(ctx, qp, n_sets, n_keys, keys, out, s);
    case 4: return launch_G<B, 4>(ctx, qp, n_sets, n_keys, keys, out, s);
    case 5: return launch_G<B, 5>(ctx, qp, n_sets, n_keys, keys, out, s);
    case 6: return launch_G<B, 6>(ctx, qp, n_sets, n_keys, keys, out, s);
    case 7: return launch_G<B, 7>(ctx, qp, n_sets, n_keys, keys, out, s);
    default: return launch_G<B, 8>(ctx, qp, n_sets, n_keys, keys, out, s);
  }
}

}  // namespace

bool logits_d128_applies(const tq_ctx& ctx, int64_t n_sets, int g, int64_t n_keys) {
  const KParams& P = ctx.kp;
  if (!(P.d == kD && P.m == kM && P.B >= 1 && P.B <= 3 && g >= 1 && g <= 8 && n_keys > 0 && n_sets > 0 &&
        ctx.use_tc))
    return false;
  // the A operand and the accumulator share a warpgroup's TMEM columns
  const int ng = (4 * g <= 16) ? 16 : 32;
  const int a_cols = 8 * (P.B * 4 + (P.B == 3 ? 4 : 0) + 4), n_cols = (P.B == 3 ? 3 : 2) * ng;
  const int cols = P.B == 3 ? 256 : 128;
  if (a_cols + n_cols > cols) return false;
  if (P.B == 3) {                       // the bit-plane form needs a symmetric codebook
    double a[4];
    if (odd_fit3(P.c, a) > 1e-6) return false;
  }
  return true;
}

int launch_logits_d128(const tq_ctx& ctx, const float* qp, int64_t n_sets, int g, const Packed& keys, int64_t n_keys,
                       float* out, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (ctx.kp.B == 1) return launch_B<1>(ctx, qp, n_sets, g, n_keys, keys, out, s);
  if (ctx.kp.B == 2) return launch_B<2>(ctx, qp, n_sets, g, n_keys, keys, out, s);
  return launch_B<3>(ctx, qp, n_sets, g, n_keys, keys, out, s);
}

}  // namespace tq
