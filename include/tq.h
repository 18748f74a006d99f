/*
 * tq.h -- C ABI of libtq, the TurboQuant KV-cache / vector quantization hot
 * path for NVIDIA B200 (sm_100a).
 *
 * TurboQuant compresses a row x in R^d in two stages and reads the result
 * back without decompressing it:
 *
 *   write half (tq_quantize)
 *     n = ||x||, u = x / n                       -- 0h-n0.github.io "ICLR 2026論文解説:
 *                                                   TurboQuant", section "Step 1: PolarQuant"
 *     y = R u, R = H_d D / sqrt(d)               -- same section (randomized Hadamard
 *                                                   transform, Rademacher D)
 *     code_i = #{k : t_k < y_i}, yhat = c[code]  -- Qiita TurboQuant explainer, section
 *                                                   "Stage 1: PolarQuant" (Lloyd-Max)
 *     r = y - yhat; bit_j = [ (S r)_j < 0 ]      -- Qiita explainer, section "Stage 2: QJL";
 *                                                   ai.spot.hk "Google TurboQuant", section
 *                                                   "無偏內積估計" ((b-1)-bit MSE + 1-bit QJL)
 *     store codes, sign bits, norm = n, rnorm = n ||r||
 *
 *   read half
 *     tq_logits:  <q,k> ~ norm <R q, yhat> + rnorm sqrt(pi/2)/m <S R q, z>,  z_j = 1 - 2 bit_j
 *                 -- Qiita explainer, "Stage 2: QJL" (the estimator formula)
 *     tq_dequant: x~ = R^T (norm yhat + sqrt(pi/2)/m rnorm S^T z)   (PROD, unbiased:
 *                 ai.spot.hk "無偏內積估計") or x~ = norm R^T yhat (MSE, Qiita "APIの構成")
 *
 * Conventions for every call
 *   - Tensor pointers are DEVICE pointers owned by the caller, unless a
 *     parameter says "host".  The library never frees them.
 *   - Compute calls are asynchronous on the CUDA stream passed as `stream`
 *     (a cudaStream_t; NULL = legacy default stream) and allocate nothing.
 *     A call that needs device scratch takes it from a caller-provided
 *     `workspace` whose size the matching *_workspace_bytes function gives
 *     (16-byte aligned; used only by that call's kernels on `stream`, so two
 *     calls in flight at once need two workspaces).
 *   - Arguments are checked on the host before any launch.  A failed check
 *     returns a status and launches nothing; tq_last_error() then gives a
 *     one-line reason (thread-local, valid until the next call on the thread).
 *   - n_rows == 0 (or n_keys == 0, n_sets == 0) is a no-op returning TQ_OK.
 *   - Inputs must be finite and ||x||^2 must be finite in fp32; the output
 *     for other inputs is unspecified (no fault: every access stays in bounds).
 *   - A tq_ctx is immutable after tq_init; one context may be used from
 *     several host threads and streams at once.  It belongs to the device
 *     that was current at tq_init; calls must be made with that device current.
 *
 * Packed row format (all little-endian, one array per field, row r at r * bytes):
 *   codes  d (b-1) / 8 bytes: LSB-first bitstream, code i in bits [B i, B i + B), B = b - 1
 *   signs  m / 8 bytes: sign j is bit (j mod 8) of byte j / 8; 1 = negative projection
 *   norm   fp32 n;  rnorm fp32 n * ||r||.   A row with n < 1e-10 is stored as all zeros.
 * At d = 128, m = 128 a row takes 40 / 56 / 72 bytes for b = 2 / 3 / 4.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size or enum */
  TQ_ERR_UNSUPPORTED = 2,  /* valid request outside what this library implements */
  TQ_ERR_NOMEM = 3,        /* device or host allocation failed (tq_init only) */
  TQ_ERR_CUDA = 4          /* a CUDA runtime call or launch failed; see tq_last_error() */
} tq_status;

typedef enum { TQ_BF16 = 0, TQ_F32 = 1 } tq_dtype;
typedef enum { TQ_DEQUANT_PROD = 0, TQ_DEQUANT_MSE = 1 } tq_dequant_mode;

typedef struct tq_ctx tq_ctx;

/* Caller-owned device arrays of one packed batch (row r at codes + r*codes_bytes
 * etc.).  codes and signs must be 16-byte aligned; norm and rnorm 4-byte aligned. */
typedef struct {
  uint8_t* codes;
  uint8_t* signs;
  float* norm;
  float* rnorm;
} tq_packed;

/* ---------------------------------------------------------------- setup -- */

/* Derive the method's fixed parameters on the host, without any CUDA call.
 *   d     row length in [32, 4096]; b in [2, 5] (b-1 MSE bits + 1 QJL bit);
 *   m     multiple of 32 in [32, 4096]; seed any 64-bit value.
 * A d that is not a power of two is zero-padded to D' = the next power of two
 * (0h-n0 "ICLR 2026論文解説: TurboQuant", "実装のポイント": the randomized
 * Hadamard rotation needs a power-of-two length); every parameter, and the
 * packed format, is that of D' (D' = d otherwise).  Rows and queries keep d
 * elements on the way in, dequantized rows and attention outputs have d on
 * the way out.
 * Outputs (host arrays, any may be NULL):
 *   centroids[2^(b-1)] ascending fp32 Lloyd-Max levels for one rotated coordinate,
 *   thresholds[2^(b-1)-1] fp32 midpoints,
 *   D[D'] int8 +-1 (Rademacher diagonal), S_bits[m*D'] binary16 bit patterns of
 *   the Gaussian projection, row-major (row j = projection j).
 * The codebook is the Lloyd-Max fixed point for the exact law of a coordinate
 * of a uniform unit vector, f_d(x) ~ (1-x^2)^((d-3)/2) (ai.spot.hk,
 * "隨機旋轉與Beta分佈": rotated coordinates follow one Beta law).  D and S come
 * from SplitMix64 used as a counter generator (stream 0: D, stream 1: S,
 * Box-Muller, rounded once to binary16). */
tq_status tq_host_params(int d, int b, int m, uint64_t seed, float* centroids, float* thresholds,
                         int8_t* D, uint16_t* S_bits);

/* Create a context on the current device: derives the parameters as above
 * and uploads them (the only host->device copy of parameters).  Requires a
 * compute capability 10.x device.  *out receives the context. */
tq_status tq_init(int d, int b, int m, uint64_t seed, tq_ctx** out);

/* Free a context's device memory.  The caller must make sure no work that
 * uses it is still in flight.  NULL is accepted. */
tq_status tq_destroy(tq_ctx* ctx);

/* Bytes per array for n_rows packed rows (norm and rnorm take 4 * n_rows each). */
tq_status tq_packed_sizes(const tq_ctx* ctx, int64_t n_rows, size_t* codes_bytes, size_t* signs_bytes);

/* Host copies of the context's parameters (formats as tq_host_params; any may be NULL). */
tq_status tq_get_params(const tq_ctx* ctx, float* centroids, float* thresholds, int8_t* D, uint16_t* S_bits);

/* ---------------------------------------------------------- write half -- */

/* Quantize n_rows rows of x (row r at x + r * ld_x elements, dtype bf16 or
 * fp32, ld_x >= d; x and ld_x * element size 16-byte aligned when d is a
 * power of two, x aligned to its element size otherwise) into `out`.
 * Per row: norm, rotation, Lloyd-Max codes, QJL signs of the residual,
 * residual norm (write half above).  At d = m = 128 a tensor-core kernel
 * does it all and marks the rows in which a projection fell inside the
 * tensor cores' error bound (one bit per row in the workspace); a second
 * kernel recomputes those rows' signs exactly (fp64).  Wide rows (d >= 256,
 * n_rows >= 4096) run per 37888-row chunk: a CUDA-core kernel (norm,
 * rotation, codes, residual halves), a tensor-core GEMM for the projections
 * and their signs, and a fix-up of the rare projections inside the GEMM's
 * error bound (recomputed in fp64); their scratch (residual halves, fix-up
 * list) is the workspace.  Other shapes run on general CUDA-core kernels.
 *   workspace: device memory of at least tq_quantize_workspace_bytes(ctx,
 *   n_rows) bytes, 16-byte aligned (may be NULL when that is 0, as it is for
 *   the general kernels). */
size_t tq_quantize_workspace_bytes(const tq_ctx* ctx, int64_t n_rows);
tq_status tq_quantize(const tq_ctx* ctx, const void* x, tq_dtype x_dtype, int64_t n_rows, int64_t ld_x,
                      tq_packed out, void* workspace, size_t workspace_bytes, void* stream);

/* ----------------------------------------------------------- read half -- */

/* Decode-time append into a paged cache: quantize n_rows rows of x (as
 * tq_quantize) and write input row i to packed row dest_rows[i] of `cache`,
 * a packed array of n_cache_rows rows (write-phase compression of the newly
 * generated tokens: Qiita TurboQuant explainer, "APIの構成", the KV-cache
 * wrapper).  dest_rows: device int64 array of n_rows indices (8-byte
 * aligned); rows not named are left untouched; an index outside
 * [0, n_cache_rows) is not written and makes the next tq_sync_status report
 * TQ_ERR_INVALID_ARG (checked on the device, no fault).  Indices should be distinct (two rows sent to one
 * slot race).  Runs one warp per row, sized for a handful of tokens
 * (32 .. 256 rows): latency, not throughput. */
tq_status tq_quantize_scatter(const tq_ctx* ctx, const void* x, tq_dtype x_dtype, int64_t n_rows, int64_t ld_x,
                              const int64_t* dest_rows, int64_t n_cache_rows, tq_packed cache, void* stream);

/* Device workspace that tq_logits needs for n_sets * g queries against
 * n_keys keys per set (bytes; 0 for an empty call): the query operands
 * (R q | S R q, fp32, per query), and on wide rows the tensor-core GEMM's
 * operands (keys decoded to binary16, 18944 at a time, and the split queries). */
size_t tq_logits_workspace_bytes(const tq_ctx* ctx, int64_t n_sets, int g, int64_t n_keys);

/* Estimated logits of queries against packed keys (estimator above; no
 * 1/sqrt(d) softmax scale).
 *   q     [n_sets, g, d] bf16 or fp32 (query j of set s at row s*g + j), 16-byte aligned;
 *   keys  packed rows, set s at rows [s*n_keys, (s+1)*n_keys);
 *   out   [n_sets, g, n_keys] fp32.
 * For grouped-query attention a set is one (batch, kv head) pair and g the
 * number of query heads sharing it; for vector search n_sets = 1 and g the
 * number of queries.  g in [1, 4096].  workspace: device memory of at least
 * tq_logits_workspace_bytes(ctx, n_sets, g, n_keys) bytes, 16-byte aligned,
 * not used concurrently by another call.  With d >= 256, m a multiple of 64,
 * g >= 64 and n_keys >= 4096 the estimates run as a tensor-core GEMM over
 * keys decoded into binary16 operands, 18944 keys at a time. */
tq_status tq_logits(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int64_t n_sets, int g,
                    tq_packed keys, int64_t n_keys, float* out, void* workspace, size_t workspace_bytes,
                    void* stream);

/* tq_logits without a caller-provided workspace, for callers that cannot
 * allocate device memory where they make the call (a component that does not
 * own the device memory pool, a plug-in barred from the CUDA allocator, a
 * latency-critical path that must not risk the synchronization an allocation
 * can cause).  The pages describe no such call: it is an interface
 * convenience of this library.  Same arguments, checks and results as
 * tq_logits, without the workspace: the per-query operands go to a 4 MiB
 * scratch array compiled into the library (held on every device that loads
 * it until the process exits), so n_sets * g * (d + m) * 4 must be at most
 * 4 MiB (else TQ_ERR_UNSUPPORTED, no launch).  On wide rows, where tq_logits
 * would decode keys into a GEMM operand, this call runs the general logit
 * kernels on the packed keys instead (results within the logit tolerance of
 * tq_logits', not bit-identical).  Allocates nothing.  The first call with a
 * given CUDA context current looks up the array's device address in that
 * context and caches it (make that call before any stream capture; a context
 * destroyed by cudaDeviceReset leaves a stale cached address, so processes
 * that reset the device should not use this call).  All calls share the
 * array: calls that may overlap on the GPU race and must be serialized by
 * the caller. */
tq_status tq_logits_noalloc(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int64_t n_sets, int g,
                            tq_packed keys, int64_t n_keys, float* out, void* stream);

/* Device workspace that tq_attention needs (bytes; 0 for an empty call):
 * query operands, the logits and per-chunk partial sums. */
size_t tq_attention_workspace_bytes(const tq_ctx* ctx, int64_t n_sets, int g, int64_t n_keys);

/* Decode attention read from packed keys and values (Qiita TurboQuant
 * explainer, "APIの構成": attention scores from the compressed keys, values
 * kept compressed):
 *   out[s*g + j] = sum_k softmax_k(scale * logit(q_{s,j}, key_{s,k})) * dequant(value_{s,k})
 * with the logit estimator of tq_logits and dequant in `mode` (PROD or MSE).
 * The weighted sum is formed in the rotated domain and rotated back once per
 * query; no value row is reconstructed in memory.
 * q [n_sets * g, d] bf16/fp32 (16-byte aligned); keys and values: rows of set
 * s at [s * n_keys, (s + 1) * n_keys) of each packed array (caller-owned
 * device pointers, as for tq_logits); out [n_sets * g, d] fp32; scale is the
 * softmax scale (1/sqrt(d) for the usual attention), finite; g in [1, 8];
 * d + m <= 2048; n_keys >= 1 when n_sets > 0.  workspace: device buffer of at
 * least tq_attention_workspace_bytes(ctx, n_sets, g, n_keys) bytes, 16-byte
 * aligned, used only by this call's kernels on `stream`.  Arguments are checked
 * before any launch (TQ_ERR_INVALID_ARG / TQ_ERR_UNSUPPORTED, nothing
 * launched).  Launches qprep, logits and two attention kernels on `stream`. */
tq_status tq_attention(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int64_t n_sets, int g,
                       tq_packed keys, tq_packed values, int64_t n_keys, float scale, tq_dequant_mode mode,
                       float* out, void* workspace, size_t workspace_bytes, void* stream);

/* Reconstruct n_rows packed rows into out [n_rows, d] (bf16 or fp32,
 * contiguous, 16-byte aligned).  mode PROD adds the QJL term (unbiased),
 * MSE uses the codes alone. */
tq_status tq_dequant(const tq_ctx* ctx, tq_packed in, int64_t n_rows, void* out, tq_dtype out_dtype,
                     tq_dequant_mode mode, void* stream);

/* Vector search: for each of n_q queries, the k packed rows (of n_keys) with
 * the largest estimated inner product (the tq_logits estimator with
 * n_sets = 1, g = n_q), larger first, equal estimates by lower row index
 * (0h-n0 "ICLR 2026論文解説: TurboQuant", "実験結果 — ベクトル検索（Recall評価）":
 * Recall@k of a 4-bit database; Qiita TurboQuant explainer, "ベクトル検索への応用").
 * When the
 * wide-row path applies (d >= 256, m a multiple of 64, n_q >= 64,
 * n_keys >= 4096) no score is written: a persistent tensor-core kernel keeps
 * each query's running top-k in registers while it streams the keys, and the
 * per-CTA lists are merged at the end; its estimates equal tq_logits' up to
 * fp32 accumulation order.  Elsewhere the scores go through the workspace
 * and tq_topk's kernel.
 *   q    [n_q, d] bf16 or fp32, 16-byte aligned; n_q in [0, 4096];
 *   idx  [n_q, k] int32 row indices; val [n_q, k] fp32 estimates (may be NULL);
 *   k in [1, 16], k <= n_keys < 2^31;
 *   workspace: device memory of at least tq_search_workspace_bytes(ctx, n_q,
 *   n_keys, k) bytes, 16-byte aligned, not used concurrently by another call. */
size_t tq_search_workspace_bytes(const tq_ctx* ctx, int64_t n_q, int64_t n_keys, int k);
tq_status tq_search(const tq_ctx* ctx, const void* q, tq_dtype q_dtype, int64_t n_q, tq_packed keys, int64_t n_keys,
                    int k, int32_t* idx, float* val, void* workspace, size_t workspace_bytes, void* stream);

/* Per row of scores [rows, cols] fp32, the k largest values, larger first,
 * equal values by lower column index first.  idx [rows, k] int32 and
 * val [rows, k] fp32 (val may be NULL).  k in [1, 64], k <= cols. */
tq_status tq_topk(const float* scores, int64_t rows, int64_t cols, int k, int32_t* idx, float* val,
                  void* stream);

/* ------------------------------------------------------------ baseline -- */

/* Plain unquantized-key logits, the comparison point for tq_logits:
 * out[s, j, t] = <q[s, j], k[s, t]> with bf16 q [n_sets, g, d], bf16 keys
 * [n_sets, n_keys, d] (contiguous, 16-byte aligned), fp32 accumulation,
 * fp32 out [n_sets, g, n_keys].  d in {64, 128, 256}, g in [1, 8], n_sets <= 65535. */
tq_status tq_logits_bf16(const void* q, const void* keys, int64_t n_sets, int g, int64_t n_keys, int d,
                         float* out, void* stream);

/* ------------------------------------------- fractional bit widths -- */

/* A channel split: channels [0, d_hi) of each row are one TurboQuant
 * instance with b_hi bits per coordinate, channels [d_hi, d) another with
 * b_lo bits (m = each part's dimension; seeds seed and seed + 1), for
 * (d_hi b_hi + (d - d_hi) b_lo) / d bits per coordinate: 2.5 bits at
 * d = 128 as 64 channels at b = 3 and 64 at b = 2, 3.5 bits as 64 at 4 and
 * 64 at 3.  The pages report 2.5- and 3.5-bit results without the split rule
 * (inlevel9 "TurboQuantのメモリ圧縮と半導体需要", "TurboQuantが実際に行っていること");
 * this is the library's reading: the estimate of <q, k> is the sum of the
 * two parts' estimates (inner products add over disjoint channels, so it
 * stays unbiased), and the caller picks the channels that get the higher
 * width by ordering them first.  d_hi and d - d_hi: multiples of 32, >= 32.
 * The part contexts (tq_split_part) give packed sizes and parameters; each
 * part has its own packed arrays. */
typedef struct tq_split tq_split;
tq_status tq_split_init(int d, int d_hi, int b_hi, int b_lo, uint64_t seed, tq_split** out);
tq_status tq_split_destroy(tq_split* sp);
/* part 0 (channels [0, d_hi)) or 1 (channels [d_hi, d)); owned by sp */
tq_status tq_split_part(const tq_split* sp, int part, const tq_ctx** out);
/* Workspace bytes of tq_split_quantize for n_rows rows: the larger of the
 * two parts' tq_quantize_workspace_bytes (the parts run one after the other
 * on the caller's stream and share it); 0 when neither part needs one. */
size_t tq_split_quantize_workspace_bytes(const tq_split* sp, int64_t n_rows);
/* x [n_rows, ld_x >= d] as tq_quantize; each part's columns into its packed
 * rows.  workspace: device memory, 16-byte aligned, at least
 * tq_split_quantize_workspace_bytes(sp, n_rows) bytes (NULL when that is 0);
 * TQ_ERR_INVALID_ARG when missing or too small. */
tq_status tq_split_quantize(const tq_split* sp, const void* x, tq_dtype x_dtype, int64_t n_rows, int64_t ld_x,
                            tq_packed out_hi, tq_packed out_lo, void* workspace, size_t workspace_bytes,
                            void* stream);
size_t tq_split_logits_workspace_bytes(const tq_split* sp, int64_t n_sets, int g, int64_t n_keys);
/* As tq_logits, with q [n_sets, g, d] and each part's packed keys; out is the
 * sum of the two parts' estimates. */
tq_status tq_split_logits(const tq_split* sp, const void* q, tq_dtype q_dtype, int64_t n_sets, int g,
                          tq_packed keys_hi, tq_packed keys_lo, int64_t n_keys, float* out, void* workspace,
                          size_t workspace_bytes, void* stream);
/* Reconstructed rows [n_rows, d] (each part's columns from its packed rows). */
tq_status tq_split_dequant(const tq_split* sp, tq_packed in_hi, tq_packed in_lo, int64_t n_rows, void* out,
                           tq_dtype out_dtype, tq_dequant_mode mode, void* stream);

/* ------------------------------------------------------------- testing -- */

/* Process-wide test settings (no counterpart on the pages; for the library's
 * own failure tests, not for production use).  Injected failures happen on
 * the host: no GPU fault is provoked.
 *   TQ_TEST_WAIT_LIMIT   limit, in SM clock cycles, of the bounded mbarrier
 *                        waits in the tile loops of the d = 128 tensor-core
 *                        kernels (quantize, logits, dequant; 0 restores the
 *                        default, about one second).  A limit shorter than the
 *                        work makes a kernel give up: it stops, waits (with
 *                        the default limit) for its own MMAs and stage loads,
 *                        frees its tensor memory and leaves an error that
 *                        tq_sync_status reports as TQ_ERR_CUDA (the quantize
 *                        kernel, whose first wait gives up, writes no
 *                        results; the logits and dequant kernels may have
 *                        written some before they gave up).  Applies to
 *                        launches made after the call.
 *   TQ_TEST_FAIL_ALLOC   the next `value` device allocations of tq_init fail
 *                        as if the device were out of memory (TQ_ERR_NOMEM,
 *                        nothing leaked).
 *   TQ_TEST_FAIL_LAUNCH  the next `value` calls that would launch quantize,
 *                        logit or dequant kernels fail with TQ_ERR_CUDA
 *                        before launching anything.
 *   TQ_TEST_FIXUP_CAP    caps the list of projections that the d = 128
 *                        quantize kernel hands to its exact fix-up at `value`
 *                        entries (0 restores the default, two per 128-row
 *                        tile): rows beyond the list take the overflow path,
 *                        which recomputes all their signs.
 * value >= 0, else TQ_ERR_INVALID_ARG. */
typedef enum {
  TQ_TEST_WAIT_LIMIT = 0,
  TQ_TEST_FAIL_ALLOC = 1,
  TQ_TEST_FAIL_LAUNCH = 2,
  TQ_TEST_FIXUP_CAP = 3
} tq_test_knob;
tq_status tq_test_set(tq_test_knob knob, int64_t value);

/* ----------------------------------------------------------- reporting -- */

const char* tq_status_str(tq_status s);
/* Wait for `stream`, then report whether any kernel of this context timed out
 * in one of its bounded device-side waits since the last check (TQ_ERR_CUDA,
 * outputs of that call invalid), found more projections inside the wide-row
 * GEMM's error bound than its fix-up list holds (TQ_ERR_CUDA, some signs not
 * recomputed), or met an out-of-range destination row in
 * tq_quantize_scatter (TQ_ERR_INVALID_ARG), and clear the record.  Blocking. */
tq_status tq_sync_status(const tq_ctx* ctx, void* stream);
/* One-line reason for the last non-OK status returned on this host thread. */
const char* tq_last_error(void);
/* Number of kernel launches this library has issued in this process (all
 * threads), for launch accounting in benchmarks. */
uint64_t tq_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
