/*
 * tq.h -- C ABI of the B200 compressed-KV (TurboQuant-style) hot path.
 *
 * Three operations, each on plain pointers and sizes:
 *
 *   tq_build_codebook  host     Lloyd-Max quantizer of N(0,1) (computed once per bit width).
 *   tq_quantize        device   rotate -> scalar-quantize -> pack -> 1-bit QJL sketch of K/V.
 *   tq_decode_attn     device   single-token attention directly over the packed cache.
 *
 * Around them: tq_decode_attn_static (decode without a caller workspace), tq_decode_step (append
 * one token, then attend), tq_sketch_rotation (the optional fp64 constant S Pi),
 * tq_build_hadamard_rotation (a structured Pi), and the tq_quantize diagnostics.
 *
 * Method sources (page and passage):
 *   - ai-news.ru TurboQuant overview, paragraphs on the first and second ideas: multiply each
 *     vector by a random orthogonal matrix so the coordinates become near-Gaussian, then apply a
 *     Lloyd-Max grid precomputed once for that distribution; static codebook, no calibration.
 *   - same page, next paragraph ("third component"): a 1-bit QJL correction of the residual.
 *   - tproger.ru "Google TurboQuant in simple words", sections "Step 1: PolarQuant" (per-coordinate
 *     Lloyd-Max with no per-group scale bits) and "Step 2: QJL" (one extra bit makes the residual
 *     error unbiased); section "Benchmarks": a TQ3 block is 52 bytes per 128 values.
 *   - inner-product estimator used for keys:
 *       <q,k> ~= <q,k_mse> + ||r|| * sqrt(pi/2)/m * <S q, sign(S r)>,   S Gaussian m x d.
 *
 * Conventions (all functions):
 *   - head_dim is 128.  Bit widths 2..4 for keys and values; qjl_m is 0 (off) or 128.
 *   - The library never allocates device memory.  All device pointers are caller-owned and must
 *     stay valid until the work enqueued on `stream` has finished.
 *   - Device work is enqueued on `stream` (a cudaStream_t passed as void*; NULL = legacy default
 *     stream) and is asynchronous.  Argument errors are detected on the host and returned before
 *     anything is enqueued.  A launch failure returns TQ_ERR_CUDA; tq_last_error() then describes it.
 *   - Every device pointer must be 16-byte aligned.
 *
 * Packed cache layout ([B, Hkv, T_cap] rows, each array contiguous, row r of (b,h,t) at
 * ((b*Hkv + h)*T_cap + t)):
 *   k_codes  uint8 [.., 16*k_bits]  key codes; v_codes uint8 [.., 16*v_bits] value codes.
 *            A row is a little-endian bit stream (row bit k = bit k%8 of byte k/8); slot s holds
 *            bits [b*s, b*s+b) = the Lloyd index (0 = most negative centroid) of one rotated
 *            coordinate.  Key rows: coordinate j = 16*a + 8*h + 2*t + e sits at slot
 *            32*t + 4*a + 2*h + e.  Value rows: coordinate j = 8*n + g sits at slot 16*g + n.
 *   k_signs  uint8 [.., 16]  QJL bits: sketch row l = 16*a + 8*h + 2*t + e at row bit
 *            32*t + (2*a + h) + 16*e; a bit is 1 when (S rho)_l >= 0.
 *   k_norm, v_norm  float [..]  ||x|| of the original vector.
 *   k_rnorm         float [..]  ||r|| = ||x|| * ||rho|| / sqrt(128), rho = u - c[idx].
 *   Rotated normalized coordinates: u = sqrt(128) * Pi x / ||x|| (u = 0 when x = 0);
 *   index = number of thresholds t_i with u >= t_i (a tie goes to the upper cell).
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or shape */
  TQ_ERR_UNSUPPORTED = 2,   /* head_dim != 128, bits outside 2..4, qjl_m not in {0,128} */
  TQ_ERR_NO_CONVERGENCE = 3,/* Lloyd iteration did not reach the tolerance */
  TQ_ERR_WORKSPACE = 4,     /* workspace smaller than tq_decode_workspace_size() */
  TQ_ERR_CUDA = 5           /* CUDA runtime error (launch or device query) */
} tq_status;

enum { TQ_F32 = 0, TQ_BF16 = 1 };

/* Static description of a status code.  Never NULL. */
const char* tq_status_string(int status);

/* Detail of the last failure on the calling thread ("" if none).  Valid until the next call
 * into this library on the same thread. */
const char* tq_last_error(void);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int tq_version(void);

/*
 * Lloyd-Max scalar quantizer of the standard normal density (host, double precision).
 * Source: ai-news.ru overview, "second idea" (optimal grid for a known distribution, computed
 * once, stored statically); tproger.ru "Step 1: PolarQuant" (per-coordinate Lloyd-Max).
 *
 *   bits        1..8
 *   max_iter    iteration cap (> 0); tol: stop when the largest centroid move is < tol (> 0)
 *   centroids   host float[1 << bits]  out: ascending, symmetric, each rounded to the nearest
 *               fp16 value (so the decode path can use them as exact half-precision operands)
 *   thresholds  host float[(1 << bits) - 1]  out: exact midpoints of adjacent stored centroids
 *   distortion  host double* or NULL  out: E[(X - Q(X))^2] of the unrounded Lloyd solution
 * Errors: TQ_ERR_INVALID_ARG (bits, max_iter, tol, null outputs), TQ_ERR_NO_CONVERGENCE.
 * The caller owns all arrays.  Thread-safe; no device work.
 */
tq_status tq_build_codebook(int bits, int max_iter, double tol, float* centroids,
                            float* thresholds, double* distortion);

/*
 * Structured alternative to a dense Haar rotation for tq_params.Pi (host, no device work):
 * Pi = D1 H D2 H D3 / 128, H the 128 x 128 Sylvester Hadamard matrix (H[i][j] = (-1)^popcount(i & j)),
 * D_k = diag(s_k) with s_k[i] = +1 when output 128k + i of a SplitMix64 generator started at
 * `seed` is even, else -1.  Orthogonal exactly; every entry is a multiple of 1/64, so it is exact
 * in fp16 and the rotation MMA needs no lo part.
 * Source: tproger.ru, section "TurboQuant in llama.cpp, MLX and PyTorch: who is already trying"
 * (the dense rotation is the slow step; its authors turn to the Hadamard transform); ai-news.ru
 * overview, paragraph on RotorQuant (the dense d x d rotation costs 16384 operations at d = 128).
 *   Pi   host float[128 * 128] out, row-major.
 * Errors: TQ_ERR_INVALID_ARG (Pi NULL).  Thread-safe.
 */
tq_status tq_build_hadamard_rotation(uint64_t seed, float* Pi);

/* Cache layouts (tq_cache.layout). */
enum { TQ_LAYOUT_PLAIN = 0, TQ_LAYOUT_MIXED = 1 };

/* Caller-owned packed cache (device pointers; see the layout above).  k_signs and k_rnorm may
 * be NULL when qjl_m == 0.
 *
 * layout = TQ_LAYOUT_MIXED: outlier-aware mixed precision.  Source: tproger.ru, section on
 * TheTom's llama.cpp fork (turbo3 = 3.5-bit KV quantization, 4.6x vs FP16); ai-manual.ru M5 Max
 * KV-cache benchmark (per-layer outlier-aware 3/4-bit quantization).  The channels split into an
 * outlier half O (tq_params.outlier_mask, 64 channels) coded with k_bits / v_bits and the other
 * half R coded with one bit less; each half is rotated on its own (tq_params.Pi must be the block
 * rotation: rows 0..63 act only on the outlier channels, rows 64..127 only on the others), has its
 * own norm and codebook (tq_params.*_lo for half R), u_g = sqrt(64) (Pi x)_g / ||x_g||.  QJL acts
 * on the whole residual r = Pi x - khat (khat_g = ||x_g|| / 8 * c_g[idx_g]): k_rnorm = ||r||, and
 * a sign bit is 1 when (S r)_l >= 0.  Supported: k_bits = v_bits = 4 (halves of 4 and 3 bits).
 *   k_codes row: the half-O bit stream (64 codes of k_bits bits; coordinate 16a + 8h + 2t + e at
 *     slot 16t + 4a + 2h + e), then the half-R stream (64 codes of k_bits - 1 bits, coordinate
 *     64 + 16a + 8h + 2t + e at slot 16t + 4a + 2h + e): 8 (2 k_bits - 1) bytes.
 *   v_codes row: likewise with value slots (coordinate 64g' + 8n + g at slot 8g + n of half g').
 *   k_norm, v_norm: float [.., 2] = (||x_O||, ||x_R||). */
typedef struct {
  int B, Hkv, T_cap, head_dim, k_bits, v_bits, qjl_m;
  uint8_t* k_codes;
  uint8_t* k_signs;
  float* k_norm;
  float* k_rnorm;
  uint8_t* v_codes;
  float* v_norm;
  int layout;  /* TQ_LAYOUT_PLAIN or TQ_LAYOUT_MIXED */
} tq_cache;

/* Per-layer constants (device pointers, caller-owned, fp32 unless stated).
 *   Pi            [128 x 128] row-major orthogonal rotation (u = sqrt(128) Pi x / ||x||)
 *   S             [qjl_m x 128] row-major Gaussian sketch, entries exactly representable in fp16
 *                 (may be NULL when qjl_m == 0)
 *   k_centroids   [1 << k_bits], k_thresholds [(1 << k_bits) - 1]  from tq_build_codebook
 *   v_centroids   [1 << v_bits], v_thresholds [(1 << v_bits) - 1]
 *   S_Pi          optional float64 [qjl_m x 128] row-major product S Pi, as written by
 *                 tq_sketch_rotation for these S and Pi; NULL is allowed.  It changes no output:
 *                 with it, tq_quantize settles a sketch value that lies near 0 with one
 *                 length-128 dot product (S r = sqrt(128)/||x|| (S Pi) x - S c[idx]) instead of
 *                 re-rotating the whole key in fp64. */
typedef struct {
  const float* Pi;
  const float* S;
  const float* k_centroids;
  const float* k_thresholds;
  const float* v_centroids;
  const float* v_thresholds;
  const double* S_Pi;
  /* TQ_LAYOUT_MIXED only (ignored otherwise): codebooks of the non-outlier half (one bit fewer),
   * device fp32 like the ones above, and the outlier channels (bit c of outlier_mask[c / 32] set
   * for channel c in O; exactly 64 bits set). */
  const float* k_centroids_lo;
  const float* k_thresholds_lo;
  const float* v_centroids_lo;
  const float* v_thresholds_lo;
  uint32_t outlier_mask[4];
} tq_params;

/*
 * S_Pi[l][j] = sum_i S[l][i] Pi[i][j] in float64 (device; every product of two fp32 values is
 * exact in fp64, summed in ascending i), for tq_params.S_Pi.  Enqueued on `stream`.
 *   Pi      device fp32 [128 x 128];  S  device fp32 [qjl_m x 128];  S_Pi  device fp64 [qjl_m x 128]
 *   qjl_m   >= 1
 * Errors: TQ_ERR_INVALID_ARG (NULL or misaligned pointer, qjl_m < 1), TQ_ERR_CUDA.
 */
tq_status tq_sketch_rotation(const float* Pi, const float* S, int qjl_m, double* S_Pi, void* stream);

/*
 * Compress T_new new tokens of K and V into cache rows [t_offset, t_offset + T_new).
 * Source: tproger.ru "Step 1: PolarQuant" and "Step 2: QJL"; ai-news.ru overview (rotation,
 * Lloyd-Max, QJL residual); the estimator above fixes what is stored for keys.
 *
 *   k, v        device [B, Hkv, T_new, 128] of `dtype` (TQ_F32 or TQ_BF16); element (b,h,t,j) at
 *               b*stride_b + h*stride_h + t*stride_t + j (strides in elements, shared by k and v;
 *               the last dimension is contiguous; stride_t * element size a multiple of 16 bytes)
 *   T_new       >= 0 (0 enqueues nothing);  0 <= t_offset, t_offset + T_new <= cache->T_cap
 * Output bits are those of the float64 definition except where a rotated coordinate lies within
 * about 1e-15 of a threshold (the kernel re-derives near-boundary cases in fp64).
 * Calls may run concurrently on different streams: the TQ_BF16 kernel keeps its queue of fp64
 * re-derivations per SM, a CTA of it occupies an SM's shared memory alone, and each CTA tags its
 * entries with a generation number drawn at its start.  Consecutive calls on one stream overlap
 * as programmatic dependent launches (the next call's set-up runs during the previous call's tail).
 * Errors: TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_CUDA.
 */
tq_status tq_quantize(const tq_params* params, const void* k, const void* v, int dtype,
                      int64_t stride_b, int64_t stride_h, int64_t stride_t, int T_new,
                      int t_offset, const tq_cache* cache, void* stream);

/*
 * Diagnostics of tq_quantize (host; synchronizes with the device).  The kernel never blocks
 * without bound: every wait on tensor-core completion gives up after about two seconds, records
 * the failure here and leaves its tile unwritten.
 *   tq_quantize_device_errors   bit 0: a completion wait timed out; bit 1: shared memory not
 *                               1024-byte aligned.  0 = no error since the library was loaded;
 *                               -1 if the device could not be queried.
 *   tq_quantize_vector_fixups   number of key vectors whose QJL sketch had a value too close to
 *                               0 for the tensor-core path and was re-derived in fp64.
 */
int tq_quantize_device_errors(void);
long long tq_quantize_vector_fixups(void);
/* Number of single coordinates whose code was re-derived in fp64 (value near a threshold). */
long long tq_quantize_code_fixups(void);
/*
 * Exemption counts of the comparison rule for codes and signs (cumulative since the library was
 * loaded; host, synchronizes with the device; -1 if the device could not be queried).  The
 * method's parity rule lets a code differ from the float64 definition only where the rotated
 * coordinate u lies within 1e-6 of a decision threshold, and asks for the fraction of such
 * cases to be reported.  The fast path's error is far inside its fp64 guard bands, so every such
 * coordinate is re-derived in fp64, where it is counted:
 *   tq_quantize_exempt_codes   coordinates (keys and values) whose exact u lies within 1e-6 of a
 *                              threshold.  Divide by 256 per (token, kv-head) quantized for the
 *                              fraction.
 *   tq_quantize_exempt_signs   QJL sketch values that the fast path flagged near 0 and whose exact
 *                              value lies within 1e-5 of 0 (normalized units).
 */
long long tq_quantize_exempt_codes(void);
long long tq_quantize_exempt_signs(void);

/*
 * Clear the error bits that tq_quantize_device_errors and tq_decode_device_errors report (host;
 * synchronizes with the device).  Returns 0, or -1 if the device could not be reached.
 */
int tq_reset_device_errors(void);

/*
 * Test hook for the failure handling of tq_quantize (bf16 inputs): while enabled, every CTA of a
 * launch skips its first tile load and every wait of the kernel gives up after `wait_cycles` SM
 * cycles instead of about two seconds.  The waits then run out one after another, the kernel
 * records bit 0 in tq_quantize_device_errors, releases its tensor memory and returns; the cache
 * rows of that launch are not valid.  enable = 0 restores normal operation.  Host-side setting,
 * read at each launch; not for concurrent use with other callers of tq_quantize.
 * Errors: TQ_ERR_INVALID_ARG (enable with wait_cycles <= 0).
 */
tq_status tq_debug_quantize_stall(int enable, long long wait_cycles);

/*
 * Bytes of device workspace tq_decode_attn needs for these sizes on the current device: the
 * split-K partials, one (max, sum, o'[128]) record of 132 floats per query head for every consumer
 * warp of every CTA that streams part of the head's tokens.  Returns 0 on invalid sizes.
 */
size_t tq_decode_workspace_size(int B, int Hq, const tq_cache* cache, int seq_len);

/*
 * Single-token decode attention over the first seq_len cached tokens.
 * Source: the estimator above (QJL-corrected scores); tproger.ru "Benchmarks" (4-bit TurboQuant
 * attention speedups), ai-manual.ru M5 Max KV-cache benchmark (decode over turbo3/turbo4 caches).
 *
 *   q           device [B, Hq, 128] of q_dtype (TQ_F32 or TQ_BF16), contiguous
 *   Hq          query heads; Hq % cache->Hkv == 0, query head h reads kv-head h / (Hq / Hkv)
 *   seq_len     0 <= seq_len <= cache->T_cap (0 writes zeros)
 *   scale       softmax scale; <= 0 selects 1/sqrt(128)
 *   out         device float [B, Hq, 128]:  o = Pi^T sum_i softmax(scale * est_i) vhat'_i
 *   workspace   device buffer of at least tq_decode_workspace_size() bytes, contents ignored
 * est_i = <Pi q, (n_i/sqrt(d)) c_K[idx_i]> + ||r_i|| sqrt(pi/2)/m <S Pi q, 2 sign_i - 1>,
 * vhat'_i = (nV_i/sqrt(d)) c_V[idxV_i]  (rotated basis).
 * Errors: TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_WORKSPACE, TQ_ERR_CUDA.
 */
tq_status tq_decode_attn(const tq_params* params, const void* q, int q_dtype, int Hq,
                         const tq_cache* cache, int seq_len, float scale, float* out,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * Diagnostics of tq_decode_attn (host; synchronizes with the device).  The split kernel's waits on
 * its shared-memory pipeline are bounded (about two seconds each); one that gives up records it
 * here and the call's output is not valid.
 *   bit 0: a pipeline wait timed out;  bit 1: the device's shared memory per block was too small
 *   for the pipeline;  bits 2 and 3 (only in the library built with -DTQ_DEBUG): a pipeline stage's
 *   cache rows or shared-memory slot, or a partial's slot, failed its bounds check and was skipped.
 *   0 = no error since the library was loaded; -1 if the device could not be queried.
 */
int tq_decode_device_errors(void);

/*
 * One autoregressive decode step: compress the new token's K and V into cache row t of every
 * (batch, kv-head), then attend q over rows [0, t].  Fused where tq_decode_step_fused says so:
 * the decode kernel quantizes row t itself (fp64, so the row equals the float64 definition's
 * except within ~1e-15 of a threshold or of 0), writes it into the cache and attends over it in
 * the same launch; otherwise tq_quantize (T_new = 1) and tq_decode_attn (seq_len = t + 1) are
 * enqueued back to back.  Either way one CUDA graph can hold a whole step (specific to t).
 * Source: ai-manual.ru MLX port, section "who needs this right now" (the method serves text
 * generation with autoregressive decoding); ai-news.ru overview, paragraph on the speed figures
 * (quantization is paid per token on top of attention).
 *   k_new, v_new  device [B, Hkv, 128] of kv_dtype (TQ_F32 or TQ_BF16), contiguous
 *   q             device [B, Hq, 128] of q_dtype (TQ_F32 or TQ_BF16), contiguous
 *   t             0 <= t < cache->T_cap;  rows [0, t) must already hold the earlier tokens
 *   scale, out    as tq_decode_attn
 *   workspace     device, at least tq_decode_workspace_size(B, Hq, cache, t + 1) bytes
 * Errors: as tq_quantize and tq_decode_attn; every argument is checked before anything is
 * enqueued.
 */
tq_status tq_decode_step(const tq_params* params, const void* k_new, const void* v_new, int kv_dtype,
                         const void* q, int q_dtype, int Hq, const tq_cache* cache, int t, float scale,
                         float* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Whether tq_decode_step runs fused for these sizes on the current device: 1 when the split
 * kernel quantizes the new row itself (in fp64, exactly as the definition reads), writes it into
 * the cache and attends over it, all in one decode launch; 0 when the call is tq_quantize followed
 * by tq_decode_attn (the mixed layout, or short contexts over many units, where a CTA's range
 * holds more than two segments or more than one unit end).  -1 on invalid sizes.  Host only.
 */
int tq_decode_step_fused(const tq_cache* cache, int Hq, int t);

/*
 * tq_decode_attn_static -- decode attention that allocates nothing and takes no workspace.
 * The pages describe no counterpart: this is a deployment aid of this library.
 *
 * For callers that cannot allocate device memory when they run decode: code running inside a
 * custom allocator or memory-pool callback (an allocation there would re-enter the allocator),
 * runtimes that fix their device footprint at start-up and forbid later cudaMalloc, and plug-in
 * hosts that pass a library only the tensors of one call.  Same arguments and results as
 * tq_decode_attn without `workspace`/`workspace_bytes`: the scratch lives in a file-scope device
 * array of tq_decode_static_workspace_limit() bytes (16 MiB) that every GPU loading the library
 * holds until the process exits.  The function itself calls no cudaMalloc or cudaFree.
 *
 *   - Sizes whose scratch (tq_decode_workspace_size) exceeds the limit are rejected with
 *     TQ_ERR_WORKSPACE before anything is enqueued; use tq_decode_attn for them.
 *   - The first call on each device looks up the array's device address (cudaGetSymbolAddress,
 *     with that device current); make that first call before any stream capture begins.
 *   - All calls on a device share the one array.  Calls whose device work may overlap (different
 *     streams without ordering, or host threads racing on one device) corrupt each other's
 *     results; order them on one stream or use tq_decode_attn with separate workspaces.
 *   - No part of the array needs to start at zero: every byte a call reads was written earlier in
 *     the same call, and the array keeps the last call's contents afterwards.
 * Errors: as tq_decode_attn, plus TQ_ERR_WORKSPACE for sizes above the limit.
 */
tq_status tq_decode_attn_static(const tq_params* params, const void* q, int q_dtype, int Hq,
                                const tq_cache* cache, int seq_len, float scale, float* out,
                                void* stream);

/* The device address of the array is looked up once per device and kept for the life of the
 * process: after a cudaDeviceReset (or any reset of the primary context) this entry point must not
 * be called again in the same process. */
/* Size in bytes of the static scratch array used by tq_decode_attn_static. */
size_t tq_decode_static_workspace_limit(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
