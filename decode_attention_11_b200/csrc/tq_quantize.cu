// tq_quantize: rotate -> Lloyd-Max scalar quantize -> bit-pack -> 1-bit QJL sketch, on the
// sm_100a tensor cores (tcgen05 + tensor memory).
//
// Method: ai-news.ru TurboQuant overview (first idea: a random orthogonal rotation makes the
// coordinates near-Gaussian; second idea: a Lloyd-Max grid precomputed for that distribution;
// third component: a 1-bit QJL correction of the residual); tproger.ru "Google TurboQuant in
// simple words", "Step 1: PolarQuant" (each coordinate quantized independently, no per-group
// scale bits) and "Step 2: QJL" (one extra bit per sketch row makes the inner-product error
// unbiased).
//
// This general kernel serves fp32 inputs and the outlier-aware mixed layout (TQ_LAYOUT_MIXED, any
// input type); bf16 inputs in the plain layout go to the pipelined kernel of tq_quantize_pipe.cu.
// One persistent 512-thread CTA per SM works on 128-token tiles of one (batch, kv-head):
//   1. cp.async brings the K and V tiles into shared memory in the UMMA 128-byte-swizzle layout
//      (fp32 as fp16 hi + lo); each thread converts one row and sums its squares in fp64 (the
//      stored norm; one norm per half in the mixed layout).
//   2. One thread issues tcgen05.mma: Y_K = X_K Pi^T and Y_V = X_V Pi^T with Pi split into fp16
//      hi + lo (about 22 significant bits; the lo pass is skipped when Pi is exact in fp16),
//      accumulated in fp32 tensor memory.
//   3. The epilogue warps read Y row by row in 32-coordinate chunks: u = sqrt(d) y / ||x||, code
//      by a branch-free binary search of the thresholds (each half its own codebook and scale in
//      the mixed layout), residual rho = u - c[code] written as fp16 hi + lo for the next MMA.
//   4. tcgen05.mma: S rho for the QJL sign bits, packed by the epilogue.
// Exactness: codes and sign bits equal those of the float64 definition.  Any coordinate whose
// fast value lies within a guard band of a decision boundary (a threshold; 0 for a sign) is
// re-derived in fp64 from the original inputs, leaving only values within ~1e-15 of a boundary.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "tq_internal.h"
#include "tq_sm100.h"

namespace tq {
namespace {

using namespace sm100;

constexpr int D = kHeadDim;
constexpr int TM = 128;          // tokens per tile (MMA M)
constexpr int THREADS = 512;     // 16 warps: each epilogue thread owns one 32-coordinate chunk
constexpr int TILE_BYTES = TM * D * 2;  // one fp16 [128 x 128] operand
constexpr uint32_t IDESC = idesc_f16_f32(128, 128);
constexpr uint32_t TMEM_COLS = 512;
// Tensor-memory columns: Y_K, Y_V and S rho (fp32, 128 each), rho hi / lo (fp16 pairs, 64 each).
constexpr uint32_t COL_K = 0, COL_V = 128, COL_S = 256, COL_RH = 384, COL_RL = 448;
constexpr long long WAIT_LIMIT = 4000000000LL;  // ~2 s of SM clock
constexpr float PI_SCALE = 256.0f;

// Fast-path guard bands (normalized units): a value closer than this to a decision boundary is
// re-derived in fp64.
struct Guards {
  float code_k, code_v, sign;
};

__device__ unsigned int g_quantize_error;          // bit 0: a wait timed out; bit 1: misaligned smem
__device__ unsigned int g_quantize_vector_fixups;  // key vectors re-derived in fp64 (diagnostic)
__device__ unsigned int g_quantize_code_fixups;    // coordinates re-derived in fp64 (diagnostic)
__device__ unsigned int g_quantize_exempt_codes;   // exact u within kExemptCodeBand of a threshold
__device__ unsigned int g_quantize_exempt_signs;   // exact sketch value within kExemptSignBand of 0

struct QArgs {
  const void* k;
  const void* v;
  int64_t sb, sh, st;
  int T_new, t_offset;
  int B, Hkv, T_cap;
  int qjl, in_f32;
  uint8_t* k_codes;
  uint8_t* k_signs;
  float* k_norm;
  float* k_rnorm;
  uint8_t* v_codes;
  float* v_norm;
  const float* Pi;
  const float* S;
  const float* kc;
  const float* kt;
  const float* vc;
  const float* vt;
  Guards guard;
  // mixed layout: codebooks of the non-outlier half (one bit fewer) and the outlier channels
  const float* kc2;
  const float* kt2;
  const float* vc2;
  const float* vt2;
  uint32_t omask[4];
};

constexpr int FL_CAP = 1024;  // deferred single-coordinate fixups per tile

// Shared memory (all operand tiles 1024-byte aligned).
struct __align__(1024) Smem {
  uint8_t xk[TILE_BYTES];   // X_K fp16 (bf16 on arrival)
  uint8_t xv[TILE_BYTES];   // X_V
  uint8_t pih[TILE_BYTES];  // Pi hi (B operand: row n = output coordinate)
  uint8_t pil[TILE_BYTES];  // Pi lo
  uint8_t sm[TILE_BYTES];   // S (exact in fp16)
  uint8_t xl[TILE_BYTES];   // X_K lo (fp32 input only: x = fp16 hi + fp16 lo)
  uint8_t kst[TM * 64];     // staged output rows: key codes (16 * k_bits bytes each)
  uint8_t vst[TM * 64];     // value codes
  uint8_t sst[TM * 16];     // sign bits
  float kn[TM], vn[TM], rn[TM];
  double nrmk[TM], nrmv[TM];
  float sclk[TM], sclv[TM];  // u = y * scl (0 for a zero row)
  float rho2[4][TM];         // ||rho||^2 partials of the four 32-coordinate chunks
  uint16_t fl[FL_CAP];      // deferred fixups: bit 15 = value side, bits 14..7 row, 6..0 coordinate
  unsigned int vflag[TM];   // bit 0: key vector to fp64 path; bit 1: key list overflow; bit 2: value
  uint8_t vfl[TM];
  double fx64[D];           // exact residual of one vector (vector path)
  double red64[THREADS / 32];
  float kcent[16], kthr[16], vcent[16], vthr[16];
  // mixed layout: half R (non-outlier channels) scales, norms and codebooks
  float sclk2[TM], sclv2[TM], kn2[TM], vn2[TM];
  double nrmk2[TM], nrmv2[TM];
  float kcent2[16], kthr2[16], vcent2[16], vthr2[16];
  uint8_t fcode[D];
  uint8_t fsign[D];
  int nfl, nvfl;
  unsigned int nexc, nexs;  // exempt codes / signs found by this tile's fp64 fixups
  uint64_t bar_kv, bar_s;
  uint32_t tmem_base;
  unsigned int err;
};

// Byte offset of 16-byte chunk c (0..15, k = 8c..8c+7) of row r of a [128 x 128] fp16 operand:
// two 64-element K atoms, 8-row groups 1024 bytes apart, chunks XOR-swizzled by (r % 8).
__device__ __forceinline__ uint32_t sw_chunk(int r, int c) {
  return (uint32_t)((c >> 3) * (TM * 128) + (r >> 3) * 1024 + (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4));
}
__device__ __forceinline__ uint32_t sw_off(int r, int k) { return sw_chunk(r, k >> 3) + (k & 7) * 2; }

__device__ __forceinline__ uint64_t desc_at(const uint8_t* tile, int kstep) {
  return desc_sw128_kmajor(smem_u32(tile) + (kstep >> 2) * (TM * 128) + (kstep & 3) * 32);
}

// Load a row-major fp32 [128 x 128] matrix, times `scale` (a power of two), into an fp16 hi
// (+ optional lo) operand tile, one 16-byte chunk (8 consecutive elements of a row) per step.
// Returns (per thread) whether any lo element it wrote is nonzero: a matrix exact in fp16 (the
// structured rotation) then needs no lo MMA pass.
__device__ bool load_matrix(const float* __restrict__ M, float scale, uint8_t* hi, uint8_t* lo) {
  bool lo_nz = false;
  for (int i = threadIdx.x; i < D * D / 8; i += THREADS) {
    const int r = i / 16, c = i % 16;
    const float4 p0 = reinterpret_cast<const float4*>(M + r * D + 8 * c)[0];
    const float4 p1 = reinterpret_cast<const float4*>(M + r * D + 8 * c)[1];
    const float v[8] = {p0.x * scale, p0.y * scale, p0.z * scale, p0.w * scale,
                        p1.x * scale, p1.y * scale, p1.z * scale, p1.w * scale};
    uint32_t h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __half2 hh = __floats2half2_rn(v[2 * e], v[2 * e + 1]);
      const float2 hf = __half22float2(hh);
      const __half2 ll = __floats2half2_rn(v[2 * e] - hf.x, v[2 * e + 1] - hf.y);
      h[e] = *reinterpret_cast<const uint32_t*>(&hh);
      l[e] = *reinterpret_cast<const uint32_t*>(&ll);
    }
    *reinterpret_cast<uint4*>(hi + sw_chunk(r, c)) = make_uint4(h[0], h[1], h[2], h[3]);
    if (lo) *reinterpret_cast<uint4*>(lo + sw_chunk(r, c)) = make_uint4(l[0], l[1], l[2], l[3]);
    lo_nz = lo_nz || ((l[0] | l[1] | l[2] | l[3]) & 0x7fff7fffu) != 0;
  }
  return lo_nz;
}

// Positive-half search: k = #{T_j <= a} over the 2^(B-1)-1 positive thresholds T[1..], and the
// distance from a to the thresholds compared (the bracket of a is always among them).
template <int B>
__device__ __forceinline__ int search_pos(float a, const float* T, float& margin) {
  if constexpr (B == 2) {
    margin = fabsf(a - T[1]);
    return a >= T[1] ? 1 : 0;
  } else if constexpr (B == 3) {
    const bool c1 = a >= T[2];
    const float t2 = c1 ? T[3] : T[1];
    const bool c2 = a >= t2;
    margin = fminf(fabsf(a - T[2]), fabsf(a - t2));
    return (c1 ? 2 : 0) + (c2 ? 1 : 0);
  } else {
    const bool c1 = a >= T[4];
    const float t2 = c1 ? T[6] : T[2];
    const bool c2 = a >= t2;
    const float t3 = c1 ? (c2 ? T[7] : T[5]) : (c2 ? T[3] : T[1]);
    const bool c3 = a >= t3;
    margin = fminf(fminf(fabsf(a - T[4]), fabsf(a - t2)), fabsf(a - t3));
    return (c1 ? 4 : 0) + (c2 ? 2 : 0) + (c3 ? 1 : 0);
  }
}

// Part q (0..3) of the exact (fp64) dot product of Pi row j with input row x: elements
// 32q..32q+31, all loads issued at once.  Four consecutive lanes form the whole sum (quad_sum).
template <typename InT>
__device__ __forceinline__ double exact_dot_part(const float* __restrict__ Pi, const InT* __restrict__ x,
                                                 int j, int q) {
  const float4* pr = reinterpret_cast<const float4*>(Pi + j * D + 32 * q);
  float4 p[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) p[c] = pr[c];
  float xv[32];
  if constexpr (sizeof(InT) == 4) {
    const float4* xr = reinterpret_cast<const float4*>(x + 32 * q);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float4 t = xr[c];
      xv[4 * c] = t.x; xv[4 * c + 1] = t.y; xv[4 * c + 2] = t.z; xv[4 * c + 3] = t.w;
    }
  } else {
    const uint4* xr = reinterpret_cast<const uint4*>(x + 32 * q);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 t = xr[c];
      const uint32_t w4[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
        xv[8 * c + 2 * e] = f.x;
        xv[8 * c + 2 * e + 1] = f.y;
      }
    }
  }
  double y0 = 0.0, y1 = 0.0;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    y0 = fma((double)p[c].x, (double)xv[4 * c + 0], y0);
    y1 = fma((double)p[c].y, (double)xv[4 * c + 1], y1);
    y0 = fma((double)p[c].z, (double)xv[4 * c + 2], y0);
    y1 = fma((double)p[c].w, (double)xv[4 * c + 3], y1);
  }
  return y0 + y1;
}
__device__ __forceinline__ double quad_sum(double v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

__device__ __forceinline__ int code_exact(double u, const float* thr, int nthr) {
  int idx = 0;
  for (int i = 0; i < nthr; ++i) idx += (u >= (double)thr[i]) ? 1 : 0;
  return idx;
}
// Whether an exact coordinate lies within kExemptCodeBand of one of the nthr thresholds.
__device__ __forceinline__ bool code_exempt_exact(double u, const float* thr, int nthr) {
  bool near = false;
  for (int i = 0; i < nthr; ++i) near = near || fabs(u - (double)thr[i]) <= kExemptCodeBand;
  return near;
}

// Read / replace the b-bit code at bit position P of a staged row (32-bit shared words; in the
// plain layout P = b * slot, in the mixed layout the position within the row's two streams).
__device__ __forceinline__ uint32_t get_code_at(const uint8_t* row, int bits, int P) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(row);
  uint64_t v = w[P >> 5];
  if ((P & 31) + bits > 32) v |= (uint64_t)w[(P >> 5) + 1] << 32;
  return (uint32_t)(v >> (P & 31)) & ((1u << bits) - 1u);
}
__device__ __forceinline__ void set_code_at(uint8_t* row, int bits, int P, uint32_t code) {
  uint32_t* w = reinterpret_cast<uint32_t*>(row);
  const int wi = P >> 5, sh = P & 31;
  const uint64_t m = (uint64_t)((1u << bits) - 1u) << sh;
  const uint64_t c = (uint64_t)code << sh;
  atomicAnd(&w[wi], ~(uint32_t)m);
  atomicOr(&w[wi], (uint32_t)c);
  if (sh + bits > 32) {
    atomicAnd(&w[wi + 1], ~(uint32_t)(m >> 32));
    atomicOr(&w[wi + 1], (uint32_t)(c >> 32));
  }
}

template <typename InT>
__device__ void issue_x_loads(Smem& s, const QArgs& a, int b, int h, int t0, int nt) {
  if constexpr (sizeof(InT) == 2) {
    const InT* srcs[2] = {reinterpret_cast<const InT*>(a.k), reinterpret_cast<const InT*>(a.v)};
    uint8_t* dsts[2] = {s.xk, s.xv};
    const int64_t base = (int64_t)b * a.sb + (int64_t)h * a.sh + (int64_t)t0 * a.st;
    for (int i = threadIdx.x; i < 2 * TM * 16; i += THREADS) {
      const int which = i / (TM * 16), rem = i % (TM * 16);
      const int r = rem / 16, c = rem % 16;
      const bool ok = r < nt;
      const InT* src = srcs[which] + (ok ? base + (int64_t)r * a.st + 8 * c : 0);
      cp_async16(smem_u32(dsts[which] + sw_chunk(r, c)), src, ok ? 16 : 0);
    }
  }
}

// Read 8 consecutive input values of chunk c of this thread's row (fp32 path: global memory;
// bf16 path: the staged tile in shared memory).
template <typename InT>
__device__ __forceinline__ void row_chunk(const InT* xrow, const uint8_t* xt, int r, int c, bool live,
                                          float (&v8)[8]) {
  if constexpr (sizeof(InT) == 4) {
    if (live) {
      const float4 p0 = *reinterpret_cast<const float4*>(xrow + 8 * c);
      const float4 p1 = *reinterpret_cast<const float4*>(xrow + 8 * c + 4);
      v8[0] = p0.x; v8[1] = p0.y; v8[2] = p0.z; v8[3] = p0.w;
      v8[4] = p1.x; v8[5] = p1.y; v8[6] = p1.z; v8[7] = p1.w;
    } else {
      for (int i = 0; i < 8; ++i) v8[i] = 0.0f;
    }
  } else {
    const uint4 q = *reinterpret_cast<const uint4*>(xt + sw_chunk(r, c));
    const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[i]));
      v8[2 * i] = f.x;
      v8[2 * i + 1] = f.y;
    }
  }
}

// MX: the outlier-aware mixed layout (TQ_LAYOUT_MIXED): chunks ch = 0, 1 (coordinates 0..63) are
// the outlier half with KB / VB bits, chunks 2, 3 the other half with one bit fewer; each half has
// its own norm, codebook and power-of-two input scale (exact, as Pi is block-diagonal).
template <int KB, int VB, typename InT, bool MX>
__global__ void __launch_bounds__(THREADS, 1) quantize_kernel(QArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5;
  // conversion: two threads per input row (K rows 0..127, V rows 128..255), 8 chunks each
  const int crow = tid >> 1, cwhich = crow >> 7, cr = crow & 127, chalf = tid & 1;
  // epilogues: thread = (tile row r = TMEM lane, 32-coordinate chunk ch)
  const int r = tid & 127, ch = tid >> 7;
  constexpr int LK = 1 << KB, LV = 1 << VB;
  constexpr int LK2 = MX ? 1 << (KB - 1) : LK, LV2 = MX ? 1 << (VB - 1) : LV;
  constexpr int K_ROW = MX ? 8 * (2 * KB - 1) : 16 * KB;  // packed row bytes
  constexpr int V_ROW = MX ? 8 * (2 * VB - 1) : 16 * VB;
  const int g = ch >> 1;  // mixed layout: half of this thread's chunk (0: outlier channels)
  // sqrt(d_half) for u: sqrt(64) per half in the mixed layout, sqrt(128) otherwise
  const double sqd_u = MX ? 8.0 : sqrt((double)D);

  if ((smem_u32(smem_raw) & 1023u) != 0) {  // operand tiles need 1024-byte alignment
    if (tid == 0) atomicOr(&g_quantize_error, 2u);
    return;
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&s.bar_kv, 1);
    mbar_init(&s.bar_s, 1);
    s.err = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (tid < LK) s.kcent[tid] = a.kc[tid];
  if (tid < LK - 1) s.kthr[tid] = a.kt[tid];
  if (tid < LV) s.vcent[tid] = a.vc[tid];
  if (tid < LV - 1) s.vthr[tid] = a.vt[tid];
  if (MX && tid < LK2) s.kcent2[tid] = a.kc2[tid];
  if (MX && tid < LK2 - 1) s.kthr2[tid] = a.kt2[tid];
  if (MX && tid < LV2) s.vcent2[tid] = a.vc2[tid];
  if (MX && tid < LV2 - 1) s.vthr2[tid] = a.vt2[tid];
  if (tid < TM) s.vflag[tid] = 0;
  // Pi enters as 2^8 Pi so that its fp16 lo part stays clear of the subnormal range (the hi + lo
  // pair then carries ~22 significant bits of every entry); the 2^-8 is folded into u's scale.
  // (a Pi exact in fp16, like the structured rotation, has no lo part: its MMA pass is skipped)
  const bool pi_lo = __syncthreads_or(load_matrix(a.Pi, PI_SCALE, s.pih, s.pil) ? 1 : 0) != 0;
  if (a.qjl) load_matrix(a.S, 1.0f, s.sm, nullptr);

  const int tiles_per_bh = (a.T_new + TM - 1) / TM;
  const int64_t total = (int64_t)a.B * a.Hkv * tiles_per_bh;
  auto tile_coords = [&](int64_t tile, int& b, int& h, int& t0, int& nt) {
    const int bh = (int)(tile / tiles_per_bh);
    t0 = (int)(tile % tiles_per_bh) * TM;
    nt = min(TM, a.T_new - t0);
    b = bh / a.Hkv;
    h = bh % a.Hkv;
  };
  if ((int64_t)blockIdx.x < total) {
    int b, h, t0, nt;
    tile_coords(blockIdx.x, b, h, t0, nt);
    issue_x_loads<InT>(s, a, b, h, t0, nt);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;  // == (r & ~31) << 16
  // positive thresholds: T[j] = t[L/2 - 1 + j] (T[0] = 0)
  float TK[8], TV[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    TK[j] = (j < LK / 2) ? s.kthr[LK / 2 - 1 + j] : INFINITY;
    TV[j] = (j < LV / 2) ? s.vthr[LV / 2 - 1 + j] : INFINITY;
  }
  // (mixed layout: the non-outlier half's thresholds)
  float TK2[8], TV2[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    TK2[j] = (MX && j < LK2 / 2) ? s.kthr2[LK2 / 2 - 1 + j] : INFINITY;
    TV2[j] = (MX && j < LV2 / 2) ? s.vthr2[LV2 / 2 - 1 + j] : INFINITY;
  }

  uint32_t phase = 0;
  for (int64_t tile = blockIdx.x; tile < total; tile += gridDim.x, phase ^= 1) {
    int b, h, t0, nt;
    tile_coords(tile, b, h, t0, nt);
    const int64_t row0 = ((int64_t)b * a.Hkv + h) * a.T_cap + a.t_offset + t0;
    const int64_t in_base = (int64_t)b * a.sb + (int64_t)h * a.sh + (int64_t)t0 * a.st;
    const bool live = r < nt;

    // ---- 1. operands ready; convert rows in place to fp16, norms in fp64 ----
    // Codes depend only on the direction of x, so each row is scaled by 2^e (exact) to bring its
    // largest element to [2^14, 2^15) before the fp16 conversion; the stored norm is unscaled.
    {
      const InT* xrow = reinterpret_cast<const InT*>(cwhich == 0 ? a.k : a.v) + in_base + (int64_t)cr * a.st;
      const bool clive = cr < nt;
      uint8_t* xt = cwhich == 0 ? s.xk : s.xv;
      if constexpr (sizeof(InT) != 4) {
        cp_async_wait_all();
        __syncthreads();
      }
      // Half membership of the eight channels 8c .. 8c + 7 (mixed layout: outlier channels).
      auto in_o = [&](int c, int i) -> bool {
        const int ch8 = 8 * c + i;
        return MX && ((a.omask[ch8 >> 5] >> (ch8 & 31)) & 1u);
      };
      double acc = 0.0, acc2 = 0.0;  // plain: acc; mixed: acc (outlier half), acc2 (other half)
      float amax = 0.0f, amax2 = 0.0f;
#pragma unroll 1
      for (int c = 8 * chalf; c < 8 * chalf + 8; ++c) {
        float v8[8];
        row_chunk<InT>(xrow, xt, cr, c, clive, v8);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (!MX || in_o(c, i)) {
            acc = fma((double)v8[i], (double)v8[i], acc);
            amax = fmaxf(amax, fabsf(v8[i]));
          } else {
            acc2 = fma((double)v8[i], (double)v8[i], acc2);
            amax2 = fmaxf(amax2, fabsf(v8[i]));
          }
        }
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      acc2 += __shfl_xor_sync(0xffffffffu, acc2, 1);
      amax2 = fmaxf(amax2, __shfl_xor_sync(0xffffffffu, amax2, 1));
      auto pow2_for = [](float am) {
        int ex = 0;
        frexpf(am, &ex);
        const int e = am > 0.0f ? max(-126, min(127, 15 - ex)) : 0;
        return __int_as_float((e + 127) << 23);  // 2^e
      };
      const float p2 = pow2_for(amax), p2b = MX ? pow2_for(amax2) : p2;
#pragma unroll 1
      for (int c = 8 * chalf; c < 8 * chalf + 8; ++c) {
        float v8[8];
        row_chunk<InT>(xrow, xt, cr, c, clive, v8);
        uint32_t o[4], ol[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float s0 = (!MX || in_o(c, 2 * i)) ? p2 : p2b, s1 = (!MX || in_o(c, 2 * i + 1)) ? p2 : p2b;
          const float x0 = v8[2 * i] * s0, x1 = v8[2 * i + 1] * s1;
          const __half2 hh = __floats2half2_rn(x0, x1);
          o[i] = *reinterpret_cast<const uint32_t*>(&hh);
          if constexpr (sizeof(InT) == 4) {
            const float2 hf = __half22float2(hh);
            const __half2 ll = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
            ol[i] = *reinterpret_cast<const uint32_t*>(&ll);
          }
        }
        *reinterpret_cast<uint4*>(xt + sw_chunk(cr, c)) = make_uint4(o[0], o[1], o[2], o[3]);
        if constexpr (sizeof(InT) == 4)
          if (cwhich == 0) *reinterpret_cast<uint4*>(s.xl + sw_chunk(cr, c)) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
      }
      if (chalf == 0) {
        const double n = sqrt(acc);
        (cwhich == 0 ? s.nrmk : s.nrmv)[cr] = n;
        (cwhich == 0 ? s.sclk : s.sclv)[cr] =
            n > 0.0 ? (float)(sqd_u / (n * (double)p2 * (double)PI_SCALE)) : 0.0f;
        if constexpr (MX) {
          const double n2 = sqrt(acc2);
          (cwhich == 0 ? s.nrmk2 : s.nrmv2)[cr] = n2;
          (cwhich == 0 ? s.sclk2 : s.sclv2)[cr] =
              n2 > 0.0 ? (float)(sqd_u / (n2 * (double)p2b * (double)PI_SCALE)) : 0.0f;
        }
      }
    }
    // sign rows (and 3-bit value rows) are assembled with shared-memory atomics: clear them
    for (int i = tid; i < TM * 4; i += THREADS) reinterpret_cast<uint32_t*>(s.sst)[i] = 0u;
    if constexpr (VB == 3 || MX)  // (the mixed layout's 3-bit value half uses atomics too)
      for (int i = tid; i < TM * V_ROW / 4; i += THREADS) reinterpret_cast<uint32_t*>(s.vst)[i] = 0u;
    if (tid == 0) {
      s.nfl = 0;
      s.nvfl = 0;
      s.nexc = 0;
      s.nexs = 0;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- 2. rotation MMAs: Y = X (Pi_hi + Pi_lo)^T ----
    if (tid == 0) {
      tc_fence_after();
#pragma unroll 1
      for (int ks = 0; ks < 8; ++ks) {
        umma_f16(tmem + COL_K, desc_at(s.xk, ks), desc_at(s.pih, ks), IDESC, ks > 0);
        if (pi_lo) umma_f16(tmem + COL_K, desc_at(s.xk, ks), desc_at(s.pil, ks), IDESC, 1);
        if constexpr (sizeof(InT) == 4) umma_f16(tmem + COL_K, desc_at(s.xl, ks), desc_at(s.pih, ks), IDESC, 1);
        umma_f16(tmem + COL_V, desc_at(s.xv, ks), desc_at(s.pih, ks), IDESC, ks > 0);
        if (pi_lo) umma_f16(tmem + COL_V, desc_at(s.xv, ks), desc_at(s.pil, ks), IDESC, 1);
      }
      umma_commit(&s.bar_kv);
    }
    if (!mbar_wait(&s.bar_kv, phase, WAIT_LIMIT)) s.err = 1;
    tc_fence_after();
    __syncthreads();
    if (s.err) break;
    // X buffers are free: prefetch the next tile while this one is finished.
    if (tile + gridDim.x < total) {
      int b2, h2, t02, nt2;
      tile_coords(tile + gridDim.x, b2, h2, t02, nt2);
      issue_x_loads<InT>(s, a, b2, h2, t02, nt2);
    }

    // ---- 3a. keys: codes, residual rho (fp16 hi + lo into tensor memory), ||rho||^2 ----
    // Chunk ch holds coordinates 32ch + i; for each tau its codes fill the 8 consecutive slots
    // 32 tau + 8 ch + q of coordinates 32ch + 2 tau + {0,1,8,9,16,17,24,25}[q]: one
    // byte-aligned field of 8 * k_bits bits at byte k_bits * (4 tau + ch).  Mixed layout: the
    // half's stream starts at byte 0 (outlier half) or 8 k_bits, and the field of chunk ch holds
    // slots 16 tau + 8 (ch & 1) + q at byte b (2 tau + (ch & 1)) of it, b the half's bit width.
    // The residual entering the sketch is, in the mixed layout, f_g rho with
    // f_g = sqrt(2) ||x_g|| / ||x||: sqrt(128) / ||x|| times the half's residual in the rotated
    // basis, so that the sketch is S r in the units of the plain method.
    {
      const bool g1 = MX && g == 1;
      const float scl = g1 ? s.sclk2[r] : s.sclk[r];
      const bool zero = scl == 0.0f;
      float fg = 1.0f;
      if constexpr (MX) {
        const double n0 = s.nrmk[r], n1 = s.nrmk2[r], nx = sqrt(n0 * n0 + n1 * n1);
        fg = nx > 0.0 ? (float)(1.4142135623730951 * (g1 ? n1 : n0) / nx) : 0.0f;
      }
      uint8_t* krow = s.kst + r * K_ROW;
      float r2 = 0.0f;
      uint32_t yr[32];
      tmem_ld32(tmem + lane_base + COL_K + 32 * ch, yr);
      tmem_wait_ld();
      uint32_t hi[16], lo[16];
      uint32_t fld[4] = {0u, 0u, 0u, 0u};
      uint32_t near = 0u;
      const int LKg = g1 ? LK2 : LK;
      const float* kcg = g1 ? s.kcent2 : s.kcent;
      const int bg = g1 ? KB - 1 : KB;
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        float rr[2];
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
          const int ii = i + e2;
          const float u = __uint_as_float(yr[ii]) * scl;
          const float aa = fabsf(u);
          float margin;
          int kpos;
          if constexpr (MX) kpos = g1 ? search_pos<KB - 1>(aa, TK2, margin) : search_pos<KB>(aa, TK, margin);
          else kpos = search_pos<KB>(aa, TK, margin);
          const int idx = zero ? LKg / 2 : (u >= 0.0f ? LKg / 2 + kpos : LKg / 2 - 1 - kpos);
          const float rho = (u - kcg[idx]) * fg;
          near |= (fminf(margin, aa) < a.guard.code_k ? 1u : 0u) << ii;
          rr[e2] = rho;
          r2 = fmaf(rho, rho, r2);
          const int tau = (ii & 7) >> 1, q = ((ii >> 4) << 2) | (((ii >> 3) & 1) << 1) | (ii & 1);
          fld[tau] |= (uint32_t)idx << (bg * q);
        }
        const __half2 hh = __floats2half2_rn(rr[0], rr[1]);
        const float2 hf = __half22float2(hh);
        const __half2 ll = __floats2half2_rn(rr[0] - hf.x, rr[1] - hf.y);
        hi[i / 2] = *reinterpret_cast<const uint32_t*>(&hh);
        lo[i / 2] = *reinterpret_cast<const uint32_t*>(&ll);
      }
#pragma unroll
      for (int tau = 0; tau < 4; ++tau) {
        if constexpr (MX) {
          uint8_t* dst = krow + (g1 ? 8 * KB : 0) + bg * (2 * tau + (ch & 1));
          if (!g1 && KB == 4) {
            *reinterpret_cast<uint32_t*>(dst) = fld[tau];
          } else {
            for (int bb = 0; bb < bg; ++bb) dst[bb] = (uint8_t)(fld[tau] >> (8 * bb));
          }
        } else {
          uint8_t* dst = krow + KB * (4 * tau + ch);
          if constexpr (KB == 4) {
            *reinterpret_cast<uint32_t*>(dst) = fld[tau];
          } else if constexpr (KB == 2) {
            *reinterpret_cast<uint16_t*>(dst) = (uint16_t)fld[tau];
          } else {
            dst[0] = (uint8_t)fld[tau];
            dst[1] = (uint8_t)(fld[tau] >> 8);
            dst[2] = (uint8_t)(fld[tau] >> 16);
          }
        }
      }
      if (a.qjl) {
        tmem_st16(tmem + lane_base + COL_RH + 16 * ch, hi);
        tmem_st16(tmem + lane_base + COL_RL + 16 * ch, lo);
        tmem_wait_st();
      }
      s.rho2[ch][r] = r2;
      if (!(live && !zero)) near = 0u;
      while (near) {  // queue coordinates near a threshold for the fp64 pass
        const int ii = __ffs(near) - 1;
        near &= near - 1;
        const int slot = atomicAdd(&s.nfl, 1);
        if (slot < FL_CAP) s.fl[slot] = (uint16_t)((r << 7) | (32 * ch + ii));
        else atomicOr(&s.vflag[r], 2u);  // list full: the key row takes the fp64 vector path
      }
    }
    // ---- 3b. values: codes.  Coordinate 32ch + i sits at slot 16 (i % 8) + 4 ch + i / 8: chunk ch
    //          gives lane group g a field of 4 codes at bit v_bits (16 g + 4 ch).  Mixed layout:
    //          within the half's stream (byte 0 or 8 v_bits), slot 8 (i % 8) + 4 (ch & 1) + i / 8. ----
    {
      const bool g1 = MX && g == 1;
      const float scl = g1 ? s.sclv2[r] : s.sclv[r];
      const bool zero = scl == 0.0f;
      uint32_t yr[32];
      tmem_ld32(tmem + lane_base + COL_V + 32 * ch, yr);
      tmem_wait_ld();
      uint32_t near = 0u;
      uint32_t f8[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      const int LVg = g1 ? LV2 : LV;
      const int bg = g1 ? VB - 1 : VB;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float u = __uint_as_float(yr[i]) * scl;
        const float aa = fabsf(u);
        float margin;
        int kpos;
        if constexpr (MX) kpos = g1 ? search_pos<VB - 1>(aa, TV2, margin) : search_pos<VB>(aa, TV, margin);
        else kpos = search_pos<VB>(aa, TV, margin);
        const int idx = zero ? LVg / 2 : (u >= 0.0f ? LVg / 2 + kpos : LVg / 2 - 1 - kpos);
        near |= (fminf(margin, aa) < a.guard.code_v ? 1u : 0u) << i;
        f8[i & 7] |= (uint32_t)idx << (bg * (i >> 3));
      }
      uint8_t* vrow = s.vst + r * V_ROW;
#pragma unroll
      for (int gg = 0; gg < 8; ++gg) {
        if constexpr (MX) {
          if (!g1 && VB == 4) {
            *reinterpret_cast<uint16_t*>(vrow + 4 * gg + 2 * (ch & 1)) = (uint16_t)f8[gg];
          } else {  // 4 codes of bg bits at bit 8 (8 VB) + bg (8 gg + 4 (ch & 1)) of the row
            const int P = (g1 ? 64 * VB : 0) + bg * (8 * gg + 4 * (ch & 1));
            uint32_t* w = reinterpret_cast<uint32_t*>(vrow);
            atomicOr(&w[P >> 5], f8[gg] << (P & 31));
            if ((P & 31) + 4 * bg > 32) atomicOr(&w[(P >> 5) + 1], f8[gg] >> (32 - (P & 31)));
          }
        } else if constexpr (VB == 4) {
          *reinterpret_cast<uint16_t*>(vrow + 8 * gg + 2 * ch) = (uint16_t)f8[gg];
        } else if constexpr (VB == 2) {
          vrow[4 * gg + ch] = (uint8_t)f8[gg];
        } else {
          const int P = 48 * gg + 12 * ch;  // 12-bit field: may straddle two words
          uint32_t* w = reinterpret_cast<uint32_t*>(vrow);
          atomicOr(&w[P >> 5], f8[gg] << (P & 31));
          if ((P & 31) > 20) atomicOr(&w[(P >> 5) + 1], f8[gg] >> (32 - (P & 31)));
        }
      }
      if (!(live && !zero)) near = 0u;
      while (near) {
        const int ii = __ffs(near) - 1;
        near &= near - 1;
        const int slot = atomicAdd(&s.nfl, 1);
        if (slot < FL_CAP) s.fl[slot] = (uint16_t)(0x8000u | (r << 7) | (32 * ch + ii));
        else atomicOr(&s.vflag[r], 4u);  // list full: this value row is re-derived whole in fp64
      }
    }
    if (ch == 0) {
      s.kn[r] = (float)s.nrmk[r];
      s.vn[r] = (float)s.nrmv[r];
      if constexpr (MX) {
        s.kn2[r] = (float)s.nrmk2[r];
        s.vn2[r] = (float)s.nrmv2[r];
      }
    }
    tc_fence_before();
    __syncthreads();

    // ---- 4. sketch MMA D_S = (rho_hi + rho_lo) S^T; meanwhile re-derive flagged coordinates ----
    if (a.qjl && tid == 0) {
      tc_fence_after();
#pragma unroll 1
      for (int ks = 0; ks < 8; ++ks) {
        umma_f16_ts(tmem + COL_S, tmem + COL_RH + 8 * ks, desc_at(s.sm, ks), IDESC, ks > 0);
        umma_f16_ts(tmem + COL_S, tmem + COL_RL + 8 * ks, desc_at(s.sm, ks), IDESC, 1);
      }
      umma_commit(&s.bar_s);
    }
    {
      // four threads per queued coordinate: one fp64 dot product each, one memory round trip
      const int nfl = min(s.nfl, FL_CAP);
      for (int f0 = 0; f0 < nfl; f0 += THREADS / 4) {
        const int f = f0 + (tid >> 2);
        const bool have = f < nfl;
        const uint32_t ent = have ? s.fl[f] : 0u;
        const bool val = ent & 0x8000u;
        const int rr = (ent >> 7) & 127, j = ent & 127;
        const InT* x = reinterpret_cast<const InT*>(val ? a.v : a.k) + in_base + (int64_t)rr * a.st;
        const double part = have ? exact_dot_part<InT>(a.Pi, x, j, tid & 3) : 0.0;
        const double dot = quad_sum(part);  // all lanes take part in the shuffle
        if (!have || (tid & 3)) continue;
        const bool hj = MX && j >= 64;  // mixed layout: coordinate of the non-outlier half
        const double nn = val ? (hj ? s.nrmv2[rr] : s.nrmv[rr]) : (hj ? s.nrmk2[rr] : s.nrmk[rr]);
        const double ud = sqd_u * dot / nn;
        const float* thr = val ? (hj ? s.vthr2 : s.vthr) : (hj ? s.kthr2 : s.kthr);
        const int nthr = (val ? (hj ? LV2 : LV) : (hj ? LK2 : LK)) - 1;
        if (code_exempt_exact(ud, thr, nthr)) atomicAdd(&s.nexc, 1u);
        const uint32_t idx = (uint32_t)code_exact(ud, thr, nthr);
        if (val) {
          uint8_t* row = s.vst + rr * V_ROW;
          const int bits = hj ? VB - 1 : VB;
          const int P = MX ? mixed_bit_pos(j, v_slot_of_coord_mixed(j), VB) : VB * v_slot_of_coord(j);
          if (get_code_at(row, bits, P) != idx) set_code_at(row, bits, P, idx);
        } else {
          uint8_t* row = s.kst + rr * K_ROW;
          const int bits = hj ? KB - 1 : KB;
          const int P = MX ? mixed_bit_pos(j, k_slot_of_coord_mixed(j), KB) : KB * k_slot_of_coord(j);
          if (get_code_at(row, bits, P) != idx) {
            set_code_at(row, bits, P, idx);
            // the residual fed to the sketch came from the other cell: redo the vector in fp64
            if (a.qjl) atomicOr(&s.vflag[rr], 1u);
          }
        }
      }
      if (tid == 0 && s.nfl) atomicAdd(&g_quantize_code_fixups, (unsigned)min(s.nfl, FL_CAP));
    }
    if (a.qjl) {
      if (!mbar_wait(&s.bar_s, phase, WAIT_LIMIT)) s.err = 1;
      tc_fence_after();
      // sketch row l = 32ch + i = 16 kap + 8 h + 2 tau + e sits at row bit 32 tau + (2 kap + h)
      // + 16 e; chunk ch fills, for each tau and e, the nibble at bit 32 tau + 16 e + 4 ch.
      uint32_t yr[32];
      tmem_ld32(tmem + lane_base + COL_S + 32 * ch, yr);
      tmem_wait_ld();
      uint32_t nib[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // [tau][e]
      bool flagged = false;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float sp = __uint_as_float(yr[i]);
        const int tau = (i >> 1) & 3, e2 = i & 1, pp = ((i >> 4) << 1) | ((i >> 3) & 1);
        nib[2 * tau + e2] |= (sp >= 0.0f ? 1u : 0u) << pp;
        flagged |= fabsf(sp) < a.guard.sign;
      }
      uint32_t* srow = reinterpret_cast<uint32_t*>(s.sst + r * 16);
#pragma unroll
      for (int tau = 0; tau < 4; ++tau)
        atomicOr(&srow[tau], (nib[2 * tau] << (4 * ch)) | (nib[2 * tau + 1] << (16 + 4 * ch)));
      if (flagged && live) atomicOr(&s.vflag[r], 1u);
    }
    tc_fence_before();
    __syncthreads();
    if (s.err) break;
    if (tid < TM) {
      if (a.qjl) {
        const double nk = MX ? sqrt(s.nrmk[tid] * s.nrmk[tid] + s.nrmk2[tid] * s.nrmk2[tid]) : s.nrmk[tid];
        s.rn[tid] = (float)(nk * sqrt((double)(s.rho2[0][tid] + s.rho2[1][tid] + s.rho2[2][tid] +
                                                s.rho2[3][tid])) / sqrt((double)D));
      }
      if (s.vflag[tid]) s.vfl[atomicAdd(&s.nvfl, 1)] = (uint8_t)tid;
    }
    __syncthreads();

    // ---- 5. rows re-derived whole in fp64: key vectors with a sketch value near 0 or a corrected
    //         code, and rows whose near-threshold list overflowed ----
    {
      const int nvf = s.nvfl;
      for (int f = 0; f < nvf; ++f) {
        const int rr = s.vfl[f];
        const unsigned int fl = s.vflag[rr];
        if (fl & 4) {  // value row
          const InT* vx = reinterpret_cast<const InT*>(a.v) + in_base + (int64_t)rr * a.st;
          {
            const int j = tid >> 2;
            const bool hj = MX && j >= 64;
            const double nv = hj ? s.nrmv2[rr] : s.nrmv[rr];
            const float* thr = hj ? s.vthr2 : s.vthr;
            const int nthr = (hj ? LV2 : LV) - 1;
            const double dot = quad_sum(exact_dot_part<InT>(a.Pi, vx, j, tid & 3));
            if ((tid & 3) == 0) {
              const int idx = nv > 0.0 ? code_exact(sqd_u * dot / nv, thr, nthr) : (nthr + 1) / 2;
              // (a row whose near-threshold list overflowed: its coordinates are counted here)
              if (nv > 0.0 && code_exempt_exact(sqd_u * dot / nv, thr, nthr)) atomicAdd(&s.nexc, 1u);
              s.fcode[MX ? (hj ? 64 : 0) + v_slot_of_coord_mixed(j) : v_slot_of_coord(j)] = (uint8_t)idx;
            }
          }
          __syncthreads();
          if (tid < V_ROW / 4) {
            uint32_t word = 0;
            for (int kk = 0; kk < 32; ++kk) {
              const int P = 32 * tid + kk;
              int code, bit;
              if (MX && P >= 64 * VB) {
                code = s.fcode[64 + (P - 64 * VB) / (VB - 1)];
                bit = (P - 64 * VB) % (VB - 1);
              } else {
                code = s.fcode[P / VB];
                bit = P % VB;
              }
              word |= (uint32_t)((code >> bit) & 1) << kk;
            }
            reinterpret_cast<uint32_t*>(s.vst + rr * V_ROW)[tid] = word;
          }
          __syncthreads();
        }
        if (!(fl & 3)) continue;  // uniform: read from shared memory after a barrier
        const InT* kx = reinterpret_cast<const InT*>(a.k) + in_base + (int64_t)rr * a.st;
        // ||x|| (mixed layout: of both halves); each coordinate's residual enters the sketch as
        // f_g rho (f_g = sqrt(2) ||x_g|| / ||x||, 1 in the plain layout)
        const double nk = MX ? sqrt(s.nrmk[rr] * s.nrmk[rr] + s.nrmk2[rr] * s.nrmk2[rr]) : s.nrmk[rr];
        {
          const int j = tid >> 2;
          const bool hj = MX && j >= 64;
          const double ng = hj ? s.nrmk2[rr] : s.nrmk[rr];
          const float* thr = hj ? s.kthr2 : s.kthr;
          const float* cen = hj ? s.kcent2 : s.kcent;
          const int nthr = (hj ? LK2 : LK) - 1;
          const double fgd = MX ? (nk > 0.0 ? 1.4142135623730951 * ng / nk : 0.0) : 1.0;
          const double dot = quad_sum(exact_dot_part<InT>(a.Pi, kx, j, tid & 3));
          double rho = 0.0;
          if ((tid & 3) == 0) {
            int idx;
            if (ng > 0.0) {
              const double ud = sqd_u * dot / ng;
              idx = code_exact(ud, thr, nthr);
              if ((fl & 2) && code_exempt_exact(ud, thr, nthr)) atomicAdd(&s.nexc, 1u);
              rho = (ud - (double)cen[idx]) * fgd;
            } else {
              idx = (nthr + 1) / 2;
              rho = -(double)cen[idx] * fgd;
            }
            s.fx64[j] = rho;
            s.fcode[MX ? (hj ? 64 : 0) + k_slot_of_coord_mixed(j) : k_slot_of_coord(j)] = (uint8_t)idx;
          }
          double q2 = rho * rho;
          for (int o = 16; o > 0; o >>= 1) q2 += __shfl_xor_sync(0xffffffffu, q2, o);
          if ((tid & 31) == 0) s.red64[tid >> 5] = q2;
        }
        __syncthreads();
        if (a.qjl) {  // (S rho)_l from the exact fp16 copy of S in shared memory
          const int l = tid >> 2, q = tid & 3;
          double sp0 = 0.0, sp1 = 0.0;
#pragma unroll 8
          for (int jj = 0; jj < 32; jj += 2) {
            const int j = 32 * q + jj;
            sp0 = fma((double)__half2float(*reinterpret_cast<const __half*>(s.sm + sw_off(l, j))), s.fx64[j], sp0);
            sp1 = fma((double)__half2float(*reinterpret_cast<const __half*>(s.sm + sw_off(l, j + 1))), s.fx64[j + 1], sp1);
          }
          const double sp = quad_sum(sp0 + sp1);
          if (q == 0) {
            s.fsign[sign_bit_of_row(l)] = sp >= 0.0 ? 1 : 0;
            if (fabs(sp) <= kExemptSignBand) atomicAdd(&s.nexs, 1u);
          }
        }
        __syncthreads();
        if (tid < K_ROW / 4) {
          uint32_t word = 0;
          for (int kk = 0; kk < 32; ++kk) {
            const int P = 32 * tid + kk;
            int code, bit;
            if (MX && P >= 64 * KB) {
              code = s.fcode[64 + (P - 64 * KB) / (KB - 1)];
              bit = (P - 64 * KB) % (KB - 1);
            } else {
              code = s.fcode[P / KB];
              bit = P % KB;
            }
            word |= (uint32_t)((code >> bit) & 1) << kk;
          }
          reinterpret_cast<uint32_t*>(s.kst + rr * K_ROW)[tid] = word;
        } else if (tid >= 32 && tid < 36 && a.qjl) {
          const int w = tid - 32;
          uint32_t word = 0;
          for (int kk = 0; kk < 32; ++kk) word |= (uint32_t)s.fsign[32 * w + kk] << kk;
          reinterpret_cast<uint32_t*>(s.sst + rr * 16)[w] = word;
        } else if (tid == 64 && a.qjl) {
          double q2 = 0.0;
          for (int w = 0; w < THREADS / 32; ++w) q2 += s.red64[w];
          s.rn[rr] = (float)(nk * sqrt(q2) / sqrt((double)D));
        }
        __syncthreads();
      }
      if (tid < TM) s.vflag[tid] = 0;
      if (tid == 0 && nvf) atomicAdd(&g_quantize_vector_fixups, (unsigned)nvf);
      if (tid == 0 && s.nexc) atomicAdd(&g_quantize_exempt_codes, s.nexc);
      if (tid == 0 && s.nexs) atomicAdd(&g_quantize_exempt_signs, s.nexs);
    }

    // ---- 6. coalesced stores of the tile's rows ----
    {
      if constexpr (MX) {  // rows of 56 bytes: 8-byte units (any row is 8-byte aligned)
        const uint2* srk = reinterpret_cast<const uint2*>(s.kst);
        uint2* dsk = reinterpret_cast<uint2*>(a.k_codes + row0 * K_ROW);
        for (int i = tid; i < nt * K_ROW / 8; i += THREADS) dsk[i] = srk[i];
        const uint2* srv = reinterpret_cast<const uint2*>(s.vst);
        uint2* dsv = reinterpret_cast<uint2*>(a.v_codes + row0 * V_ROW);
        for (int i = tid; i < nt * V_ROW / 8; i += THREADS) dsv[i] = srv[i];
      } else {
        const uint4* srk = reinterpret_cast<const uint4*>(s.kst);
        uint4* dsk = reinterpret_cast<uint4*>(a.k_codes + row0 * K_ROW);
        for (int i = tid; i < nt * KB; i += THREADS) dsk[i] = srk[i];
        const uint4* srv = reinterpret_cast<const uint4*>(s.vst);
        uint4* dsv = reinterpret_cast<uint4*>(a.v_codes + row0 * V_ROW);
        for (int i = tid; i < nt * VB; i += THREADS) dsv[i] = srv[i];
      }
      const uint4* src;
      uint4* dst;
      if (a.qjl) {
        src = reinterpret_cast<const uint4*>(s.sst);
        dst = reinterpret_cast<uint4*>(a.k_signs + row0 * 16);
        for (int i = tid; i < nt; i += THREADS) dst[i] = src[i];
      }
      for (int i = tid; i < nt; i += THREADS) {
        if constexpr (MX) {
          reinterpret_cast<float2*>(a.k_norm)[row0 + i] = make_float2(s.kn[i], s.kn2[i]);
          reinterpret_cast<float2*>(a.v_norm)[row0 + i] = make_float2(s.vn[i], s.vn2[i]);
        } else {
          a.k_norm[row0 + i] = s.kn[i];
          a.v_norm[row0 + i] = s.vn[i];
        }
        if (a.qjl) a.k_rnorm[row0 + i] = s.rn[i];
      }
    }
    __syncthreads();
  }
  cp_async_wait_all();
  tc_fence_before();
  __syncthreads();
  if (s.err && tid == 0) atomicOr(&g_quantize_error, s.err);
  if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

template <int KB, int VB, typename InT, bool MX = false>
tq_status launch3(const QArgs& a, int sms, cudaStream_t stream) {
  const size_t smem = sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(quantize_kernel<KB, VB, InT, MX>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "smem attribute: %s", cudaGetErrorString(e));
  const int64_t total = (int64_t)a.B * a.Hkv * ((a.T_new + TM - 1) / TM);
  const int grid = (int)(total < sms ? total : sms);
  quantize_kernel<KB, VB, InT, MX><<<grid, THREADS, smem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "quantize launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}

template <typename InT>
tq_status launch(int kb, int vb, const QArgs& a, int sms, cudaStream_t s) {
#define TQ_V(KB)                                        \
  switch (vb) {                                         \
    case 2: return launch3<KB, 2, InT>(a, sms, s);      \
    case 3: return launch3<KB, 3, InT>(a, sms, s);      \
    default: return launch3<KB, 4, InT>(a, sms, s);     \
  }
  switch (kb) {
    case 2: TQ_V(2)
    case 3: TQ_V(3)
    default: TQ_V(4)
  }
#undef TQ_V
}

// S_Pi = S Pi in fp64: block l, thread j; products of fp32 values are exact in fp64 and are
// summed in ascending i.
__global__ void __launch_bounds__(kHeadDim) sketch_rotation_kernel(const float* __restrict__ Pi,
                                                                   const float* __restrict__ S,
                                                                   double* __restrict__ S_Pi) {
  __shared__ double srow[kHeadDim];
  const int l = blockIdx.x, j = threadIdx.x;
  srow[j] = (double)S[(int64_t)l * kHeadDim + j];
  __syncthreads();
  double acc = 0.0;
#pragma unroll 8
  for (int i = 0; i < kHeadDim; ++i) acc = fma(srow[i], (double)Pi[i * kHeadDim + j], acc);
  S_Pi[(int64_t)l * kHeadDim + j] = acc;
}

}  // namespace
}  // namespace tq

extern "C" tq_status tq_sketch_rotation(const float* Pi, const float* S, int qjl_m, double* S_Pi,
                                        void* stream) {
  using namespace tq;
  clear_error();
  if (!Pi || !S || !S_Pi) return fail(TQ_ERR_INVALID_ARG, "Pi / S / S_Pi is NULL");
  if (!aligned16(Pi) || !aligned16(S) || !aligned16(S_Pi))
    return fail(TQ_ERR_INVALID_ARG, "Pi / S / S_Pi must be 16-byte aligned");
  if (qjl_m < 1) return fail(TQ_ERR_INVALID_ARG, "qjl_m %d < 1", qjl_m);
  sketch_rotation_kernel<<<qjl_m, kHeadDim, 0, reinterpret_cast<cudaStream_t>(stream)>>>(Pi, S, S_Pi);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "sketch rotation launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}

extern "C" tq_status tq_quantize(const tq_params* params, const void* k, const void* v, int dtype,
                                 int64_t stride_b, int64_t stride_h, int64_t stride_t, int T_new,
                                 int t_offset, const tq_cache* cache, void* stream) {
  using namespace tq;
  const NvtxRange nvtx_range("tq_quantize");
  clear_error();
  tq_status st = check_cache(cache);
  if (st != TQ_OK) return st;
  st = check_params(params, cache);
  if (st != TQ_OK) return st;
  if (dtype != TQ_F32 && dtype != TQ_BF16) return fail(TQ_ERR_UNSUPPORTED, "dtype %d", dtype);
  if (T_new < 0 || t_offset < 0 || (int64_t)t_offset + T_new > cache->T_cap)
    return fail(TQ_ERR_INVALID_ARG, "token range [%d, %d) outside T_cap %d", t_offset,
                t_offset + T_new, cache->T_cap);
  if (T_new == 0) return TQ_OK;
  if (!k || !v) return fail(TQ_ERR_INVALID_ARG, "k / v is NULL");
  const int64_t esz = dtype == TQ_F32 ? 4 : 2;
  if (!aligned16(k) || !aligned16(v)) return fail(TQ_ERR_INVALID_ARG, "k / v must be 16-byte aligned");
  if (stride_t < kHeadDim || stride_b < 0 || stride_h < 0 || (stride_t * esz) % 16 ||
      (stride_h * esz) % 16 || (stride_b * esz) % 16)
    return fail(TQ_ERR_INVALID_ARG, "strides (%lld, %lld, %lld) invalid", (long long)stride_b,
                (long long)stride_h, (long long)stride_t);
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "device query: %s", cudaGetErrorString(e));
  QArgs a;
  a.k = k;
  a.v = v;
  a.sb = stride_b;
  a.sh = stride_h;
  a.st = stride_t;
  a.T_new = T_new;
  a.t_offset = t_offset;
  a.B = cache->B;
  a.Hkv = cache->Hkv;
  a.T_cap = cache->T_cap;
  a.qjl = cache->qjl_m ? 1 : 0;
  a.in_f32 = dtype == TQ_F32;
  a.k_codes = cache->k_codes;
  a.k_signs = cache->k_signs;
  a.k_norm = cache->k_norm;
  a.k_rnorm = cache->k_rnorm;
  a.v_codes = cache->v_codes;
  a.v_norm = cache->v_norm;
  a.Pi = params->Pi;
  a.S = params->S;
  a.kc = params->k_centroids;
  a.kt = params->k_thresholds;
  a.vc = params->v_centroids;
  a.vt = params->v_thresholds;
  // Fast-path error, measured on B200 over 1.5e7 coordinates with every guard off: a code differed
  // from the float64 one only within 6.3e-7 of a threshold, a sign only for |S rho| <= 7.8e-6
  // (exact fp16 operands: bf16 input, or fp32 keys as fp16 hi + lo; Pi as fp16 hi + lo).  The
  // bands below are >= 4x those.  fp32 values enter as fp16(x) alone (relative 2^-12, ~2e-4 in u).
  a.guard = dtype == TQ_F32 ? Guards{4e-6f, 4e-3f, 3e-5f} : Guards{4e-6f, 4e-6f, 3e-5f};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cache->layout == TQ_LAYOUT_MIXED) {  // 4-bit outlier half, 3-bit other half (checked above)
    a.kc2 = params->k_centroids_lo;
    a.kt2 = params->k_thresholds_lo;
    a.vc2 = params->v_centroids_lo;
    a.vt2 = params->v_thresholds_lo;
    for (int w = 0; w < 4; ++w) a.omask[w] = params->outlier_mask[w];
    return dtype == TQ_F32 ? launch3<4, 4, float, true>(a, sms, s) : launch3<4, 4, __nv_bfloat16, true>(a, sms, s);
  }
  if (dtype == TQ_BF16) {
    bool handled = false;
    st = quantize_bf16_pipeline(params, k, v, stride_b, stride_h, stride_t, T_new, t_offset, cache, sms, s,
                                &handled);
    if (handled || st != TQ_OK) return st;
  }
  return dtype == TQ_F32 ? launch<float>(cache->k_bits, cache->v_bits, a, sms, s)
                         : launch<__nv_bfloat16>(cache->k_bits, cache->v_bits, a, sms, s);
}

extern "C" int tq_quantize_device_errors(void) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, tq::g_quantize_error, sizeof(v)) != cudaSuccess) return -1;
  const unsigned int p = tq::pipe_device_errors();
  if (p == 0xffffffffu) return -1;
  return (int)(v | p);
}

extern "C" long long tq_quantize_vector_fixups(void) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, tq::g_quantize_vector_fixups, sizeof(v)) != cudaSuccess) return -1;
  const long long p = tq::pipe_vector_fixups();
  return p < 0 ? -1 : (long long)v + p;
}

extern "C" long long tq_quantize_code_fixups(void) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, tq::g_quantize_code_fixups, sizeof(v)) != cudaSuccess) return -1;
  const long long p = tq::pipe_code_fixups();
  return p < 0 ? -1 : (long long)v + p;
}

extern "C" long long tq_quantize_exempt_codes(void) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, tq::g_quantize_exempt_codes, sizeof(v)) != cudaSuccess) return -1;
  const long long p = tq::pipe_exempt_codes();
  return p < 0 ? -1 : (long long)v + p;
}

extern "C" long long tq_quantize_exempt_signs(void) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, tq::g_quantize_exempt_signs, sizeof(v)) != cudaSuccess) return -1;
  const long long p = tq::pipe_exempt_signs();
  return p < 0 ? -1 : (long long)v + p;
}

extern "C" tq_status tq_debug_quantize_stall(int enable, long long wait_cycles) {
  tq::clear_error();
  if (enable && wait_cycles <= 0) return tq::fail(TQ_ERR_INVALID_ARG, "wait_cycles %lld must be > 0", wait_cycles);
  tq::pipe_set_test_stall(enable, wait_cycles);
  return TQ_OK;
}

extern "C" int tq_reset_device_errors(void) {
  const unsigned int z = 0;
  if (cudaMemcpyToSymbol(tq::g_quantize_error, &z, sizeof(z)) != cudaSuccess) return -1;
  if (tq::pipe_reset_errors() != 0) return -1;
  return tq::decode_reset_errors();
}
