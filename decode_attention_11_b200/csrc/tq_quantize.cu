// tq_quantize: rotate -> Lloyd-Max scalar quantize -> bit-pack -> 1-bit QJL sketch.
//
// Method: ai-news.ru TurboQuant overview (first idea: random orthogonal rotation makes the
// coordinates near-Gaussian; second idea: a Lloyd-Max grid precomputed for that distribution;
// third component: 1-bit QJL correction of the residual), tproger.ru "Google TurboQuant in simple
// words", "Step 1: PolarQuant" (every coordinate quantized independently, no per-group scale
// bits) and "Step 2: QJL" (one extra bit per sketch row makes the inner-product error unbiased).
//
// Exactness: codes and sign bits must equal those of the float64 definition.  The fast path
// computes the rotation and the sketch in fp32; any coordinate whose fp32 value lies within a
// guard band of a decision boundary (a threshold, or 0 for a sign) is re-derived in fp64 from the
// original inputs, which leaves only values within ~1e-15 of a boundary undecided.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr int D = kHeadDim;
constexpr int TILE = 16;                 // tokens per tile (one CTA step)
constexpr int THREADS = 128;             // thread j owns coordinate j / sketch row j
// fp32 error of u = sqrt(d) * (Pi x) / ||x|| is ~4e-7 (rms) for d = 128; the bands are >= 100x it.
constexpr float kGuardCode = 4e-5f;
// fp32 error of (S rho)_l is ~5e-6 (rms), dominated by the rounding of rho.
constexpr float kGuardSign = 2e-4f;

struct QArgs {
  const void* k;
  const void* v;
  int64_t sb, sh, st;
  int T_new, t_offset;
  int B, Hkv, T_cap;
  int kb, vb, qjl;
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
};

struct __align__(16) Smem {
  float PiT[D][D];        // PiT[k][j] = Pi[j][k]
  float ST[D][D];         // ST[j][l]  = S[l][j]
  float xT[D][TILE];      // input tile, transposed
  float rhoT[D][TILE];    // residuals, transposed
  double rho64[D];        // exact residual of one vector (fixup path)
  double nrm[TILE];       // ||x|| (fp64, exact sum of squares)
  double red64[4];
  float cent[16];
  float thr[16];
  float red[TILE][4];
  int flag[TILE];
  uint8_t codes[TILE][D];  // code by slot
  uint8_t sbits[TILE][D];  // sign bit by row-bit position
};

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// index = #{i : u >= t_i}; margin = distance to the nearest threshold.
__device__ __forceinline__ int code_of(float u, const float* thr, int nthr, float& margin) {
  int idx = 0;
  float m = INFINITY;
  for (int i = 0; i < nthr; ++i) {
    idx += (u >= thr[i]) ? 1 : 0;
    m = fminf(m, fabsf(u - thr[i]));
  }
  margin = m;
  return idx;
}

__device__ __forceinline__ int code_of_d(double u, const float* thr, int nthr) {
  int idx = 0;
  for (int i = 0; i < nthr; ++i) idx += (u >= (double)thr[i]) ? 1 : 0;
  return idx;
}

// Exact (fp64) rotated coordinate j of tile vector v.
__device__ __forceinline__ double exact_u(const Smem& s, int j, int v, double n) {
  double y0 = 0.0, y1 = 0.0;
#pragma unroll 4
  for (int k = 0; k < D; k += 2) {
    y0 = fma((double)s.PiT[k][j], (double)s.xT[k][v], y0);
    y1 = fma((double)s.PiT[k + 1][j], (double)s.xT[k + 1][v], y1);
  }
  return sqrt((double)D) * (y0 + y1) / n;
}

template <typename InT>
__device__ void quantize_side(Smem& s, const QArgs& a, int which, int b, int h, int t0, int nt) {
  const int j = threadIdx.x;
  const int lane = j & 31, warp = j >> 5;
  const bool isK = which == 0;
  const int bits = isK ? a.kb : a.vb;
  const int L = 1 << bits;
  const bool qjl = isK && a.qjl;
  const InT* src = reinterpret_cast<const InT*>(isK ? a.k : a.v);

  __syncthreads();  // previous users of xT / codes / sbits are done
  const int64_t base = (int64_t)b * a.sb + (int64_t)h * a.sh + (int64_t)t0 * a.st;
#pragma unroll 4
  for (int v = 0; v < TILE; ++v)
    s.xT[j][v] = v < nt ? to_f32<InT>(src[base + (int64_t)v * a.st + j]) : 0.0f;
  if (j < L) s.cent[j] = (isK ? a.kc : a.vc)[j];
  if (j < L - 1) s.thr[j] = (isK ? a.kt : a.vt)[j];
  if (j < TILE) s.flag[j] = 0;
  __syncthreads();

  // ||x|| in fp64: the squares of bf16/fp32 values and their sum are exact or nearly so.
#pragma unroll
  for (int vv = 0; vv < 4; ++vv) {
    const int v = warp * 4 + vv;
    double acc = 0.0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const double x = (double)s.xT[lane + 32 * q][v];
      acc = fma(x, x, acc);
    }
    acc = warp_sum_d(acc);
    if (lane == 0) s.nrm[v] = sqrt(acc);
  }
  __syncthreads();

  // y_j = sum_k Pi[j][k] x_k for the 16 tile vectors (fp32).
  float acc[TILE];
#pragma unroll
  for (int v = 0; v < TILE; ++v) acc[v] = 0.0f;
#pragma unroll 4
  for (int k = 0; k < D; ++k) {
    const float p = s.PiT[k][j];
    const float4* xr = reinterpret_cast<const float4*>(&s.xT[k][0]);
#pragma unroll
    for (int q = 0; q < TILE / 4; ++q) {
      const float4 x4 = xr[q];
      acc[4 * q + 0] = fmaf(p, x4.x, acc[4 * q + 0]);
      acc[4 * q + 1] = fmaf(p, x4.y, acc[4 * q + 1]);
      acc[4 * q + 2] = fmaf(p, x4.z, acc[4 * q + 2]);
      acc[4 * q + 3] = fmaf(p, x4.w, acc[4 * q + 3]);
    }
  }

  const int slot = isK ? k_slot_of_coord(j) : v_slot_of_coord(j);
  float rho2[TILE];
#pragma unroll
  for (int v = 0; v < TILE; ++v) {
    const double n = s.nrm[v];
    const float scl = n > 0.0 ? (float)(sqrt((double)D) / n) : 0.0f;
    const float u = acc[v] * scl;
    float margin;
    int idx = code_of(u, s.thr, L - 1, margin);
    float rho;
    if (margin < kGuardCode && n > 0.0) {
      const double ud = exact_u(s, j, v, n);
      idx = code_of_d(ud, s.thr, L - 1);
      rho = (float)(ud - (double)s.cent[idx]);
    } else {
      rho = u - s.cent[idx];
    }
    s.codes[v][slot] = (uint8_t)idx;
    s.rhoT[j][v] = rho;
    rho2[v] = rho * rho;
  }

  if (qjl) {
#pragma unroll
    for (int v = 0; v < TILE; ++v) {
      const float r = warp_sum_f(rho2[v]);
      if (lane == 0) s.red[v][warp] = r;
    }
    __syncthreads();
    // (S rho)_l for row l = j
    float sp[TILE];
#pragma unroll
    for (int v = 0; v < TILE; ++v) sp[v] = 0.0f;
#pragma unroll 4
    for (int jj = 0; jj < D; ++jj) {
      const float sv = s.ST[jj][j];
      const float4* rr = reinterpret_cast<const float4*>(&s.rhoT[jj][0]);
#pragma unroll
      for (int q = 0; q < TILE / 4; ++q) {
        const float4 r4 = rr[q];
        sp[4 * q + 0] = fmaf(sv, r4.x, sp[4 * q + 0]);
        sp[4 * q + 1] = fmaf(sv, r4.y, sp[4 * q + 1]);
        sp[4 * q + 2] = fmaf(sv, r4.z, sp[4 * q + 2]);
        sp[4 * q + 3] = fmaf(sv, r4.w, sp[4 * q + 3]);
      }
    }
    const int sbit = sign_bit_of_row(j);
#pragma unroll
    for (int v = 0; v < TILE; ++v) {
      s.sbits[v][sbit] = sp[v] >= 0.0f ? 1 : 0;
      if (fabsf(sp[v]) < kGuardSign && v < nt) s.flag[v] = 1;
    }
    __syncthreads();
    float rnorm_fast = 0.0f;
    if (j < TILE) {
      const float r2 = s.red[j][0] + s.red[j][1] + s.red[j][2] + s.red[j][3];
      rnorm_fast = (float)(s.nrm[j] * sqrt((double)r2) / sqrt((double)D));
    }
    // Vectors with a near-zero sketch value: redo the whole vector in fp64.
    for (int v = 0; v < nt; ++v) {
      if (!s.flag[v]) continue;  // uniform: flag read after a barrier
      const double n = s.nrm[v];
      double r = 0.0;
      if (n > 0.0) {
        const double ud = exact_u(s, j, v, n);
        const int idx = code_of_d(ud, s.thr, L - 1);
        r = ud - (double)s.cent[idx];
        s.codes[v][slot] = (uint8_t)idx;
      } else {
        r = -(double)s.cent[s.codes[v][slot]];
      }
      s.rho64[j] = r;
      const double r2 = warp_sum_d(r * r);
      if (lane == 0) s.red64[warp] = r2;
      __syncthreads();
      double spd0 = 0.0, spd1 = 0.0;
      for (int jj = 0; jj < D; jj += 2) {
        spd0 = fma((double)s.ST[jj][j], s.rho64[jj], spd0);
        spd1 = fma((double)s.ST[jj + 1][j], s.rho64[jj + 1], spd1);
      }
      s.sbits[v][sbit] = (spd0 + spd1) >= 0.0 ? 1 : 0;
      if (j == v) {
        const double rr = s.red64[0] + s.red64[1] + s.red64[2] + s.red64[3];
        rnorm_fast = (float)(n * sqrt(rr) / sqrt((double)D));
      }
      __syncthreads();
    }
    if (j < nt) {
      const int64_t row = ((int64_t)b * a.Hkv + h) * a.T_cap + a.t_offset + t0 + j;
      a.k_rnorm[row] = rnorm_fast;
    }
  }
  __syncthreads();

  // Pack code rows (little-endian bit stream, slot s at bits [bits*s, bits*s + bits)).
  const int wpr = 4 * bits;  // 32-bit words per row
  uint8_t* dst = isK ? a.k_codes : a.v_codes;
  for (int w = j; w < nt * wpr; w += THREADS) {
    const int v = w / wpr, ww = w % wpr;
    uint32_t word = 0;
    for (int kk = 0; kk < 32; ++kk) {
      const int P = 32 * ww + kk;
      word |= (uint32_t)((s.codes[v][P / bits] >> (P % bits)) & 1) << kk;
    }
    const int64_t row = ((int64_t)b * a.Hkv + h) * a.T_cap + a.t_offset + t0 + v;
    reinterpret_cast<uint32_t*>(dst + row * (16 * bits))[ww] = word;
  }
  if (qjl) {
    for (int w = j; w < nt * 4; w += THREADS) {
      const int v = w / 4, ww = w % 4;
      uint32_t word = 0;
      for (int kk = 0; kk < 32; ++kk) word |= (uint32_t)s.sbits[v][32 * ww + kk] << kk;
      const int64_t row = ((int64_t)b * a.Hkv + h) * a.T_cap + a.t_offset + t0 + v;
      reinterpret_cast<uint32_t*>(a.k_signs + row * 16)[ww] = word;
    }
  }
  if (j < nt) {
    const int64_t row = ((int64_t)b * a.Hkv + h) * a.T_cap + a.t_offset + t0 + j;
    (isK ? a.k_norm : a.v_norm)[row] = (float)s.nrm[j];
  }
}

template <typename InT>
__global__ void __launch_bounds__(THREADS, 1) quantize_kernel(QArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw);
  const int tid = threadIdx.x;
  for (int i = tid; i < D * D; i += THREADS) {
    const int r = i / D, c = i % D;
    s.PiT[c][r] = a.Pi[i];
    if (a.qjl) s.ST[c][r] = a.S[i];
  }
  const int tiles_per_bh = (a.T_new + TILE - 1) / TILE;
  const int64_t total = (int64_t)a.B * a.Hkv * tiles_per_bh;
  for (int64_t tile = blockIdx.x; tile < total; tile += gridDim.x) {
    const int bh = (int)(tile / tiles_per_bh);
    const int t0 = (int)(tile % tiles_per_bh) * TILE;
    const int nt = min(TILE, a.T_new - t0);
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    quantize_side<InT>(s, a, 0, b, h, t0, nt);
    quantize_side<InT>(s, a, 1, b, h, t0, nt);
  }
}

template <typename InT>
tq_status launch(const QArgs& a, cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "device query: %s", cudaGetErrorString(e));
  const size_t smem = sizeof(Smem);
  e = cudaFuncSetAttribute(quantize_kernel<InT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "smem attribute: %s", cudaGetErrorString(e));
  const int tiles_per_bh = (a.T_new + TILE - 1) / TILE;
  const int64_t total = (int64_t)a.B * a.Hkv * tiles_per_bh;
  const int grid = (int)(total < sms ? total : sms);
  quantize_kernel<InT><<<grid, THREADS, smem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "quantize launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}

}  // namespace
}  // namespace tq

extern "C" tq_status tq_quantize(const tq_params* params, const void* k, const void* v, int dtype,
                                 int64_t stride_b, int64_t stride_h, int64_t stride_t, int T_new,
                                 int t_offset, const tq_cache* cache, void* stream) {
  using namespace tq;
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
  a.kb = cache->k_bits;
  a.vb = cache->v_bits;
  a.qjl = cache->qjl_m ? 1 : 0;
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
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return dtype == TQ_F32 ? launch<float>(a, s) : launch<__nv_bfloat16>(a, s);
}
