// tq_decode_attn: single-token decode attention directly over the packed cache.
//
// Scores follow the QJL-corrected inner-product estimator,
//   est_i = <q', khat'_i> + ||r_i|| sqrt(pi/2)/m <S q', 2 sign_i - 1>,  q' = Pi q,
// with khat'_i = (n_i / sqrt(d)) c_K[idx_i] in the rotated basis (ai-news.ru overview, first and
// second ideas plus the third, QJL, component; tproger.ru "Step 1: PolarQuant", "Step 2: QJL").
// Softmax and the value sum also run in the rotated basis; one final o = Pi^T o' per head.
//
// Kernels (all on the caller's stream; split and merge are programmatic dependent launches):
//   prep    q' = Pi q and sq = S q' per (batch, query head), fp32, into the workspace: clusters of
//           eight CTAs, each CTA holding 16 rows of Pi and S for a batch of up to 16 heads.
//   split   grid (splits, Hkv * head_groups, B).  A 4-warp CTA streams its token range through a
//           4-stage cp.async pipeline (64 tokens per stage).  Each warp takes 16 tokens per stage:
//           codes are turned into fp16 pairs by a lane-replicated shared-memory table (one load per
//           two coordinates, no bank conflicts), and m16n8k16 tensor-core MMAs compute q'.khat,
//           the QJL sign dot (q' and S q' split into fp16 hi + lo rows; signs -> +-0.5 by one
//           half2 FMA) and P.vhat (P split into hi + lo rows).  Online softmax runs in log2 units.
//           The CTA merges its warps and writes one (max, sum, o'[128]) partial per head.
//   merge   one CTA per (batch, query head), a programmatic dependent of split: log-sum-exp
//           merge of the head's split partials, then o = Pi^T o'.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr int D = kHeadDim;
// CTA shape per code widths.  With 4-bit keys and values the pair tables take 64 KB, so two CTAs
// share an SM: six warps and three stages each (12 warps per SM).  Smaller tables leave room for
// three four-warp CTAs with four stages (register-bound).
template <int KB, int VB>
struct Cfg {
  static constexpr bool kPacked = KB == 4 && VB == 4;
  static constexpr int W = kPacked ? 6 : 4;
  static constexpr int THREADS = 32 * W;
  static constexpr int STAGE_TOK = 16 * W;  // 16 tokens per warp per stage
  static constexpr int NSTAGE = kPacked ? 3 : 4;
  static constexpr int MIN_BLOCKS = kPacked ? 2 : 3;
};
inline int stage_tokens(int kb, int vb) { return (kb == 4 && vb == 4) ? 96 : 64; }
constexpr int HG = 8;                  // query heads per MMA row block (hi rows 0-7, lo rows 8-15)
constexpr int PART = 4 + D;            // (max, sum, pad, pad, o'[128]) per partial: o' 16-byte aligned
constexpr int SPLITS_MAX = 512;        // CTAs per (batch, kv-head, head group)
constexpr unsigned FULL = 0xffffffffu;

struct DArgs {
  int B, Hq, Hkv, g, hgroups, T_cap, seq_len, splits, tps;
  float sK;   // scale*log2e/sqrt(d)                     (times n_i)
  float sQ;   // scale*log2e*2*sqrt(pi/2)/m              (times ||r_i||; 2 undoes the +-0.5 signs)
  const uint8_t* k_codes;
  const uint8_t* k_signs;
  const float* k_norm;
  const float* k_rnorm;
  const uint8_t* v_codes;
  const float* v_norm;
  const float* kc;
  const float* vc;
  const float* qrot;
  const float* sq;
  float* part;
};

// ------------------------------------------------------------------------------------------ PTX

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// 16-byte async copy; src_bytes < 16 zero-fills the rest (src_bytes = 0: no global read).
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __halves2half2(__float2half_rn(lo), __float2half_rn(hi));
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Split x into fp16 hi + lo with x ~= hi + lo (about 22 significant bits).
__device__ __forceinline__ void split_half(float x, float& hi, float& lo) {
  hi = __half2float(__float2half_rn(x));
  lo = x - hi;
}

// Sign bits -> +-0.5 fp16 pair: bits q and q+16 of w (1 <= q <= 9) placed in the mantissa of 1.0
// (fp16 0x3C00: mantissa bits 0-9 are zero, bit 10 is already an exponent bit), then one exact
// half2 FMA maps 1 + b*2^(q-10) to b - 0.5.
template <int Q>
__device__ __forceinline__ uint32_t sign_half2(uint32_t w) {
  static_assert(Q >= 1 && Q <= 9, "mantissa position");
  const uint32_t x = (w & (0x00010001u << Q)) | 0x3C003C00u;
  const __half2 hx = *reinterpret_cast<const __half2*>(&x);
  const float m = (float)(1 << (10 - Q));
  const __half2 r = __hfma2(hx, __float2half2_rn(m), __float2half2_rn(-(m + 0.5f)));
  return *reinterpret_cast<const uint32_t*>(&r);
}
// Pair p of a thread's 32-bit sign word (bits p and p+16).
template <int P>
__device__ __forceinline__ uint32_t sign_pair(uint32_t w) {
  if constexpr (P == 0) return sign_half2<1>(w << 1);
  else if constexpr (P <= 9) return sign_half2<P>(w);
  else return sign_half2<P - 9>(w >> 9);
}

// Pair p (0..15) of a thread's key-code chunk: 2*KB bits starting at bit 2*KB*p.
template <int KB, int P>
__device__ __forceinline__ uint32_t k_pair_index(const uint32_t (&c)[KB]) {
  constexpr int off = 2 * KB * P;
  constexpr int w = off / 32, sh = off % 32;
  constexpr uint32_t mask = (1u << (2 * KB)) - 1u;
  if constexpr (KB == 4) {
    return __byte_perm(c[w], 0u, 0x4440u | (uint32_t)(sh / 8));  // byte sh/8, zero-extended
  } else if constexpr (sh + 2 * KB <= 32) {
    return (c[w] >> sh) & mask;
  } else {
    return __funnelshift_r(c[w], c[w + 1], sh) & mask;
  }
}

// Value-code pair indices of tokens a and b (one lane group's 16 codes each): index of code nu is
// code_a(nu) | code_b(nu) << VB.  For 4- and 2-bit codes the two chunks are interleaved field by
// field with a few logic operations, after which every index is one byte / nibble extract.
template <int VB>
struct VPairs {
  uint32_t w[VB == 3 ? 4 : 2 * (VB == 4 ? 2 : 1)];
  __device__ __forceinline__ void build(uint64_t ca, uint64_t cb) {
    if constexpr (VB == 4) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t a = (uint32_t)(h ? ca >> 32 : ca), b = (uint32_t)(h ? cb >> 32 : cb);
        w[2 * h + 0] = (a & 0x0F0F0F0Fu) | ((b << 4) & 0xF0F0F0F0u);   // nu = 8h + 2k
        w[2 * h + 1] = ((a >> 4) & 0x0F0F0F0Fu) | (b & 0xF0F0F0F0u);   // nu = 8h + 2k + 1
      }
    } else if constexpr (VB == 2) {
      const uint32_t a = (uint32_t)ca, b = (uint32_t)cb;
      w[0] = (a & 0x33333333u) | ((b << 2) & 0xCCCCCCCCu);   // nibble k: nu = 2k
      w[1] = ((a >> 2) & 0x33333333u) | (b & 0xCCCCCCCCu);   // nibble k: nu = 2k + 1
    } else {
      w[0] = (uint32_t)ca;
      w[1] = (uint32_t)(ca >> 32);
      w[2] = (uint32_t)cb;
      w[3] = (uint32_t)(cb >> 32);
    }
  }
  template <int NU>
  __device__ __forceinline__ uint32_t index() const {
    if constexpr (VB == 4) {
      return __byte_perm(w[2 * (NU >> 3) + (NU & 1)], 0u, 0x4440u | (uint32_t)((NU & 7) >> 1));
    } else if constexpr (VB == 2) {
      return (w[NU & 1] >> (4 * (NU >> 1))) & 0xFu;
    } else {
      const uint64_t ca = (uint64_t)w[0] | ((uint64_t)w[1] << 32);
      const uint64_t cb = (uint64_t)w[2] | ((uint64_t)w[3] << 32);
      return (uint32_t)((ca >> (3 * NU)) & 7u) | ((uint32_t)((cb >> (3 * NU)) & 7u) << 3);
    }
  }
};

// Value code nu (0..15) of a thread's 16-code value chunk held in a 64-bit integer.
template <int VB, int NU>
__device__ __forceinline__ uint32_t v_code(uint64_t c) {
  return (uint32_t)(c >> (VB * NU)) & ((1u << VB) - 1u);
}

// ------------------------------------------------------------------------------------------ prep

// Clusters of eight 128-thread CTAs; cluster k handles query heads hb*k .. hb*k + hb - 1 (flattened
// over the batch; hb <= 16 is chosen on the host so that there are enough clusters to spread the
// work) and CTA c of it rows 16c .. 16c+15 of q' = Pi q and of sq = S q', eight threads per row
// with 16 columns each.  Each CTA loads its rows of Pi and S once (one memory round trip,
// together with the query vectors) and reuses them for all its heads; the full q' of every head
// reaches the other CTAs of the cluster through distributed shared memory.  The split kernel is
// launched as a programmatic dependent of this one and starts its prologue early.
constexpr int PREP_CLUSTER = 8, PREP_THREADS = 128, PREP_ROWS = D / PREP_CLUSTER, PREP_HB = 16;

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
// Shared-memory float at the same offset as `p` in CTA `rank` of this cluster.
__device__ __forceinline__ float ld_cluster_f32(const float* p, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(remote) : "r"(smem_u32(p)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];\n" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

template <typename QT>
__global__ void __cluster_dims__(PREP_CLUSTER, 1, 1) __launch_bounds__(PREP_THREADS)
    prep_kernel(const QT* __restrict__ q, int BH, int hb, const float* __restrict__ Pi, const float* __restrict__ S,
                int qjl, float* __restrict__ qrot, float* __restrict__ sq) {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  __shared__ __align__(16) float qs[PREP_HB][D];           // query vectors, then q' of the cluster
  __shared__ __align__(16) float qpart[PREP_HB][PREP_ROWS];  // this CTA's rows of q'
  const int tid = threadIdx.x;
  const uint32_t c = blockIdx.x % PREP_CLUSTER;  // rank in the cluster (clusters are consecutive CTAs)
  const int h0 = (int)(blockIdx.x / PREP_CLUSTER) * hb;
  const int nhb = min(hb, BH - h0);
  const int rl = tid >> 3, part = tid & 7;
  const int row = PREP_ROWS * (int)c + rl;
  float4 p[4], s4[4];
  const float4* pr = reinterpret_cast<const float4*>(Pi + row * D + 16 * part);
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = pr[i];
  if (qjl) {
    const float4* sr = reinterpret_cast<const float4*>(S + row * D + 16 * part);
#pragma unroll
    for (int i = 0; i < 4; ++i) s4[i] = sr[i];
  }
  for (int h = 0; h < nhb; ++h) {
    if constexpr (sizeof(QT) == 4) qs[h][tid] = (float)q[(int64_t)(h0 + h) * D + tid];
    else qs[h][tid] = __bfloat162float(q[(int64_t)(h0 + h) * D + tid]);
  }
  __syncthreads();
  auto dot16 = [&](const float4 (&m)[4], const float* vec) {
    const float4* v4 = reinterpret_cast<const float4*>(vec + 16 * part);
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 x = v4[i];
      acc = fmaf(m[i].x, x.x, acc);
      acc = fmaf(m[i].y, x.y, acc);
      acc = fmaf(m[i].z, x.z, acc);
      acc = fmaf(m[i].w, x.w, acc);
    }
    acc += __shfl_xor_sync(FULL, acc, 1);
    acc += __shfl_xor_sync(FULL, acc, 2);
    acc += __shfl_xor_sync(FULL, acc, 4);
    return acc;
  };
  for (int h = 0; h < nhb; ++h) {
    const float v = dot16(p, qs[h]);
    if (part == 0) {
      qpart[h][rl] = v;
      qrot[(int64_t)(h0 + h) * D + row] = v;
    }
  }
  if (!qjl) return;  // uniform over the cluster: no CTA waits at the barriers below
  cluster_sync_all();
  for (int h = 0; h < nhb; ++h)
    qs[h][tid] = ld_cluster_f32(&qpart[h][tid % PREP_ROWS], (uint32_t)(tid / PREP_ROWS));
  cluster_sync_all();  // every remote read is done before any CTA of the cluster exits
  for (int h = 0; h < nhb; ++h) {
    const float w = dot16(s4, qs[h]);
    if (part == 0) sq[(int64_t)(h0 + h) * D + row] = w;
  }
}

// ------------------------------------------------------------------------------------------ split

template <int KB, int VB, bool QJL>
struct Layout {
  static constexpr int W = Cfg<KB, VB>::W;
  static constexpr int STAGE_TOK = Cfg<KB, VB>::STAGE_TOK;
  static constexpr int NSTAGE = Cfg<KB, VB>::NSTAGE;
  static constexpr int K_ROW = 16 * KB;
  static constexpr int V_ROW = 16 * VB;
  static constexpr bool kPackedLut = KB == 4 && VB == 4;
  static constexpr int OFF_KC = 0;
  static constexpr int OFF_SG = OFF_KC + STAGE_TOK * K_ROW;
  static constexpr int OFF_VC = OFF_SG + (QJL ? STAGE_TOK * 16 : 0);
  static constexpr int OFF_NK = OFF_VC + STAGE_TOK * V_ROW;
  static constexpr int OFF_RN = OFF_NK + STAGE_TOK * 4;
  static constexpr int OFF_NV = OFF_RN + (QJL ? STAGE_TOK * 4 : 0);
  static constexpr int STAGE_BYTES = OFF_NV + STAGE_TOK * 4;
  static constexpr int LUT_BYTES = kPackedLut ? 256 * 256 : ((1 << (2 * KB)) + (1 << (2 * VB))) * 128;
  // After the main loop the pipeline buffers hold the CTA's own warp merge.
  static constexpr int WARP_MERGE_BYTES = 4 * (W * HG * 2 + W * HG * D);
  static constexpr int PIPE_BYTES = NSTAGE * STAGE_BYTES;
  static constexpr int SMEM = LUT_BYTES + (PIPE_BYTES > WARP_MERGE_BYTES ? PIPE_BYTES : WARP_MERGE_BYTES);
  static_assert(STAGE_BYTES % 16 == 0, "stage alignment");
};

template <int KB, int VB, bool QJL>
__device__ __forceinline__ void load_stage(const DArgs& a, unsigned char* stage, int64_t row0,
                                           int count) {
  using Lay = Layout<KB, VB, QJL>;
  constexpr int THREADS = Cfg<KB, VB>::THREADS, STAGE_TOK = Cfg<KB, VB>::STAGE_TOK;
  const int tid = threadIdx.x;
  // key codes: KB 16-byte chunks per token
  {
    const uint8_t* src = a.k_codes + row0 * Lay::K_ROW;
    for (int i = tid; i < STAGE_TOK * KB; i += THREADS) {
      const bool ok = i < count * KB;
      cp_async16(stage + Lay::OFF_KC + 16 * i, ok ? src + 16 * i : a.k_codes, ok ? 16 : 0);
    }
  }
  if constexpr (QJL) {
    const uint8_t* src = a.k_signs + row0 * 16;
    for (int i = tid; i < STAGE_TOK; i += THREADS) {
      const bool ok = i < count;
      cp_async16(stage + Lay::OFF_SG + 16 * i, ok ? src + 16 * i : a.k_signs, ok ? 16 : 0);
    }
  }
  {
    const uint8_t* src = a.v_codes + row0 * Lay::V_ROW;
    for (int i = tid; i < STAGE_TOK * VB; i += THREADS) {
      const bool ok = i < count * VB;
      cp_async16(stage + Lay::OFF_VC + 16 * i, ok ? src + 16 * i : a.v_codes, ok ? 16 : 0);
    }
  }
  for (int i = tid; i < STAGE_TOK; i += THREADS) {
    const bool ok = i < count;
    cp_async4(stage + Lay::OFF_NK + 4 * i, ok ? a.k_norm + row0 + i : a.k_norm, ok ? 4 : 0);
    if constexpr (QJL)
      cp_async4(stage + Lay::OFF_RN + 4 * i, ok ? a.k_rnorm + row0 + i : a.k_rnorm, ok ? 4 : 0);
    cp_async4(stage + Lay::OFF_NV + 4 * i, ok ? a.v_norm + row0 + i : a.v_norm, ok ? 4 : 0);
  }
}

// Value chunk of one token for this lane group (16 codes of VB bits) as a 64-bit integer.
template <int VB>
__device__ __forceinline__ uint64_t load_v_chunk(const unsigned char* row, int gid) {
  if constexpr (VB == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(row + 8 * gid);
    return (uint64_t)w.x | ((uint64_t)w.y << 32);
  } else if constexpr (VB == 2) {
    return (uint64_t)*reinterpret_cast<const uint32_t*>(row + 4 * gid);
  } else {  // 6 bytes per lane group: read the aligned 12 bytes of the group pair
    const uint32_t* p = reinterpret_cast<const uint32_t*>(row + 12 * (gid >> 1));
    const uint32_t w0 = p[0], w1 = p[1], w2 = p[2];
    if (gid & 1) return (uint64_t)((w1 >> 16) | (w2 << 16)) | ((uint64_t)(w2 >> 16) << 32);
    return (uint64_t)w0 | ((uint64_t)(w1 & 0xffffu) << 32);
  }
}

// ------------------------------------------------------------------------------------------ merge

// One 512-thread CTA per (batch, query head), a programmatic dependent of the split kernel: it
// waits for the split grid, merges the head's split partials by log-sum-exp and writes
// o = Pi^T o'.  Thread (d, q), d = tid % 128 and q = tid / 128, sums the splits s = q (mod 4) of
// dimension d; the un-rotation gives thread (i, q) the rows 32q .. 32q + 31 of Pi.  Each phase
// issues its loads at once (one L2 round trip each).
constexpr int MERGE_THREADS = 4 * D;

__device__ __forceinline__ float block_reduce(float v, float* red, bool is_max) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float x = __shfl_xor_sync(FULL, v, o);
    v = is_max ? fmaxf(v, x) : v + x;
  }
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = red[lane < MERGE_THREADS / 32 ? lane : 0];
  if (lane >= MERGE_THREADS / 32) v = is_max ? -INFINITY : 0.0f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {  // every lane ends with the full result
    const float x = __shfl_xor_sync(FULL, v, o);
    v = is_max ? fmaxf(v, x) : v + x;
  }
  __syncthreads();  // red is reused by the next reduction
  return v;
}

// (The partials are written by the still-running split grid: they are read with ld.global.cg,
// through L2 only, never through the non-coherent read-only path.)
__global__ void __launch_bounds__(MERGE_THREADS) merge_kernel(const float* part,
                                                              const float* __restrict__ Pi,
                                                              float* __restrict__ out, int S) {
  extern __shared__ __align__(16) float msm[];  // [S] weights, [S] sums, [4][D] partial o', [D] o', [4][D]
  __shared__ float red[32];
  const int tid = threadIdx.x, d = tid % D, q = tid / D;
  // Pi is an input, not an output of split: its rows load while the split grid finishes
  float pj[32];
#pragma unroll
  for (int jj = 0; jj < 32; ++jj) pj[jj] = __ldg(Pi + (32 * q + jj) * D + d);
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  const int64_t bh = blockIdx.x;
  const float* p = part + bh * S * PART;
  float* wts = msm;
  float* ls = wts + S;
  float* osum = ls + ((S + 3) & ~3);
  float* ob = osum + 4 * D;
  float* rsum = ob + D;
  // phase 1: (max, sum) of every partial
  float m = -INFINITY;
  for (int s2 = tid; s2 < S; s2 += MERGE_THREADS) {
    const float2 ml = __ldcg(reinterpret_cast<const float2*>(p + (int64_t)s2 * PART));
    wts[s2] = ml.x;
    ls[s2] = ml.y;
    m = fmaxf(m, ml.x);
  }
  const float M = block_reduce(m, red, true);
  // phase 2: weights 2^(m_s - M) and L = sum_s w_s l_s
  float l = 0.0f;
  for (int s2 = tid; s2 < S; s2 += MERGE_THREADS) {
    const float ms = wts[s2];
    const float f = (ms == -INFINITY) ? 0.0f : ex2(ms - M);
    wts[s2] = f;
    l = fmaf(f, ls[s2], l);
  }
  const float L = block_reduce(l, red, false);  // also makes the weights visible
  // phase 3: thread (d, q) sums splits q, q + 4, ...
  float acc = 0.0f;
#pragma unroll 16
  for (int s2 = q; s2 < S; s2 += 4) acc = fmaf(wts[s2], __ldcg(p + (int64_t)s2 * PART + 4 + d), acc);
  osum[q * D + d] = acc;
  __syncthreads();
  if (tid < D) {
    const float o = osum[d] + osum[D + d] + osum[2 * D + d] + osum[3 * D + d];
    ob[d] = L > 0.0f ? o / L : 0.0f;
  }
  __syncthreads();
  // phase 4: o_i = sum_j Pi[j][i] o'_j, thread (i = d, q) over rows 32q .. 32q + 31
  float r = 0.0f;
#pragma unroll
  for (int jj = 0; jj < 32; ++jj) r = fmaf(pj[jj], ob[32 * q + jj], r);
  rsum[q * D + d] = r;
  __syncthreads();
  if (tid < D) out[bh * D + d] = rsum[d] + rsum[D + d] + rsum[2 * D + d] + rsum[3 * D + d];
}

inline size_t merge_smem_bytes(int S) { return sizeof(float) * ((size_t)S + ((S + 3) & ~3) + 9 * D); }

// Transpose an 8x8 matrix of 16-bit elements held one row pair per lane (m8n8 fragment layout).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// Pair-table lookups.  With 4-bit keys and values the K and V pair tables share 256-byte entry
// slots (K replicas at +0, V replicas at +128): one byte permute turns a code byte e and the lane
// offset into the byte address (e << 8) | 4 lane, so a pair costs one PRMT and one LDS.  Other bit
// widths use separate tables with 128-byte entries (lane-replicated, bank = lane).
template <int KB, int VB>
struct PairLut {
  static constexpr bool kPacked = KB == 4 && VB == 4;
  static constexpr int K_BYTES = kPacked ? 0 : (1 << (2 * KB)) * 128;
  static constexpr int V_BYTES = kPacked ? 0 : (1 << (2 * VB)) * 128;
  static constexpr int BYTES = kPacked ? 256 * 256 : K_BYTES + V_BYTES;
  uint32_t base;   // shared-window address of the tables
  uint32_t lane4;  // 4 * lane
  __device__ __forceinline__ static uint32_t lds(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(addr));
    return v;
  }
  __device__ __forceinline__ uint32_t k(uint32_t e) const { return lds(base + ((e << 7) | lane4)); }
  __device__ __forceinline__ uint32_t v(uint32_t e) const { return lds(base + K_BYTES + ((e << 7) | lane4)); }
  // byte `Bt` of word w as the pair index (packed layout only)
  template <int Bt>
  __device__ __forceinline__ uint32_t k_byte(uint32_t w) const {
    return lds(base + __byte_perm(w, lane4, 0x5504u | (Bt << 4)));
  }
  template <int Bt>
  __device__ __forceinline__ uint32_t v_byte(uint32_t w) const {
    return lds(base + 128 + __byte_perm(w, lane4, 0x5504u | (Bt << 4)));
  }
};

// Key pair P (0..15) of a thread's code chunk, as a half2 of centroids.
template <int KB, int VB, int P>
__device__ __forceinline__ uint32_t k_pair(const PairLut<KB, VB>& L, const uint32_t (&c)[KB]) {
  if constexpr (PairLut<KB, VB>::kPacked) {
    return L.template k_byte<P & 3>(c[P >> 2]);
  } else {
    return L.k(k_pair_index<KB, P>(c));
  }
}
// Value pair NU of a token pair, as a half2 of centroids.
template <int KB, int VB, int NU>
__device__ __forceinline__ uint32_t v_pair(const PairLut<KB, VB>& L, const VPairs<VB>& p) {
  if constexpr (PairLut<KB, VB>::kPacked) {
    return L.template v_byte<((NU & 7) >> 1)>(p.w[2 * (NU >> 3) + (NU & 1)]);
  } else {
    return L.v(p.template index<NU>());
  }
}

// Split-K decode over one token range.  Transposed MMAs: tokens are the M dimension and the
// columns are (head, part) pairs, part 0 = fp16 hi and part 1 = fp16 lo of the query-side operand,
// so one m16n8k16 covers 16 tokens of four heads:
//   scores   D[tok x (h,p)] += Khat[tok x dim] . Q'[dim x (h,p)]        (A from the pair tables)
//   QJL      D[tok x (h,p)] += sign[tok x row] . SQ'[row x (h,p)]        (A = +-0.5 from the bits)
//   values   O'[dim x (h,p)] += Vhat^T[dim x tok] . P~[tok x (h,p)]      (B = P~ transposed in
//                                                                          registers by movmatrix)
// NB = 1 (up to 4 heads per kv-head) or 2 (up to 8): n-blocks of four heads share the A operands.
template <int KB, int VB, bool QJL, int NB>
__global__ void __launch_bounds__(Cfg<KB, VB>::THREADS, Cfg<KB, VB>::MIN_BLOCKS) split_kernel(DArgs a) {
  using Lay = Layout<KB, VB, QJL>;
  using Lut = PairLut<KB, VB>;
  constexpr int THREADS = Cfg<KB, VB>::THREADS, STAGE_TOK = Cfg<KB, VB>::STAGE_TOK;
  constexpr int NSTAGE = Cfg<KB, VB>::NSTAGE, WARPS = Cfg<KB, VB>::W;
  static_assert(Lay::LUT_BYTES == Lut::BYTES && Lut::K_BYTES + Lut::V_BYTES <= Lut::BYTES, "pair tables");
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned char* pipe = smem + Lay::LUT_BYTES;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, t = lane & 3;
  const int split = blockIdx.x;
  const int kvh = blockIdx.y / a.hgroups, hg = blockIdx.y % a.hgroups;
  const int b = blockIdx.z;
  const int h0 = kvh * a.g + hg * HG;
  const int nh = min(HG, a.g - hg * HG);
  const int tok_begin = split * a.tps;
  const int tok_end = min(a.seq_len, tok_begin + a.tps);
  const int ntok = max(0, tok_end - tok_begin);
  const int nstages = (ntok + STAGE_TOK - 1) / STAGE_TOK;
  const int64_t row_base = ((int64_t)b * a.Hkv + kvh) * a.T_cap;

  // Start the pipeline before building the tables.
#pragma unroll
  for (int s = 0; s < NSTAGE - 1; ++s) {
    if (s < nstages)
      load_stage<KB, VB, QJL>(a, pipe + s * Lay::STAGE_BYTES, row_base + tok_begin + s * STAGE_TOK,
                              min(STAGE_TOK, ntok - s * STAGE_TOK));
    cp_commit();
  }

  // Pair tables: entry e = lo | hi << B  ->  half2(c[lo], c[hi]), replicated per lane (bank = lane).
  if constexpr (Lut::kPacked) {
    for (int i = tid; i < 256 * 64; i += THREADS) {
      const int e = i >> 6, half = (i >> 5) & 1, ln = i & 31;
      const float* c = half ? a.vc : a.kc;
      *reinterpret_cast<uint32_t*>(smem + e * 256 + half * 128 + 4 * ln) = pack_half2(c[e & 15], c[e >> 4]);
    }
  } else {
    for (int i = tid; i < Lut::K_BYTES / 4; i += THREADS) {
      const int e = i >> 5;
      reinterpret_cast<uint32_t*>(smem)[i] = pack_half2(a.kc[e & ((1 << KB) - 1)], a.kc[e >> KB]);
    }
    for (int i = tid; i < Lut::V_BYTES / 4; i += THREADS) {
      const int e = i >> 5;
      reinterpret_cast<uint32_t*>(smem + Lut::K_BYTES)[i] = pack_half2(a.vc[e & ((1 << VB) - 1)], a.vc[e >> VB]);
    }
  }
  Lut L;
  L.base = smem_u32(smem);
  L.lane4 = 4u * (uint32_t)lane;

  // Everything above reads only the cache; the rotated queries come from the prep kernel.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  // the merge kernel may launch now; its CTAs wait for this grid to finish before reading
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  // B operands: column gq of n-block nb = head 4 nb + gq/2, part gq%2 (0: fp16 hi, 1: fp16 lo);
  // k-step kk: dims 16kk + 2t, +1 (reg 0) and 16kk + 8 + 2t, +1 (reg 1).
  uint32_t bq[NB][8][2], bsq[NB][8][2];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int hh = 4 * nb + (gq >> 1);
    const bool live = hh < nh;
    const bool lo = gq & 1;
    const float* qp = a.qrot + ((int64_t)b * a.Hq + h0 + (live ? hh : 0)) * D;
    const float* sp = a.sq + ((int64_t)b * a.Hq + h0 + (live ? hh : 0)) * D;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int c0 = 16 * kk + 8 * r + 2 * t;
        float hx, lx, hy, ly;
        split_half(live ? qp[c0] : 0.0f, hx, lx);
        split_half(live ? qp[c0 + 1] : 0.0f, hy, ly);
        bq[nb][kk][r] = lo ? pack_half2(lx, ly) : pack_half2(hx, hy);
        if constexpr (QJL) {
          split_half(live ? sp[c0] : 0.0f, hx, lx);
          split_half(live ? sp[c0 + 1] : 0.0f, hy, ly);
          bsq[nb][kk][r] = lo ? pack_half2(lx, ly) : pack_half2(hx, hy);
        } else {
          bsq[nb][kk][r] = 0u;
        }
      }
    }
  }

  // Output accumulators: n-block nb, dim block db: (dim 16db + gq, head 4nb + t) hi/lo in [0]/[1],
  // (dim 16db + 8 + gq) in [2]/[3].
  float oacc[NB][8][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int i = 0; i < 8; ++i) oacc[nb][i][0] = oacc[nb][i][1] = oacc[nb][i][2] = oacc[nb][i][3] = 0.0f;
  float m_run[NB], l_run[NB];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    m_run[nb] = -INFINITY;
    l_run[nb] = 0.0f;
  }

  for (int st = 0; st < nstages; ++st) {
    cp_wait<NSTAGE - 2>();
    __syncthreads();
    {
      const int s = st + NSTAGE - 1;
      if (s < nstages)
        load_stage<KB, VB, QJL>(a, pipe + (s % NSTAGE) * Lay::STAGE_BYTES,
                                row_base + tok_begin + s * STAGE_TOK,
                                min(STAGE_TOK, ntok - s * STAGE_TOK));
      cp_commit();
    }
    const int wtok0 = st * STAGE_TOK + 16 * warp;  // first token of this warp, relative to range
    if (wtok0 >= ntok) continue;                    // warp-uniform
    const unsigned char* stage = pipe + (st % NSTAGE) * Lay::STAGE_BYTES;
    const int r0 = 16 * warp + gq, r1 = r0 + 8;    // this lane's token rows in the stage

    // ---- scores for tokens r0, r1 and heads 4nb + t ----
    float kacc[NB][4], qacc[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) kacc[nb][e] = qacc[nb][e] = 0.0f;
    {
      uint32_t c0[KB], c1[KB];
      const uint32_t* k0 = reinterpret_cast<const uint32_t*>(stage + Lay::OFF_KC + r0 * Lay::K_ROW + 4 * KB * t);
      const uint32_t* k1 = reinterpret_cast<const uint32_t*>(stage + Lay::OFF_KC + r1 * Lay::K_ROW + 4 * KB * t);
#pragma unroll
      for (int i = 0; i < KB; ++i) {
        c0[i] = k0[i];
        c1[i] = k1[i];
      }
#define TQ_KSTEP(KK)                                                                         \
      {                                                                                      \
        const uint32_t A[4] = {k_pair<KB, VB, 2 * (KK)>(L, c0), k_pair<KB, VB, 2 * (KK)>(L, c1), \
                               k_pair<KB, VB, 2 * (KK) + 1>(L, c0),                          \
                               k_pair<KB, VB, 2 * (KK) + 1>(L, c1)};                         \
        _Pragma("unroll") for (int nb = 0; nb < NB; ++nb)                                    \
            mma16816(kacc[nb], A, bq[nb][KK][0], bq[nb][KK][1]);                              \
      }
      TQ_KSTEP(0) TQ_KSTEP(1) TQ_KSTEP(2) TQ_KSTEP(3) TQ_KSTEP(4) TQ_KSTEP(5) TQ_KSTEP(6) TQ_KSTEP(7)
#undef TQ_KSTEP
    }
    if constexpr (QJL) {
      const uint32_t s0 = *reinterpret_cast<const uint32_t*>(stage + Lay::OFF_SG + r0 * 16 + 4 * t);
      const uint32_t s1 = *reinterpret_cast<const uint32_t*>(stage + Lay::OFF_SG + r1 * 16 + 4 * t);
#define TQ_SSTEP(KK)                                                                         \
      {                                                                                      \
        const uint32_t A[4] = {sign_pair<2 * (KK)>(s0), sign_pair<2 * (KK)>(s1),             \
                               sign_pair<2 * (KK) + 1>(s0), sign_pair<2 * (KK) + 1>(s1)};    \
        _Pragma("unroll") for (int nb = 0; nb < NB; ++nb)                                    \
            mma16816(qacc[nb], A, bsq[nb][KK][0], bsq[nb][KK][1]);                            \
      }
      TQ_SSTEP(0) TQ_SSTEP(1) TQ_SSTEP(2) TQ_SSTEP(3) TQ_SSTEP(4) TQ_SSTEP(5) TQ_SSTEP(6) TQ_SSTEP(7)
#undef TQ_SSTEP
    }

    // ---- online softmax (log2 units) per head 4nb + t over this warp's 16 tokens ----
    const float nk0 = *reinterpret_cast<const float*>(stage + Lay::OFF_NK + 4 * r0);
    const float nk1 = *reinterpret_cast<const float*>(stage + Lay::OFF_NK + 4 * r1);
    float rn0 = 0.0f, rn1 = 0.0f;
    if constexpr (QJL) {
      rn0 = *reinterpret_cast<const float*>(stage + Lay::OFF_RN + 4 * r0);
      rn1 = *reinterpret_cast<const float*>(stage + Lay::OFF_RN + 4 * r1);
    }
    const float nv0 = *reinterpret_cast<const float*>(stage + Lay::OFF_NV + 4 * r0) * 0.08838834764831845f;
    const float nv1 = *reinterpret_cast<const float*>(stage + Lay::OFF_NV + 4 * r1) * 0.08838834764831845f;
    const bool v0ok = wtok0 + gq < ntok, v1ok = wtok0 + 8 + gq < ntok;
    uint32_t bp[NB][2];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      float s0 = (kacc[nb][0] + kacc[nb][1]) * (nk0 * a.sK);
      float s1 = (kacc[nb][2] + kacc[nb][3]) * (nk1 * a.sK);
      if constexpr (QJL) {
        s0 = fmaf(qacc[nb][0] + qacc[nb][1], rn0 * a.sQ, s0);
        s1 = fmaf(qacc[nb][2] + qacc[nb][3], rn1 * a.sQ, s1);
      }
      s0 = v0ok ? s0 : -INFINITY;
      s1 = v1ok ? s1 : -INFINITY;
      float mx = fmaxf(s0, s1);
      mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 16));
      const float m_new = fmaxf(m_run[nb], mx);
      if (m_new > m_run[nb]) {  // uniform over the 8 lanes of head 4nb + t
        const float alpha = ex2(m_run[nb] - m_new);  // ex2(-inf) = 0
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          oacc[nb][i][0] *= alpha;
          oacc[nb][i][1] *= alpha;
          oacc[nb][i][2] *= alpha;
          oacc[nb][i][3] *= alpha;
        }
        l_run[nb] *= alpha;
        m_run[nb] = m_new;
      }
      const float p0 = m_run[nb] == -INFINITY ? 0.0f : ex2(s0 - m_run[nb]);
      const float p1 = m_run[nb] == -INFINITY ? 0.0f : ex2(s1 - m_run[nb]);
      l_run[nb] += p0 + p1;
      // P~ = p nV / sqrt(d) as fp16 hi + lo: row token, columns (head t, hi) and (head t, lo)
      float hx, lx, hy, ly;
      split_half(p0 * nv0, hx, lx);
      split_half(p1 * nv1, hy, ly);
      bp[nb][0] = movmatrix_trans(pack_half2(hx, lx));  // tokens 2t, 2t+1 of column gq
      bp[nb][1] = movmatrix_trans(pack_half2(hy, ly));  // tokens 2t+8, 2t+9
    }

    // ---- O'^T += Vhat^T P~: dim blocks of 16; A holds token pairs (2t,2t+1), (2t+8,2t+9) ----
    {
      const unsigned char* vbase = stage + Lay::OFF_VC + (16 * warp) * Lay::V_ROW;
      const uint64_t cv0 = load_v_chunk<VB>(vbase + (2 * t) * Lay::V_ROW, gq);
      const uint64_t cv1 = load_v_chunk<VB>(vbase + (2 * t + 1) * Lay::V_ROW, gq);
      const uint64_t cv2 = load_v_chunk<VB>(vbase + (2 * t + 8) * Lay::V_ROW, gq);
      const uint64_t cv3 = load_v_chunk<VB>(vbase + (2 * t + 9) * Lay::V_ROW, gq);
      VPairs<VB> p01, p89;
      p01.build(cv0, cv1);
      p89.build(cv2, cv3);
#define TQ_VSTEP(DB)                                                                          \
      {                                                                                       \
        const uint32_t A[4] = {v_pair<KB, VB, 2 * (DB)>(L, p01), v_pair<KB, VB, 2 * (DB) + 1>(L, p01), \
                               v_pair<KB, VB, 2 * (DB)>(L, p89), v_pair<KB, VB, 2 * (DB) + 1>(L, p89)}; \
        _Pragma("unroll") for (int nb = 0; nb < NB; ++nb)                                     \
            mma16816(oacc[nb][DB], A, bp[nb][0], bp[nb][1]);                                   \
      }
      TQ_VSTEP(0) TQ_VSTEP(1) TQ_VSTEP(2) TQ_VSTEP(3) TQ_VSTEP(4) TQ_VSTEP(5) TQ_VSTEP(6) TQ_VSTEP(7)
#undef TQ_VSTEP
    }
  }
  cp_wait<0>();
  __syncthreads();  // pipeline buffers are reused for the merge below

  // ---- merge the 4 warps of this CTA ----
  float* mw = reinterpret_cast<float*>(pipe);  // [WARPS][HG]
  float* lw = mw + WARPS * HG;                 // [WARPS][HG]
  float* ow = lw + WARPS * HG;                 // [WARPS][HG][D]
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int hh = 4 * nb + t;
    float lq = l_run[nb];
    lq += __shfl_xor_sync(FULL, lq, 4);
    lq += __shfl_xor_sync(FULL, lq, 8);
    lq += __shfl_xor_sync(FULL, lq, 16);
    if (gq == 0) {
      mw[warp * HG + hh] = m_run[nb];
      lw[warp * HG + hh] = lq;
    }
    float* o = ow + (warp * HG + hh) * D;
#pragma unroll
    for (int db = 0; db < 8; ++db) {
      o[16 * db + gq] = oacc[nb][db][0] + oacc[nb][db][1];
      o[16 * db + 8 + gq] = oacc[nb][db][2] + oacc[nb][db][3];
    }
  }
  __syncthreads();
  for (int r = 0; r < nh && tid < D; ++r) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) M = fmaxf(M, mw[w * HG + r]);
    float Ls = 0.0f, O = 0.0f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      const float mwr = mw[w * HG + r];
      const float f = (mwr == -INFINITY) ? 0.0f : ex2(mwr - M);
      Ls += f * lw[w * HG + r];
      O += f * ow[(w * HG + r) * D + tid];
    }
    float* dst = a.part + (((int64_t)b * a.Hq + h0 + r) * a.splits + split) * PART;
    dst[4 + tid] = O;
    if (tid == 0) {
      dst[0] = M;
      dst[1] = Ls;
    }
  }

}

// ------------------------------------------------------------------------------------------ host

struct Plan {
  int hgroups, splits, tps;
};

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;
  }
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
    cudaGetLastError();
    return 148;
  }
  return sms;
}

// Resident split CTAs per SM: the 4-bit pair tables (64 KB) allow two, the smaller ones three
// (register-bound, see split_kernel's launch bounds).
int resident_ctas(int kb, int vb) { return (kb == 4 && vb == 4) ? 2 : 3; }
// (two six-warp CTAs with the 4-bit tables, three four-warp CTAs otherwise)

Plan make_plan(int B, int Hq, int Hkv, int seq_len, int sms, int resident, int stage_tok) {
  const int STAGE_TOK = stage_tok;
  Plan p;
  const int g = Hq / Hkv;
  p.hgroups = (g + HG - 1) / HG;
  const int64_t units = (int64_t)B * Hkv * p.hgroups;
  if (seq_len <= 0) {
    p.splits = 1;
    p.tps = STAGE_TOK;
    return p;
  }
  // One wave of resident CTAs: the largest split count whose grid still fits it.
  const int64_t slots = (int64_t)resident * sms;
  int64_t splits = slots / units;
  const int64_t max_splits = (seq_len + 4 * STAGE_TOK - 1) / (4 * STAGE_TOK);  // >= 4 stages each
  if (splits > max_splits) splits = max_splits;
  if (splits > SPLITS_MAX) splits = SPLITS_MAX;
  if (splits < 1) splits = 1;
  int64_t tps = (seq_len + splits - 1) / splits;
  tps = (tps + STAGE_TOK - 1) / STAGE_TOK * STAGE_TOK;
  p.tps = (int)tps;
  p.splits = (int)((seq_len + tps - 1) / tps);
  return p;
}

// Workspace: q' and S q' [B*Hq][128] fp32, then the split partials [B*Hq][splits][132] fp32.
size_t workspace_bytes(int B, int Hq, int Hkv, const Plan& p) {
  (void)Hkv;
  return sizeof(float) * ((size_t)2 * B * Hq * D + (size_t)B * Hq * p.splits * PART);
}

template <int KB, int VB, bool QJL, int NB>
tq_status launch_split_nb(const DArgs& a, dim3 grid, cudaStream_t stream) {
  using Lay = Layout<KB, VB, QJL>;
  cudaError_t e = cudaFuncSetAttribute(split_kernel<KB, VB, QJL, NB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::SMEM);
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "smem attribute: %s", cudaGetErrorString(e));
  // programmatic dependent launch: the prologue (tables, first cache stages) overlaps prep
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(Cfg<KB, VB>::THREADS);
  cfg.dynamicSmemBytes = Lay::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, split_kernel<KB, VB, QJL, NB>, a);
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "split launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}

// One n-block of four heads when a group has at most four query heads, else two.
template <int KB, int VB, bool QJL>
tq_status launch_split(const DArgs& a, dim3 grid, cudaStream_t stream) {
  return a.g <= 4 ? launch_split_nb<KB, VB, QJL, 1>(a, grid, stream) : launch_split_nb<KB, VB, QJL, 2>(a, grid, stream);
}

template <int KB, bool QJL>
tq_status dispatch_v(int vb, const DArgs& a, dim3 grid, cudaStream_t s) {
  switch (vb) {
    case 2: return launch_split<KB, 2, QJL>(a, grid, s);
    case 3: return launch_split<KB, 3, QJL>(a, grid, s);
    default: return launch_split<KB, 4, QJL>(a, grid, s);
  }
}

template <bool QJL>
tq_status dispatch(int kb, int vb, const DArgs& a, dim3 grid, cudaStream_t s) {
  switch (kb) {
    case 2: return dispatch_v<2, QJL>(vb, a, grid, s);
    case 3: return dispatch_v<3, QJL>(vb, a, grid, s);
    default: return dispatch_v<4, QJL>(vb, a, grid, s);
  }
}

}  // namespace
}  // namespace tq

extern "C" size_t tq_decode_workspace_size(int B, int Hq, const tq_cache* cache, int seq_len) {
  using namespace tq;
  if (!cache || B < 1 || Hq < 1 || cache->Hkv < 1 || Hq % cache->Hkv || seq_len < 0) return 0;
  const Plan p = make_plan(B, Hq, cache->Hkv, seq_len, device_sms(),
                           resident_ctas(cache->k_bits, cache->v_bits), stage_tokens(cache->k_bits, cache->v_bits));
  return workspace_bytes(B, Hq, cache->Hkv, p);
}

extern "C" tq_status tq_decode_attn(const tq_params* params, const void* q, int q_dtype, int Hq,
                                    const tq_cache* cache, int seq_len, float scale, float* out,
                                    void* workspace, size_t ws_bytes, void* stream) {
  using namespace tq;
  clear_error();
  tq_status st = check_cache(cache);
  if (st != TQ_OK) return st;
  st = check_params(params, cache);
  if (st != TQ_OK) return st;
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return fail(TQ_ERR_UNSUPPORTED, "q_dtype %d", q_dtype);
  if (Hq < 1 || Hq % cache->Hkv) return fail(TQ_ERR_INVALID_ARG, "Hq %d vs Hkv %d", Hq, cache->Hkv);
  if (seq_len < 0 || seq_len > cache->T_cap)
    return fail(TQ_ERR_INVALID_ARG, "seq_len %d outside [0, %d]", seq_len, cache->T_cap);
  if (!q || !out || !workspace) return fail(TQ_ERR_INVALID_ARG, "q / out / workspace is NULL");
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace))
    return fail(TQ_ERR_INVALID_ARG, "q / out / workspace must be 16-byte aligned");
  const int B = cache->B;
  const Plan plan = make_plan(B, Hq, cache->Hkv, seq_len, device_sms(),
                              resident_ctas(cache->k_bits, cache->v_bits), stage_tokens(cache->k_bits, cache->v_bits));
  const size_t need = workspace_bytes(B, Hq, cache->Hkv, plan);
  if (ws_bytes < need)
    return fail(TQ_ERR_WORKSPACE, "workspace %zu bytes, need %zu", ws_bytes, need);

  const float sc = scale > 0.0f ? scale : 1.0f / sqrtf((float)D);
  float* ws = reinterpret_cast<float*>(workspace);
  DArgs a;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = cache->Hkv;
  a.g = Hq / cache->Hkv;
  a.hgroups = plan.hgroups;
  a.T_cap = cache->T_cap;
  a.seq_len = seq_len;
  a.splits = plan.splits;
  a.tps = plan.tps;
  a.sK = (float)((double)sc * 1.4426950408889634 / sqrt((double)D));
  a.sQ = cache->qjl_m ? (float)((double)sc * 1.4426950408889634 * 2.0 * sqrt(M_PI / 2.0) / cache->qjl_m)
                      : 0.0f;
  a.k_codes = cache->k_codes;
  a.k_signs = cache->k_signs;
  a.k_norm = cache->k_norm;
  a.k_rnorm = cache->k_rnorm;
  a.v_codes = cache->v_codes;
  a.v_norm = cache->v_norm;
  a.kc = params->k_centroids;
  a.vc = params->v_centroids;
  a.qrot = ws;
  a.sq = ws + (size_t)B * Hq * D;
  a.part = ws + (size_t)2 * B * Hq * D;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  const int BH = B * Hq;
  // heads per cluster: about 16 clusters at least (one CTA on each of 128 SMs), at most PREP_HB
  const int hb = std::max(1, std::min(PREP_HB, BH / 16));
  const int prep_ctas = (BH + hb - 1) / hb * PREP_CLUSTER;
  if (q_dtype == TQ_F32)
    prep_kernel<float><<<prep_ctas, PREP_THREADS, 0, s>>>(reinterpret_cast<const float*>(q), BH, hb, params->Pi,
                                                           params->S, cache->qjl_m ? 1 : 0, ws, ws + (size_t)BH * D);
  else
    prep_kernel<__nv_bfloat16><<<prep_ctas, PREP_THREADS, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16*>(q), BH, hb, params->Pi, params->S, cache->qjl_m ? 1 : 0, ws,
        ws + (size_t)BH * D);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "prep launch: %s", cudaGetErrorString(e));

  const dim3 grid(plan.splits, cache->Hkv * plan.hgroups, B);
  st = cache->qjl_m ? dispatch<true>(cache->k_bits, cache->v_bits, a, grid, s)
                    : dispatch<false>(cache->k_bits, cache->v_bits, a, grid, s);
  if (st != TQ_OK) return st;
  // merge: programmatic dependent of split (its CTAs wait for the split grid before reading)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(BH);
  cfg.blockDim = dim3(MERGE_THREADS);
  cfg.dynamicSmemBytes = merge_smem_bytes(plan.splits);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, merge_kernel, (const float*)a.part, params->Pi, out, plan.splits);
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "merge launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}

// One decode step: append the new token (tq_quantize with T_new = 1), then attend over t + 1
// tokens.  The decode arguments are checked first so that an invalid call enqueues nothing.
extern "C" tq_status tq_decode_step(const tq_params* params, const void* k_new, const void* v_new,
                                    int kv_dtype, const void* q, int q_dtype, int Hq, const tq_cache* cache,
                                    int t, float scale, float* out, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  using namespace tq;
  clear_error();
  tq_status st = check_cache(cache);
  if (st != TQ_OK) return st;
  st = check_params(params, cache);
  if (st != TQ_OK) return st;
  if (t < 0 || t >= cache->T_cap) return fail(TQ_ERR_INVALID_ARG, "t %d outside [0, %d)", t, cache->T_cap);
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return fail(TQ_ERR_UNSUPPORTED, "q_dtype %d", q_dtype);
  if (Hq < 1 || Hq % cache->Hkv) return fail(TQ_ERR_INVALID_ARG, "Hq %d vs Hkv %d", Hq, cache->Hkv);
  if (!q || !out || !workspace) return fail(TQ_ERR_INVALID_ARG, "q / out / workspace is NULL");
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace))
    return fail(TQ_ERR_INVALID_ARG, "q / out / workspace must be 16-byte aligned");
  const size_t need = tq_decode_workspace_size(cache->B, Hq, cache, t + 1);
  if (workspace_bytes < need)
    return fail(TQ_ERR_WORKSPACE, "workspace %zu bytes, need %zu", workspace_bytes, need);
  const int64_t sh = kHeadDim, sb = (int64_t)cache->Hkv * kHeadDim;
  st = tq_quantize(params, k_new, v_new, kv_dtype, sb, sh, kHeadDim, 1, t, cache, stream);
  if (st != TQ_OK) return st;
  return tq_decode_attn(params, q, q_dtype, Hq, cache, t + 1, scale, out, workspace, workspace_bytes,
                        stream);
}

// ------------------------------------------------------------------------------------------------
// Allocation-free decode: the same kernels, with the scratch space in a fixed device array.
//
// Some callers cannot allocate device memory at the point where they run decode: code inside a
// custom allocator or memory-pool callback (which would re-enter itself), runtimes that forbid
// cudaMalloc after start-up so that the memory footprint stays fixed, and plug-in hosts that hand
// a library only the tensors of one call.  For them the scratch lives in this array, which every
// GPU that loads the library holds until the process exits.
// ------------------------------------------------------------------------------------------------

#include <mutex>

namespace tq {
namespace {

constexpr size_t kStaticWorkspaceBytes = (size_t)4 << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_static_ws[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_ws_mutex;
void* g_static_ws_ptr[kMaxDevices] = {};

// Device address of g_static_ws on the current device, looked up once per device.
tq_status static_workspace(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(TQ_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lock(g_static_ws_mutex);
  if (!g_static_ws_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_ws);
    if (e != cudaSuccess || !p)
      return fail(TQ_ERR_CUDA, "cudaGetSymbolAddress(static workspace): %s", cudaGetErrorString(e));
    g_static_ws_ptr[dev] = p;
  }
  *out = g_static_ws_ptr[dev];
  return TQ_OK;
}

}  // namespace
}  // namespace tq

extern "C" size_t tq_decode_static_workspace_limit(void) { return tq::kStaticWorkspaceBytes; }

extern "C" tq_status tq_decode_attn_static(const tq_params* params, const void* q, int q_dtype,
                                           int Hq, const tq_cache* cache, int seq_len,
                                           float scale, float* out, void* stream) {
  using namespace tq;
  clear_error();
  if (!cache) return fail(TQ_ERR_INVALID_ARG, "cache is NULL");
  const size_t need = tq_decode_workspace_size(cache->B, Hq, cache, seq_len);
  if (need == 0) return fail(TQ_ERR_INVALID_ARG, "invalid sizes B=%d Hq=%d Hkv=%d seq_len=%d",
                             cache->B, Hq, cache->Hkv, seq_len);
  if (need > kStaticWorkspaceBytes)
    return fail(TQ_ERR_WORKSPACE,
                "decode needs %zu bytes of scratch, above the %zu-byte static workspace; "
                "use tq_decode_attn with a caller-allocated workspace",
                need, kStaticWorkspaceBytes);
  void* ws = nullptr;
  const tq_status st = static_workspace(&ws);
  if (st != TQ_OK) return st;
  return tq_decode_attn(params, q, q_dtype, Hq, cache, seq_len, scale, out, ws,
                        kStaticWorkspaceBytes, stream);
}
