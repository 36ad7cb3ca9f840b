// tq_decode_attn: single-token decode attention directly over the packed cache.
//
// Scores follow the QJL-corrected inner-product estimator,
//   est_i = <q', khat'_i> + ||r_i|| sqrt(pi/2)/m <S q', 2 sign_i - 1>,  q' = Pi q,
// with khat'_i = (n_i / sqrt(d)) c_K[idx_i] in the rotated basis (ai-news.ru overview, first and
// second ideas plus the third, QJL, component; tproger.ru "Step 1: PolarQuant", "Step 2: QJL").
// Softmax and the value sum also run in the rotated basis; one final o = Pi^T o' per head.
//
// Kernels (on the caller's stream; merge is a programmatic dependent of split):
//   split   one persistent CTA per SM over an even share of all (unit, token) pairs.  Up front the
//           CTA computes q' = Pi q and sq = S q' of the heads of its first four segments in fp32
//           (shared memory), while a producer warp already streams stages of the packed cache into
//           a ring of shared-memory slots with bulk copies (mbarrier completion).  11 (7 for groups
//           of 5-8 heads) consumer warps take 16 tokens each per stage: codes become fp16 pairs
//           through a lane-replicated shared-memory table (one permute + one load per two
//           coordinates), and m16n8k16 tensor-core MMAs compute q'.khat, the QJL sign dot (sign bits
//           placed in fp16 mantissas by a shift and one logic op, B rows pre-scaled to match) and
//           P.vhat (P split into fp16 hi + lo).  Online softmax runs in log2 units; at a segment's
//           end every consumer warp writes its own (max, sum, o'[128]) partial per head, so no
//           barrier stops the CTA between segments.
//   merge   one CTA per (batch, query head): log-sum-exp merge of the head's partials, then
//           o = Pi^T o'.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr int D = kHeadDim;
constexpr int HG = 8;                  // query heads per MMA row block (hi rows 0-7, lo rows 8-15)
constexpr int PART = 4 + D;            // (max, sum, pad, pad, o'[128]) per partial: o' 16-byte aligned
constexpr unsigned FULL = 0xffffffffu;


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

// 4-byte async copy (src_bytes = 0: no global read, zero fill).
__device__ __forceinline__ void cp_async4(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(smem_u32(dst)), "l"(src));
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

// ------------------------------------------------------------------------------------------ split
//
// Persistent split-K kernel.  The B * Hkv * head_groups (batch, kv-head, head group) units, each
// seq_len tokens long, are laid end to end and cut into one contiguous range per CTA (one CTA per
// SM), so every CTA streams the same number of tokens.  A range that crosses a unit boundary is
// processed as two segments; each segment ends with one (max, sum, o') partial per query head.
//
// Per CTA: warp NW (the producer) moves stages of ST = 16 * NW tokens into a ring of shared-memory
// slots: the key codes, sign bits and value codes of a stage are three contiguous blocks of the
// cache, fetched with one bulk copy each (cp.async.bulk, completion counted in bytes on the slot's
// "full" mbarrier), and the three per-token norms go through 4-byte cp.async whose completion the
// same mbarrier tracks.  Warps 0..NW-1 consume 16 tokens of every stage each and release the slot
// on its "empty" mbarrier.

// CTA shape: NW consumer warps + 1 producer.  The register file is split between the SM's four
// schedulers, so 12 warps (three per scheduler) leave 168 registers a thread: enough for one n-block
// of four heads (NB = 1).  Two n-blocks (five to eight heads per kv-head) need more registers and
// run with 8 warps (two per scheduler, up to 255 registers).
template <int NB>
struct Shape {
  static constexpr int NW = NB == 1 ? 11 : 7;
  static constexpr int THREADS = 32 * (NW + 1);
  static constexpr int ST = 16 * NW;        // tokens per stage
};
constexpr int NS_MAX = 8;                   // ring slots
constexpr int NSEG_PRE = 2;                 // segments whose query prep is computed in one pass
constexpr int MIN_TOK_PER_CTA = 256;        // fewer CTAs than SMs below this much work each
constexpr int CTRL_BYTES = 256;             // mbarriers, slot offsets, flags (end of dynamic smem)
constexpr long long WAIT_LIMIT = 4000000000LL;  // ~2 s of SM clock per wait

// Flat partition of N = units * seq_len tokens over C CTAs: CTA c takes [start(c), start(c + 1)).
__host__ __device__ inline int64_t part_start(int64_t N, int C, int c) { return (int64_t)c * N / C; }
__host__ __device__ inline int part_cta_of(int64_t N, int C, int64_t f) { return (int)(((f + 1) * C - 1) / N); }

// Shared-memory plan of a split CTA: absolute shared-window addresses (tables) and offsets from
// the start of dynamic shared memory (the rest), for dynamic shared memory starting at `base`.
struct SmemPlan {
  uint32_t base, tbl, tbl2, prep_off, merge_off;
  int ns;
  uint32_t stage_off[NS_MAX];
};

struct DArgs {
  SmemPlan plan;  // computed on the host for the usual base of dynamic shared memory
  int B, Hq, Hkv, g, hgroups, T_cap, seq_len;
  int units, ctas, pmax, dyn_smem;
  int64_t ntot;  // units * seq_len
  float sK;      // scale*log2e/sqrt(d)                (times n_i)
  float sQ;      // scale*log2e*2*sqrt(pi/2)/m         (times ||r_i||)
  const uint8_t* k_codes;
  const uint8_t* k_signs;
  const float* k_norm;
  const float* k_rnorm;
  const uint8_t* v_codes;
  const float* v_norm;
  const float* kc;
  const float* vc;
  const float* kc2;  // mixed layout: codebooks of the non-outlier half (3 bits)
  const float* vc2;
  const void* q;    // [B, Hq, 128] fp32 or bf16 (q_bf16)
  int q_bf16;
  const float* Pi;  // [128 x 128]
  const float* S;   // [128 x 128] (QJL)
  float* part;
  // Decode step (step = 1): row seq_len - 1 of every unit is quantized in the kernel from k_new /
  // v_new ([B, Hkv, 128], fp32 or bf16) in fp64, written to the cache and attended.
  int step, kv_bf16;
  const void* k_new;
  const void* v_new;
  const float* kt;  // thresholds of the codebooks
  const float* vt;
};

// bit 0: a wait timed out; bit 1: shared memory too small; bit 2 (TQ_DEBUG builds): a stage's rows
// or slot out of range; bit 3 (TQ_DEBUG): a partial slot out of range
__device__ unsigned int g_decode_error;

// MX: the outlier-aware mixed layout (TQ_LAYOUT_MIXED, KB = VB = 4): rows of 56 bytes (a 4-bit
// outlier half, then a 3-bit half) and two norms per token; the 4-bit halves use the packed pair
// table, the 3-bit halves two more 64-entry tables.
template <int KB, int VB, bool QJL, int NB, bool MX = false>
struct Layout {
  static constexpr int ST = Shape<NB>::ST, HGN = 4 * NB;
  static constexpr int K_ROW = MX ? 8 * (2 * KB - 1) : 16 * KB;
  static constexpr int V_ROW = MX ? 8 * (2 * VB - 1) : 16 * VB;
  static constexpr int NORM = MX ? 8 : 4;  // norm bytes per token
  static constexpr int OFF_KC = 0;
  static constexpr int OFF_SG = OFF_KC + ST * K_ROW;
  static constexpr int OFF_VC = OFF_SG + (QJL ? ST * 16 : 0);
  static constexpr int OFF_NK = OFF_VC + ST * V_ROW;
  static constexpr int OFF_RN = OFF_NK + ST * NORM;
  static constexpr int OFF_NV = OFF_RN + (QJL ? ST * 4 : 0);
  static constexpr int STAGE_BYTES = (OFF_NV + ST * NORM + 127) / 128 * 128;
  // bulk-copied bytes (mixed rows of 56 bytes go through 8-byte cp.async instead)
  static constexpr int TX_PER_TOKEN = (QJL ? 16 : 0) + (MX ? 0 : K_ROW + V_ROW);
  static constexpr bool kPacked = KB == 4 && VB == 4;
  static constexpr int K_TBL = kPacked ? 0 : (1 << (2 * KB)) * 128;
  static constexpr int V_TBL = kPacked ? 0 : (1 << (2 * VB)) * 128;
  static constexpr int TBL_BYTES = kPacked ? 65536 : K_TBL + V_TBL;
  static constexpr int TBL2_BYTES = MX ? 2 * 64 * 128 : 0;  // 3-bit K and V pair tables
  // query prep of NSEG_PRE segments: q' and S q' of their heads (the raw q is staged in the
  // latter), 64 codebook floats, the MMA B fragments of every lane ([segment][n-block][word / 4]
  // [lane][word % 4], 32 words) and (fK, fQ, Kh, 2^-e) per head
  static constexpr int FRAG_WORDS = NSEG_PRE * NB * 32 * 32;
  static constexpr int PREP_WORDS = 2 * NSEG_PRE * HGN * D + 64 + FRAG_WORDS + NSEG_PRE * HGN * 4;
  // decode step: the packed new row (key codes 16, signs 4, value codes 16, norms 4 words); its
  // scratch (8 * 2D + 4 * 2D + 32 bytes) lives in the B-fragment area
  static constexpr int STEP_BYTES = 4 * 40;
  static_assert(4 * FRAG_WORDS >= 8 * 2 * D + 4 * 2 * D + 8 * 4, "step scratch");
  static constexpr int PREP_BYTES = 4 * PREP_WORDS + STEP_BYTES;
  // the merge of the warps at the CTA's last segment end, one n-block at a time, in ring memory:
  // (max, sum) and o' of four heads per warp
  static constexpr int MERGE_BYTES = 4 * (Shape<NB>::NW * 4 * 2 + Shape<NB>::NW * 4 * D);
  static_assert(STAGE_BYTES % 16 == 0 && OFF_SG % 16 == 0 && OFF_VC % 16 == 0 && OFF_NK % 16 == 0,
                "bulk-copy granularity");
  static_assert(MX || (K_ROW % 16 == 0 && V_ROW % 16 == 0), "bulk-copy granularity");
  static_assert(!MX || kPacked, "mixed layout: 4-bit outlier halves");
};

// Control block at the end of the dynamic shared memory.
struct Ctrl {
  uint64_t full[NS_MAX];
  uint64_t empty[NS_MAX];
  uint32_t stage_off[NS_MAX];  // byte offsets of the ring slots from the start of dynamic smem
  uint32_t tbl_addr;           // shared-window address of the pair tables
  uint32_t tbl2_addr;          // mixed layout: the 3-bit pair tables
  uint32_t prep_off;
  uint32_t merge_off;          // the warps' merge area at the CTA's end (inside the ring)
  int ns;
  unsigned int err;
};
static_assert(sizeof(Ctrl) <= CTRL_BYTES, "control block");

__device__ __forceinline__ void mbar_init_(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive_(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx_(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// The thread's earlier cp.async copies arrive on the mbarrier when they land (counted in its init).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}
// One bulk copy global -> shared (sizes and addresses multiples of 16), completion in bytes.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t addr, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(addr), "r"(parity), "r"(100000u)
      : "memory");
  return done != 0;
}
// Bounded wait of a whole warp on an mbarrier phase (every lane returns the same answer).  Gives up
// at once when another warp has recorded an error, or after WAIT_LIMIT cycles (then records one).
__device__ __forceinline__ bool wait_w(Ctrl& c, uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_u32(bar);
  const long long t0 = clock64();
  while (true) {
    if (__any_sync(FULL, mbar_try(addr, parity))) return true;
    const bool stop = *reinterpret_cast<volatile unsigned int*>(&c.err) != 0 || clock64() - t0 > WAIT_LIMIT;
    if (__any_sync(FULL, stop)) {
      if ((threadIdx.x & 31) == 0) atomicOr(&c.err, 1u);
      return false;
    }
  }
}
// Named barrier of the NW consumer warps (the producer warp never takes part).
template <int NW>
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;\n" ::"n"(NW * 32) : "memory");
}

// QJL sign operand: pair P (bits P and P + 16 of the lane's sign word, sketch rows 2t + e of
// k-half P % 2 of k-step P / 2) as a half2 of 1 + b 2^(q - 10), b the sign bit: the word, shifted
// so that the pair lands on mantissa bits q and q + 16 (q = 6 + P % 4), masked and ORed into 1.0.
// The B operand rows of such a pair are pre-scaled by 2^(10 - q), so the MMA yields
// C + sum_l b_l sq_l with the per-head constant C = sum_l 2^(10 - q_l) sq_l.
template <int P>
__device__ __forceinline__ uint32_t sgn(uint32_t w) {
  constexpr int q = 6 + (P & 3);
  uint32_t x;
  if constexpr (P < 4) x = w << 6;
  else if constexpr (P < 8) x = w << 2;
  else if constexpr (P < 12) x = w >> 2;
  else x = w >> 6;
  return (x & (0x00010001u << q)) | 0x3C003C00u;
}
// 2^(10 - q) of pair P: the B-row scale that undoes the mantissa position.
__host__ __device__ constexpr float sgn_scale(int P) { return (float)(16 >> (P & 3)); }

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

// Transpose an 8x8 matrix of 16-bit elements held one row pair per lane (m8n8 fragment layout).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(addr));
  return v;
}
// Vector shared loads at addresses the caller guarantees aligned (stage rows are 16-byte aligned).
__device__ __forceinline__ uint4 lds128(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(smem_u32(p)));
  return v;
}
__device__ __forceinline__ uint2 lds64(const void* p) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(smem_u32(p)));
  return v;
}
// x as fp16 hi + lo (about 22 significant bits) packed into one half2 (hi in the low half).
__device__ __forceinline__ uint32_t hilo_half2(float x) {
  const float hi = __half2float(__float2half_rn(x));
  const __half2 h = __floats2half2_rn(hi, x - hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Pair tables: a pair of codes -> half2 of centroids, replicated per lane (bank = lane).
// 4-bit keys and values: 256 entries of 256 bytes (K replicas at +0, V at +128) starting at a
// 64 KB-aligned address, so one byte permute of the code word and of rk / rv (table address |
// lane offset) is the entry's address.  Other widths: separate K and V tables of 128-byte entries,
// address = (index << 7) + rk / rv.
template <int KB, int VB>
struct PairLut {
  static constexpr bool kPacked = KB == 4 && VB == 4;
  uint32_t rk, rv;
  uint32_t rk2, rv2;  // mixed layout: the 3-bit tables of the non-outlier half
  __device__ __forceinline__ uint32_t k2(uint32_t e) const { return lds32((e << 7) + rk2); }
  __device__ __forceinline__ uint32_t v2(uint32_t e) const { return lds32((e << 7) + rv2); }
  __device__ __forceinline__ uint32_t k(uint32_t e) const { return lds32((e << 7) + rk); }
  __device__ __forceinline__ uint32_t v(uint32_t e) const { return lds32((e << 7) + rv); }
  template <int Bt>
  __device__ __forceinline__ uint32_t k_byte(uint32_t w) const { return lds32(__byte_perm(w, rk, 0x7604u | (Bt << 4))); }
  template <int Bt>
  __device__ __forceinline__ uint32_t v_byte(uint32_t w) const { return lds32(__byte_perm(w, rv, 0x7604u | (Bt << 4))); }
};

// Key pair P (0..15) of a thread's code chunk, as a half2 of centroids.
template <int KB, int VB, int P>
__device__ __forceinline__ uint32_t k_pair(const PairLut<KB, VB>& L, const uint32_t (&c)[KB]) {
  if constexpr (PairLut<KB, VB>::kPacked) return L.template k_byte<P & 3>(c[P >> 2]);
  else return L.k(k_pair_index<KB, P>(c));
}
// Value pair NU of a token pair, as a half2 of centroids.
template <int KB, int VB, int NU>
__device__ __forceinline__ uint32_t v_pair(const PairLut<KB, VB>& L, const VPairs<VB>& p) {
  if constexpr (PairLut<KB, VB>::kPacked) return L.template v_byte<((NU & 7) >> 1)>(p.w[2 * (NU >> 3) + (NU & 1)]);
  else return L.v(p.template index<NU>());
}

// Shared-memory plan: the pair tables (at a 64 KB boundary for the packed tables) split the rest
// into two free regions; the most ring slots (up to NS_MAX) are placed first-fit such that the
// query-prep area (and the mixed layout's second tables) still fit around them.  The warps' merge
// at the CTA's end goes into adjacent ring slots.  ns = 0 when nothing fits (never with the 227 KB
// of an sm_100 CTA).  The host computes it once per launch for the usual start of dynamic shared
// memory; a CTA whose dynamic shared memory starts elsewhere computes its own.
struct Regions {
  uint32_t base, r0, r0e, r1, r1e;
  __host__ __device__ bool take(uint32_t bytes, uint32_t& off) {
    if (r0e - r0 >= bytes) {
      off = r0 - base;
      r0 += bytes;
      return true;
    }
    if (r1e - r1 >= bytes) {
      off = r1 - base;
      r1 += bytes;
      return true;
    }
    return false;
  }
};

template <int KB, int VB, bool QJL, int NB, bool MX>
__host__ __device__ void plan_layout(uint32_t base, int dyn, SmemPlan& p) {
  using Lay = Layout<KB, VB, QJL, NB, MX>;
  const uint32_t end = base + (uint32_t)dyn - CTRL_BYTES;
  const uint32_t tbl = Lay::kPacked ? ((base + 0xFFFFu) & ~0xFFFFu) : base;
  p.base = base;
  p.tbl = tbl;
  p.tbl2 = 0;
  p.ns = 0;
  if (tbl + Lay::TBL_BYTES > end) return;
  for (int ns = NS_MAX; ns >= 2; --ns) {
    Regions r{base, base, tbl, tbl + (uint32_t)Lay::TBL_BYTES, end};  // [base, tbl) and [tbl + TBL, end)
    bool ok = true;
    for (int i = 0; i < ns && ok; ++i) ok = r.take(Lay::STAGE_BYTES, p.stage_off[i]);
    ok = ok && r.take(Lay::PREP_BYTES, p.prep_off);
    if (ok && Lay::TBL2_BYTES) {
      uint32_t off = 0;
      ok = r.take(Lay::TBL2_BYTES, off);
      p.tbl2 = base + off;
    }
    if (!ok) continue;
    // the warps' merge at the CTA's end reuses ring memory: a run of adjacent slots large enough
    p.merge_off = 0xFFFFFFFFu;
    for (int k = 0; k < ns && p.merge_off == 0xFFFFFFFFu; ++k) {
      uint32_t run = Lay::STAGE_BYTES;
      for (int i = k + 1; i < ns && run < (uint32_t)Lay::MERGE_BYTES &&
                          p.stage_off[i] == p.stage_off[i - 1] + Lay::STAGE_BYTES; ++i)
        run += Lay::STAGE_BYTES;
      if (run >= (uint32_t)Lay::MERGE_BYTES) p.merge_off = p.stage_off[k];
    }
    if (p.merge_off == 0xFFFFFFFFu) continue;
    p.ns = ns;
    return;
  }
}

// 64-bit division that takes the 32-bit path when both operands fit (every realistic size).
__device__ __forceinline__ int64_t div_s(int64_t x, int64_t y) {
  return (x <= 0x7fffffff && y <= 0x7fffffff) ? (int64_t)((uint32_t)x / (uint32_t)y) : x / y;
}

// Decode step, by the consumer warps of a CTA whose range ends a unit: the unit's new key and value
// (k_new / v_new) quantized in fp64 exactly as the definition reads -- n = ||x||,
// u = sqrt(d) Pi x / n, idx = #{t_i <= u}, rho = u - c[idx], ||r|| = n ||rho|| / sqrt(d), sign
// bits of S rho -- packed into `row` (key codes [0,16), signs [16,20), value codes [20,36), norms
// [36,39) words) and, for the unit's first head group, written into cache row seq_len - 1.
// Matrix rows are read eight lanes per row as in the prologue.  Kept out of line: its registers
// must not weigh on the main loop.
template <int KB, int VB, bool QJL, int NB>
__device__ __noinline__ void quantize_step_row(const DArgs& a, float* x, double* y, double* nrm, uint32_t* row,
                                      const float* cbs, int64_t bk, int hg, int64_t L) {
  constexpr int NW = Shape<NB>::NW, PR = (D + 4 * NW - 1) / (4 * NW);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, e = lane & 7;
  for (int i = tid; i < 2 * D; i += NW * 32) {  // i < D: key element i; D <= i: value element i - D
    const void* src = i < D ? a.k_new : a.v_new;
    const int64_t off = bk * D + (i % D);
    x[i] = a.kv_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(src)[off])
                     : reinterpret_cast<const float*>(src)[off];
  }
  if (tid < 40) row[tid] = 0u;
  consumers_sync<NW>();
  // vout[v][r] = sum_k M[r][k] vin[v][k] in fp64 (vin: fp32 at vf or fp64 at vd), nv vectors
  auto matvec = [&](const float* M, const float* vf, const double* vd, double* vout, int nv) {
    for (int j = 0; j < PR; ++j) {
      const int r = 4 * warp + (lane >> 3) + 4 * NW * j;
      if (4 * NW * j + 4 * warp >= D) break;  // warp-uniform
      const float4* mr = reinterpret_cast<const float4*>(M + r * D) + e;
      float4 m[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) m[k] = __ldg(mr + 8 * k);
      for (int v = 0; v < nv; ++v) {
        double acc = 0.0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int c0 = v * D + 4 * (e + 8 * k);
          acc = fma((double)m[k].x, vd ? vd[c0] : (double)vf[c0], acc);
          acc = fma((double)m[k].y, vd ? vd[c0 + 1] : (double)vf[c0 + 1], acc);
          acc = fma((double)m[k].z, vd ? vd[c0 + 2] : (double)vf[c0 + 2], acc);
          acc = fma((double)m[k].w, vd ? vd[c0 + 3] : (double)vf[c0 + 3], acc);
        }
        acc += __shfl_xor_sync(FULL, acc, 1);
        acc += __shfl_xor_sync(FULL, acc, 2);
        acc += __shfl_xor_sync(FULL, acc, 4);
        if (e == 0) vout[v * D + r] = acc;
      }
    }
  };
  auto sumsq = [&](const float* vf, const double* vd) -> double {  // one warp, fixed order
    double acc = 0.0;
    for (int k = 0; k < D / 32; ++k) {
      const double v = vd ? vd[lane + 32 * k] : (double)vf[lane + 32 * k];
      acc = fma(v, v, acc);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(FULL, acc, o);
    return acc;
  };
  matvec(a.Pi, x, nullptr, y, 2);  // y = Pi k, Pi v
  if (warp < 2) {
    const double ss = sumsq(x + D * warp, nullptr);
    if (lane == 0) nrm[warp] = sqrt(ss);
  }
  consumers_sync<NW>();
  for (int i = tid; i < 2 * D; i += NW * 32) {  // coordinate i % D of the key (i < D) or the value
    const bool isv = i >= D;
    const int j = i % D;
    const double n = nrm[isv ? 1 : 0];
    const double u = n > 0.0 ? sqrt((double)D) * y[i] / n : 0.0;
    const int bits = isv ? VB : KB;
    const float* th = isv ? a.vt : a.kt;
    int idx = 0;
    for (int c = 0; c < (1 << bits) - 1; ++c) idx += u >= (double)th[c] ? 1 : 0;
    if (!isv) y[j] = u - (double)cbs[idx];  // rho, in place of this thread's own y element
    const int bit = bits * (isv ? v_slot_of_coord(j) : k_slot_of_coord(j));
    uint32_t* w = row + (isv ? 20 : 0);
    atomicOr(w + (bit >> 5), (uint32_t)idx << (bit & 31));
    if ((bit & 31) + bits > 32) atomicOr(w + (bit >> 5) + 1, (uint32_t)idx >> (32 - (bit & 31)));
  }
  consumers_sync<NW>();
  if constexpr (QJL) {
    matvec(a.S, nullptr, y, y + D, 1);  // S rho, over the value's y (read before the barrier)
    if (warp == 0) {
      const double rr = sumsq(nullptr, y);
      if (lane == 0) nrm[2] = nrm[0] * sqrt(rr) / sqrt((double)D);
    }
    consumers_sync<NW>();
    for (int l = tid; l < kQjlRows; l += NW * 32) {
      const int bit = sign_bit_of_row(l);
      if (y[D + l] >= 0.0) atomicOr(row + 16 + (bit >> 5), 1u << (bit & 31));
    }
  }
  if (tid == 0) {
    reinterpret_cast<float*>(row)[36] = (float)nrm[0];
    reinterpret_cast<float*>(row)[37] = QJL ? (float)nrm[2] : 0.0f;
    reinterpret_cast<float*>(row)[38] = (float)nrm[1];
  }
  consumers_sync<NW>();  // the packed row is complete
  if (hg == 0 && warp == 0) {  // one copy of the row into the cache
    constexpr int K_ROW = 16 * KB, V_ROW = 16 * VB;
    const int64_t r = bk * a.T_cap + L - 1;
    if (lane < K_ROW / 4) reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(a.k_codes) + r * K_ROW)[lane] = row[lane];
    if (lane < V_ROW / 4) reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(a.v_codes) + r * V_ROW)[lane] = row[20 + lane];
    if (QJL && lane < 4) reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(a.k_signs) + r * 16)[lane] = row[16 + lane];
    if (lane == 0) {
      const_cast<float*>(a.k_norm)[r] = reinterpret_cast<const float*>(row)[36];
      if (QJL) const_cast<float*>(a.k_rnorm)[r] = reinterpret_cast<const float*>(row)[37];
      const_cast<float*>(a.v_norm)[r] = reinterpret_cast<const float*>(row)[38];
    }
  }
}

// STEP: the decode-step variant (a separate instantiation, so that plain decode carries none of it).
template <int KB, int VB, bool QJL, int NB, bool MX, bool STEP>
__global__ void __launch_bounds__(Shape<NB>::THREADS, 1) split_kernel(const __grid_constant__ DArgs a) {
  using Lay = Layout<KB, VB, QJL, NB, MX>;
  using Lut = PairLut<KB, VB>;
  constexpr int NW = Shape<NB>::NW, ST = Shape<NB>::ST, HGN = 4 * NB;
  extern __shared__ __align__(1024) unsigned char smem[];
  Ctrl& ctl = *reinterpret_cast<Ctrl*>(smem + a.dyn_smem - CTRL_BYTES);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x;
  const int64_t f_begin = part_start(a.ntot, a.ctas, c), f_end = part_start(a.ntot, a.ctas, c + 1);
  const int64_t L = a.seq_len;

  if (tid == 0) {
    SmemPlan p;
    if (smem_u32(smem) == a.plan.base) p = a.plan;
    else plan_layout<KB, VB, QJL, NB, MX>(smem_u32(smem), a.dyn_smem, p);
    ctl.tbl_addr = p.tbl;
    ctl.tbl2_addr = p.tbl2;
    ctl.prep_off = p.prep_off;
    ctl.merge_off = p.merge_off;
    ctl.ns = p.ns;
    for (int i = 0; i < p.ns; ++i) ctl.stage_off[i] = p.stage_off[i];
    ctl.err = 0;
    for (int i = 0; i < ctl.ns; ++i) {
      mbar_init_(&ctl.full[i], 1 + 32);  // producer's expect_tx + the noinc arrivals of its 32 lanes
      mbar_init_(&ctl.empty[i], NW);
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  __syncthreads();
  const int ns = ctl.ns;
  if (ns == 0) {
    if (tid == 0) atomicOr(&g_decode_error, 2u);
    return;  // uniform: every thread read the same ns
  }

  if (warp == NW) {
    // ================================================================ producer
    // the consumers' prologue loads go to memory first (named barrier 2, arrived at by them)
    asm volatile("bar.sync 2, %0;\n" ::"n"((NW + 1) * 32) : "memory");
    int it = 0, issued = 0, slot = 0, round = 0;  // stage count, ring slot, times round the ring
    for (int64_t f = f_begin; f < f_end;) {
      const int64_t u = div_s(f, L);
      const int t0 = (int)(f - u * L);
      const int t1 = (int)(L < t0 + (f_end - f) ? L : t0 + (f_end - f));
      f += t1 - t0;
      const int bk = (int)div_s(u, a.hgroups);  // b * Hkv + kv-head
      const int64_t rowb = (int64_t)bk * a.T_cap;
      // decode step: this segment ends its unit, whose last row is the new token, quantized by
      // the consumers in the prologue; the producer writes it into the stage itself
      const bool step_seg = STEP && !MX && t1 == L;
      for (int s0 = t0; s0 < t1; s0 += ST, ++it) {
        const int cur = slot, cur_round = round;  // this stage's slot, and its earlier uses
        if (++slot == ns) {
          slot = 0;
          ++round;
        }
        // the slot's previous contents (use cur_round - 1) have been consumed
        if (cur_round > 0 && !wait_w(ctl, &ctl.empty[cur], (cur_round - 1) & 1)) continue;
        if (*reinterpret_cast<volatile unsigned int*>(&ctl.err)) continue;
        const int ntok = min(ST, t1 - s0);
        const int64_t row0 = rowb + s0;
        unsigned char* st = smem + ctl.stage_off[cur];
#ifdef TQ_DEBUG
        // debug build: the stage's cache rows and its ring slot lie inside their arrays; otherwise
        // nothing is copied, the error is recorded and every wait of the CTA gives up
        if (ntok <= 0 || row0 < 0 || row0 + ntok > (int64_t)a.B * a.Hkv * a.T_cap ||
            ctl.stage_off[cur] + (uint32_t)Lay::STAGE_BYTES > (uint32_t)(a.dyn_smem - CTRL_BYTES)) {
          if (lane == 0) {
            atomicOr(&g_decode_error, 4u);
            atomicOr(&ctl.err, 1u);
          }
          // the consumers' arrival on the new-row barrier still needs its partner
          if (STEP && step_seg && s0 + ntok == t1) asm volatile("bar.sync 3, %0;\n" ::"n"((NW + 1) * 32) : "memory");
          continue;
        }
#endif
        if (STEP && step_seg && s0 + ntok == t1) {  // the stage with the new row (its last one)
          const int nb = ntok - 1;          // rows copied from the cache
          if (lane == 0 && nb > 0) {
            if constexpr (!MX) {
              bulk_g2s(st + Lay::OFF_KC, a.k_codes + row0 * Lay::K_ROW, nb * Lay::K_ROW, &ctl.full[cur]);
              if constexpr (QJL) bulk_g2s(st + Lay::OFF_SG, a.k_signs + row0 * 16, nb * 16, &ctl.full[cur]);
              bulk_g2s(st + Lay::OFF_VC, a.v_codes + row0 * Lay::V_ROW, nb * Lay::V_ROW, &ctl.full[cur]);
            }
          }
          for (int i = lane; i < nb; i += 32) {
            cp_async4(st + Lay::OFF_NK + 4 * i, a.k_norm + row0 + i, 4);
            if constexpr (QJL) cp_async4(st + Lay::OFF_RN + 4 * i, a.k_rnorm + row0 + i, 4);
            cp_async4(st + Lay::OFF_NV + 4 * i, a.v_norm + row0 + i, 4);
          }
          // wait (once) until the consumers have the packed row
          asm volatile("bar.sync 3, %0;\n" ::"n"((NW + 1) * 32) : "memory");
          const uint32_t* row = reinterpret_cast<const uint32_t*>(smem + ctl.prep_off + 4 * Lay::PREP_WORDS);
          const int p = nb;
          if (lane < Lay::K_ROW / 4) reinterpret_cast<uint32_t*>(st + Lay::OFF_KC + p * Lay::K_ROW)[lane] = row[lane];
          if (QJL && lane < 4) reinterpret_cast<uint32_t*>(st + Lay::OFF_SG + p * 16)[lane] = row[16 + lane];
          if (lane < Lay::V_ROW / 4) reinterpret_cast<uint32_t*>(st + Lay::OFF_VC + p * Lay::V_ROW)[lane] = row[20 + lane];
          if (lane == 0) {
            reinterpret_cast<float*>(st + Lay::OFF_NK)[p] = reinterpret_cast<const float*>(row)[36];
            if (QJL) reinterpret_cast<float*>(st + Lay::OFF_RN)[p] = reinterpret_cast<const float*>(row)[37];
            reinterpret_cast<float*>(st + Lay::OFF_NV)[p] = reinterpret_cast<const float*>(row)[38];
          }
          __syncwarp();  // (the lanes' stores are ordered before lane 0's release arrive)
          if (lane == 0) mbar_expect_tx_(&ctl.full[cur], (uint32_t)(nb * Lay::TX_PER_TOKEN));
          cp_async_arrive_noinc(&ctl.full[cur]);
          issued = it + 1;
          continue;
        }
        if (lane == 0) {
          mbar_expect_tx_(&ctl.full[cur], (uint32_t)(ntok * Lay::TX_PER_TOKEN));
          if constexpr (!MX)
            bulk_g2s(st + Lay::OFF_KC, a.k_codes + row0 * Lay::K_ROW, ntok * Lay::K_ROW, &ctl.full[cur]);
          if constexpr (QJL) bulk_g2s(st + Lay::OFF_SG, a.k_signs + row0 * 16, ntok * 16, &ctl.full[cur]);
          if constexpr (!MX)
            bulk_g2s(st + Lay::OFF_VC, a.v_codes + row0 * Lay::V_ROW, ntok * Lay::V_ROW, &ctl.full[cur]);
        }
        if constexpr (MX) {  // 56-byte rows: seven 8-byte copies per row (every row is 8-byte aligned)
          const uint8_t* kg = a.k_codes + row0 * Lay::K_ROW;
          const uint8_t* vg = a.v_codes + row0 * Lay::V_ROW;
          for (int i = lane; i < ntok * (Lay::K_ROW / 8); i += 32) {
            cp_async8(st + Lay::OFF_KC + 8 * i, kg + 8 * i);
            cp_async8(st + Lay::OFF_VC + 8 * i, vg + 8 * i);
          }
          for (int i = lane; i < ntok; i += 32) {
            cp_async8(st + Lay::OFF_NK + 8 * i, a.k_norm + 2 * (row0 + i));
            if constexpr (QJL) cp_async4(st + Lay::OFF_RN + 4 * i, a.k_rnorm + row0 + i, 4);
            cp_async8(st + Lay::OFF_NV + 8 * i, a.v_norm + 2 * (row0 + i));
          }
        } else {
          for (int i = lane; i < ntok; i += 32) {
            cp_async4(st + Lay::OFF_NK + 4 * i, a.k_norm + row0 + i, 4);
            if constexpr (QJL) cp_async4(st + Lay::OFF_RN + 4 * i, a.k_rnorm + row0 + i, 4);
            cp_async4(st + Lay::OFF_NV + 4 * i, a.v_norm + row0 + i, 4);
          }
        }
        cp_async_arrive_noinc(&ctl.full[cur]);
        issued = it + 1;
      }
    }
    // every copy issued has landed before the CTA may exit (bounded)
    for (int j = max(0, issued - ns); j < issued; ++j) {
      const uint32_t addr = smem_u32(&ctl.full[j % ns]);
      const long long t0 = clock64();
      while (!__all_sync(FULL, mbar_try(addr, (j / ns) & 1)) && clock64() - t0 < WAIT_LIMIT) {
      }
    }
    if (lane == 0 && *reinterpret_cast<volatile unsigned int*>(&ctl.err)) atomicOr(&g_decode_error, 1u);
    return;
  }

  // ================================================================ consumers (warps 0 .. NW-1)
  // Prologue: q' = Pi q and sq = S q' of the heads of the CTA's first NSEG_PRE segments (fp32, the
  // prep area [NSEG_PRE][HGN][D] each; the raw q is staged where sq goes), then the pair tables.
  // Every global load it needs is issued first, so they share one memory round trip: the
  // thread's rows of Pi and S (see prologue_pass), its share of the queries and one codebook
  // entry.  The producer starts its copies once the consumers have these loads (named barrier 2).
  float* qpm = reinterpret_cast<float*>(smem + ctl.prep_off);
  float* sqm = qpm + NSEG_PRE * HGN * D;
  float* cbs = sqm + NSEG_PRE * HGN * D;  // [64]: c_K at 0, c_V at 16, mixed layout c_K lo at 32, c_V lo at 40
  int nhs[NSEG_PRE];  // heads of each segment of the chunk (0 past the CTA's range)
  constexpr int QPT = (NSEG_PRE * HGN * D + NW * 32 - 1) / (NW * 32);  // query values per thread
  // segments of the chunk starting at fc: heads and query offsets
  auto chunk_info = [&](int64_t fc, int64_t (&qbase)[NSEG_PRE]) {
    int64_t f = fc;
#pragma unroll
    for (int si = 0; si < NSEG_PRE; ++si) {
      nhs[si] = 0;
      qbase[si] = 0;
      if (f < f_end) {
        const int64_t u = div_s(f, L);
        const int64_t t0 = f - u * L;
        f += (L - t0 < f_end - f) ? L - t0 : f_end - f;
        const int bk = (int)div_s(u, a.hgroups), hg = (int)(u - (int64_t)bk * a.hgroups);
        const int b = bk / a.Hkv, h0 = (bk % a.Hkv) * a.g + hg * HG;
        nhs[si] = min(HG, a.g - hg * HG);
        qbase[si] = ((int64_t)b * a.Hq + h0) * D;
      }
    }
  };
  auto load_q = [&](const int64_t (&qbase)[NSEG_PRE], int i) -> float {
    const int si = i / (HGN * D), hh = (i / D) % HGN, d = i % D;
    const int64_t qi = qbase[si] + hh * D + d;
    return a.q_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.q)[qi])
                    : reinterpret_cast<const float*>(a.q)[qi];
  };
  auto q_live = [&](int i) { return (i % (HGN * D)) / D < nhs[i / (HGN * D)]; };
  // Prologue pass: eight lanes per matrix row, lane (row, e) holding the 16-byte chunks e, e + 8,
  // e + 16, e + 24 of the row, so that each load instruction of a warp reads four whole 128-byte
  // lines; warp w takes rows 4w + r + 4 NW j in round j.  A row's dot product is summed over its
  // eight lanes.
  constexpr int PR = (D + 4 * NW - 1) / (4 * NW);  // rounds
  auto prologue_pass = [&](const float4 (&r4)[PR][4], const float* vin, float* vout) {
    const int e = lane & 7;
#pragma unroll 1
    for (int si = 0; si < NSEG_PRE; ++si) {
#pragma unroll 1
      for (int hh = 0; hh < nhs[si]; ++hh) {
        const float4* v4 = reinterpret_cast<const float4*>(vin + (si * HGN + hh) * D) + e;
        float4 x[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) x[k] = v4[8 * k];
#pragma unroll
        for (int j = 0; j < PR; ++j) {
          const int row = 4 * warp + (lane >> 3) + 4 * NW * j;
          if (4 * NW * j + 4 * warp < D) {  // warp-uniform: this round has rows for the warp
            float c0 = 0.0f, c1 = 0.0f;
#pragma unroll
            for (int k = 0; k < 4; k += 2) {
              c0 = fmaf(r4[j][k].x, x[k].x, c0);
              c1 = fmaf(r4[j][k + 1].x, x[k + 1].x, c1);
              c0 = fmaf(r4[j][k].y, x[k].y, c0);
              c1 = fmaf(r4[j][k + 1].y, x[k + 1].y, c1);
              c0 = fmaf(r4[j][k].z, x[k].z, c0);
              c1 = fmaf(r4[j][k + 1].z, x[k + 1].z, c1);
              c0 = fmaf(r4[j][k].w, x[k].w, c0);
              c1 = fmaf(r4[j][k + 1].w, x[k + 1].w, c1);
            }
            float acc = c0 + c1;
            acc += __shfl_xor_sync(FULL, acc, 1);
            acc += __shfl_xor_sync(FULL, acc, 2);
            acc += __shfl_xor_sync(FULL, acc, 4);
            if (e == 0 && row < D) vout[(si * HGN + hh) * D + row] = acc;
          }
        }
      }
    }
  };
  // Decode step: the new key / value of the CTA's segment that ends its unit (at most one; the
  // host keeps the step on this path only then), quantized in fp64 exactly as the definition
  // reads (norm, u = sqrt(d) Pi x / n, idx = #{t_i <= u}, rho = u - c[idx], ||r|| and the signs
  // of S rho), so that no guard band is needed.  The matrix rows are the prologue's registers.
  // Scratch of the step in the B-fragment area, which prep_frags fills only afterwards: y (fp64
  // [2][D]: Pi k, Pi v; then rho, S rho), the new vectors (fp32 [2][D]) and the fp64 norms; the
  // packed row stays until its stage is patched.
  double* sty = reinterpret_cast<double*>(cbs + 64);
  float* stx = reinterpret_cast<float*>(sty + 2 * D);
  double* stn = reinterpret_cast<double*>(stx + 2 * D);
  uint32_t* strow = reinterpret_cast<uint32_t*>(smem + ctl.prep_off + 4 * Lay::PREP_WORDS);  // [0,16) K codes, [16,20) signs, [20,36) V codes, [36,39) norms
  // B operands of the main loop's MMAs, built once per chunk for all consumer warps.  Column gq of
  // n-block nb = head 4 nb + gq / 2, part gq % 2 (0: fp16 hi, 1: fp16 lo); k-step kk holds
  // k = 16kk + 2t, +1 (reg 0), +8, +9 (reg 1) of lane (gq, t).  Word 2kk + r of a lane holds the q'
  // fragment (kk, r), word 16 + 2kk + r the S q' one.  Each head is scaled by a power of two 2^-e
  // so that q' and 16 S q' stay far inside fp16 range.
  uint32_t* frg = reinterpret_cast<uint32_t*>(cbs + 64);
  float4* hcon = reinterpret_cast<float4*>(frg + Lay::FRAG_WORDS);  // [NSEG_PRE][HGN]
  auto prep_frags = [&]() {
    // per head: the scale, then the QJL constant Kh = -C - 0.5 sum_k sq_k 2^-e with C the sum of the
    // fp16 parts of the pre-scaled S q' (sum_l sq_l (2 b_l - 1) = 2 (D_hi + D_lo + Kh) in the MMA)
    for (int hx = warp; hx < NSEG_PRE * HGN; hx += NW) {  // warp-uniform
      const int si = hx / HGN, hh = hx % HGN;
      if (hh >= nhs[si]) {
        if (lane == 0) hcon[hx] = make_float4(a.sK, a.sQ, 0.0f, 1.0f);
        continue;
      }
      const float* qp = qpm + hx * D;
      const float* sp = sqm + hx * D;
      float mx = 0.0f;
#pragma unroll
      for (int k = lane; k < D; k += 32)
        mx = fmaxf(mx, fmaxf(fabsf(qp[k]), QJL ? 16.0f * fabsf(sp[k]) : 0.0f));
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
      // 2^-e with mx 2^-e < 2^14 (e >= 0); inf / nan stay inf / nan
      const int ex = (mx < 16384.0f || !(mx < INFINITY)) ? 0 : ((__float_as_int(mx) >> 23) & 255) - 127 - 13;
      const float dn = __int_as_float((127 - ex) << 23);
      float ch = 0.0f, sh = 0.0f;
      if constexpr (QJL) {
#pragma unroll
        for (int k = lane; k < D; k += 32) {
          const float scl = (float)(16 >> ((k >> 3) & 3));  // sgn_scale of the k-step pair
          const float v = sp[k] * dn * scl;
          const float hi = __half2float(__float2half_rn(v));
          const float lo = __half2float(__float2half_rn(v - hi));
          ch += hi + lo;
          sh += (hi + lo) * (1.0f / scl);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          ch += __shfl_xor_sync(FULL, ch, o);
          sh += __shfl_xor_sync(FULL, sh, o);
        }
      }
      if (lane == 0) {
        const float up = __int_as_float((127 + ex) << 23);
        hcon[hx] = make_float4(a.sK * up, a.sQ * up, -ch - 0.5f * sh, dn);
      }
    }
    consumers_sync<NW>();
    for (int i = tid; i < Lay::FRAG_WORDS; i += NW * 32) {
      const int word = ((i >> 7) & 7) * 4 + (i & 3), ln = (i >> 2) & 31;
      const int nb = (i >> 10) % NB, si = i / (1024 * NB);
      const int kk = (word >> 1) & 7, r = word & 1, sq = word >> 4;
      const int hh = 4 * nb + (ln >> 3), tt = ln & 3;
      const bool lo = (ln >> 2) & 1;
      uint32_t v = 0u;
      if (hh < nhs[si] && (!sq || QJL)) {
        const float* src = (sq ? sqm : qpm) + (si * HGN + hh) * D + 16 * kk + 8 * r + 2 * tt;
        const float f = hcon[si * HGN + hh].w * (sq ? sgn_scale(2 * kk + r) : 1.0f);
        float h0, l0, h1, l1;
        split_half(src[0] * f, h0, l0);
        split_half(src[1] * f, h1, l1);
        v = lo ? pack_half2(l0, l1) : pack_half2(h0, h1);
      }
      frg[i] = v;
    }
    consumers_sync<NW>();
  };
  // A later chunk (a CTA whose range holds more than NSEG_PRE segments: short contexts) comes in the
  // middle of the stream, where every consumer warp is at the same segment boundary and the loop
  // state holds registers: there the matrix rows are read 16 values at a time.
  auto prep_chunk = [&](int64_t fc) {
    int64_t qbase[NSEG_PRE];
    chunk_info(fc, qbase);
#pragma unroll 1
    for (int i = tid; i < NSEG_PRE * HGN * D; i += NW * 32)
      if (q_live(i)) sqm[i] = load_q(qbase, i);
    consumers_sync<NW>();
#pragma unroll 1
    for (int pass = 0; pass < (QJL ? 2 : 1); ++pass) {
      const float* vin = pass ? qpm : sqm;
      float* vout = pass ? sqm : qpm;
#pragma unroll 1
      for (int task = tid; task < 2 * D; task += NW * 32) {  // whole warps
        const int row = task >> 1, half = task & 1;
        const float4* mr = reinterpret_cast<const float4*>((pass ? a.S : a.Pi) + row * D + 64 * half);
#pragma unroll 1
        for (int si2 = 0; si2 < NSEG_PRE; ++si2) {
#pragma unroll 1
          for (int hh = 0; hh < nhs[si2]; ++hh) {
            const float4* v4 = reinterpret_cast<const float4*>(vin + (si2 * HGN + hh) * D + 64 * half);
            float acc = 0.0f;
#pragma unroll 1
            for (int k0 = 0; k0 < 16; k0 += 4) {
#pragma unroll
              for (int k = k0; k < k0 + 4; ++k) {
                const float4 mm = __ldg(mr + k), x = v4[k];
                acc = fmaf(mm.x, x.x, acc);
                acc = fmaf(mm.y, x.y, acc);
                acc = fmaf(mm.z, x.z, acc);
                acc = fmaf(mm.w, x.w, acc);
              }
            }
            acc += __shfl_xor_sync(FULL, acc, 1);
            if (half == 0) vout[(si2 * HGN + hh) * D + row] = acc;
          }
        }
      }
      consumers_sync<NW>();
    }
    prep_frags();
  };

  Lut lut;
  {
    // ---- issue the loads
    int64_t qbase[NSEG_PRE];
    chunk_info(f_begin, qbase);
    float qr[QPT];
#pragma unroll
    for (int k = 0; k < QPT; ++k) {
      const int i = tid + k * NW * 32;
      qr[k] = (i < NSEG_PRE * HGN * D && q_live(i)) ? load_q(qbase, i) : 0.0f;
    }
    float4 m4[PR][4], s4[PR][4];
#pragma unroll
    for (int j = 0; j < PR; ++j) {
      const int row = 4 * warp + (lane >> 3) + 4 * NW * j;
      const float4* pr = reinterpret_cast<const float4*>(a.Pi + (row < D ? row : 0) * D) + (lane & 7);
      const float4* sr = reinterpret_cast<const float4*>(a.S + (row < D ? row : 0) * D) + (lane & 7);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        m4[j][k] = __ldg(pr + 8 * k);
        if constexpr (QJL) s4[j][k] = __ldg(sr + 8 * k);
      }
    }
    // decode step: the segment of this CTA that ends its unit (its last token is the new one)
    int64_t step_bk = -1;  // b * Hkv + kv-head of that unit, -1: none
    int step_hg = 0;
    if constexpr (STEP && !MX) {
      for (int64_t f = f_begin; f < f_end;) {
        const int64_t u = div_s(f, L);
        const int64_t t0 = f - u * L;
        const int64_t len = (L - t0 < f_end - f) ? L - t0 : f_end - f;
        if (t0 + len == L) {
          step_bk = div_s(u, a.hgroups);
          step_hg = (int)(u - step_bk * a.hgroups);
        }
        f += len;
      }
    }
    float cbv = 0.0f;
    if (tid < 16) cbv = tid < (1 << KB) ? a.kc[tid] : 0.0f;
    else if (tid < 32) cbv = tid - 16 < (1 << VB) ? a.vc[tid - 16] : 0.0f;
    else if (MX && tid < 40) cbv = a.kc2[tid - 32];
    else if (MX && tid < 48) cbv = a.vc2[tid - 40];
    asm volatile("bar.arrive 2, %0;\n" ::"n"((NW + 1) * 32) : "memory");  // the producer may start
    // ---- stage them in shared memory
#pragma unroll
    for (int k = 0; k < QPT; ++k) {
      const int i = tid + k * NW * 32;
      if (i < NSEG_PRE * HGN * D) sqm[i] = qr[k];
    }
    if (tid < 64) cbs[tid] = cbv;
    consumers_sync<NW>();
    // ---- q' = Pi q, then sq = S q'
    prologue_pass(m4, sqm, qpm);
    consumers_sync<NW>();
    if constexpr (QJL) {
      prologue_pass(s4, qpm, sqm);
      consumers_sync<NW>();
    }
    // ---- decode step: the new row of this CTA's unit end (its scratch is the B-fragment area,
    // which prep_frags fills only afterwards)
    if constexpr (STEP) {
      if (step_bk >= 0) {
        quantize_step_row<KB, VB, QJL, NB>(a, stx, sty, stn, strow, cbs, step_bk, step_hg, L);
        asm volatile("bar.arrive 3, %0;\n" ::"n"((NW + 1) * 32) : "memory");  // the producer may place it
      }
    }

    // ---- pair tables: entry e = lo | hi << b -> half2(c[lo], c[hi]), four lane replicas per
    // 16-byte store
    const uint32_t tbl = ctl.tbl_addr;
    unsigned char* tp = smem + (tbl - smem_u32(smem));
    if constexpr (Lut::kPacked) {
      for (int i = tid; i < 256 * 2 * 8; i += NW * 32) {  // (entry, half, group of four lanes)
        const int e = i >> 4, half = (i >> 3) & 1, q4 = i & 7;
        const float* cb = cbs + 16 * half;
        const uint32_t v = pack_half2(cb[e & 15], cb[e >> 4]);
        *reinterpret_cast<uint4*>(tp + e * 256 + half * 128 + 16 * q4) = make_uint4(v, v, v, v);
      }
      lut.rk = tbl | (4u * lane);
      lut.rv = tbl | 128u | (4u * lane);
      if constexpr (MX) {  // 3-bit pair tables of the other half: K at +0, V at +8 KB
        unsigned char* tp2 = smem + (ctl.tbl2_addr - smem_u32(smem));
        for (int i = tid; i < 2 * 64 * 8; i += NW * 32) {  // (table, entry, group of four lanes)
          const int isv = i >> 9, e = (i >> 3) & 63, q4 = i & 7;
          const float* cb = cbs + 32 + 8 * isv;
          const uint32_t v = pack_half2(cb[e & 7], cb[e >> 3]);
          *reinterpret_cast<uint4*>(tp2 + isv * 8192 + e * 128 + 16 * q4) = make_uint4(v, v, v, v);
        }
        lut.rk2 = ctl.tbl2_addr + 4u * lane;
        lut.rv2 = ctl.tbl2_addr + 8192u + 4u * lane;
      }
    } else {
      for (int i = tid; i < (Lay::K_TBL + Lay::V_TBL) / 16; i += NW * 32) {
        const bool isv = i >= Lay::K_TBL / 16;
        const int j = isv ? i - Lay::K_TBL / 16 : i;
        const int e = j >> 3;
        const int bits = isv ? VB : KB;
        const float* cb = cbs + (isv ? 16 : 0);
        const uint32_t v = pack_half2(cb[e & ((1 << bits) - 1)], cb[e >> bits]);
        *reinterpret_cast<uint4*>(tp + 16 * i) = make_uint4(v, v, v, v);
      }
      lut.rk = tbl + 4u * lane;
      lut.rv = tbl + Lay::K_TBL + 4u * lane;
    }
  }
  prep_frags();  // (its barriers also order the table stores before the first lookup)
  // the merge kernel may launch now; its CTAs wait for this grid to finish before reading
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  const int gq = lane >> 2, t = lane & 3;
  int slot = 0;
  uint32_t phase = 0;  // parity of the ring round being consumed
  int si = 0;          // this segment's index in the prep chunk
  for (int64_t f = f_begin; f < f_end; ++si) {
    if (si == NSEG_PRE) {  // the next chunk (every consumer warp is at this segment boundary)
      consumers_sync<NW>();  // the previous chunk's q' / S q' are read
      prep_chunk(f);
      si = 0;
    }
    const int64_t u = div_s(f, L);
    const int t0 = (int)(f - u * L);
    const int t1 = (int)(L < t0 + (f_end - f) ? L : t0 + (f_end - f));
    f += t1 - t0;
    const int bk = (int)div_s(u, a.hgroups), hg = (int)(u - (int64_t)bk * a.hgroups);
    const int b = bk / a.Hkv, kvh = bk % a.Hkv;
    const int h0 = kvh * a.g + hg * HG;
    const int nh = min(HG, a.g - hg * HG);

    // ---- B operands and per-head constants of this segment (built by prep_frags)
    uint32_t bq[NB][8][2], bsq[NB][8][2];
    float fK[NB], fQ[NB], Kh[NB];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const uint4* fp = reinterpret_cast<const uint4*>(frg) + (si * NB + nb) * 8 * 32 + lane;
#pragma unroll
      for (int w4 = 0; w4 < 8; ++w4) {
        const uint4 v = fp[w4 * 32];
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int word = 4 * w4 + j;
          if (word < 16) bq[nb][word >> 1][word & 1] = wv[j];
          else bsq[nb][(word >> 1) & 7][word & 1] = wv[j];
        }
      }
      const float4 hc = hcon[si * HGN + 4 * nb + t];
      fK[nb] = hc.x;
      fQ[nb] = hc.y;
      Kh[nb] = hc.z;
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
      m_run[nb] = -1e30f;  // finite: ex2(s - m) and ex2(m_old - m_new) never see inf - inf
      l_run[nb] = 0.0f;
    }

    for (int s0 = t0; s0 < t1; s0 += ST) {
      const bool ok = wait_w(ctl, &ctl.full[slot], phase);
      const int nvalid = min(16, t1 - s0 - 16 * warp);
      if (ok && nvalid > 0) {
        const unsigned char* stage = smem + ctl.stage_off[slot];
        const int r0 = 16 * warp + gq, r1 = r0 + 8;  // this lane's token rows in the stage

        // Value codes of the lane's four tokens (rows 2t, 2t+1, 2t+8, 2t+9 of the warp's 16), paired
        // for the value MMAs.  With 4-bit values and one n-block they are loaded before the score
        // MMAs, which do not depend on them, so they fill the MMA chains' latency (2% at 128K x 4);
        // otherwise (measured slower with two n-blocks) they are loaded after the softmax.
        constexpr bool EARLY_V = VB == 4 && NB == 1;
        VPairs<VB> p01, p89;
        auto load_vpairs = [&]() {
          const unsigned char* vbase = stage + Lay::OFF_VC + (16 * warp) * Lay::V_ROW;
          uint64_t cv0, cv1, cv2, cv3;
          if constexpr (VB == 4) {
            // lanes with odd t read their odd row first, so that in each load the four t-lanes
            // of a column group hit two bank groups instead of one (64-byte rows)
            const int sw = t & 1;
            const uint2 a0 = lds64(vbase + (2 * t + sw) * Lay::V_ROW + 8 * gq);
            const uint2 a1 = lds64(vbase + (2 * t + 1 - sw) * Lay::V_ROW + 8 * gq);
            const uint2 a2 = lds64(vbase + (2 * t + 8 + sw) * Lay::V_ROW + 8 * gq);
            const uint2 a3 = lds64(vbase + (2 * t + 9 - sw) * Lay::V_ROW + 8 * gq);
            const uint64_t x0 = (uint64_t)a0.x | ((uint64_t)a0.y << 32), x1 = (uint64_t)a1.x | ((uint64_t)a1.y << 32);
            const uint64_t x2 = (uint64_t)a2.x | ((uint64_t)a2.y << 32), x3 = (uint64_t)a3.x | ((uint64_t)a3.y << 32);
            cv0 = sw ? x1 : x0;
            cv1 = sw ? x0 : x1;
            cv2 = sw ? x3 : x2;
            cv3 = sw ? x2 : x3;
          } else {
            cv0 = load_v_chunk<VB>(vbase + (2 * t) * Lay::V_ROW, gq);
            cv1 = load_v_chunk<VB>(vbase + (2 * t + 1) * Lay::V_ROW, gq);
            cv2 = load_v_chunk<VB>(vbase + (2 * t + 8) * Lay::V_ROW, gq);
            cv3 = load_v_chunk<VB>(vbase + (2 * t + 9) * Lay::V_ROW, gq);
          }
          p01.build(cv0, cv1);
          p89.build(cv2, cv3);
        };
        if constexpr (!MX && EARLY_V) load_vpairs();

        // ---- scores for tokens r0, r1 and heads 4nb + t ----
        // two accumulators per product (even / odd k-steps) halve the dependent MMA chains
        float kacc[NB][4], qacc[NB][4], kacc2[NB][4], qacc2[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
          for (int e = 0; e < 4; ++e) kacc[nb][e] = qacc[nb][e] = kacc2[nb][e] = qacc2[nb][e] = 0.0f;
        if constexpr (MX) {
          // outlier half: 16 4-bit codes at byte 8t (k-steps 0..3, the packed table, accumulated in
          // kacc); other half: 16 3-bit codes at byte 32 + 6t (k-steps 4..7, kacc2)
          const unsigned char* k0 = stage + Lay::OFF_KC + r0 * Lay::K_ROW;
          const unsigned char* k1 = stage + Lay::OFF_KC + r1 * Lay::K_ROW;
          const uint2 o0 = lds64(k0 + 8 * t), o1 = lds64(k1 + 8 * t);
          const uint32_t c0[2] = {o0.x, o0.y}, c1[2] = {o1.x, o1.y};
          const int rb = 32 + 6 * t, ra = rb & ~3, rsh = 8 * (rb & 3);  // (rb & 3) is 0 or 2
          const uint64_t g0 = ((uint64_t)lds32(smem_u32(k0 + ra + 4)) << 32 | lds32(smem_u32(k0 + ra))) >> rsh;
          const uint64_t g1 = ((uint64_t)lds32(smem_u32(k1 + ra + 4)) << 32 | lds32(smem_u32(k1 + ra))) >> rsh;
#define TQ_KSTEP_O(KK)                                                                       \
          {                                                                                  \
            const uint32_t A[4] = {lut.template k_byte<(2 * (KK)) & 3>(c0[(2 * (KK)) >> 2]),   \
                                   lut.template k_byte<(2 * (KK)) & 3>(c1[(2 * (KK)) >> 2]),   \
                                   lut.template k_byte<(2 * (KK) + 1) & 3>(c0[(2 * (KK) + 1) >> 2]), \
                                   lut.template k_byte<(2 * (KK) + 1) & 3>(c1[(2 * (KK) + 1) >> 2])}; \
            _Pragma("unroll") for (int nb = 0; nb < NB; ++nb)                                \
                mma16816(kacc[nb], A, bq[nb][KK][0], bq[nb][KK][1]);                           \
          }
#define TQ_KSTEP_R(KK)                                                                       \
          {                                                                                  \
            const uint32_t A[4] = {lut.k2((uint32_t)(g0 >> (12 * ((KK) - 4))) & 63u),          \
                                   lut.k2((uint32_t)(g1 >> (12 * ((KK) - 4))) & 63u),          \
                                   lut.k2((uint32_t)(g0 >> (12 * ((KK) - 4) + 6)) & 63u),      \
                                   lut.k2((uint32_t)(g1 >> (12 * ((KK) - 4) + 6)) & 63u)};     \
            _Pragma("unroll") for (int nb = 0; nb < NB; ++nb)                                \
                mma16816(kacc2[nb], A, bq[nb][KK][0], bq[nb][KK][1]);                          \
          }
          TQ_KSTEP_O(0) TQ_KSTEP_O(1) TQ_KSTEP_O(2) TQ_KSTEP_O(3) TQ_KSTEP_R(4) TQ_KSTEP_R(5) TQ_KSTEP_R(6) TQ_KSTEP_R(7)
#undef TQ_KSTEP_O
#undef TQ_KSTEP_R
        } else {
          uint32_t c0[KB], c1[KB];
          const unsigned char* k0 = stage + Lay::OFF_KC + r0 * Lay::K_ROW + 4 * KB * t;
          const unsigned char* k1 = stage + Lay::OFF_KC + r1 * Lay::K_ROW + 4 * KB * t;
          if constexpr (KB == 4) {
            const uint4 x0 = lds128(k0), x1 = lds128(k1);
            c0[0] = x0.x; c0[1] = x0.y; c0[2] = x0.z; c0[3] = x0.w;
            c1[0] = x1.x; c1[1] = x1.y; c1[2] = x1.z; c1[3] = x1.w;
          } else if constexpr (KB == 2) {
            const uint2 x0 = lds64(k0), x1 = lds64(k1);
            c0[0] = x0.x; c0[1] = x0.y;
            c1[0] = x1.x; c1[1] = x1.y;
          } else {
#pragma unroll
            for (int i = 0; i < KB; ++i) {
              c0[i] = reinterpret_cast<const uint32_t*>(k0)[i];
              c1[i] = reinterpret_cast<const uint32_t*>(k1)[i];
            }
          }
#define TQ_KSTEP(KK)                                                                         \
          {                                                                                  \
            const uint32_t A[4] = {k_pair<KB, VB, 2 * (KK)>(lut, c0), k_pair<KB, VB, 2 * (KK)>(lut, c1), \
                                   k_pair<KB, VB, 2 * (KK) + 1>(lut, c0),                    \
                                   k_pair<KB, VB, 2 * (KK) + 1>(lut, c1)};                   \
            _Pragma("unroll") for (int nb = 0; nb < NB; ++nb)                                \
                mma16816((KK) & 1 ? kacc2[nb] : kacc[nb], A, bq[nb][KK][0], bq[nb][KK][1]);    \
          }
          TQ_KSTEP(0) TQ_KSTEP(1) TQ_KSTEP(2) TQ_KSTEP(3) TQ_KSTEP(4) TQ_KSTEP(5) TQ_KSTEP(6) TQ_KSTEP(7)
#undef TQ_KSTEP
        }
        if constexpr (QJL) {
          const uint32_t w0 = *reinterpret_cast<const uint32_t*>(stage + Lay::OFF_SG + r0 * 16 + 4 * t);
          const uint32_t w1 = *reinterpret_cast<const uint32_t*>(stage + Lay::OFF_SG + r1 * 16 + 4 * t);
#define TQ_SSTEP(KK)                                                                         \
          {                                                                                  \
            const uint32_t A[4] = {sgn<2 * (KK)>(w0), sgn<2 * (KK)>(w1), sgn<2 * (KK) + 1>(w0), \
                                   sgn<2 * (KK) + 1>(w1)};                                   \
            _Pragma("unroll") for (int nb = 0; nb < NB; ++nb)                                \
                mma16816((KK) & 1 ? qacc2[nb] : qacc[nb], A, bsq[nb][KK][0], bsq[nb][KK][1]);  \
          }
          TQ_SSTEP(0) TQ_SSTEP(1) TQ_SSTEP(2) TQ_SSTEP(3) TQ_SSTEP(4) TQ_SSTEP(5) TQ_SSTEP(6) TQ_SSTEP(7)
#undef TQ_SSTEP
        }

        // ---- online softmax (log2 units) per head 4nb + t over this warp's 16 tokens ----
        const bool v0ok = gq < nvalid, v1ok = gq + 8 < nvalid;
        // (mixed layout: two norms per token, the outlier half's first)
        const float nk0 = *reinterpret_cast<const float*>(stage + Lay::OFF_NK + Lay::NORM * r0);
        const float nk1 = *reinterpret_cast<const float*>(stage + Lay::OFF_NK + Lay::NORM * r1);
        const float nk0b = MX ? *reinterpret_cast<const float*>(stage + Lay::OFF_NK + Lay::NORM * r0 + 4) : 0.0f;
        const float nk1b = MX ? *reinterpret_cast<const float*>(stage + Lay::OFF_NK + Lay::NORM * r1 + 4) : 0.0f;
        float rn0 = 0.0f, rn1 = 0.0f;
        if constexpr (QJL) {
          rn0 = *reinterpret_cast<const float*>(stage + Lay::OFF_RN + 4 * r0);
          rn1 = *reinterpret_cast<const float*>(stage + Lay::OFF_RN + 4 * r1);
        }
        // rows past the segment's end hold stale or uninitialised words: their weight is 0 and
        // their value scale too, so nothing of them reaches the sums
        // value scale ||v|| / sqrt(128) (mixed layout: ||v_g|| / 8 of each half)
        constexpr float VSC = MX ? 0.125f : 0.08838834764831845f;
        const float nv0 = v0ok ? *reinterpret_cast<const float*>(stage + Lay::OFF_NV + Lay::NORM * r0) * VSC : 0.0f;
        const float nv1 = v1ok ? *reinterpret_cast<const float*>(stage + Lay::OFF_NV + Lay::NORM * r1) * VSC : 0.0f;
        const float nv0b = (MX && v0ok) ? *reinterpret_cast<const float*>(stage + Lay::OFF_NV + Lay::NORM * r0 + 4) * VSC : 0.0f;
        const float nv1b = (MX && v1ok) ? *reinterpret_cast<const float*>(stage + Lay::OFF_NV + Lay::NORM * r1 + 4) * VSC : 0.0f;
        uint32_t bp[NB][2], bp2[NB][2];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          float s0v, s1v;
          if constexpr (MX) {  // the halves carry their own norms
            s0v = fmaf(kacc2[nb][0] + kacc2[nb][1], nk0b * fK[nb], (kacc[nb][0] + kacc[nb][1]) * (nk0 * fK[nb]));
            s1v = fmaf(kacc2[nb][2] + kacc2[nb][3], nk1b * fK[nb], (kacc[nb][2] + kacc[nb][3]) * (nk1 * fK[nb]));
          } else {
            s0v = ((kacc[nb][0] + kacc2[nb][0]) + (kacc[nb][1] + kacc2[nb][1])) * (nk0 * fK[nb]);
            s1v = ((kacc[nb][2] + kacc2[nb][2]) + (kacc[nb][3] + kacc2[nb][3])) * (nk1 * fK[nb]);
          }
          if constexpr (QJL) {
            s0v = fmaf(((qacc[nb][0] + qacc2[nb][0]) + (qacc[nb][1] + qacc2[nb][1])) + Kh[nb], rn0 * fQ[nb], s0v);
            s1v = fmaf(((qacc[nb][2] + qacc2[nb][2]) + (qacc[nb][3] + qacc2[nb][3])) + Kh[nb], rn1 * fQ[nb], s1v);
          }
          s0v = v0ok ? s0v : -INFINITY;
          s1v = v1ok ? s1v : -INFINITY;
          float mx = fmaxf(s0v, s1v);
          mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 16));
          if (mx > m_run[nb]) {  // uniform over the 8 lanes of head 4nb + t
            const float alpha = ex2(m_run[nb] - mx);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              oacc[nb][i][0] *= alpha;
              oacc[nb][i][1] *= alpha;
              oacc[nb][i][2] *= alpha;
              oacc[nb][i][3] *= alpha;
            }
            l_run[nb] *= alpha;
            m_run[nb] = mx;
          }
          const float p0 = ex2(s0v - m_run[nb]);  // ex2(-inf) = 0 for rows past the end
          const float p1 = ex2(s1v - m_run[nb]);
          l_run[nb] += p0 + p1;
          // P~ = p nV / sqrt(d) as fp16 hi + lo: row token, columns (head t, hi) and (head t, lo)
          bp[nb][0] = movmatrix_trans(hilo_half2(p0 * nv0));  // tokens 2t, 2t+1 of column gq
          bp[nb][1] = movmatrix_trans(hilo_half2(p1 * nv1));  // tokens 2t+8, 2t+9
          if constexpr (MX) {  // the other half's values: their own scale
            bp2[nb][0] = movmatrix_trans(hilo_half2(p0 * nv0b));
            bp2[nb][1] = movmatrix_trans(hilo_half2(p1 * nv1b));
          }
        }

        // ---- O'^T += Vhat^T P~: dim blocks of 16; A holds token pairs (2t,2t+1), (2t+8,2t+9) ----
        if constexpr (MX) {
          // lane group gq: outlier half, 8 4-bit codes at byte 4gq (dim blocks 0..3); other half,
          // 8 3-bit codes at byte 32 + 3gq (dim blocks 4..7)
          const unsigned char* vbase = stage + Lay::OFF_VC + (16 * warp) * Lay::V_ROW;
          const int rb = 32 + 3 * gq, ra = rb & ~3, rsh = 8 * (rb & 3);
          uint32_t vo[4], vr[4];
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const unsigned char* row = vbase + (2 * t + (k4 & 1) + 8 * (k4 >> 1)) * Lay::V_ROW;
            vo[k4] = lds32(smem_u32(row + 4 * gq));
            vr[k4] = (uint32_t)((((uint64_t)lds32(smem_u32(row + ra + 4)) << 32) | lds32(smem_u32(row + ra))) >> rsh);
          }
          // token pairs (2t, 2t+1) and (2t+8, 2t+9): codes of both tokens interleaved per byte
          const uint32_t w01e = (vo[0] & 0x0F0F0F0Fu) | ((vo[1] << 4) & 0xF0F0F0F0u);
          const uint32_t w01o = ((vo[0] >> 4) & 0x0F0F0F0Fu) | (vo[1] & 0xF0F0F0F0u);
          const uint32_t w89e = (vo[2] & 0x0F0F0F0Fu) | ((vo[3] << 4) & 0xF0F0F0F0u);
          const uint32_t w89o = ((vo[2] >> 4) & 0x0F0F0F0Fu) | (vo[3] & 0xF0F0F0F0u);
#define TQ_VSTEP_O(DB)                                                                        \
          {                                                                                   \
            const uint32_t A[4] = {lut.template v_byte<DB>(w01e), lut.template v_byte<DB>(w01o), \
                                   lut.template v_byte<DB>(w89e), lut.template v_byte<DB>(w89o)}; \
            _Pragma("unroll") for (int nb = 0; nb < NB; ++nb)                                 \
                mma16816(oacc[nb][DB], A, bp[nb][0], bp[nb][1]);                               \
          }
#define TQ_VPAIR_R(X, Y, NU) (((X >> (3 * (NU))) & 7u) | (((Y >> (3 * (NU))) & 7u) << 3))
#define TQ_VSTEP_R(DB)                                                                        \
          {                                                                                   \
            const uint32_t A[4] = {lut.v2(TQ_VPAIR_R(vr[0], vr[1], 2 * ((DB) - 4))),           \
                                   lut.v2(TQ_VPAIR_R(vr[0], vr[1], 2 * ((DB) - 4) + 1)),       \
                                   lut.v2(TQ_VPAIR_R(vr[2], vr[3], 2 * ((DB) - 4))),           \
                                   lut.v2(TQ_VPAIR_R(vr[2], vr[3], 2 * ((DB) - 4) + 1))};      \
            _Pragma("unroll") for (int nb = 0; nb < NB; ++nb)                                 \
                mma16816(oacc[nb][DB], A, bp2[nb][0], bp2[nb][1]);                             \
          }
          TQ_VSTEP_O(0) TQ_VSTEP_O(1) TQ_VSTEP_O(2) TQ_VSTEP_O(3) TQ_VSTEP_R(4) TQ_VSTEP_R(5) TQ_VSTEP_R(6) TQ_VSTEP_R(7)
#undef TQ_VSTEP_O
#undef TQ_VSTEP_R
#undef TQ_VPAIR_R
        } else {
          if constexpr (!EARLY_V) load_vpairs();
#define TQ_VSTEP(DB)                                                                          \
          {                                                                                   \
            const uint32_t A[4] = {v_pair<KB, VB, 2 * (DB)>(lut, p01), v_pair<KB, VB, 2 * (DB) + 1>(lut, p01), \
                                   v_pair<KB, VB, 2 * (DB)>(lut, p89), v_pair<KB, VB, 2 * (DB) + 1>(lut, p89)}; \
            _Pragma("unroll") for (int nb = 0; nb < NB; ++nb)                                 \
                mma16816(oacc[nb][DB], A, bp[nb][0], bp[nb][1]);                               \
          }
          TQ_VSTEP(0) TQ_VSTEP(1) TQ_VSTEP(2) TQ_VSTEP(3) TQ_VSTEP(4) TQ_VSTEP(5) TQ_VSTEP(6) TQ_VSTEP(7)
#undef TQ_VSTEP
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_(&ctl.empty[slot]);
      if (++slot == ns) {
        slot = 0;
        phase ^= 1u;
      }
    }

    // ---- partials.  Per head, slots 0 .. pmax-1 hold one (max, sum, o') partial per CTA that ends
    // inside the head's unit (slot j: the CTA's index among the unit's CTAs), and slots pmax ..
    // pmax + NW - 1 the per-warp partials of the one CTA that streams the unit's last token and
    // goes on to the next unit.  So a segment that is not the CTA's last costs no barrier, and
    // the CTA's last one merges its warps through the (then free) ring memory.
    const int64_t hstride = (int64_t)(a.pmax + NW) * PART;
    if (f < f_end) {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const int hh = 4 * nb + t;
        float lq = l_run[nb];
        lq += __shfl_xor_sync(FULL, lq, 4);
        lq += __shfl_xor_sync(FULL, lq, 8);
        lq += __shfl_xor_sync(FULL, lq, 16);
#ifdef TQ_DEBUG
        if (hh < nh && (int64_t)b * a.Hq + h0 + hh >= (int64_t)a.B * a.Hq) {
          if (gq == 0) atomicOr(&g_decode_error, 8u);
          continue;
        }
#endif
        if (hh < nh) {
          float* dst = a.part + ((int64_t)b * a.Hq + h0 + hh) * hstride + (a.pmax + warp) * PART;
          if (gq == 0) {
            dst[0] = m_run[nb];
            dst[1] = lq;
          }
#pragma unroll
          for (int db = 0; db < 8; ++db) {
            dst[4 + 16 * db + gq] = oacc[nb][db][0] + oacc[nb][db][1];
            dst[4 + 16 * db + 8 + gq] = oacc[nb][db][2] + oacc[nb][db][3];
          }
        }
      }
    } else {
      const int j = c - part_cta_of(a.ntot, a.ctas, u * L);
      float* mw = reinterpret_cast<float*>(smem + ctl.merge_off);  // [NW][4]
      float* lw = mw + NW * 4;                                       // [NW][4]
      float* ow = lw + NW * 4;                                       // [NW][4][D]
      consumers_sync<NW>();  // every warp is past its last stage: the ring is free
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        float lq = l_run[nb];
        lq += __shfl_xor_sync(FULL, lq, 4);
        lq += __shfl_xor_sync(FULL, lq, 8);
        lq += __shfl_xor_sync(FULL, lq, 16);
        if (gq == 0) {
          mw[warp * 4 + t] = m_run[nb];
          lw[warp * 4 + t] = lq;
        }
        float* o = ow + (warp * 4 + t) * D;
#pragma unroll
        for (int db = 0; db < 8; ++db) {
          o[16 * db + gq] = oacc[nb][db][0] + oacc[nb][db][1];
          o[16 * db + 8 + gq] = oacc[nb][db][2] + oacc[nb][db][3];
        }
        consumers_sync<NW>();
        for (int idx = tid; idx < 4 * D; idx += NW * 32) {
          const int r = idx / D, dd = idx % D;
#ifdef TQ_DEBUG
          if (4 * nb + r < nh && (j < 0 || j >= a.pmax || (int64_t)b * a.Hq + h0 + 4 * nb + r >= (int64_t)a.B * a.Hq)) {
            atomicOr(&g_decode_error, 8u);
            continue;
          }
#endif
          if (4 * nb + r < nh) {
            float M = -1e30f;
#pragma unroll
            for (int w = 0; w < NW; ++w) M = fmaxf(M, mw[w * 4 + r]);
            float Ls = 0.0f, O = 0.0f;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
              const float fw = ex2(mw[w * 4 + r] - M);
              Ls = fmaf(fw, lw[w * 4 + r], Ls);
              O = fmaf(fw, ow[(w * 4 + r) * D + dd], O);
            }
            float* dst = a.part + ((int64_t)b * a.Hq + h0 + 4 * nb + r) * hstride + (int64_t)j * PART;
            dst[4 + dd] = O;
            if (dd == 0) {
              dst[0] = M;
              dst[1] = Ls;
            }
          }
        }
        if (nb + 1 < NB) consumers_sync<NW>();  // the area is reused by the next n-block
      }
    }
  }
  if (tid == 0 && *reinterpret_cast<volatile unsigned int*>(&ctl.err)) atomicOr(&g_decode_error, 1u);
}

// ------------------------------------------------------------------------------------------ merge

// One 1024-thread CTA per (batch, query head), a programmatic dependent of the split kernel: it
// waits for the split grid, merges the head's partials (see the split kernel's end) by
// log-sum-exp and writes o = Pi^T o'.  Thread (d, q),
// d = tid % 128 and q = tid / 128, takes the partials s = q (mod 8) of dimension d with a running
// maximum; its loads do not depend on one another, so they issue together.  The eight groups are
// then combined per dimension.  The un-rotation gives thread (i, q) the rows 16q .. 16q + 15 of Pi,
// loaded before the wait.
constexpr int MERGE_GROUPS = 8;
constexpr int MERGE_THREADS = MERGE_GROUPS * D;
constexpr int MERGE_ROWS = D / MERGE_GROUPS;

// (The partials are written by the still-running split grid: they are read with ld.global.cg,
// through L2 only, never through the non-coherent read-only path.)
__global__ void __launch_bounds__(MERGE_THREADS) merge_kernel(const float* part, const float* __restrict__ Pi,
                                                              float* __restrict__ out, int Hq, int g, int Hkv,
                                                              int hgroups, int64_t seq_len, int64_t ntot, int ctas,
                                                              int pmax, int nw) {
  __shared__ float mq[MERGE_GROUPS][D], lq[MERGE_GROUPS][D], oq[MERGE_GROUPS][D], ob[D];
  const int tid = threadIdx.x, d = tid % D, q = tid / D;
  const int64_t bh = blockIdx.x;
  if (seq_len == 0) {  // empty context: the output is zero (no split grid ran)
    if (tid < D) out[bh * D + d] = 0.0f;
    return;
  }
  // Pi is an input, not an output of split: its rows load while the split grid finishes
  float pj[MERGE_ROWS];
#pragma unroll
  for (int jj = 0; jj < MERGE_ROWS; ++jj) pj[jj] = __ldg(Pi + (MERGE_ROWS * q + jj) * D + d);
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  const int b = (int)(bh / Hq), h = (int)(bh % Hq);
  const int64_t u = ((int64_t)b * Hkv + h / g) * hgroups + (h % g) / HG;
  const int first = part_cta_of(ntot, ctas, u * seq_len);
  const int last = part_cta_of(ntot, ctas, u * seq_len + seq_len - 1);
  // the last CTA wrote per-warp partials (slots pmax ..) when its range goes on past the unit
  const bool past = part_start(ntot, ctas, last + 1) > (u + 1) * seq_len;
  const int S = last - first + (past ? nw : 1);
  const float* p = part + bh * (pmax + nw) * PART;
  float M = -1e30f, Ls = 0.0f, O = 0.0f;
#pragma unroll 4
  for (int s2 = q; s2 < S; s2 += MERGE_GROUPS) {
    const int slot = s2 < last - first ? s2 : (past ? pmax + s2 - (last - first) : s2);
    const float2 ml = __ldcg(reinterpret_cast<const float2*>(p + (int64_t)slot * PART));
    const float o = __ldcg(p + (int64_t)slot * PART + 4 + d);
    const float Mn = fmaxf(M, ml.x);
    const float a0 = ex2(M - Mn), a1 = ex2(ml.x - Mn);
    Ls = fmaf(a1, ml.y, Ls * a0);
    O = fmaf(a1, o, O * a0);
    M = Mn;
  }
  mq[q][d] = M;
  lq[q][d] = Ls;
  oq[q][d] = O;
  __syncthreads();
  if (tid < D) {
    float Mx = mq[0][d];
#pragma unroll
    for (int k = 1; k < MERGE_GROUPS; ++k) Mx = fmaxf(Mx, mq[k][d]);
    float Lt = 0.0f, Ot = 0.0f;
#pragma unroll
    for (int k = 0; k < MERGE_GROUPS; ++k) {
      const float w = ex2(mq[k][d] - Mx);
      Lt = fmaf(w, lq[k][d], Lt);
      Ot = fmaf(w, oq[k][d], Ot);
    }
    ob[d] = Lt > 0.0f ? Ot / Lt : 0.0f;
  }
  __syncthreads();
  // o_i = sum_j Pi[j][i] o'_j, thread (i = d, q) over rows MERGE_ROWS q ..
  float r = 0.0f;
#pragma unroll
  for (int jj = 0; jj < MERGE_ROWS; ++jj) r = fmaf(pj[jj], ob[MERGE_ROWS * q + jj], r);
  mq[q][d] = r;  // (the combine above has read mq: a barrier separates them)
  __syncthreads();
  if (tid < D) {
    float acc = 0.0f;
#pragma unroll
    for (int k = 0; k < MERGE_GROUPS; ++k) acc += mq[k][d];
    out[bh * D + d] = acc;
  }
}

// ------------------------------------------------------------------------------------------ host

struct Plan {
  int hgroups, units, ctas, pmax;
  int64_t ntot;
};

int device_attr(cudaDeviceAttr attr, int fallback) {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&v, attr, dev) != cudaSuccess || v <= 0) {
    cudaGetLastError();
    return fallback;
  }
  return v;
}
int device_sms() { return device_attr(cudaDevAttrMultiProcessorCount, 148); }
// Dynamic shared memory of a split CTA: all an SM gives one block, in whole 256-byte units.
int split_dyn_smem() { return device_attr(cudaDevAttrMaxSharedMemoryPerBlockOptin, 232448) / 256 * 256; }

Plan make_plan(int B, int Hq, int Hkv, int seq_len, int sms) {
  Plan p;
  const int g = Hq / Hkv;
  p.hgroups = (g + HG - 1) / HG;
  p.units = B * Hkv * p.hgroups;
  p.ntot = (int64_t)p.units * seq_len;
  if (seq_len <= 0) {
    p.ctas = 0;
    p.pmax = 0;
    return p;
  }
  int64_t c = p.ntot / MIN_TOK_PER_CTA;
  if (c > sms) c = sms;
  if (c < 1) c = 1;
  p.ctas = (int)c;
  // partial slots per head: the most CTA ranges one unit meets (exact for up to 2^16 units)
  if (p.units <= (1 << 16)) {
    int pm = 1;
    for (int64_t u = 0; u < p.units; ++u) {
      const int n = part_cta_of(p.ntot, p.ctas, u * seq_len + seq_len - 1) - part_cta_of(p.ntot, p.ctas, u * seq_len) + 1;
      pm = n > pm ? n : pm;
    }
    p.pmax = pm;
  } else {  // ranges are at least floor(N / C) >= MIN_TOK_PER_CTA long
    const int64_t minlen = p.ntot / p.ctas;
    p.pmax = (int)std::min<int64_t>(p.ctas, (seq_len + minlen - 1) / minlen + 1);
  }
  return p;
}

// Consumer warps of a split CTA for groups of g query heads per kv-head.
int split_warps(int g) { return g <= 4 ? Shape<1>::NW : Shape<2>::NW; }

// Workspace: the partials [B*Hq][pmax + NW][132] fp32: one per CTA that ends inside the head's
// unit, plus one per consumer warp of the CTA that streams past the unit's end.
size_t workspace_bytes(int B, int Hq, int g, const Plan& p) {
  return sizeof(float) * (size_t)B * Hq * (p.pmax + split_warps(g)) * PART;
}

template <int KB, int VB, bool QJL, int NB, bool MX, bool STEP>
tq_status launch_split_nb(const DArgs& a0, cudaStream_t stream) {
  DArgs a = a0;
  // dynamic shared memory usually starts right after the per-block reserved bytes
  plan_layout<KB, VB, QJL, NB, MX>((uint32_t)device_attr(cudaDevAttrReservedSharedMemoryPerBlock, 1024),
                                   a.dyn_smem, a.plan);
  cudaError_t e = cudaFuncSetAttribute(split_kernel<KB, VB, QJL, NB, MX, STEP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       a.dyn_smem);
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "smem attribute: %s", cudaGetErrorString(e));
  // an ordinary launch: the cache it reads may come from the kernel just before (tq_quantize)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.ctas);
  cfg.blockDim = dim3(Shape<NB>::THREADS);
  cfg.dynamicSmemBytes = a.dyn_smem;
  cfg.stream = stream;
  e = cudaLaunchKernelEx(&cfg, split_kernel<KB, VB, QJL, NB, MX, STEP>, a);
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "split launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}

// One n-block of four heads when a group has at most four query heads, else two (split_warps).
template <int KB, int VB, bool QJL, bool MX = false>
tq_status launch_split(const DArgs& a, cudaStream_t stream) {
  if constexpr (!MX) {
    if (a.step)
      return a.g <= 4 ? launch_split_nb<KB, VB, QJL, 1, false, true>(a, stream)
                      : launch_split_nb<KB, VB, QJL, 2, false, true>(a, stream);
  }
  return a.g <= 4 ? launch_split_nb<KB, VB, QJL, 1, MX, false>(a, stream)
                  : launch_split_nb<KB, VB, QJL, 2, MX, false>(a, stream);
}

template <int KB, bool QJL>
tq_status dispatch_v(int vb, const DArgs& a, cudaStream_t s) {
  switch (vb) {
    case 2: return launch_split<KB, 2, QJL>(a, s);
    case 3: return launch_split<KB, 3, QJL>(a, s);
    default: return launch_split<KB, 4, QJL>(a, s);
  }
}

template <bool QJL>
tq_status dispatch(int kb, int vb, bool mixed, const DArgs& a, cudaStream_t s) {
  if (mixed) return launch_split<4, 4, QJL, true>(a, s);  // (the mixed layout is checked to be 4 / 4)
  switch (kb) {
    case 2: return dispatch_v<2, QJL>(vb, a, s);
    case 3: return dispatch_v<3, QJL>(vb, a, s);
    default: return dispatch_v<4, QJL>(vb, a, s);
  }
}

}  // namespace
}  // namespace tq

extern "C" size_t tq_decode_workspace_size(int B, int Hq, const tq_cache* cache, int seq_len) {
  using namespace tq;
  if (!cache || B < 1 || Hq < 1 || cache->Hkv < 1 || Hq % cache->Hkv || seq_len < 0) return 0;
  const Plan p = make_plan(B, Hq, cache->Hkv, seq_len, device_sms());
  return workspace_bytes(B, Hq, Hq / cache->Hkv, p);
}

namespace tq {
int decode_reset_errors() {
  const unsigned int z = 0;
  return cudaMemcpyToSymbol(g_decode_error, &z, sizeof(z)) == cudaSuccess ? 0 : -1;
}
}  // namespace tq

extern "C" int tq_decode_device_errors(void) {
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, tq::g_decode_error, sizeof(v)) != cudaSuccess) return -1;
  return (int)v;
}

namespace tq {
namespace {
// The new token of a fused decode step: [B, Hkv, 128] key and value of kv_dtype.
struct StepIn {
  const void* k_new;
  const void* v_new;
  int kv_dtype;
};

// A decode step runs fused (the new row quantized inside the split kernel) when every CTA's range
// holds at most NSEG_PRE segments and at most one unit end: the prologue then computes the one new
// row the CTA needs.  Other sizes (short contexts over many units) take quantize + decode.
bool step_fusable(const Plan& p, int64_t L) {
  if (p.ctas <= 0 || L <= 0) return false;
  for (int c = 0; c < p.ctas; ++c) {
    const int64_t f0 = part_start(p.ntot, p.ctas, c), f1 = part_start(p.ntot, p.ctas, c + 1);
    if (f1 <= f0) continue;
    if ((f1 - 1) / L - f0 / L + 1 > NSEG_PRE || f1 / L - f0 / L > 1) return false;
  }
  return true;
}

tq_status decode_impl(const tq_params* params, const void* q, int q_dtype, int Hq, const tq_cache* cache,
                      int seq_len, float scale, float* out, void* workspace, size_t ws_bytes, void* stream,
                      const StepIn* step);
}  // namespace
}  // namespace tq

extern "C" tq_status tq_decode_attn(const tq_params* params, const void* q, int q_dtype, int Hq,
                                    const tq_cache* cache, int seq_len, float scale, float* out,
                                    void* workspace, size_t ws_bytes, void* stream) {
  using namespace tq;
  const NvtxRange nvtx_range("tq_decode_attn");
  clear_error();
  return decode_impl(params, q, q_dtype, Hq, cache, seq_len, scale, out, workspace, ws_bytes, stream, nullptr);
}

namespace tq {
namespace {
tq_status decode_impl(const tq_params* params, const void* q, int q_dtype, int Hq, const tq_cache* cache,
                      int seq_len, float scale, float* out, void* workspace, size_t ws_bytes, void* stream,
                      const StepIn* step) {
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
  const Plan plan = make_plan(B, Hq, cache->Hkv, seq_len, device_sms());
  const size_t need = workspace_bytes(B, Hq, Hq / cache->Hkv, plan);
  if (ws_bytes < need)
    return fail(TQ_ERR_WORKSPACE, "workspace %zu bytes, need %zu", ws_bytes, need);

  const float sc = scale > 0.0f ? scale : 1.0f / sqrtf((float)D);
  float* ws = reinterpret_cast<float*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int BH = B * Hq;
  const int g = Hq / cache->Hkv;
  cudaError_t e = cudaSuccess;
  if (seq_len > 0) {
    DArgs a;
    a.B = B;
    a.Hq = Hq;
    a.Hkv = cache->Hkv;
    a.g = g;
    a.hgroups = plan.hgroups;
    a.T_cap = cache->T_cap;
    a.seq_len = seq_len;
    a.units = plan.units;
    a.ctas = plan.ctas;
    a.pmax = plan.pmax;
    a.ntot = plan.ntot;
    a.dyn_smem = split_dyn_smem();
    // (a.plan is filled per layout at launch)
    // k-hat = ||k|| / sqrt(128) c (mixed layout: ||k_g|| / sqrt(64) c_g of each half)
    a.sK = (float)((double)sc * 1.4426950408889634 / sqrt(cache->layout == TQ_LAYOUT_MIXED ? 64.0 : (double)D));
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
    a.kc2 = params->k_centroids_lo;
    a.vc2 = params->v_centroids_lo;
    a.q = q;
    a.q_bf16 = q_dtype == TQ_BF16 ? 1 : 0;
    a.Pi = params->Pi;
    a.S = params->S;
    a.part = ws;
    a.step = step ? 1 : 0;
    a.kv_bf16 = step && step->kv_dtype == TQ_BF16 ? 1 : 0;
    a.k_new = step ? step->k_new : nullptr;
    a.v_new = step ? step->v_new : nullptr;
    a.kt = params->k_thresholds;
    a.vt = params->v_thresholds;
    const bool mixed = cache->layout == TQ_LAYOUT_MIXED;
    st = cache->qjl_m ? dispatch<true>(cache->k_bits, cache->v_bits, mixed, a, s)
                      : dispatch<false>(cache->k_bits, cache->v_bits, mixed, a, s);
    if (st != TQ_OK) return st;
  }
  // merge: programmatic dependent of split (its CTAs wait for the split grid before reading); with
  // an empty context it only writes zeros
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(BH);
  cfg.blockDim = dim3(MERGE_THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = seq_len > 0 ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, merge_kernel, (const float*)ws, params->Pi, out, Hq, g,
                         cache->Hkv, plan.hgroups, (int64_t)seq_len, plan.ntot, plan.ctas, plan.pmax,
                         split_warps(g));
  if (e != cudaSuccess) return fail(TQ_ERR_CUDA, "merge launch: %s", cudaGetErrorString(e));
  return TQ_OK;
}
}  // namespace
}  // namespace tq

// One decode step: append the new token (tq_quantize with T_new = 1), then attend over t + 1
// tokens.  The decode arguments are checked first so that an invalid call enqueues nothing.
extern "C" int tq_decode_step_fused(const tq_cache* cache, int Hq, int t) {
  using namespace tq;
  if (!cache || cache->Hkv < 1 || Hq < 1 || Hq % cache->Hkv || t < 0 || t >= cache->T_cap) return -1;
  return cache->layout == TQ_LAYOUT_PLAIN &&
                 step_fusable(make_plan(cache->B, Hq, cache->Hkv, t + 1, device_sms()), (int64_t)t + 1)
             ? 1
             : 0;
}

extern "C" tq_status tq_decode_step(const tq_params* params, const void* k_new, const void* v_new,
                                    int kv_dtype, const void* q, int q_dtype, int Hq, const tq_cache* cache,
                                    int t, float scale, float* out, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  using namespace tq;
  const NvtxRange nvtx_range("tq_decode_step");
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
  if (cache->layout == TQ_LAYOUT_PLAIN &&
      step_fusable(make_plan(cache->B, Hq, cache->Hkv, t + 1, device_sms()), (int64_t)t + 1)) {
    // one launch sequence: the split kernel quantizes row t itself (fp64), writes it and attends
    if (!k_new || !v_new) return fail(TQ_ERR_INVALID_ARG, "k_new / v_new is NULL");
    if (kv_dtype != TQ_F32 && kv_dtype != TQ_BF16) return fail(TQ_ERR_UNSUPPORTED, "kv_dtype %d", kv_dtype);
    const size_t es = kv_dtype == TQ_BF16 ? 2 : 4;
    if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new)) % es)
      return fail(TQ_ERR_INVALID_ARG, "k_new / v_new not aligned to their element size");
    const StepIn in{k_new, v_new, kv_dtype};
    return decode_impl(params, q, q_dtype, Hq, cache, t + 1, scale, out, workspace, workspace_bytes, stream, &in);
  }
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

constexpr size_t kStaticWorkspaceBytes = (size_t)16 << 20;  // 16 MiB
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
  const NvtxRange nvtx_range("tq_decode_attn_static");
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
