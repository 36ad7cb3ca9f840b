// Internal helpers shared by the host entry points and the kernels of the tq library.
#pragma once

#include <cstdarg>
#include <cstddef>
#include <cstdint>

#include "tq.h"

#ifndef __CUDACC__
#define __host__
#define __device__
#endif

namespace tq {

constexpr int kHeadDim = 128;
constexpr int kQjlRows = 128;
// Comparison bands of the parity rules: a coordinate within kExemptCodeBand of a threshold (in u
// units), or a sketch value within kExemptSignBand of 0, is decided by rounding; the quantize
// kernels count such cases (tq_quantize_exempt_codes / _signs).
constexpr double kExemptCodeBand = 1e-6;
constexpr double kExemptSignBand = 1e-5;

// NVTX range around an entry point (header-only NVTX 3: a no-op unless a profiler is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name);
  ~NvtxRange();
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Thread-local error detail; returns `st` so callers can `return fail(...)`.
tq_status fail(tq_status st, const char* fmt, ...);
void clear_error();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Packed-row slot maps (the cache layout documented in tq.h).
// Key-code rows and sign rows are ordered for the decode kernel's m16n8k16 B fragments:
// thread tau of a quad owns coordinates 16*a + 8*h + 2*tau + e.
__host__ __device__ inline int k_slot_of_coord(int j) {
  const int a = j >> 4, h = (j >> 3) & 1, t = (j >> 1) & 3, e = j & 1;
  return 32 * t + 4 * a + 2 * h + e;
}
// Value-code rows: lane group g of a warp owns coordinates 8*n + g.
__host__ __device__ inline int v_slot_of_coord(int j) {
  const int n = j >> 3, g = j & 7;
  return 16 * g + n;
}
// Mixed layout (TQ_LAYOUT_MIXED): each half g = j / 64 is its own bit stream; within it the key
// coordinate 16a + 8h + 2t + e (a < 4) sits at slot 16t + 4a + 2h + e, the value coordinate
// 8n + g' at slot 8g' + n.  Bit position of coordinate j in the row (half O of `bits_o` bits first):
__host__ __device__ inline int k_slot_of_coord_mixed(int j) {
  const int jj = j & 63;
  const int a = jj >> 4, h = (jj >> 3) & 1, t = (jj >> 1) & 3, e = jj & 1;
  return 16 * t + 4 * a + 2 * h + e;
}
__host__ __device__ inline int v_slot_of_coord_mixed(int j) {
  const int jj = j & 63;
  return 8 * (jj & 7) + (jj >> 3);
}
__host__ __device__ inline int mixed_bit_pos(int j, int slot, int bits_o) {
  return j < 64 ? bits_o * slot : 64 * bits_o + (bits_o - 1) * slot;
}

__host__ __device__ inline int sign_bit_of_row(int l) {
  const int a = l >> 4, h = (l >> 3) & 1, t = (l >> 1) & 3, e = l & 1;
  return 32 * t + (2 * a + h) + 16 * e;
}

// bf16 quantize pipeline (tq_quantize_pipe.cu).  Sets *handled = false, and enqueues nothing,
// when the inputs cannot be described by a TMA tensor map.
tq_status quantize_bf16_pipeline(const tq_params* p, const void* k, const void* v, int64_t sb, int64_t sh,
                                 int64_t st, int T_new, int t_offset, const tq_cache* c, int sms,
                                 struct CUstream_st* stream, bool* handled);
unsigned int pipe_device_errors();
long long pipe_vector_fixups();
long long pipe_code_fixups();
long long pipe_exempt_codes();
void pipe_set_test_stall(int enable, long long wait_cycles);
int decode_reset_errors();
int pipe_reset_errors();
long long pipe_exempt_signs();

// Validation shared by tq_quantize / tq_decode_attn.
tq_status check_params(const tq_params* p, const tq_cache* c);
tq_status check_cache(const tq_cache* c);

}  // namespace tq
