// Device helpers shared by the fdllm kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/fdllm.h"

namespace fdllm {

// ---------------------------------------------------------------------------
// workspace header: the first 256 bytes of every workspace.
struct WsHeader {
  int status;  // first device-detected error (fdllm_status), 0 = none
  int pad[63];
};
constexpr size_t kWsHeaderBytes = 256;

__device__ __forceinline__ void set_status(int* status, int code) {
  atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------------------
// storage types
template <typename T> struct Store;
template <> struct Store<float> {
  static __device__ __forceinline__ float ld(const float* p) { return *p; }
  static __device__ __forceinline__ void st(float* p, float v) { *p = v; }
};
template <> struct Store<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

// ---------------------------------------------------------------------------
// RoPE: pair (j, j + dh/2) of a head is turned by pos * base^(-2j/dh).
// The angle is formed and reduced to [-pi, pi] in double so that large slot
// indices keep full float accuracy; sin/cos are then taken in float.
__device__ __forceinline__ double rope_inv_freq(int j, int dh, double log2_base) {
  return exp2(-(2.0 * (double)j / (double)dh) * log2_base);
}
__device__ __forceinline__ void rope_cos_sin(int pos, double inv_freq, float* c, float* s) {
  const double two_pi = 6.283185307179586476925286766559;
  double a = (double)pos * inv_freq;
  a -= two_pi * rint(a / two_pi);
  sincosf((float)a, s, c);
}

// ---------------------------------------------------------------------------
// Flash-Verify visibility.  Keys are cache slots or side slots.
//   row_view: 0 T_v, 1 draft, 2 mask.  key_draft_rank: rank of the draft row
//   written at this cache slot, or -1 when the slot is not a draft position.
//   For a side slot, side_rank is the rank of the mask row that wrote it.
__device__ __forceinline__ bool visible_cache(int row_view, int row_rank, int key_draft_rank,
                                              int causal_cross) {
  if (row_view != 2 || key_draft_rank < 0) return true;
  return causal_cross ? (key_draft_rank < row_rank) : false;
}
__device__ __forceinline__ bool visible_side(int row_view, int row_rank, int side_rank,
                                             int causal_cross) {
  if (row_view != 2) return false;
  return causal_cross ? (side_rank >= row_rank) : true;
}

// ---------------------------------------------------------------------------
// bounded waits: every spin in these kernels gives up after this many
// nanoseconds of %globaltimer, records FDLLM_ERR_TIMEOUT and lets the kernel
// leave.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

}  // namespace fdllm
