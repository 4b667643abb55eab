// The last step of the projection epilogue, shared by both projection kernels:
// one chunk of 32 tokens of a 128-feature block, already summed in shared
// memory, is rotated (RoPE on the q and k heads) and stored as 16-byte rows.
//
// Flash-dLLM review, "How It Works", Step 1: Draft: the step writes k, v into
// the cache at the slots of Q (verify: mask-view rows into side slots); q goes
// to the staging buffer the attention reads.  RoPE turns the pair (j, j + dh/2)
// of a head by pos * theta_j: both elements of a pair are produced by the same
// work item from one sine and cosine.
#pragma once

#include "common.cuh"

namespace fdllm {
namespace epi {

constexpr int kBM = 128;            // features of a block (TMEM lanes)
constexpr int kChunk = 32;          // tokens per chunk
constexpr int kPitch = kChunk + 1;  // staging pitch (floats)
constexpr double kTwoPi = 6.283185307179586476925286766559;
constexpr double kInvTwoPi = 0.15915494309189533576888376337251;

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void store8(__nv_bfloat16* dst, const float* o) {
  uint4 pk;
  pk.x = pack_bf16x2(o[0], o[1]);
  pk.y = pack_bf16x2(o[2], o[3]);
  pk.z = pack_bf16x2(o[4], o[5]);
  pk.w = pack_bf16x2(o[6], o[7]);
  *reinterpret_cast<uint4*>(dst) = pk;
}

// staging[f * kPitch + n]: feature f (0..127) of block fbase, token m0 + cc + n.
// Token routing (per column of the tile): tok_slot (cache or side slot, -1 =
// write no k, v), tok_flag (bit0: q valid, bit1: side buffer), tok_b
// (sequence), tok_pos (RoPE position).  theta[j] = base^(-2j/dh).
template <class P>
__device__ __forceinline__ void rope_store_chunk(const P& p, const float* staging, int fbase,
                                                 int m0, int cc, int BN, const int* tok_slot,
                                                 const int* tok_flag, const int* tok_b,
                                                 const int* tok_pos, const double* theta,
                                                 int etid, int nthreads) {
  const int half = p.dh >> 1;
  const int dh_log2 = p.dh == 128 ? 7 : 6;  // dh is 64 or 128
  // 32 tokens x 16 groups of 8 features; a warp covers 32 tokens of one group
  for (int itm = etid; itm < kChunk * (kBM / 8); itm += nthreads) {
    const int g = itm / kChunk, n = itm % kChunk;
    const int m = m0 + cc + n;
    if (cc + n >= BN || m >= p.M) continue;
    const int f0 = g * 8;
    const int fg = fbase + f0;
    if (fg >= p.F) continue;
    // no integer division: F = 3E and dh is 64 or 128
    const int blk = fg >= 2 * p.E ? 2 : (fg >= p.E ? 1 : 0);
    const int rem = fg - blk * p.E;
    const int h = rem >> dh_log2, j0 = rem & (p.dh - 1);
    const int slot = tok_slot[cc + n], flag = tok_flag[cc + n];
    if (blk != 0 && slot < 0) continue;
    // a rotated head's upper half is written by the group of its lower half
    // (heads start at multiples of dh, so both halves are in this block)
    if (blk != 2 && j0 >= half) continue;
    __nv_bfloat16* dst;
    if (blk == 0) {
      dst = p.q_out + (size_t)m * p.E + h * p.dh + j0;
    } else {
      const bool side = (flag & 2) != 0;
      __nv_bfloat16* base = (blk == 1) ? (side ? p.k_side : p.k_cache)
                                       : (side ? p.v_side : p.v_cache);
      const int nslots = side ? p.S_max : p.N;
      dst = base + (((size_t)tok_b[cc + n] * p.H + h) * nslots + slot) * p.dh + j0;
    }
    float o[8];
    if (blk == 2) {
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = staging[(f0 + i) * kPitch + n];
      store8(dst, o);
    } else if (blk == 0 && !(flag & 1)) {
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = 0.f;  // a skipped query attends with q = 0
      store8(dst, o);
      store8(dst + half, o);
    } else {
      float o2[8];
      const double pos = (double)tok_pos[cc + n];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float x = staging[(f0 + i) * kPitch + n];
        const float xp = staging[(f0 + half + i) * kPitch + n];
        // angle mod 2 pi in double, then the fast sine/cosine on [-pi, pi]
        const double ang = pos * theta[j0 + i];
        const double k = rint(ang * kInvTwoPi);
        float sn, cs;
        __sincosf((float)fma(-k, kTwoPi, ang), &sn, &cs);
        o[i] = x * cs - xp * sn;
        o2[i] = xp * cs + x * sn;
      }
      store8(dst, o);
      store8(dst + half, o2);
    }
  }
}

}  // namespace epi
}  // namespace fdllm
