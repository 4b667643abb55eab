// QKV projection + RoPE + cache scatter on the 5th-generation tensor cores (bf16).
//
// Flash-dLLM review, "How It Works", Step 1: Draft (Alg. 1): the step reads only
// the hidden rows x[Q], builds q, k, v on chip and writes k, v into the cache at
// exactly the slots of Q.
//
// Shape of the work: Y = x[Q] * W^T with few rows (B*|Q| = 32..2048) and a wide
// W (3E x D = 12288 x 4096, 100 MB), so for small batches the kernel streams W
// once from HBM.  It is computed transposed (swap-AB): Y^T[128 features x BN
// tokens] = W_tile[128 x K] * X[BN x K]^T, so W rows fill the MMA's M = 128 and
// the gathered tokens are its N (16..256).
//
// Fused step: two kernels, the second launched as a programmatic dependent of
// the first (verify rows arrive packed, so the verify pass runs the second only):
//   proj_prep    one CTA per row: packs x[Q] into the workspace.
//   proj_tc      persistent stream-K GEMM.  Its W loads do not depend on the
//                prep kernel and are issued before the grid-dependency wait.
//
// Persistent stream-K: one CTA per SM.  The (tile, k-step) units are laid out
// tile after tile and every CTA takes an equal contiguous range of them, so the
// load is balanced whatever the tile count.  Tiles are numbered feature tile
// first (tile = token tile * feature tiles + feature tile): the CTAs that work
// on the token tiles of one feature tile then run side by side, so W streams
// from HBM once and the other token tiles find it in L2.  A CTA's range covers whole tiles
// and at most one partial tile at each end; a partial tile is written as an
// fp32 partial and the last of its contributors (atomic counter) sums the
// partials in k order (results do not depend on timing) and runs the epilogue.
// No CTA ever waits on another.  A k-step loads `subs` 64-wide sub-blocks at
// once (up to 512 contiguous bytes of every W row).
//
//   warp 0      TMA producer: W boxes [64 x 128] and X boxes [64 x BN]
//   warp 1      TMEM allocation; lane 0 issues tcgen05.mma into one of two
//               TMEM accumulators (the epilogue drains the other)
//   warps 2-9   epilogue, two warps per TMEM lane quarter: TMEM (or the summed
//               partials) -> shared memory -> RoPE on the q and k heads (cos
//               and sin computed in place: the angle reduced modulo 2 pi in
//               double, then the fast single-precision sine and cosine) ->
//               16-byte stores of q, k, v rows
#include "common.cuh"
#include "kernels.h"
#include "proj_epilogue.cuh"
#include "tc_common.cuh"
#include "tmap.h"

namespace fdllm {

namespace {

constexpr int kBM = 128;            // W rows (features) per tile = MMA M
constexpr int kSub = 64;            // bf16 K elements per sub-block = one 128-byte swizzle row
constexpr int kThreads = 320;
constexpr int kEpiThreads = 256;    // two warps per TMEM lane quarter
constexpr int kChunk = 32;          // tokens per epilogue pass
constexpr int kPitch = kChunk + 1;  // staging pitch (floats)
constexpr int kMaxBN = 256;
constexpr uint32_t kASubBytes = kBM * kSub * 2;  // 16 KB


struct ProjTcParams {
  int M, F, D, E, N, H, dh, rows_per_seq, S_max, verify;
  int check_repeats;   // report a repeated index (packed fused rows; the prep kernel does it otherwise)
  int BN, n_tt, n_ft, tiles, nks, subs, nsub_total, nstage;
  long long total_units;
  const int32_t* idx;
  const int8_t* view;
  double log2_base;        // log2 of the RoPE base
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  __nv_bfloat16* k_side;
  __nv_bfloat16* v_side;
  __nv_bfloat16* q_out;
  int* status;
  float* partials;     // [grid][2][BN][128]
  unsigned* tile_cnt;  // [tiles], zero between calls
};

__device__ __forceinline__ long long unit_lo(long long total, int G, int c) {
  return total * c / G;
}
// The CTA whose unit range holds unit u: the largest c with unit_lo(c) <= u,
// i.e. total * c < (u + 1) * G.  A double-precision estimate is corrected with
// exact 64-bit products (64-bit integer division is a long software routine).
__device__ __forceinline__ int owner_of(long long u, long long total, int G) {
  const long long lim = (u + 1) * (long long)G;
  int c = (int)((double)(lim - 1) / (double)total);
  c = c < 0 ? 0 : (c >= G ? G - 1 : c);
  while (c + 1 < G && total * (c + 1) < lim) ++c;
  while (c > 0 && total * c >= lim) --c;
  return c;
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* ptr) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
  return v;
}

// One CTA per projection row m of the fused step: xq[m] = x[b, q_idx[m]] (zeros
// when the index is out of range); a repeated index sets FDLLM_ERR_BAD_INDEX.
__global__ void __launch_bounds__(128) proj_prep_kernel(const __nv_bfloat16* __restrict__ x,
                                                        const int32_t* __restrict__ idx, int N,
                                                        int D, int rows_per_seq,
                                                        __nv_bfloat16* __restrict__ xq,
                                                        int* __restrict__ status) {
  tc::griddep_launch_dependents();
  const int m = blockIdx.x;
  const int ps = idx[m];
  const bool ok = ps >= 0 && ps < N;
  const int b = m / rows_per_seq;
  // Q is a set: an index that repeats an earlier row of the sequence is
  // reported (both rows would write the same cache slot)
  for (int r = b * rows_per_seq + threadIdx.x; r < m; r += blockDim.x)
    if (idx[r] == ps) set_status(status, FDLLM_ERR_BAD_INDEX);
  const uint4* src = reinterpret_cast<const uint4*>(x + ((size_t)b * N + (ok ? ps : 0)) * D);
  uint4* dst = reinterpret_cast<uint4*>(xq + (size_t)m * D);
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  for (int i = threadIdx.x; i < D / 8; i += blockDim.x) dst[i] = ok ? __ldg(src + i) : zero;
}

__global__ void __launch_bounds__(kThreads, 1)
proj_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
               ProjTcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int BN = p.BN;
  const uint32_t bsub_bytes = (uint32_t)BN * 128u;
  const uint32_t stage_bytes = (uint32_t)p.subs * (kASubBytes + bsub_bytes);
  float* staging = reinterpret_cast<float*>(smem + p.nstage * stage_bytes);
  uint8_t* misc = reinterpret_cast<uint8_t*>(staging + kBM * kPitch);
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* empty = full + p.nstage;
  uint64_t* acc_full = empty + p.nstage;   // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* last_flag = abort_flag + 1;
  int* tok_slot = reinterpret_cast<int*>(misc + 256);  // -1: skip k, v
  int* tok_flag = tok_slot + kMaxBN;                   // bit0: q valid, bit1: side buffer
  int* tok_b = tok_flag + kMaxBN;                      // sequence of the token
  int* tok_pos = tok_b + kMaxBN;                       // RoPE position (0 for a skipped row)
  double* theta = reinterpret_cast<double*>(tok_pos + kMaxBN);  // [dh/2] RoPE frequencies

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const long long u_begin = unit_lo(p.total_units, G, c);
  const long long u_end = unit_lo(p.total_units, G, c + 1);
  // (tile, k-step) of the first unit; later units are reached by stepping
  const int tile_begin = (int)(u_begin / p.nks);
  const int ks_begin = (int)(u_begin - (long long)tile_begin * p.nks);

  // two accumulators of BN columns; a chunk load never reaches past them
  uint32_t ncols = 32;
  while ((int)ncols < 2 * BN || (int)ncols < BN + kChunk) ncols <<= 1;

  if (tid == 0) {
    for (int s = 0; s < p.nstage; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&acc_full[b], 1);
      tc::mbar_init(&acc_empty[b], kEpiThreads / 32);  // one arrival per epilogue warp
    }
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, ncols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the attention kernel that follows may start its prologue on SMs this grid
  // leaves; it reads nothing of ours before its own grid-dependency wait
  tc::griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tc::prefetch_tmap(&tm_w);
      tc::prefetch_tmap(&tm_x);
      const uint64_t pol_w = p.n_tt > 1 ? tc::policy_evict_normal() : tc::policy_evict_first();
      const uint64_t pol_x = tc::policy_evict_last();
      const long long n_units = u_end - u_begin;
      // W does not depend on the prep kernel: fill the first stages before
      // waiting for it, then add their X boxes.
      const int pre = (int)(n_units < p.nstage ? n_units : p.nstage);
      int tile = tile_begin, ks = ks_begin;
      for (int i = 0; i < pre; ++i) {
        if (i > 0 && ++ks == p.nks) {
          ks = 0;
          ++tile;
        }
        const int sb0 = ks * p.subs, nsub = min(p.subs, p.nsub_total - sb0);
        uint8_t* a_s = smem + i * stage_bytes;
        tc::mbar_arrive_expect_tx(&full[i], (uint32_t)nsub * (kASubBytes + bsub_bytes));
        for (int q = 0; q < nsub; ++q)
          tc::tma_load_2d(a_s + q * kASubBytes, &tm_w, &full[i], (sb0 + q) * kSub,
                          (tile % p.n_ft) * kBM, pol_w);
      }
      tc::griddep_wait();
      tile = tile_begin;
      ks = ks_begin;
      for (int i = 0; i < pre; ++i) {
        if (i > 0 && ++ks == p.nks) {
          ks = 0;
          ++tile;
        }
        const int sb0 = ks * p.subs, nsub = min(p.subs, p.nsub_total - sb0);
        uint8_t* b_s = smem + i * stage_bytes + p.subs * kASubBytes;
        for (int q = 0; q < nsub; ++q)
          tc::tma_load_2d(b_s + q * bsub_bytes, &tm_x, &full[i], (sb0 + q) * kSub,
                          (tile / p.n_ft) * BN, pol_x);
      }
      for (int it = pre; it < (int)n_units; ++it) {
        if (++ks == p.nks) {
          ks = 0;
          ++tile;
        }
        const int s = it % p.nstage;
        const uint32_t ph = (uint32_t)(it / p.nstage) & 1u;
        if (!tc::mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status)) break;
        const int sb0 = ks * p.subs, nsub = min(p.subs, p.nsub_total - sb0);
        uint8_t* a_s = smem + s * stage_bytes;
        uint8_t* b_s = a_s + p.subs * kASubBytes;
        // rows of X past M are outside the tensor: TMA fills them with zeros
        tc::mbar_arrive_expect_tx(&full[s], (uint32_t)nsub * (kASubBytes + bsub_bytes));
        for (int q = 0; q < nsub; ++q) {
          tc::tma_load_2d(a_s + q * kASubBytes, &tm_w, &full[s], (sb0 + q) * kSub,
                          (tile % p.n_ft) * kBM, pol_w);
          tc::tma_load_2d(b_s + q * bsub_bytes, &tm_x, &full[s], (sb0 + q) * kSub,
                          (tile / p.n_ft) * BN, pol_x);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(kBM, BN);
      int it = 0, j = 0;
      bool ok = true;
      for (long long u = u_begin; u < u_end && ok; ++j) {
        const int ks0 = (u == u_begin) ? ks_begin : 0;  // later segments start a tile
        const int ks1 = (int)min((long long)p.nks, ks0 + (u_end - u));
        u += ks1 - ks0;
        const int buf = j & 1;
        if (!tc::mbar_wait(&acc_empty[buf], ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag, p.status)) break;
        tc::tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(buf * BN);
        for (int ks = ks0; ks < ks1; ++ks, ++it) {
          const int s = it % p.nstage;
          const uint32_t ph = (uint32_t)(it / p.nstage) & 1u;
          if (!tc::mbar_wait(&full[s], ph, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const int nsub = min(p.subs, p.nsub_total - ks * p.subs);
          const uint32_t a_addr = tc::smem_u32(smem + s * stage_bytes);
          const uint32_t b_addr = a_addr + p.subs * kASubBytes;
          for (int q = 0; q < nsub; ++q) {
#pragma unroll
            for (int kk = 0; kk < kSub / 16; ++kk) {
              const uint64_t da = tc::smem_desc(a_addr + q * kASubBytes + kk * 32, 16, 1024, 2);
              const uint64_t db = tc::smem_desc(b_addr + q * bsub_bytes + kk * 32, 16, 1024, 2);
              tc::mma_bf16(d_tmem, da, db, idesc, (ks != ks0 || q != 0 || kk != 0) ? 1u : 0u);
            }
          }
          tc::mma_commit(&empty[s]);
        }
        tc::mma_commit(&acc_full[buf]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    tc::griddep_wait();
    const int etid = tid - 64;
    // theta_j = base^(-2j/dh), in double: the angle pos * theta_j is reduced
    // modulo 2 pi in double before the single-precision sine and cosine
    for (int jj = etid; jj < (p.dh >> 1); jj += kEpiThreads)
      theta[jj] = exp2(-(2.0 * (double)jj / (double)p.dh) * p.log2_base);
    tc::named_bar_sync(1, kEpiThreads);
    const int quarter = warp & 3;
    const int f_loc = quarter * 32 + lane;
    const int n_half = ((warp - 2) >> 2) * (kChunk / 2);  // this warp's 16 tokens of a chunk
    float* my_parts = p.partials + (size_t)c * 2 * BN * kBM;
    int j = 0;
    for (long long u = u_begin; u < u_end; ++j) {
      const int tile = tile_begin + j;  // a segment is the part of one tile
      const int ks0 = (j == 0) ? ks_begin : 0;
      const int ks1 = (int)min((long long)p.nks, ks0 + (u_end - u));
      u += ks1 - ks0;
      const int buf = j & 1;
      const int ft = tile % p.n_ft, tt = tile / p.n_ft;
      const int m0 = tt * BN;
      const bool whole = (ks0 == 0 && ks1 == p.nks);
      const uint32_t t_acc = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);

      // token routing of this tile, ahead of the accumulator
      for (int n = etid; n < BN; n += kEpiThreads) {
        const int m = m0 + n;
        int slot = -1, flag = 0;
        if (m < p.M) {
          const int ps = p.idx[m];
          const bool in_range = ps >= 0 && ps < p.N;
          if (in_range) flag |= 1;
          if (p.verify && p.view[m] == 2) {
            int s = 0;
            const int b = m / p.rows_per_seq;
            for (int r = b * p.rows_per_seq; r < m; ++r) s += (p.view[r] == 2);
            flag |= 2;
            slot = (in_range && s < p.S_max) ? s : -1;
          } else {
            slot = in_range ? ps : -1;
          }
        }
        // Q is a set: a packed fused row repeating an earlier row's slot is
        // reported once, by the first feature tile
        if (p.check_repeats && ft == 0 && m < p.M) {
          const int ps = p.idx[m];
          for (int r = (m / p.rows_per_seq) * p.rows_per_seq; r < m; ++r)
            if (p.idx[r] == ps) set_status(p.status, FDLLM_ERR_BAD_INDEX);
        }
        tok_slot[n] = slot;
        tok_flag[n] = flag;
        tok_b[n] = m < p.M ? m / p.rows_per_seq : 0;
        tok_pos[n] = (flag & 1) ? p.idx[m] : 0;
      }

      // after a timeout every later wait returns at once: keep going so that all
      // epilogue threads still meet at the same named barriers
      tc::mbar_wait(&acc_full[buf], (uint32_t)(j >> 1) & 1u, abort_flag, p.status);
      tc::tc_fence_after();

      bool run = true;
      bool own_in_tmem = true;  // this CTA's part of the tile is still (only) in TMEM
      int c_first = c, c_last = c;
      const long long tu0 = (long long)tile * p.nks;
      if (!whole) {
        c_first = owner_of(tu0, p.total_units, G);
        c_last = owner_of(tu0 + p.nks - 1, p.total_units, G);
        // The other contributors count up after storing their parts.  When they
        // all have, this CTA is the last one and merges its own part straight
        // from TMEM: no store, fence or atomic of its own.
        if (etid == 0) {
          const unsigned done = ld_acquire(&p.tile_cnt[tile]);
          *last_flag = (done == (unsigned)(c_last - c_first)) ? 2 : 0;
          if (*last_flag == 2) p.tile_cnt[tile] = 0u;  // reset for the next call
        }
        tc::named_bar_sync(1, kEpiThreads);
      }
      if (!whole && *last_flag != 2) {
        own_in_tmem = false;
        // partial tile: store it, free the accumulator, and see who is last
        const int slot = (j == 0) ? 0 : 1;
        float* dst = my_parts + (size_t)slot * BN * kBM;
        for (int cc = n_half; cc < BN; cc += kChunk) {
          float v[kChunk / 2];
          tc::tmem_ld16(t_acc + cc, v);
          tc::tmem_wait_ld();
#pragma unroll
          for (int n = 0; n < kChunk / 2; ++n) dst[(size_t)(cc + n) * kBM + f_loc] = v[n];
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&acc_empty[buf]);
        __threadfence();
        tc::named_bar_sync(1, kEpiThreads);
        if (etid == 0) {
          const unsigned prev = atomicAdd(&p.tile_cnt[tile], 1u);
          *last_flag = (prev == (unsigned)(c_last - c_first));
          if (*last_flag) p.tile_cnt[tile] = 0u;
        }
        tc::named_bar_sync(1, kEpiThreads);
        run = *last_flag != 0;
        if (run) __threadfence();
      }
      if (run) {
        if (ft == 0) {
          for (int n = etid; n < BN; n += kEpiThreads)
            if (m0 + n < p.M && tok_slot[n] < 0) set_status(p.status, FDLLM_ERR_BAD_INDEX);
        }
        // The part of contributor cb for this thread's feature row and 16 tokens
        // from column c (slot 0 when the tile is cb's first: unit_lo(cb) >= tu0).
        auto load_part = [&](int cb, int c, float* t) {
          const int sl = (p.total_units * cb >= tu0 * (long long)G) ? 0 : 1;
          const float* ps = p.partials + ((size_t)cb * 2 + sl) * BN * kBM + (size_t)c * kBM + f_loc;
#pragma unroll
          for (int n = 0; n < kChunk / 2; ++n) t[n] = __ldcg(ps + (size_t)n * kBM);
        };
        // The first contributor whose part is in global memory has its next
        // chunk loaded while this chunk is rotated and stored, so the merge
        // does not wait out an L2 round trip per chunk.
        const int cb_pf = (c_first == c && own_in_tmem) ? c_first + 1 : c_first;
        float pf[kChunk / 2];
        if (!whole && cb_pf <= c_last && n_half < BN) load_part(cb_pf, n_half, pf);
        for (int cc = 0; cc < BN; cc += kChunk) {
          if (whole) {
            // BN is a multiple of 16: a warp's 16 columns are all in the tile or none
            if (cc + n_half < BN) {
              float v[kChunk / 2];
              tc::tmem_ld16(t_acc + cc + n_half, v);
              tc::tmem_wait_ld();
#pragma unroll
              for (int n = 0; n < kChunk / 2; ++n) staging[f_loc * kPitch + n_half + n] = v[n];
            }
          } else if (cc + n_half < BN) {
            // sum the parts of every contributor in CTA (k) order, the thread's
            // feature row over its 16 tokens: this CTA's part from TMEM when it
            // was never stored, the others' from global memory
            float cur[kChunk / 2];
#pragma unroll
            for (int n = 0; n < kChunk / 2; ++n) cur[n] = pf[n];
            if (cb_pf <= c_last && cc + kChunk + n_half < BN)
              load_part(cb_pf, cc + kChunk + n_half, pf);
            float v[kChunk / 2];
#pragma unroll
            for (int n = 0; n < kChunk / 2; ++n) v[n] = 0.f;
            for (int cb = c_first; cb <= c_last; ++cb) {
              float t[kChunk / 2];
              if (cb == c && own_in_tmem) {
                tc::tmem_ld16(t_acc + cc + n_half, t);
                tc::tmem_wait_ld();
              } else if (cb == cb_pf) {
#pragma unroll
                for (int n = 0; n < kChunk / 2; ++n) t[n] = cur[n];
              } else {
                load_part(cb, cc + n_half, t);
              }
#pragma unroll
              for (int n = 0; n < kChunk / 2; ++n) v[n] += t[n];
            }
#pragma unroll
            for (int n = 0; n < kChunk / 2; ++n) staging[f_loc * kPitch + n_half + n] = v[n];
          }
          tc::named_bar_sync(1, kEpiThreads);
          epi::rope_store_chunk(p, staging, ft * kBM, m0, cc, BN, tok_slot, tok_flag, tok_b, tok_pos,
                                theta, etid, kEpiThreads);
          tc::named_bar_sync(1, kEpiThreads);
        }
      }
      if (whole || own_in_tmem) {
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&acc_empty[buf]);
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc(tmem, ncols);
  }
}

struct ProjPlan {
  int BN, n_tt, n_ft, tiles, nks, subs, nsub_total, nstage, grid;
  long long total_units;
  size_t smem_bytes, partial_bytes, counter_bytes, xq_bytes;
};

constexpr size_t kSmemBudget = 227 * 1024;

ProjPlan plan(int M, int D, int H, int dh, int num_sms) {
  ProjPlan q{};
  const int F = 3 * H * dh;
  q.n_tt = (M + kMaxBN - 1) / kMaxBN;
  const int per = (M + q.n_tt - 1) / q.n_tt;
  q.BN = ((per + 15) / 16) * 16;
  q.n_ft = (F + kBM - 1) / kBM;
  q.tiles = q.n_ft * q.n_tt;
  q.nsub_total = D / kSub;
  const size_t fixed = 1024 /*align*/ + (size_t)kBM * kPitch * 4 + 256 + 4 * kMaxBN * 4 + 64 * 8;
  // the widest k-step (most contiguous bytes per W row) that keeps two stages
  const int cand[3] = {4, 2, 1};
  for (int i = 0; i < 3; ++i) {
    const int subs = cand[i];
    const size_t stage = (size_t)subs * (kASubBytes + (size_t)q.BN * 128);
    const int ns = (int)((kSmemBudget - fixed) / stage);
    if (ns >= 2 || subs == 1) {
      q.subs = subs;
      q.nstage = ns < 8 ? ns : 8;
      break;
    }
  }
  if (q.subs > q.nsub_total) q.subs = q.nsub_total;
  const size_t stage = (size_t)q.subs * (kASubBytes + (size_t)q.BN * 128);
  if ((int)((kSmemBudget - fixed) / stage) < q.nstage) q.nstage = (int)((kSmemBudget - fixed) / stage);
  q.nks = (q.nsub_total + q.subs - 1) / q.subs;
  q.total_units = (long long)q.tiles * q.nks;
  q.grid = (int)(q.total_units < num_sms ? q.total_units : num_sms);
  q.smem_bytes = (size_t)q.nstage * stage + fixed;
  // sized by min(256, M rounded up to 16) >= BN, not by BN itself: BN is not
  // monotone in M, and a workspace sized for the most rows must serve fewer
  const int bn_bound = (int)(((M + 15) / 16) * 16 < kMaxBN ? ((M + 15) / 16) * 16 : kMaxBN);
  q.partial_bytes = align_up((size_t)q.grid * 2 * bn_bound * kBM * sizeof(float), 256);
  q.counter_bytes = align_up((size_t)q.tiles * sizeof(unsigned), 256);
  q.xq_bytes = align_up((size_t)M * D * 2, 256);
  return q;
}

}  // namespace

cudaError_t launch_proj_prep(const ProjArgs& a, __nv_bfloat16* xq, cudaStream_t stream) {
  const int M = a.B * a.rows_per_seq;
  proj_prep_kernel<<<M, 128, 0, stream>>>(static_cast<const __nv_bfloat16*>(a.x), a.idx, a.N, a.D,
                                          a.rows_per_seq, xq, a.status);
  count_launches(1);
  return cudaGetLastError();
}

size_t proj_tc_workspace_bytes(int M, int D, int H, int dh, int num_sms) {
  if (M <= 0) return 256;
  const ProjPlan q = plan(M, D, H, dh, num_sms);
  return q.partial_bytes + q.counter_bytes + q.xq_bytes;
}

cudaError_t launch_proj_tc(const ProjArgs& a, cudaStream_t stream) {
  const int M = a.B * a.rows_per_seq;
  if (M == 0) return cudaSuccess;
  const int E = a.H * a.dh, F = 3 * E;
  const ProjPlan q = plan(M, a.D, a.H, a.dh, device_sm_count());
  if (q.partial_bytes + q.counter_bytes + q.xq_bytes > a.ws_bytes)
    return cudaErrorInvalidValue;
  char* ws = static_cast<char*>(a.ws);
  __nv_bfloat16* xq = reinterpret_cast<__nv_bfloat16*>(ws + q.partial_bytes + q.counter_bytes);

  CUtensorMap tm_w, tm_x;
  {
    const uint64_t dims[2] = {(uint64_t)a.D, (uint64_t)F};
    const uint64_t strides[1] = {(uint64_t)a.D * 2};
    const uint32_t box[2] = {kSub, kBM};
    if (!encode_bf16_map(&tm_w, 2, a.w, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
      return cudaErrorInvalidValue;
  }
  // X: rows the caller packed (verify rows, or fused rows given as x[Q]), or
  // x[Q] packed into the workspace by the prep kernel
  const bool packed = a.verify || a.packed;
  const void* xsrc = packed ? a.x : static_cast<const void*>(xq);
  {
    const uint64_t dims[2] = {(uint64_t)a.D, (uint64_t)M};
    const uint64_t strides[1] = {(uint64_t)a.D * 2};
    const uint32_t box[2] = {kSub, (uint32_t)q.BN};
    if (!encode_bf16_map(&tm_x, 2, xsrc, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B))
      return cudaErrorInvalidValue;
  }
  ProjTcParams p{};
  p.M = M; p.F = F; p.D = a.D; p.E = E; p.N = a.N; p.H = a.H; p.dh = a.dh;
  p.rows_per_seq = a.rows_per_seq; p.S_max = a.S_max; p.verify = a.verify;
  p.check_repeats = (!a.verify && a.packed) ? 1 : 0;
  p.BN = q.BN; p.n_tt = q.n_tt; p.n_ft = q.n_ft; p.tiles = q.tiles; p.nks = q.nks; p.subs = q.subs;
  p.nsub_total = q.nsub_total; p.nstage = q.nstage; p.total_units = q.total_units;
  p.idx = a.idx; p.view = a.view; p.log2_base = a.log2_base;
  p.k_cache = static_cast<__nv_bfloat16*>(a.k_cache);
  p.v_cache = static_cast<__nv_bfloat16*>(a.v_cache);
  p.k_side = static_cast<__nv_bfloat16*>(a.k_side);
  p.v_side = static_cast<__nv_bfloat16*>(a.v_side);
  p.q_out = static_cast<__nv_bfloat16*>(a.q_out);
  p.status = a.status;
  p.partials = reinterpret_cast<float*>(ws);
  p.tile_cnt = reinterpret_cast<unsigned*>(ws + q.partial_bytes);

  cudaError_t e;
  if (!packed) {
    // the fused step gathers x[Q] into a packed operand
    e = launch_proj_prep(a, xq, stream);
    if (e != cudaSuccess) return e;
  }

  e = cudaFuncSetAttribute(proj_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)q.smem_bytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(q.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = q.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, proj_tc_kernel, tm_w, tm_x, p);
  count_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fdllm
