// QKV projection + RoPE + cache scatter for many rows (M >= 512) on CTA pairs.
//
// Flash-dLLM review, "How It Works", Step 1: Draft (Alg. 1), and the
// Flash-Verify pass over packed rows: the same projection, rotation and cache
// writes as proj_tc.cu, for the row counts where the tile shape, not the W
// stream, decides the time.
//
// Y^T [features x tokens] = W_tile * X^T on tcgen05 with cta_group::2: the two
// CTAs of a cluster share each MMA (M = 256 features, 128 from each CTA's
// shared memory; N <= 256 tokens, N/2 rows from each), so each CTA loads half
// of the x[Q] rows a feature tile needs, and the L2 -> shared-memory bytes are
// what bound these shapes.
//   Up to 512 rows: one token tile (two MMAs of N = BN/2 beyond 256 rows) and,
//     when there are no more tiles than pairs, one whole tile per pair: W
//     streams once and no tile is split, so nothing is merged.
//   More rows: tiles of up to 256 tokens with two accumulators, so that each
//     tile's epilogue overlaps the next tile's MMAs, spread by stream-K.
//
// Both CTAs' TMA loads complete on the rank-0 CTA's stage barrier (the load's
// cta_group::2 form, no multicast); rank 0 issues the MMAs, and each MMA
// completion arrives on the barrier at the same offset in both CTAs
// (tcgen05.commit multicast), which frees the stage in both.  Each CTA's
// epilogue drains its own 128 feature rows of the accumulator and arrives on
// rank 0's accumulator-empty barrier.
//
// Work split: persistent stream-K over pairs (one CTA pair per two SMs), units
// (tile, k-step) in equal contiguous ranges, tiles numbered feature pair first.
// A tile split between pairs is merged per CTA rank by its last contributor
// (atomic counter), summing the parts in pair order.  No pair waits on another.
//
//   warp 0      TMA producer (both CTAs: their own A and B boxes)
//   warp 1      TMEM allocation (pair); rank 0, lane 0 issues the MMAs
//   warps 2-9   epilogue, two warps per TMEM lane quarter, as in proj_tc.cu
#include "common.cuh"
#include "kernels.h"
#include "proj_epilogue.cuh"
#include "tc_common.cuh"
#include "tmap.h"


namespace fdllm {

namespace {

constexpr int kBM = 128;            // W rows per CTA (the pair's MMA has M = 256)
constexpr int kSub = 64;            // bf16 K elements per sub-block = one 128-byte swizzle row
constexpr int kThreads = 320;
constexpr int kEpiThreads = 256;    // two warps per TMEM lane quarter
constexpr int kChunk = 32;          // tokens per epilogue pass
constexpr int kPitch = kChunk + 1;  // staging pitch (floats)
constexpr int kMaxBN = 512;         // tokens of one accumulator (two MMAs of N <= 256)
constexpr int kMaxBNStreamK = 256;  // tokens per tile when tiles outnumber the pairs
constexpr uint32_t kASubBytes = kBM * kSub * 2;  // 16 KB

struct PairParams {
  int M, F, D, E, N, H, dh, rows_per_seq, S_max, verify, check_repeats;
  int BN, NM, nmma, nbuf, n_tt, n_fp, tiles, nks, subs, nsub_total, nstage;
  long long total_units;
  const int32_t* idx;
  const int8_t* view;
  double log2_base;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  __nv_bfloat16* k_side;
  __nv_bfloat16* v_side;
  __nv_bfloat16* q_out;
  int* status;
  float* partials;     // [CTA][2][BN][128]
  unsigned* tile_cnt;  // [tiles][2], zero between calls
};

__device__ __forceinline__ long long unit_lo(long long total, int G, int c) {
  return total * c / G;
}
// The pair whose unit range holds unit u (see proj_tc.cu).
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

__global__ void __launch_bounds__(kThreads, 1)
proj_pair_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                 PairParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int BN = p.BN, NM = p.NM, HB = p.NM / 2;  // HB: token rows of one MMA in this CTA
  const uint32_t bsub_bytes = (uint32_t)HB * 128u;  // one MMA's B rows for one 64-wide sub
  const uint32_t sub_bytes = kASubBytes + (uint32_t)p.nmma * bsub_bytes;
  const uint32_t stage_bytes = (uint32_t)p.subs * sub_bytes;
  float* staging = reinterpret_cast<float*>(smem + p.nstage * stage_bytes);
  uint8_t* misc = reinterpret_cast<uint8_t*>(staging + kBM * kPitch);
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* empty = full + p.nstage;
  uint64_t* acc_full = empty + p.nstage;   // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2], used in rank 0
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
  const int rank = (int)tc::cluster_ctarank();
  const int P = gridDim.x >> 1, pair = blockIdx.x >> 1;
  const long long u_begin = unit_lo(p.total_units, P, pair);
  const long long u_end = unit_lo(p.total_units, P, pair + 1);
  const int tile_begin = (int)(u_begin / p.nks);
  const int ks_begin = (int)(u_begin - (long long)tile_begin * p.nks);

  uint32_t ncols = 32;
  while ((int)ncols < p.nbuf * BN) ncols <<= 1;

  if (tid == 0) {
    for (int s = 0; s < p.nstage; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&acc_full[b], 1);
      tc::mbar_init(&acc_empty[b], 2 * (kEpiThreads / 32));  // both CTAs' epilogue warps
    }
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc_pair(tmem_slot, ncols);
  tc::tc_fence_before();
  __syncthreads();
  // the peer's barriers are initialised before anything of ours arrives on them
  tc::cluster_sync();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  tc::griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tc::prefetch_tmap(&tm_w);
      tc::prefetch_tmap(&tm_x);
      const uint64_t pol_w = p.n_tt > 1 ? tc::policy_evict_normal() : tc::policy_evict_first();
      const uint64_t pol_x = tc::policy_evict_last();
      const long long n_units = u_end - u_begin;
      auto leader_full = [&](int s) { return tc::map_peer(tc::smem_u32(&full[s]), 0u); };
      auto load_a = [&](int s, int tile, int ks, int nsub) {
        const int sb0 = ks * p.subs;
        uint8_t* st = smem + s * stage_bytes;
        for (int q = 0; q < nsub; ++q)
          tc::tma_load_2d_pair(st + q * sub_bytes, &tm_w, leader_full(s), (sb0 + q) * kSub,
                               (tile % p.n_fp) * (2 * kBM) + rank * kBM, pol_w);
      };
      auto load_b = [&](int s, int tile, int ks, int nsub) {
        const int sb0 = ks * p.subs;
        uint8_t* st = smem + s * stage_bytes;
        const int t0 = (tile / p.n_fp) * BN + rank * HB;
        for (int q = 0; q < nsub; ++q)
          for (int j = 0; j < p.nmma; ++j)
            tc::tma_load_2d_pair(st + q * sub_bytes + kASubBytes + j * bsub_bytes, &tm_x,
                                 leader_full(s), (sb0 + q) * kSub, t0 + j * NM, pol_x);
      };
      // W does not depend on an earlier kernel: fill the first stages' W boxes
      // before waiting for it, then add their X boxes
      const int pre = (int)(n_units < p.nstage ? n_units : p.nstage);
      int tile = tile_begin, ks = ks_begin;
      for (int i = 0; i < pre; ++i) {
        if (i > 0 && ++ks == p.nks) {
          ks = 0;
          ++tile;
        }
        const int nsub = min(p.subs, p.nsub_total - ks * p.subs);
        // rank 0 expects both CTAs' bytes on its barrier; the other CTA's loads
        // may land first (the phase cannot complete before this arrival)
        if (rank == 0) tc::mbar_arrive_expect_tx(&full[i], 2u * (uint32_t)nsub * sub_bytes);
        load_a(i, tile, ks, nsub);
      }
      tc::griddep_wait();
      tile = tile_begin;
      ks = ks_begin;
      for (int i = 0; i < pre; ++i) {
        if (i > 0 && ++ks == p.nks) {
          ks = 0;
          ++tile;
        }
        load_b(i, tile, ks, min(p.subs, p.nsub_total - ks * p.subs));
      }
      for (int it = pre; it < (int)n_units; ++it) {
        if (++ks == p.nks) {
          ks = 0;
          ++tile;
        }
        const int s = it % p.nstage;
        const uint32_t ph = (uint32_t)(it / p.nstage) & 1u;
        // the MMA that read this stage (in both CTAs) has completed
        if (!tc::mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status)) break;
        const int nsub = min(p.subs, p.nsub_total - ks * p.subs);
        if (rank == 0) tc::mbar_arrive_expect_tx(&full[s], 2u * (uint32_t)nsub * sub_bytes);
        load_a(s, tile, ks, nsub);
        load_b(s, tile, ks, nsub);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (rank 0)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = tc::idesc_bf16(2 * kBM, NM);
      int it = 0, j = 0;
      bool ok = true;
      for (long long u = u_begin; u < u_end && ok; ++j) {
        const int ks0 = (u == u_begin) ? ks_begin : 0;  // later segments start a tile
        const int ks1 = (int)min((long long)p.nks, ks0 + (u_end - u));
        u += ks1 - ks0;
        const int buf = p.nbuf == 2 ? (j & 1) : 0;
        const uint32_t use = p.nbuf == 2 ? (uint32_t)(j >> 1) : (uint32_t)j;
        // both CTAs' epilogues have drained this accumulator
        if (!tc::mbar_wait(&acc_empty[buf], (use & 1u) ^ 1u, abort_flag, p.status)) break;
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
          const uint32_t st = tc::smem_u32(smem + s * stage_bytes);
          for (int q = 0; q < nsub; ++q) {
            const uint32_t a_addr = st + q * sub_bytes;
            for (int jm = 0; jm < p.nmma; ++jm) {
              const uint32_t b_addr = a_addr + kASubBytes + jm * bsub_bytes;
#pragma unroll
              for (int kk = 0; kk < kSub / 16; ++kk) {
                const uint64_t da = tc::smem_desc(a_addr + kk * 32, 16, 1024, 2);
                const uint64_t db = tc::smem_desc(b_addr + kk * 32, 16, 1024, 2);
                tc::mma_bf16_pair(d_tmem + (uint32_t)(jm * NM), da, db, idesc,
                                  (ks != ks0 || q != 0 || kk != 0) ? 1u : 0u);
              }
            }
          }
          tc::mma_commit_pair(&empty[s]);
        }
        tc::mma_commit_pair(&acc_full[buf]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    tc::griddep_wait();
    const int etid = tid - 64;
    for (int jj = etid; jj < (p.dh >> 1); jj += kEpiThreads)
      theta[jj] = exp2(-(2.0 * (double)jj / (double)p.dh) * p.log2_base);
    tc::named_bar_sync(1, kEpiThreads);
    const int quarter = warp & 3;
    const int f_loc = quarter * 32 + lane;
    const int n_half = ((warp - 2) >> 2) * (kChunk / 2);  // this warp's 16 tokens of a chunk
    float* my_parts = p.partials + (size_t)blockIdx.x * 2 * BN * kBM;
    const uint32_t leader_acc_empty0 = tc::map_peer(tc::smem_u32(&acc_empty[0]), 0u);
    int j = 0;
    for (long long u = u_begin; u < u_end; ++j) {
      const int tile = tile_begin + j;
      const int ks0 = (j == 0) ? ks_begin : 0;
      const int ks1 = (int)min((long long)p.nks, ks0 + (u_end - u));
      u += ks1 - ks0;
      const int buf = p.nbuf == 2 ? (j & 1) : 0;
      const uint32_t use = p.nbuf == 2 ? (uint32_t)(j >> 1) : (uint32_t)j;
      const int fp = tile % p.n_fp, tt = tile / p.n_fp;
      const int m0 = tt * BN;
      const int fbase = fp * (2 * kBM) + rank * kBM;  // this CTA's first feature
      const bool whole = (ks0 == 0 && ks1 == p.nks);
      const uint32_t t_acc = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN);
      auto release_acc = [&]() {
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0)
            tc::mbar_arrive(&acc_empty[buf]);
          else
            tc::mbar_arrive_cluster(leader_acc_empty0 + (uint32_t)(buf * 8));
        }
      };

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
          // Q is a set: a packed fused row repeating an earlier row's slot is
          // reported once, by rank 0 of the first feature pair
          if (p.check_repeats && fp == 0 && rank == 0)
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
      tc::mbar_wait(&acc_full[buf], use & 1u, abort_flag, p.status);
      tc::tc_fence_after();

      bool run = true;
      bool own_in_tmem = true;  // this CTA's part of the tile is still (only) in TMEM
      int c_first = pair, c_last = pair;
      const long long tu0 = (long long)tile * p.nks;
      unsigned* cnt = &p.tile_cnt[(size_t)tile * 2 + rank];
      if (!whole) {
        c_first = owner_of(tu0, p.total_units, P);
        c_last = owner_of(tu0 + p.nks - 1, p.total_units, P);
        // The other contributors count up after storing their parts.  When they
        // all have, this CTA is the last one and merges its own part straight
        // from TMEM: no store, fence or atomic of its own.
        if (etid == 0) {
          const unsigned done = ld_acquire(cnt);
          *last_flag = (done == (unsigned)(c_last - c_first)) ? 2 : 0;
          if (*last_flag == 2) *cnt = 0u;  // reset for the next call
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
        release_acc();
        __threadfence();
        tc::named_bar_sync(1, kEpiThreads);
        if (etid == 0) {
          const unsigned prev = atomicAdd(cnt, 1u);
          *last_flag = (prev == (unsigned)(c_last - c_first));
          if (*last_flag) *cnt = 0u;
        }
        tc::named_bar_sync(1, kEpiThreads);
        run = *last_flag != 0;
        if (run) __threadfence();
      }
      if (run) {
        if (fp == 0 && rank == 0) {
          for (int n = etid; n < BN; n += kEpiThreads)
            if (m0 + n < p.M && tok_slot[n] < 0) set_status(p.status, FDLLM_ERR_BAD_INDEX);
        }
        // The part of contributor cb for this thread's feature row and 16 tokens
        // from column c (slot 0 when the tile is cb's first: unit_lo(cb) >= tu0).
        auto load_part = [&](int cb, int c, float* t) {
          const int sl = (p.total_units * cb >= tu0 * (long long)P) ? 0 : 1;
          const float* ps = p.partials + ((size_t)(2 * cb + rank) * 2 + sl) * BN * kBM +
                            (size_t)c * kBM + f_loc;
#pragma unroll
          for (int n = 0; n < kChunk / 2; ++n) t[n] = __ldcg(ps + (size_t)n * kBM);
        };
        // The first contributor whose part is in global memory has its next
        // chunk loaded while this chunk is rotated and stored, so the merge
        // does not wait out an L2 round trip per chunk.
        const int cb_pf = (c_first == pair && own_in_tmem) ? c_first + 1 : c_first;
        float pf[kChunk / 2];
        if (!whole && cb_pf <= c_last) load_part(cb_pf, n_half, pf);
        for (int cc = 0; cc < BN; cc += kChunk) {
          if (whole) {
            // BN is a multiple of 32: a warp's 16 columns are all in the tile
            float v[kChunk / 2];
            tc::tmem_ld16(t_acc + cc + n_half, v);
            tc::tmem_wait_ld();
#pragma unroll
            for (int n = 0; n < kChunk / 2; ++n) staging[f_loc * kPitch + n_half + n] = v[n];
          } else {
            // sum the parts of every contributor in pair order, the thread's
            // feature row over its 16 tokens: this CTA's part from TMEM when it
            // was never stored, the others' from global memory
            float cur[kChunk / 2];
#pragma unroll
            for (int n = 0; n < kChunk / 2; ++n) cur[n] = pf[n];
            if (cb_pf <= c_last && cc + kChunk < BN) load_part(cb_pf, cc + kChunk + n_half, pf);
            float v[kChunk / 2];
#pragma unroll
            for (int n = 0; n < kChunk / 2; ++n) v[n] = 0.f;
            for (int cb = c_first; cb <= c_last; ++cb) {
              float t[kChunk / 2];
              if (cb == pair && own_in_tmem) {
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
          epi::rope_store_chunk(p, staging, fbase, m0, cc, BN, tok_slot, tok_flag, tok_b, tok_pos,
                                theta, etid, kEpiThreads);
          tc::named_bar_sync(1, kEpiThreads);
        }
      }
      if (whole || own_in_tmem) release_acc();
    }
  }

  // every MMA that read this CTA's shared memory has completed (the epilogues
  // waited for them) and no arrival on the peer's barriers is still to come
  tc::tc_fence_before();
  __syncthreads();
  tc::cluster_sync();
  tc::tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc_pair(tmem, ncols);
  }
}

struct PairPlan {
  int BN, NM, nmma, nbuf, n_tt, n_fp, tiles, nks, subs, nsub_total, nstage, grid;
  long long total_units;
  size_t smem_bytes, partial_bytes, counter_bytes, xq_bytes;
};

constexpr size_t kSmemBudget = 227 * 1024;

// How many CTA pairs of the kernel can be resident at once with this much
// shared memory (cached; 0 when the query fails).
int max_pairs(size_t smem_bytes) {
  static size_t cached_smem = 0;
  static int cached = 0;
  if (smem_bytes != cached_smem) {
    cudaLaunchConfig_t c = {};
    c.gridDim = dim3(2);
    c.blockDim = dim3(kThreads);
    c.dynamicSmemBytes = smem_bytes;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    c.attrs = at;
    c.numAttrs = 1;
    int n = 0;
    if (cudaFuncSetAttribute(proj_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_bytes) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, proj_pair_kernel, &c) != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
    cached_smem = smem_bytes;
    cached = n;
  }
  return cached;
}

PairPlan plan_bn(int M, int D, int H, int dh, int num_sms, bool resident, int max_bn) {
  PairPlan q{};
  const int F = 3 * H * dh;
  q.n_tt = (M + max_bn - 1) / max_bn;
  const int per = (M + q.n_tt - 1) / q.n_tt;
  q.BN = ((per + 31) / 32) * 32;
  q.nmma = q.BN > 256 ? 2 : 1;
  q.NM = q.BN / q.nmma;
  q.nbuf = 2 * q.BN <= 512 ? 2 : 1;
  q.n_fp = (F + 2 * kBM - 1) / (2 * kBM);
  q.tiles = q.n_fp * q.n_tt;
  q.nsub_total = D / kSub;
  const size_t fixed = 1024 /*align*/ + (size_t)kBM * kPitch * 4 + 256 + 4 * kMaxBN * 4 + 64 * 8;
  const size_t sub = kASubBytes + (size_t)q.nmma * (q.NM / 2) * 128;
  // the k-step width (1, 2 or 4 subs) that keeps the most bytes in flight, at
  // least two stages and at most eight; ties go to the wider step
  size_t best = 0;
  for (int subs : {4, 2, 1}) {
    if (subs > q.nsub_total) continue;
    int ns = (int)((kSmemBudget - fixed) / (subs * sub));
    ns = ns < 8 ? ns : 8;
    if (ns < 2) continue;
    if ((size_t)ns * subs * sub > best) {
      best = (size_t)ns * subs * sub;
      q.subs = subs;
      q.nstage = ns;
    }
  }
  q.nks = (q.nsub_total + q.subs - 1) / q.subs;
  q.total_units = (long long)q.tiles * q.nks;
  q.smem_bytes = (size_t)q.nstage * q.subs * sub + fixed;
  // one wave of pairs: as many as are resident at once (clusters of two need
  // two SMs of one GPC), at most one per two SMs
  int pairs = num_sms / 2;
  if (resident) {
    const int mp = max_pairs(q.smem_bytes);
    if (mp > 0 && mp < pairs) pairs = mp;
  }
  if ((long long)pairs > q.total_units) pairs = (int)q.total_units;
  if (max_bn > kMaxBNStreamK && q.tiles <= pairs) pairs = q.tiles;  // whole tiles
  q.grid = 2 * pairs;
  // sized by the most columns a split tile has and one pair per two SMs, so
  // that one workspace serves every row count this kernel takes
  q.partial_bytes = align_up((size_t)(num_sms / 2) * 2 * 2 * kMaxBNStreamK * kBM * sizeof(float), 256);
  q.counter_bytes = align_up((size_t)q.tiles * 2 * sizeof(unsigned), 256);
  q.xq_bytes = align_up((size_t)M * D * 2, 256);
  return q;
}

// Up to 512 rows whose feature tiles fit in one wave of pairs: one token tile
// (two MMAs beyond 256 rows) and one whole tile per pair, so that W streams
// once and no tile is split or merged.  Otherwise: tiles of up to 256 tokens
// with two accumulators, so that each tile's epilogue overlaps the next tile's
// MMAs, spread over the pairs by stream-K.  The stream-K plan has at least as
// many tiles as the whole-tile one, so its workspace serves both.
PairPlan plan(int M, int D, int H, int dh, int num_sms, bool resident) {
  if (M <= kMaxBN) {
    PairPlan w = plan_bn(M, D, H, dh, num_sms, resident, kMaxBN);
    if (2LL * w.tiles == w.grid) return w;
  }
  return plan_bn(M, D, H, dh, num_sms, resident, kMaxBNStreamK);
}

}  // namespace

size_t proj_pair_workspace_bytes(int M, int D, int H, int dh, int num_sms) {
  if (M <= 0) return 256;
  const PairPlan q = plan_bn(M, D, H, dh, num_sms, false, kMaxBNStreamK);
  return q.partial_bytes + q.counter_bytes + q.xq_bytes;
}

cudaError_t launch_proj_pair(const ProjArgs& a, cudaStream_t stream) {
  const int M = a.B * a.rows_per_seq;
  if (M == 0) return cudaSuccess;
  const int E = a.H * a.dh, F = 3 * E;
  const int sms = device_sm_count();
  if (sms < 2) return cudaErrorInvalidValue;
  const PairPlan q = plan(M, a.D, a.H, a.dh, sms, true);
  if (q.partial_bytes + q.counter_bytes + q.xq_bytes > a.ws_bytes) return cudaErrorInvalidValue;
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
  const bool packed = a.verify || a.packed;
  const void* xsrc = packed ? a.x : static_cast<const void*>(xq);
  {
    // rows past M are outside the tensor: TMA fills them with zeros
    const uint64_t dims[2] = {(uint64_t)a.D, (uint64_t)M};
    const uint64_t strides[1] = {(uint64_t)a.D * 2};
    const uint32_t box[2] = {kSub, (uint32_t)(q.NM / 2)};
    if (!encode_bf16_map(&tm_x, 2, xsrc, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B))
      return cudaErrorInvalidValue;
  }
  PairParams p{};
  p.M = M; p.F = F; p.D = a.D; p.E = E; p.N = a.N; p.H = a.H; p.dh = a.dh;
  p.rows_per_seq = a.rows_per_seq; p.S_max = a.S_max; p.verify = a.verify;
  p.check_repeats = (!a.verify && a.packed) ? 1 : 0;
  p.BN = q.BN; p.NM = q.NM; p.nmma = q.nmma; p.nbuf = q.nbuf; p.n_tt = q.n_tt; p.n_fp = q.n_fp;
  p.tiles = q.tiles; p.nks = q.nks; p.subs = q.subs; p.nsub_total = q.nsub_total;
  p.nstage = q.nstage; p.total_units = q.total_units;
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
    e = launch_proj_prep(a, xq, stream);
    if (e != cudaSuccess) return e;
  }
  e = cudaFuncSetAttribute(proj_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)q.smem_bytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(q.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = q.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, proj_pair_kernel, tm_w, tm_x, p);
  count_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fdllm
