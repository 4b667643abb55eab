// Full-cache attention on the 5th-generation tensor cores (bf16 storage).
//
// Flash-dLLM review, "How It Works", Step 1: Draft: after the new k, v are
// written, every query of Q attends over the whole bidirectional cache; with
// the verify metadata the Flash-Verify view rule applies ("Flash-Verify",
// sec. 2.3; Step 1: Verification): draft and mask views share positions, each
// hidden from the other, and the mask view's keys live in side slots.
//
// The work is a stream over the cache (HBM-bound), with few queries per head
// (16..64).  Layout chosen so the tensor core wastes nothing on padding:
//   S^T [128 keys x NQ queries] = K_tile [128 x dh] . Q^T       (M = keys)
//   O^T [dh x NQ]              += V_tile^T [dh x 128] . P^T      (M = dh)
// so one thread owns one key of a tile (its row of S^T) and, later, one head
// dimension of O^T.  Softmax keeps a running max per query column that is
// raised only when a tile's max exceeds it by more than 2^8 (the accumulators
// are then rescaled), so most tiles need no rescaling; P goes to shared memory
// as bf16 in the MN-major swizzled layout the PV MMA reads.
//
// Persistent stream-K: one CTA per SM; units (item = (sequence, head, query
// chunk), 128-key tile) are laid out item after item and every CTA takes an
// equal contiguous range, so the cache stream is balanced whatever B, H, N.
// An item split between CTAs leaves (O, m, l) partials; its last contributor
// (atomic counter) merges them in CTA order and writes the output.
//
//   warp 0      TMA producer: Q chunk per item, K and V tiles (128 x 64 boxes)
//   warp 1      TMEM allocation; lane 0 issues QK (ahead by one tile) and PV
//   warps 2-5   softmax over S^T, P, accumulator rescale, epilogue
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"
#include "tmap.h"

namespace fdllm {

namespace {

constexpr int kKT = 128;  // keys per tile
constexpr int kThreads = 192;
constexpr int kSmx = 128;  // softmax threads
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kThresh = 8.f;  // lazy rescale threshold (log2 units)
constexpr int kMaxRows = 512;   // verify rows per sequence held in shared memory

struct AttnTcParams {
  int B, N, H, rows, S_max, causal;
  int n_qc, n_cache_tiles, n_side_tiles, tpi, nstage;
  long long total_units;
  float qk_scale;  // log2(e) / sqrt(dh)
  const int32_t* pos;
  const int8_t* view;
  const int32_t* rank;
  __nv_bfloat16* out;
  int* status;
  float* partials;     // [grid][2][NQ*DH + 2*NQ]
  unsigned* item_cnt;  // [items], zero between calls
};

__device__ __forceinline__ long long unit_lo(long long total, int G, int c) {
  return total * c / G;
}
__device__ __forceinline__ int owner_of(long long u, long long total, int G) {
  int c = (int)(((u + 1) * G - 1) / total);
  if (c >= G) c = G - 1;
  while (c > 0 && unit_lo(total, G, c) > u) --c;
  while (c + 1 < G && unit_lo(total, G, c + 1) <= u) ++c;
  return c;
}

__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
// OR of a predicate over `n` threads at named barrier `id`.
__device__ __forceinline__ bool bar_any(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

template <int NQ>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, float* v) {
#pragma unroll
  for (int c = 0; c < NQ; c += 16) tc::tmem_ld16(taddr + c, v + c);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Shared-memory layout of one CTA (offsets from a 1024-aligned base).
template <int NQ, int DH>
struct Smem {
  static constexpr int kBoxes = DH / 64;
  static constexpr uint32_t kTileBytes = kBoxes * 16384;         // K or V tile
  static constexpr uint32_t kStageBytes = 2 * kTileBytes;        // K then V
  static constexpr uint32_t kQBytes = kBoxes * NQ * 128;         // one Q chunk
  static constexpr uint32_t kPRow = NQ * 2;                      // bytes per key row of P
  static constexpr uint32_t kPBytes = kKT * kPRow;
};

template <int NQ, int DH, bool VERIFY>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_ks,
               const __grid_constant__ CUtensorMap tm_vs, AttnTcParams p) {
  using L = Smem<NQ, DH>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int NS = p.nstage;
  uint8_t* q_buf = smem + NS * L::kStageBytes;
  uint8_t* p_buf = q_buf + 2 * L::kQBytes;  // 1024-aligned (kQBytes is a multiple of 1024)
  uint8_t* misc = p_buf + ((L::kPBytes + 1023) / 1024) * 1024;
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* kv_empty = kv_full + 8;
  uint64_t* q_full = kv_empty + 8;   // [2]
  uint64_t* q_empty = q_full + 2;    // [2]
  uint64_t* s_full = q_empty + 2;    // [2]
  uint64_t* s_empty = s_full + 2;    // [2]
  uint64_t* p_full = s_empty + 2;
  uint64_t* pv_done = p_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pv_done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* last_flag = abort_flag + 1;
  int* n_draft_s = last_flag + 1;
  int* n_side_s = n_draft_s + 1;
  float* m_run = reinterpret_cast<float*>(misc + 512);      // [NQ]
  float* alpha = m_run + 128;                               // [NQ]
  float* wred = alpha + 128;                                // [4][NQ]
  int* col_meta = reinterpret_cast<int*>(wred + 4 * 128);   // [NQ] view | rank << 2
  int* draft_pos = reinterpret_cast<int*>(misc + 4096);     // [kMaxRows]
  int* draft_rank = draft_pos + kMaxRows;                   // [kMaxRows]
  int* side_rank = draft_rank + kMaxRows;                   // [kMaxRows]

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const long long u0 = unit_lo(p.total_units, G, cta);
  const long long u1 = unit_lo(p.total_units, G, cta + 1);
  const int T = (int)(u1 - u0);
  const int tpi = p.tpi;

  uint32_t ncols = 32;
  while ((int)ncols < 3 * NQ) ncols <<= 1;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(&kv_full[s], 1);
      tc::mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&q_full[b], 1);
      tc::mbar_init(&q_empty[b], 1);
      tc::mbar_init(&s_full[b], 1);
      tc::mbar_init(&s_empty[b], kSmx);
    }
    tc::mbar_init(p_full, kSmx);
    tc::mbar_init(pv_done, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, ncols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_o = tmem + 2 * NQ;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      const uint64_t pol_kv = tc::policy_evict_first();
      const uint64_t pol_q = tc::policy_evict_last();
      int seg = -1;
      for (int i = 0; i < T; ++i) {
        const long long u = u0 + i;
        const int item = (int)(u / tpi), t = (int)(u % tpi);
        const int qc = item % p.n_qc, bh = item / p.n_qc;
        const int b = bh / p.H, h = bh % p.H;
        if (i == 0 || t == 0) {
          ++seg;
          const int qb = seg & 1;
          if (!tc::mbar_wait(&q_empty[qb], ((uint32_t)(seg >> 1) & 1u) ^ 1u, abort_flag, p.status)) break;
          tc::mbar_arrive_expect_tx(&q_full[qb], L::kQBytes);
#pragma unroll
          for (int x = 0; x < L::kBoxes; ++x)
            tc::tma_load_4d(q_buf + qb * L::kQBytes + x * NQ * 128, &tm_q, &q_full[qb], x * 64, h,
                            qc * NQ, b, pol_q);
        }
        const int s = i % NS;
        if (!tc::mbar_wait(&kv_empty[s], ((uint32_t)(i / NS) & 1u) ^ 1u, abort_flag, p.status)) break;
        uint8_t* kd = smem + s * L::kStageBytes;
        uint8_t* vd = kd + L::kTileBytes;
        tc::mbar_arrive_expect_tx(&kv_full[s], L::kStageBytes);
        const bool side = VERIFY && t >= p.n_cache_tiles;
        const int key0 = (side ? t - p.n_cache_tiles : t) * kKT;
#pragma unroll
        for (int x = 0; x < L::kBoxes; ++x) {
          tc::tma_load_3d(kd + x * 16384, side ? &tm_ks : &tm_k, &kv_full[s], x * 64, key0, bh, pol_kv);
          tc::tma_load_3d(vd + x * 16384, side ? &tm_vs : &tm_v, &kv_full[s], x * 64, key0, bh, pol_kv);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc::idesc_bf16(kKT, NQ, false, false);
      constexpr uint32_t idesc_pv = tc::idesc_bf16(kKT, NQ, true, true);
      constexpr uint32_t p_swz = NQ == 64 ? 2u : (NQ == 32 ? 4u : 6u);
      const uint32_t p_addr = tc::smem_u32(p_buf);
      int seg = -1;
      bool ok = true;
      for (int i = 0; i <= T && ok; ++i) {
        if (i < T) {
          const long long u = u0 + i;
          const int t = (int)(u % tpi);
          const bool first = (i == 0 || t == 0);
          const bool last = (i == T - 1 || t == tpi - 1);
          if (first) ++seg;
          const int qb = seg & 1;
          const int s = i % NS;
          if (!tc::mbar_wait(&kv_full[s], (uint32_t)(i / NS) & 1u, abort_flag, p.status)) { ok = false; break; }
          if (first && !tc::mbar_wait(&q_full[qb], (uint32_t)(seg >> 1) & 1u, abort_flag, p.status)) { ok = false; break; }
          const int sb = i & 1;
          if (!tc::mbar_wait(&s_empty[sb], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag, p.status)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t k_addr = tc::smem_u32(smem + s * L::kStageBytes);
          const uint32_t q_addr = tc::smem_u32(q_buf + qb * L::kQBytes);
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {
            const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t qo = (kk >> 2) * NQ * 128 + (kk & 3) * 32;
            tc::mma_bf16(tmem + sb * NQ, tc::smem_desc(k_addr + ko, 16, 1024, 2),
                         tc::smem_desc(q_addr + qo, 16, 1024, 2), idesc_qk, kk != 0);
          }
          tc::mma_commit(&s_full[sb]);
          if (last) tc::mma_commit(&q_empty[qb]);
        }
        if (i >= 1) {
          const int j = i - 1;
          const long long u = u0 + j;
          const bool first = (j == 0 || (u % tpi) == 0);
          if (!tc::mbar_wait(p_full, (uint32_t)j & 1u, abort_flag, p.status)) { ok = false; break; }
          tc::tc_fence_after();
          const int s = j % NS;
          const uint32_t v_addr = tc::smem_u32(smem + s * L::kStageBytes + L::kTileBytes);
#pragma unroll
          for (int kk = 0; kk < kKT / 16; ++kk) {
            const uint64_t da = tc::smem_desc(v_addr + kk * 2048, DH == 128 ? 16384 : 0, 1024, 2);
            const uint64_t db = tc::smem_desc(p_addr + kk * 16 * L::kPRow, 0, 8 * L::kPRow, p_swz);
            tc::mma_bf16(tmem_o, da, db, idesc_pv, (first && kk == 0) ? 0u : 1u);
          }
          tc::mma_commit(pv_done);
          tc::mma_commit(&kv_empty[s]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int st = tid - 64;           // 0..127
    const int quarter = warp & 3;
    const int kl = quarter * 32 + lane;  // TMEM lane: key of S^T, dh row of O^T
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const size_t part_floats = (size_t)NQ * DH + 2 * NQ;
    float l[NQ];
    int seg = -1;
    int n_draft = 0, n_side = 0;
    int pv_waited = -1;  // index of the last PV this thread waited for
    int seg_t0 = 0;      // tile index at which the current segment started
    for (int i = 0; i < T; ++i) {
      const long long u = u0 + i;
      const int item = (int)(u / tpi), t = (int)(u % tpi);
      const bool first = (i == 0 || t == 0);
      const bool last = (i == T - 1 || t == tpi - 1);
      const int qc = item % p.n_qc, bh = item / p.n_qc;
      const int b = bh / p.H;
      if (first) {
        ++seg;
        seg_t0 = t;
        // segment metadata: running max reset, verify tables of sequence b
        if (st < NQ) m_run[st] = -INFINITY;
        if (VERIFY) {
          const int r0 = b * p.rows;
          if (st < NQ) {
            const int r = qc * NQ + st;
            col_meta[st] = (r < p.rows) ? ((int)p.view[r0 + r] | (p.rank[r0 + r] << 2)) : 0;
          }
          if (warp == 2 || warp == 3) {
            // ballot compaction of draft rows (warp 2) and mask rows (warp 3)
            const int want = warp == 2 ? 1 : 2;
            int base = 0;
            for (int r = lane; r - lane < p.rows; r += 32) {
              const int vw = r < p.rows ? (int)p.view[r0 + r] : -1;
              const unsigned bal = __ballot_sync(0xffffffffu, vw == want);
              const int at = base + __popc(bal & ((1u << lane) - 1u));
              if (vw == want && at < kMaxRows) {
                if (want == 1) {
                  draft_pos[at] = p.pos[r0 + r];
                  draft_rank[at] = p.rank[r0 + r];
                } else {
                  side_rank[at] = p.rank[r0 + r];
                }
              }
              base += __popc(bal);
            }
            if (lane == 0) {
              if (want == 1) *n_draft_s = min(base, kMaxRows);
              else *n_side_s = min(min(base, p.S_max), kMaxRows);
            }
          }
        }
#pragma unroll
        for (int c = 0; c < NQ; ++c) l[c] = 0.f;
        tc::named_bar_sync(1, kSmx);
        if (VERIFY) {
          n_draft = *n_draft_s;
          n_side = *n_side_s;
        }
      }

      // ---- scores of this tile (thread = key kl)
      const int sb = i & 1;
      // after a timeout every later wait returns at once: keep going so that all
      // softmax threads still meet at the same named barriers
      tc::mbar_wait(&s_full[sb], (uint32_t)(i >> 1) & 1u, abort_flag, p.status);
      tc::tc_fence_after();
      float s[NQ];
      tmem_ld_row<NQ>(tmem + lane_off + sb * NQ, s);
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      tc::mbar_arrive(&s_empty[sb]);

      const bool side_tile = VERIFY && t >= p.n_cache_tiles;
      const int key = (side_tile ? t - p.n_cache_tiles : t) * kKT + kl;
      const bool valid = key < (side_tile ? n_side : p.N);
#pragma unroll
      for (int c = 0; c < NQ; ++c) s[c] = valid ? s[c] * p.qk_scale : -INFINITY;
      if (VERIFY && valid) {
        if (side_tile) {
          const int srank = side_rank[key];
#pragma unroll
          for (int c = 0; c < NQ; ++c) {
            const int cm = col_meta[c];
            if (!visible_side(cm & 3, cm >> 2, srank, p.causal)) s[c] = -INFINITY;
          }
        } else {
          int kdr = -1;
          for (int d = 0; d < n_draft; ++d)
            if (draft_pos[d] == key) kdr = draft_rank[d];
          if (kdr >= 0) {
#pragma unroll
            for (int c = 0; c < NQ; ++c) {
              const int cm = col_meta[c];
              if (!visible_cache(cm & 3, cm >> 2, kdr, p.causal)) s[c] = -INFINITY;
            }
          }
        }
      }

      // ---- running max: raised only when a column's tile max exceeds it by 2^8
      bool need = false;
#pragma unroll
      for (int c = 0; c < NQ; ++c) need |= warp_max(s[c]) > m_run[c] + kThresh;
      const bool any = bar_any(2, kSmx, need);
      if (any) {
#pragma unroll
        for (int c = 0; c < NQ; ++c) {
          const float wm = warp_max(s[c]);
          if (lane == (c & 31)) wred[quarter * NQ + c] = wm;
        }
        tc::named_bar_sync(1, kSmx);
        if (st < NQ) {
          const float mo = m_run[st];
          const float tm = fmaxf(fmaxf(wred[st], wred[NQ + st]), fmaxf(wred[2 * NQ + st], wred[3 * NQ + st]));
          const float mn = (tm > mo + kThresh) ? tm : mo;
          alpha[st] = (mo == -INFINITY) ? 0.f : exp2f(mo - mn);
          m_run[st] = mn;
        }
        tc::named_bar_sync(1, kSmx);
#pragma unroll
        for (int c = 0; c < NQ; ++c) l[c] *= alpha[c];
      }

      // ---- the previous PV must be complete: P buffer free, O stable
      if (i > 0 && pv_waited < i - 1) {
        tc::mbar_wait(pv_done, (uint32_t)(i - 1) & 1u, abort_flag, p.status);
        pv_waited = i - 1;
      }
      tc::tc_fence_after();
      if (any && !first) {
        // rescale the O^T accumulator, column c by alpha[c]
        float o[16];
#pragma unroll
        for (int c0 = 0; c0 < NQ; c0 += 16) {
          tc::tmem_ld16(tmem_o + lane_off + c0, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) o[c] *= alpha[c0 + c];
          tc::tmem_st16(tmem_o + lane_off + c0, o);
        }
        tc::tmem_wait_st();
      }
      // a side tile's key rows past the used slots may hold anything: zero them
      if (side_tile && !valid) {
        uint8_t* vrow = smem + (i % NS) * L::kStageBytes + L::kTileBytes + kl * 128;
#pragma unroll
        for (int x = 0; x < L::kBoxes; ++x)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<uint4*>(vrow + x * 16384 + q * 16) = make_uint4(0u, 0u, 0u, 0u);
      }

      // ---- P = exp2(s - m), row kl of the MN-major swizzled P^T tile
      {
        uint32_t pk[NQ / 2];
#pragma unroll
        for (int c = 0; c < NQ; c += 2) {
          const float m0 = m_run[c], m1 = m_run[c + 1];
          const float p0 = (m0 == -INFINITY) ? 0.f : exp2f(s[c] - m0);
          const float p1 = (m1 == -INFINITY) ? 0.f : exp2f(s[c + 1] - m1);
          l[c] += p0;
          l[c + 1] += p1;
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
        uint8_t* prow = p_buf + kl * L::kPRow;
        constexpr uint32_t mask = L::kPRow / 16 - 1;  // swizzle span: row bytes
#pragma unroll
        for (int ch = 0; ch < NQ / 8; ++ch) {
          const uint32_t off = (uint32_t)(kl * L::kPRow + ch * 16);
          const uint32_t sw = off ^ (((off >> 7) & mask) << 4);
          *reinterpret_cast<uint4*>(p_buf + sw) =
              make_uint4(pk[ch * 4], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
        }
        (void)prow;
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(p_full);

      if (last) {
        // ---- segment done: O^T complete after this tile's PV
        tc::mbar_wait(pv_done, (uint32_t)i & 1u, abort_flag, p.status);
        pv_waited = i;
        tc::tc_fence_after();
        // total l per column: butterfly within each warp, then across warps
#pragma unroll
        for (int c = 0; c < NQ; ++c) {
          float v = l[c];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == (c & 31)) wred[quarter * NQ + c] = v;
        }
        tc::named_bar_sync(1, kSmx);
        float o[NQ];
        tmem_ld_row<NQ>(tmem_o + lane_off, o);
        tc::tmem_wait_ld();
        const bool whole = (seg_t0 == 0) && (t == tpi - 1);
        const int h = bh % p.H;
        if (whole) {
          if (kl < DH) {
#pragma unroll
            for (int c = 0; c < NQ; ++c) {
              const int r = qc * NQ + c;
              if (r < p.rows) {
                const float lt = wred[c] + wred[NQ + c] + wred[2 * NQ + c] + wred[3 * NQ + c];
                p.out[(((size_t)b * p.rows + r) * p.H + h) * DH + kl] = __float2bfloat16_rn(o[c] / lt);
              }
            }
          }
        } else {
          // partial item: (O, m, l) to this CTA's slot; the last contributor merges
          const int slot = (item == (int)(u0 / tpi)) ? 0 : 1;
          float* part = p.partials + ((size_t)cta * 2 + slot) * part_floats;
          if (kl < DH) {
#pragma unroll
            for (int c = 0; c < NQ; ++c) part[(size_t)c * DH + kl] = o[c];
          }
          if (st < NQ) {
            part[(size_t)NQ * DH + st] = m_run[st];
            part[(size_t)NQ * DH + NQ + st] = wred[st] + wred[NQ + st] + wred[2 * NQ + st] + wred[3 * NQ + st];
          }
          __threadfence();
          tc::named_bar_sync(1, kSmx);
          const long long iu0 = (long long)item * tpi;
          const int c_first = owner_of(iu0, p.total_units, G);
          const int c_last = owner_of(iu0 + tpi - 1, p.total_units, G);
          if (st == 0) {
            const unsigned prev = atomicAdd(&p.item_cnt[item], 1u);
            *last_flag = (prev == (unsigned)(c_last - c_first));
            if (*last_flag) p.item_cnt[item] = 0u;
          }
          tc::named_bar_sync(1, kSmx);
          if (*last_flag) {
            __threadfence();
            // merge the contributors' (O, m, l) in CTA order, 16 at a time:
            // weights 2^(m - M) per column first, then every column's loads
            // of one contributor in flight together
            float* wts = reinterpret_cast<float*>(draft_pos);  // [16][NQ], free here
            float M = -INFINITY;
            if (st < NQ) {
              for (int cb = c_first; cb <= c_last; ++cb) {
                const int sl = (item == (int)(unit_lo(p.total_units, G, cb) / tpi)) ? 0 : 1;
                M = fmaxf(M, __ldcg(p.partials + ((size_t)cb * 2 + sl) * part_floats + (size_t)NQ * DH + st));
              }
            }
            float lt = 0.f;
            float acc[NQ];
#pragma unroll
            for (int c = 0; c < NQ; ++c) acc[c] = 0.f;
            for (int g0 = c_first; g0 <= c_last; g0 += 16) {
              const int g1 = min(c_last + 1, g0 + 16);
              if (st < NQ) {
                for (int cb = g0; cb < g1; ++cb) {
                  const int sl = (item == (int)(unit_lo(p.total_units, G, cb) / tpi)) ? 0 : 1;
                  const float* pc = p.partials + ((size_t)cb * 2 + sl) * part_floats;
                  const float mc = __ldcg(pc + (size_t)NQ * DH + st);
                  const float w = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
                  lt += w * __ldcg(pc + (size_t)NQ * DH + NQ + st);
                  wts[(cb - g0) * NQ + st] = w;
                }
              }
              tc::named_bar_sync(1, kSmx);
              if (kl < DH) {
                for (int cb = g0; cb < g1; ++cb) {
                  const int sl = (item == (int)(unit_lo(p.total_units, G, cb) / tpi)) ? 0 : 1;
                  const float* pc = p.partials + ((size_t)cb * 2 + sl) * part_floats + kl;
                  float ov[NQ];
#pragma unroll
                  for (int c = 0; c < NQ; ++c) ov[c] = __ldcg(pc + (size_t)c * DH);
#pragma unroll
                  for (int c = 0; c < NQ; ++c) acc[c] += wts[(cb - g0) * NQ + c] * ov[c];
                }
              }
              tc::named_bar_sync(1, kSmx);
            }
            if (st < NQ) alpha[st] = lt;
            tc::named_bar_sync(1, kSmx);
            if (kl < DH) {
#pragma unroll
              for (int c = 0; c < NQ; ++c) {
                const int r = qc * NQ + c;
                if (r < p.rows)
                  p.out[(((size_t)b * p.rows + r) * p.H + h) * DH + kl] = __float2bfloat16_rn(acc[c] / alpha[c]);
              }
            }
          }
        }
        tc::tc_fence_before();
        tc::named_bar_sync(1, kSmx);
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

struct AttnPlan {
  int NQ, n_qc, nct, nst, tpi, nstage, grid;
  long long items, total_units;
  size_t smem_bytes, partial_bytes, counter_bytes;
};

constexpr size_t kSmemBudget = 227 * 1024;

AttnPlan plan(int B, int N, int H, int dh, int rows, int S_max, int verify, int num_sms) {
  AttnPlan q{};
  q.NQ = rows <= 16 ? 16 : (rows <= 32 ? 32 : 64);
  q.n_qc = (rows + q.NQ - 1) / q.NQ;
  q.nct = (N + kKT - 1) / kKT;
  q.nst = (verify && S_max > 0) ? (S_max + kKT - 1) / kKT : 0;
  q.tpi = q.nct + q.nst;
  q.items = (long long)B * H * q.n_qc;
  q.total_units = q.items * q.tpi;
  q.grid = (int)(q.total_units < num_sms ? q.total_units : num_sms);
  const size_t boxes = dh / 64;
  const size_t stage = 2 * boxes * 16384;
  const size_t qbytes = boxes * q.NQ * 128;
  const size_t pbytes = ((size_t)kKT * q.NQ * 2 + 1023) / 1024 * 1024;
  const size_t fixed = 1024 + 2 * qbytes + pbytes + 4096 + 3 * kMaxRows * 4;
  int ns = (int)((kSmemBudget - fixed) / stage);
  if (ns > 8) ns = 8;
  q.nstage = ns;
  q.smem_bytes = fixed + (size_t)ns * stage;
  q.partial_bytes = align_up((size_t)q.grid * 2 * ((size_t)q.NQ * dh + 2 * q.NQ) * sizeof(float), 256);
  q.counter_bytes = align_up((size_t)q.items * sizeof(unsigned), 256);
  return q;
}

template <int NQ, int DH, bool VERIFY>
cudaError_t launch_t(const AttnArgs& a, const AttnPlan& q, AttnTcParams prm, const CUtensorMap* maps,
                     cudaStream_t stream) {
  auto kern = attn_tc_kernel<NQ, DH, VERIFY>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)q.smem_bytes);
  if (e != cudaSuccess) return e;
  kern<<<q.grid, kThreads, q.smem_bytes, stream>>>(maps[0], maps[1], maps[2], maps[3], maps[4], prm);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

size_t attn_tc_workspace_bytes(int B, int N, int H, int dh, int rows, int S_max, int verify,
                               int num_sms) {
  if (B * rows <= 0) return 256;
  const AttnPlan q = plan(B, N, H, dh, rows, S_max, verify, num_sms);
  return q.partial_bytes + q.counter_bytes;
}

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t stream) {
  if (a.B * a.rows_per_seq == 0) return cudaSuccess;
  if (a.verify && a.rows_per_seq > kMaxRows) return cudaErrorInvalidValue;
  const AttnPlan q = plan(a.B, a.N, a.H, a.dh, a.rows_per_seq, a.S_max, a.verify, device_sm_count());
  if (q.nstage < 2) return cudaErrorInvalidValue;
  if (q.partial_bytes + q.counter_bytes > a.ws_bytes) return cudaErrorInvalidValue;
  const int dh = a.dh, E = a.H * a.dh;
  CUtensorMap maps[5];
  {
    // q [B, rows, H, dh]: box {64 dh, 1 head, NQ rows, 1 sequence}
    const uint64_t dims[4] = {(uint64_t)dh, (uint64_t)a.H, (uint64_t)a.rows_per_seq, (uint64_t)a.B};
    const uint64_t strides[3] = {(uint64_t)dh * 2, (uint64_t)E * 2, (uint64_t)a.rows_per_seq * E * 2};
    const uint32_t box[4] = {64, 1, (uint32_t)q.NQ, 1};
    if (!encode_bf16_map(&maps[0], 4, a.q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B))
      return cudaErrorInvalidValue;
  }
  const void* srcs[4] = {a.k_cache, a.v_cache, a.verify ? a.k_side : a.k_cache,
                         a.verify ? a.v_side : a.v_cache};
  for (int i = 0; i < 4; ++i) {
    const bool side = i >= 2 && a.verify;
    const uint64_t n = side ? (uint64_t)(a.S_max > 0 ? a.S_max : 1) : (uint64_t)a.N;
    const uint64_t dims[3] = {(uint64_t)dh, n, (uint64_t)a.B * a.H};
    const uint64_t strides[2] = {(uint64_t)dh * 2, n * dh * 2};
    const uint32_t box[3] = {64, kKT, 1};
    const void* base = srcs[i];
    if (side && a.S_max == 0) base = a.k_cache;  // never read: no side tiles
    if (!encode_bf16_map(&maps[1 + i], 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
      return cudaErrorInvalidValue;
  }
  AttnTcParams prm{};
  prm.B = a.B; prm.N = a.N; prm.H = a.H; prm.rows = a.rows_per_seq; prm.S_max = a.S_max;
  prm.causal = a.causal_cross;
  prm.n_qc = q.n_qc; prm.n_cache_tiles = q.nct; prm.n_side_tiles = q.nst; prm.tpi = q.tpi;
  prm.nstage = q.nstage; prm.total_units = q.total_units;
  prm.qk_scale = kLog2e / sqrtf((float)dh);
  prm.pos = a.pos; prm.view = a.view; prm.rank = a.rank;
  prm.out = static_cast<__nv_bfloat16*>(a.out);
  prm.status = a.status;
  prm.partials = static_cast<float*>(a.ws);
  prm.item_cnt = reinterpret_cast<unsigned*>(static_cast<char*>(a.ws) + q.partial_bytes);

#define FDLLM_ATTN_CASE(NQv, DHv)                                                           \
  if (q.NQ == NQv && dh == DHv)                                                            \
    return a.verify ? launch_t<NQv, DHv, true>(a, q, prm, maps, stream)                    \
                    : launch_t<NQv, DHv, false>(a, q, prm, maps, stream);
  FDLLM_ATTN_CASE(16, 64)
  FDLLM_ATTN_CASE(32, 64)
  FDLLM_ATTN_CASE(64, 64)
  FDLLM_ATTN_CASE(16, 128)
  FDLLM_ATTN_CASE(32, 128)
  FDLLM_ATTN_CASE(64, 128)
#undef FDLLM_ATTN_CASE
  return cudaErrorInvalidValue;
}

}  // namespace fdllm
