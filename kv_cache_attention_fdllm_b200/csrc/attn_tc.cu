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
// Three ways to spread the units (item = (sequence, head, query chunk),
// 128-key tile) over the SMs:
//   cluster mode (at most SMs/2 items): one thread-block cluster of cs <= 8
//     CTAs per item, each CTA an equal share of its tiles.  The CTAs leave
//     their (O, m, l) partials in their own shared memory and, after a cluster
//     barrier, each merges a slice of the head dimension reading the others'
//     partials through distributed shared memory.
//   whole items (up to two waves, when no slower by the plan's cost model):
//     one CTA per item, no merge.
//   persistent stream-K (the rest): one CTA per SM; units are laid out item
//     after item and every CTA takes an equal contiguous range, so the cache
//     stream is balanced whatever B, H, N.  An item split between CTAs leaves
//     (O, m, l) partials in global memory; its last contributor (atomic
//     counter) merges them in CTA order and writes the output.
//
//   warp 0      TMA producer: Q chunk per item, K and V tiles (128 x 64 boxes)
//   warp 1      TMEM allocation; lane 0 issues QK (ahead by one tile) and PV
//   warps 2..   softmax over S^T, P, accumulator rescale, epilogue: NQ/kCols
//               groups of 4 warps (8 warps at NQ = 32, 48 and 64, 4 at NQ = 16)
//   last warp   finisher: the item counts of partial segments (stream-K)
//
// The O^T accumulator is double-buffered in TMEM by segment (the tiles of one
// item in a CTA's range), so a segment's end costs the softmax warps only the
// reduction of l: its output or partial is written at the end of a later tile,
// once its last PV is done, while the next segment's PVs accumulate in the
// other buffer.  A partial's writers signal the finisher, which fences and takes the
// item count off the softmax warps' path; the items this CTA completes last
// are merged after its range.
//
// Launched as a programmatic dependent: the prologue and an L2 prefetch of
// the first cache tiles run before the grid-dependency wait; every thread
// waits before it reads anything an earlier kernel wrote.  The kernel leaves
// each row's log2 softmax normaliser (per head) for the tracked-set selection.
#include <limits.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"
#include "tmap.h"

namespace fdllm {

namespace {

constexpr int kKT = 128;  // keys per tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kThresh = 8.f;  // lazy rescale threshold (log2 units)
constexpr int kMaxRows = 512;   // verify rows per sequence held in shared memory
constexpr int kDraftTab = 2048; // cache slots a segment's draft-rank table covers
constexpr int kL2PrefetchTiles = 4;  // cache tiles per CTA warmed in L2 before the dependency wait
// Costs in tiles of time, for choosing between one CTA per whole item and
// stream-K: an item boundary inside a stream-K range (its result is written
// later, off the softmax warps' path), a CTA's cold start, and the merge of the
// items a stream-K CTA completes last
constexpr double kBoundaryTiles = 1.0;
constexpr double kStartTiles = 3.0;
constexpr double kMergeTiles = 3.0;
// work splits (the values fdllm_attention_split reports)
constexpr int kSplitStreamK = 1, kSplitWholeItems = 2, kSplitClusters = 3;

struct AttnTcParams {
  int B, N, H, rows, S_max, causal;
  int n_qc, n_cache_tiles, n_side_tiles, tpi, nk, nv;
  long long total_units;
  float qk_scale;  // log2(e) / sqrt(dh)
  const int32_t* pos;
  const int8_t* view;
  const int32_t* rank;
  const __nv_bfloat16* k_cache;  // [B, H, N, DH], for the L2 prefetch
  const __nv_bfloat16* v_cache;
  __nv_bfloat16* out;
  float* lse;          // [B, rows, H] log2 softmax denominators, or null
  int* status;
  int cs;              // cluster size in cluster mode, 0 in stream-K mode
  float* partials;     // [grid][2][NQ*DH + 2*NQ]
  unsigned* item_cnt;  // [items], zero between calls
};

__device__ __forceinline__ long long unit_lo(long long total, int G, int c) {
  const long long a = total * c;
  return a <= INT_MAX ? (long long)((int)a / G) : a / G;
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

// a / b for a unit index: 32-bit division when a fits (64-bit integer division
// is a long software routine)
__device__ __forceinline__ int unit_div(long long a, int b) {
  return a <= INT_MAX ? (int)a / b : (int)(a / b);
}

// (item, tile within the item, query chunk, sequence*head) of a unit, advanced
// one unit at a time without division.
struct UnitCursor {
  int item, t, qc, bh;
  __device__ __forceinline__ void init(long long u, int tpi, int n_qc) {
    item = unit_div(u, tpi);
    t = (int)(u - (long long)item * tpi);
    bh = item / n_qc;
    qc = item - bh * n_qc;
  }
  __device__ __forceinline__ void next(int tpi, int n_qc) {
    if (++t == tpi) {
      t = 0;
      ++item;
      if (++qc == n_qc) {
        qc = 0;
        ++bh;
      }
    }
  }
};

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

// Bookkeeping for polling loops: after kWaitLimitNs without progress the
// loop gives up (records FDLLM_ERR_TIMEOUT and sets the abort flag).
struct IdleClock {
  uint64_t t0 = 0;
  uint32_t spins = 0;
  __device__ __forceinline__ void reset() { t0 = 0; spins = 0; }
  __device__ __forceinline__ bool idle(volatile int* abort, int* status) {
    if ((++spins & 63u) != 0) return true;
    if (*abort) return false;
    const uint64_t now = global_ns();
    if (t0 == 0) {
      t0 = now;
    } else if (now - t0 > kWaitLimitNs) {
      *abort = 1;
      set_status(status, FDLLM_ERR_TIMEOUT);
      return false;
    }
    return true;
  }
};

// 2^x on the special-function unit (flush-to-zero; 2^-inf = 0)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// w (16, or 8 for the last chunk of 24 columns) columns of this thread's TMEM
// row; w is a constant once the caller's loop is unrolled
__device__ __forceinline__ void tmem_ld_chunk(uint32_t taddr, float* v, int w) {
  if (w >= 16)
    tc::tmem_ld16(taddr, v);
  else
    tc::tmem_ld8(taddr, v);
}
__device__ __forceinline__ void tmem_st_chunk(uint32_t taddr, const float* v, int w) {
  if (w >= 16)
    tc::tmem_st16(taddr, v);
  else
    tc::tmem_st8(taddr, v);
}

template <int NQ>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, float* v) {
#pragma unroll
  for (int c = 0; c < NQ; c += 16) tmem_ld_chunk(taddr + c, v + c, NQ - c < 16 ? NQ - c : 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Columns a query chunk occupies in TMEM and in P's swizzled layout: 48
// queries run the MMAs with N = 48 but keep the 64-column layout (P rows of
// 128 bytes, one 128-byte swizzle atom; TMEM buffers 64 columns apart).
template <int NQ>
struct NQP {
  static constexpr int v = NQ == 48 ? 64 : NQ;
};

// Shared-memory layout of one CTA (offsets from a 1024-aligned base).
template <int NQ, int DH>
struct Smem {
  static constexpr int kBoxes = DH / 64;
  static constexpr uint32_t kTileBytes = kBoxes * 16384;         // K or V tile
  static constexpr uint32_t kQBytes = kBoxes * NQ * 128;         // one Q chunk
  static constexpr uint32_t kPRow = NQP<NQ>::v * 2;              // bytes per key row of P
  static constexpr uint32_t kPBytes = kKT * kPRow;
  static constexpr uint32_t kPBufBytes = (kPBytes + 1023) / 1024 * 1024;  // one of two P buffers
};

// Softmax threads: NQ/kCols groups of 4 warps; a thread owns one key (one dh
// row) and kCols query columns: 16, or 24 at NQ = 48 and 32 at NQ = 64, so that
// those run 8 softmax warps, whose registers hold a tile's scores without
// spilling.  One more warp, the finisher, takes the item counts of the partial
// segments.
template <int NQ>
struct Threads {
  static constexpr int kCols = NQ == 64 ? 32 : (NQ == 48 ? 24 : 16);
  static constexpr int kSmx = 128 * NQ / kCols;
  static constexpr int kFinisher = 2 + kSmx / 32;  // warp index
  static constexpr int kAll = 64 + kSmx + 32;
};

// Shared-memory offsets inside the misc block.
constexpr int kMiscSeg = 4096;    // seg_m[2][64], seg_l[2][64]: (m, l) of a finished segment
constexpr int kMiscTables = 5120; // verify tables, or the merge weights [8][NQ]

template <int NQ, int DH, bool VERIFY>
__global__ void __launch_bounds__(Threads<NQ>::kAll, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_ks,
               const __grid_constant__ CUtensorMap tm_vs, AttnTcParams p) {
  using L = Smem<NQ, DH>;
  constexpr int kSmx = Threads<NQ>::kSmx;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int NK = p.nk, NV = p.nv;
  uint8_t* k_ring = smem;
  uint8_t* v_ring = smem + NK * L::kTileBytes;
  uint8_t* q_buf = v_ring + NV * L::kTileBytes;
  uint8_t* p_buf = q_buf + L::kQBytes;  // 1024-aligned (kQBytes is a multiple of 1024)
  uint8_t* misc = p_buf + 2 * L::kPBufBytes;
  uint64_t* k_full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* k_empty = k_full + 8;
  uint64_t* v_full = k_empty + 8;
  uint64_t* v_empty = v_full + 8;
  uint64_t* q_full = v_empty + 8;    // [2], [0] used: the one Q buffer
  uint64_t* q_empty = q_full + 2;    // [2], [0] used
  uint64_t* s_full = q_empty + 2;    // [2]
  uint64_t* s_empty = s_full + 2;    // [2]
  uint64_t* p_full = s_empty + 2;    // [2]
  uint64_t* pv_done = p_full + 2;    // [2]
  uint64_t* fin_full = pv_done + 2;  // [2] a partial segment's stores are issued (slot 0, 1)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin_full + 2);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* n_draft_s = abort_flag + 1;
  int* n_side_s = n_draft_s + 1;
  int* d_lo_s = n_side_s + 1;  // smallest and largest draft position of the segment
  int* d_hi_s = d_lo_s + 1;
  int* merge_item = d_hi_s + 1;    // [2] item of partial slot s this CTA merges, or -1
  int* seg_info = merge_item + 2;  // [2][3] item, first and last tile of a finished segment
  float* m_run = reinterpret_cast<float*>(misc + 512);      // [NQ]
  float* alpha = m_run + 128;                               // [NQ]
  float* wred = alpha + 128;                                // [4][NQ]
  int* col_meta = reinterpret_cast<int*>(wred + 4 * 128);   // [NQ] view | rank << 2
  float* seg_m = reinterpret_cast<float*>(misc + kMiscSeg); // [2][64] (O buffer = segment & 1)
  float* seg_l = seg_m + 2 * 64;                            // [2][64]
  int* draft_pos = reinterpret_cast<int*>(misc + kMiscTables);  // [kMaxRows]
  int* draft_rank = draft_pos + kMaxRows;                   // [kMaxRows]
  int* side_rank = draft_rank + kMaxRows;                   // [kMaxRows]
  // draft rank of each cache slot in [d_lo, d_lo + kDraftTab), -1 for no draft
  int16_t* kdr_tab = reinterpret_cast<int16_t*>(side_rank + kMaxRows);  // [kDraftTab]

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int tpi = p.tpi;
  const bool clustered = p.cs > 1;
  int crank = 0;
  long long u0, u1;
  if (clustered) {
    // cluster (cs, 1, 1): item blockIdx.x / cs, this CTA's share of its tiles
    crank = (int)tc::cluster_ctarank();
    const long long base = (long long)(cta / p.cs) * tpi;
    u0 = base + (crank * tpi) / p.cs;
    u1 = base + ((crank + 1) * tpi) / p.cs;
  } else {
    u0 = unit_lo(p.total_units, G, cta);
    u1 = unit_lo(p.total_units, G, cta + 1);
  }
  const int T = (int)(u1 - u0);

  // two S buffers and two O buffers of NQP columns each
  uint32_t ncols = 32;
  while ((int)ncols < 4 * NQP<NQ>::v) ncols <<= 1;

  if (tid == 0) {
    for (int s = 0; s < NK; ++s) {
      tc::mbar_init(&k_full[s], 1);
      tc::mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < NV; ++s) {
      tc::mbar_init(&v_full[s], 1);
      tc::mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&q_full[b], 1);
      tc::mbar_init(&q_empty[b], 1);
      tc::mbar_init(&s_full[b], 1);
      tc::mbar_init(&s_empty[b], kSmx / 32);  // one arrival per softmax warp
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&p_full[b], kSmx / 32);
      tc::mbar_init(&pv_done[b], 1);
      tc::mbar_init(&fin_full[b], kSmx / 32);
    }
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, ncols);
  if (tid == 32 * 2) {
    // Launched as a programmatic dependent of the projection: warm L2 with the
    // first cache tiles of this CTA while that grid finishes (safe before the
    // wait: L2 is where the projection's k, v writes land), then wait for it.
    tc::prefetch_tmap(&tm_q);
    tc::prefetch_tmap(&tm_k);
    tc::prefetch_tmap(&tm_v);
    UnitCursor cur;
    cur.init(u0, tpi, p.n_qc);
    const int npre = T < kL2PrefetchTiles ? T : kL2PrefetchTiles;
    for (int i = 0; i < npre; ++i, cur.next(tpi, p.n_qc)) {
      if (cur.t < p.n_cache_tiles) {
        const int key0 = cur.t * kKT;
        const int rows = p.N - key0 < kKT ? p.N - key0 : kKT;
        const size_t off = ((size_t)cur.bh * p.N + key0) * DH;
        tc::prefetch_l2(p.k_cache + off, (uint32_t)rows * DH * 2u);
        tc::prefetch_l2(p.v_cache + off, (uint32_t)rows * DH * 2u);
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_o = tmem + 2 * NQP<NQ>::v;  // O buffer b at tmem_o + b * NQP
  // every thread: nothing written by an earlier kernel is read before this
  tc::griddep_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // K and V have their own rings; each is filled as soon as its stage frees
    // (a K stage right after its QK, a V stage after its PV), polling both so
    // that neither stream waits behind the other.  The one Q buffer takes the
    // next segment's chunk as soon as the last QK of the current one is done.
    if (lane == 0) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      const uint64_t pol_kv = tc::policy_evict_first();
      const uint64_t pol_q = tc::policy_evict_last();
      const int item_a = unit_div(u0, tpi);
      const int n_seg = unit_div(u1 - 1, tpi) - item_a + 1;  // segments of this range
      int ik = 0, iv = 0, qn = 0;
      UnitCursor ck, cv;
      ck.init(u0, tpi, p.n_qc);
      cv = ck;
      IdleClock clk;
      while (iv < T || qn < n_seg) {
        bool progressed = false;
        if (qn < n_seg && tc::mbar_test(&q_empty[0], ((uint32_t)qn & 1u) ^ 1u)) {
          const int item = item_a + qn;
          const int bh = item / p.n_qc, qc = item - bh * p.n_qc;
          tc::mbar_arrive_expect_tx(&q_full[0], L::kQBytes);
#pragma unroll
          for (int x = 0; x < L::kBoxes; ++x)
            tc::tma_load_4d(q_buf + x * NQ * 128, &tm_q, &q_full[0], x * 64, bh % p.H, qc * NQ,
                            bh / p.H, pol_q);
          ++qn;
          progressed = true;
        }
        if (ik < T) {
          const int ks = ik % NK;
          if (tc::mbar_test(&k_empty[ks], ((uint32_t)(ik / NK) & 1u) ^ 1u)) {
            const int t = ck.t, bh = ck.bh;
            const bool side = VERIFY && t >= p.n_cache_tiles;
            const int key0 = (side ? t - p.n_cache_tiles : t) * kKT;
            uint8_t* kd = k_ring + ks * L::kTileBytes;
            tc::mbar_arrive_expect_tx(&k_full[ks], L::kTileBytes);
#pragma unroll
            for (int x = 0; x < L::kBoxes; ++x)
              tc::tma_load_3d(kd + x * 16384, side ? &tm_ks : &tm_k, &k_full[ks], x * 64, key0, bh, pol_kv);
            ++ik;
            ck.next(tpi, p.n_qc);
            progressed = true;
          }
        }
        if (iv < ik) {
          const int vs = iv % NV;
          if (tc::mbar_test(&v_empty[vs], ((uint32_t)(iv / NV) & 1u) ^ 1u)) {
            const int t = cv.t, bh = cv.bh;
            const bool side = VERIFY && t >= p.n_cache_tiles;
            const int key0 = (side ? t - p.n_cache_tiles : t) * kKT;
            uint8_t* vd = v_ring + vs * L::kTileBytes;
            tc::mbar_arrive_expect_tx(&v_full[vs], L::kTileBytes);
#pragma unroll
            for (int x = 0; x < L::kBoxes; ++x)
              tc::tma_load_3d(vd + x * 16384, side ? &tm_vs : &tm_v, &v_full[vs], x * 64, key0, bh, pol_kv);
            ++iv;
            cv.next(tpi, p.n_qc);
            progressed = true;
          }
        }
        if (!progressed && !clk.idle(abort_flag, p.status)) break;
        if (progressed) clk.reset();
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Two in-order streams, QK(i) and PV(j), each issued as soon as its inputs
    // are ready, so neither waits behind the other.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = tc::idesc_bf16(kKT, NQ, false, false);
      constexpr uint32_t idesc_pv = tc::idesc_bf16(kKT, NQ, true, true);
      constexpr uint32_t p_swz = L::kPRow == 128 ? 2u : (L::kPRow == 64 ? 4u : 6u);
      const uint32_t p_addr = tc::smem_u32(p_buf);
      int iq = 0, ip = 0, seg = -1, pseg = -1;
      UnitCursor cq, cpv;
      cq.init(u0, tpi, p.n_qc);
      cpv = cq;
      IdleClock clk;
      while (ip < T) {
        bool progressed = false;
        if (iq < T) {
          const int t = cq.t;
          const bool first = (iq == 0 || t == 0);
          const bool last = (iq == T - 1 || t == tpi - 1);
          const int qseg = first ? seg + 1 : seg;
          const int ks = iq % NK, sb = iq & 1;
          if (tc::mbar_test(&k_full[ks], (uint32_t)(iq / NK) & 1u) &&
              tc::mbar_test(&s_empty[sb], ((uint32_t)(iq >> 1) & 1u) ^ 1u) &&
              (!first || tc::mbar_test(&q_full[0], (uint32_t)qseg & 1u))) {
            seg = qseg;
            tc::tc_fence_after();
            const uint32_t k_addr = tc::smem_u32(k_ring + ks * L::kTileBytes);
            const uint32_t q_addr = tc::smem_u32(q_buf);
#pragma unroll
            for (int kk = 0; kk < DH / 16; ++kk) {
              const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
              const uint32_t qo = (kk >> 2) * NQ * 128 + (kk & 3) * 32;
              tc::mma_bf16(tmem + sb * NQP<NQ>::v, tc::smem_desc(k_addr + ko, 16, 1024, 2),
                           tc::smem_desc(q_addr + qo, 16, 1024, 2), idesc_qk, kk != 0);
            }
            tc::mma_commit(&s_full[sb]);
            tc::mma_commit(&k_empty[ks]);
            if (last) tc::mma_commit(&q_empty[0]);
            ++iq;
            cq.next(tpi, p.n_qc);
            progressed = true;
          }
        }
        if (ip < iq) {
          const int vs = ip % NV;
          if (tc::mbar_test(&p_full[ip & 1], (uint32_t)(ip >> 1) & 1u) &&
              tc::mbar_test(&v_full[vs], (uint32_t)(ip / NV) & 1u)) {
            const bool first = (ip == 0 || cpv.t == 0);
            if (first) ++pseg;
            tc::tc_fence_after();
            const uint32_t v_addr = tc::smem_u32(v_ring + vs * L::kTileBytes);
            const uint32_t pb_addr = p_addr + (ip & 1) * L::kPBufBytes;
            const uint32_t o_addr = tmem_o + (uint32_t)((pseg & 1) * NQP<NQ>::v);
#pragma unroll
            for (int kk = 0; kk < kKT / 16; ++kk) {
              const uint64_t da = tc::smem_desc(v_addr + kk * 2048, DH == 128 ? 16384 : 0, 1024, 2);
              const uint64_t db = tc::smem_desc(pb_addr + kk * 16 * L::kPRow, 0, 8 * L::kPRow, p_swz);
              tc::mma_bf16(o_addr, da, db, idesc_pv, (first && kk == 0) ? 0u : 1u);
            }
            tc::mma_commit(&pv_done[ip & 1]);
            tc::mma_commit(&v_empty[vs]);
            ++ip;
            cpv.next(tpi, p.n_qc);
            progressed = true;
          }
        }
        if (!progressed && !clk.idle(abort_flag, p.status)) break;
        if (progressed) clk.reset();
      }
    }
  } else if (warp < Threads<NQ>::kFinisher) {
    // ------------------------------------------------------------ softmax / epilogue
    // NQ/NQH groups of 4 warps: the warps that share a TMEM lane quarter split
    // the query columns, so a thread owns one key (later one dh row) and the
    // NQH columns [c0, c0 + NQH).
    constexpr int NQH = Threads<NQ>::kCols;
    const int st = tid - 64;                 // 0..kSmx-1
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;        // column group
    const int c0 = half * NQH;
    const int kl = quarter * 32 + lane;      // TMEM lane: key of S^T, dh row of O^T
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const size_t part_floats = (size_t)NQ * DH + 2 * NQ;
    const float scale = p.qk_scale;
    float l[NQH], mrun[NQH];
#pragma unroll
    for (int c = 0; c < NQH; ++c) {
      l[c] = 0.f;
      mrun[c] = -INFINITY;
    }
    int seg = -1;
    int n_draft = 0, n_side = 0, d_lo = INT_MAX, d_hi = INT_MIN;
    bool tab = false;      // the segment's draft positions are in kdr_tab
    uint32_t v2cols = 0;   // bit c: this thread's column c0 + c is a mask-view row
    int meta_key = -1;     // (sequence, query chunk) whose verify tables are loaded
    int pv_waited = -1;    // index of the last PV this thread waited for
    int seg_t0 = 0;        // tile index at which the current segment started
    int n_done = 0;        // segments whose last tile is through
    int n_fin = 0;         // segments whose output or partial is written
    int end0 = 0, end1 = 0;  // last tile (range index) of the segment in O buffer 0 / 1
    UnitCursor cs;
    cs.init(u0, tpi, p.n_qc);
    const int item0 = cs.item;

    // Writes segment s's result from its O buffer, once its last PV is done:
    // the output of a whole item, or this CTA's partial (O, m, l) of a split
    // one, whose arrival on fin_full hands the item count to the finisher.
    auto finish = [&](int s) {
      const int sl = s & 1;
      const int item = seg_info[sl * 3], t0 = seg_info[sl * 3 + 1], tl = seg_info[sl * 3 + 2];
      const int bh = item / p.n_qc, qc = item - bh * p.n_qc;
      const int b = bh / p.H, h = bh - b * p.H;
      const uint32_t t_o = tmem_o + (uint32_t)(sl * NQP<NQ>::v) + lane_off + (uint32_t)c0;
      const float* sm = seg_m + sl * 64;
      const float* sls = seg_l + sl * 64;
      if (t0 == 0 && tl == tpi - 1) {
#pragma unroll
        for (int cc = 0; cc < NQH; cc += 16) {
          const int w = NQH - cc < 16 ? NQH - cc : 16;
          float o[16];
          tmem_ld_chunk(t_o + cc, o, w);
          tc::tmem_wait_ld();
          if (kl < DH) {
#pragma unroll
            for (int c = 0; c < w; ++c) {
              const int cq = c0 + cc + c, r = qc * NQ + cq;
              if (r < p.rows) {
                const float lt = sls[cq];
                p.out[(((size_t)b * p.rows + r) * p.H + h) * DH + kl] = __float2bfloat16_rn(o[c] / lt);
                if (kl == 0 && p.lse) p.lse[((size_t)b * p.rows + r) * p.H + h] = sm[cq] + log2f(lt);
              }
            }
          }
        }
      } else {
        // slot 0 for the item the range starts in, 1 for the one it ends in
        // (a split item is only ever one of those two)
        const int slot = (item == item0) ? 0 : 1;
        float* part = p.partials + ((size_t)cta * 2 + slot) * part_floats;
#pragma unroll
        for (int cc = 0; cc < NQH; cc += 16) {
          const int w = NQH - cc < 16 ? NQH - cc : 16;
          float o[16];
          tmem_ld_chunk(t_o + cc, o, w);
          tc::tmem_wait_ld();
          if (kl < DH) {
            // O as [dh row][NQ columns]: a thread's columns are contiguous
            float4* dst = reinterpret_cast<float4*>(part + (size_t)kl * NQ + c0 + cc);
#pragma unroll
            for (int v = 0; v < w / 4; ++v)
              dst[v] = make_float4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
          }
        }
        if (st < NQ) {
          part[(size_t)NQ * DH + st] = sm[st];
          part[(size_t)NQ * DH + NQ + st] = sls[st];
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&fin_full[slot]);
      }
    };

    for (int i = 0; i < T; ++i, cs.next(tpi, p.n_qc)) {
      const int item = cs.item, t = cs.t, qc = cs.qc, bh = cs.bh;
      const bool first = (i == 0 || t == 0);
      const bool last = (i == T - 1 || t == tpi - 1);
      const int b = bh / p.H;
      if (first) {
        ++seg;
        seg_t0 = t;
        // segment metadata: verify tables of sequence b, query chunk qc (kept
        // while consecutive segments share them)
        if (VERIFY && b * p.n_qc + qc != meta_key) {
          meta_key = b * p.n_qc + qc;
          const int r0 = b * p.rows;
          if (st < NQ) {
            const int r = qc * NQ + st;
            col_meta[st] = (r < p.rows) ? ((int)p.view[r0 + r] | (p.rank[r0 + r] << 2)) : 0;
          }
          if (warp == 2 || warp == 3) {
            // ballot compaction of draft rows (warp 2) and mask rows (warp 3)
            const int want = warp == 2 ? 1 : 2;
            int base = 0, lo = INT_MAX, hi = INT_MIN;
            for (int r = lane; r - lane < p.rows; r += 32) {
              const int vw = r < p.rows ? (int)p.view[r0 + r] : -1;
              const unsigned bal = __ballot_sync(0xffffffffu, vw == want);
              const int at = base + __popc(bal & ((1u << lane) - 1u));
              if (vw == want && at < kMaxRows) {
                if (want == 1) {
                  const int ps = p.pos[r0 + r];
                  draft_pos[at] = ps;
                  draft_rank[at] = p.rank[r0 + r];
                  lo = min(lo, ps);
                  hi = max(hi, ps);
                } else {
                  side_rank[at] = p.rank[r0 + r];
                }
              }
              base += __popc(bal);
            }
            lo = __reduce_min_sync(0xffffffffu, lo);
            hi = __reduce_max_sync(0xffffffffu, hi);
            if (lane == 0) {
              if (want == 1) {
                *n_draft_s = min(base, kMaxRows);
                *d_lo_s = lo;
                *d_hi_s = hi;
              } else {
                *n_side_s = min(min(base, p.S_max), kMaxRows);
              }
            }
          }
          tc::named_bar_sync(1, kSmx);
          n_draft = *n_draft_s;
          n_side = *n_side_s;
          d_lo = *d_lo_s;
          d_hi = *d_hi_s;
          // slot -> draft rank, one shared-memory load per key instead of a scan
          // of the drafts, when their positions span at most kDraftTab slots
          tab = n_draft > 0 && d_hi - d_lo < kDraftTab;
          if (tab) {
            for (int j = st; j <= d_hi - d_lo; j += kSmx) kdr_tab[j] = -1;
            tc::named_bar_sync(1, kSmx);
            for (int d = st; d < n_draft; d += kSmx) kdr_tab[draft_pos[d] - d_lo] = (int16_t)draft_rank[d];
            tc::named_bar_sync(1, kSmx);
          }
          v2cols = 0;
#pragma unroll
          for (int c = 0; c < NQH; ++c)
            if ((col_meta[c0 + c] & 3) == 2) v2cols |= 1u << c;
        }
      }
      const uint32_t t_oc = tmem_o + (uint32_t)((seg & 1) * NQP<NQ>::v);  // this segment's O

      // ---- raw scores of this tile: row kl of S^T, this thread's columns
      const int sb = i & 1;
      // after a timeout every later wait returns at once: keep going so that all
      // softmax threads still meet at the same named barriers
      tc::mbar_wait(&s_full[sb], (uint32_t)(i >> 1) & 1u, abort_flag, p.status);
      tc::tc_fence_after();
      float s[NQH];
      tmem_ld_row<NQH>(tmem + lane_off + sb * NQP<NQ>::v + c0, s);
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s_empty[sb]);

      const bool side_tile = VERIFY && t >= p.n_cache_tiles;
      const int key = (side_tile ? t - p.n_cache_tiles : t) * kKT + kl;
      const bool valid = key < (side_tile ? n_side : p.N);
      if (!valid) {
#pragma unroll
        for (int c = 0; c < NQH; ++c) s[c] = -INFINITY;
      } else if (VERIFY) {
        // The view rule (visible_side / visible_cache).  In the mutual reading
        // it depends only on whether the column is a mask-view row, a bit of
        // v2cols; the causal reading also compares ranks.
        if (side_tile) {
          if (!p.causal) {
#pragma unroll
            for (int c = 0; c < NQH; ++c)
              if (!((v2cols >> c) & 1u)) s[c] = -INFINITY;
          } else {
            const int srank = side_rank[key];
#pragma unroll
            for (int c = 0; c < NQH; ++c) {
              const int cm = col_meta[c0 + c];
              if (!visible_side(cm & 3, cm >> 2, srank, 1)) s[c] = -INFINITY;
            }
          }
        } else {
          // only keys within the draft positions' range need the lookup
          int kdr = -1;
          if (key >= d_lo && key <= d_hi) {
            if (tab) {
              kdr = kdr_tab[key - d_lo];
            } else {
              for (int d = 0; d < n_draft; ++d)
                if (draft_pos[d] == key) kdr = draft_rank[d];
            }
          }
          if (kdr >= 0) {
            if (!p.causal) {
#pragma unroll
              for (int c = 0; c < NQH; ++c)
                if ((v2cols >> c) & 1u) s[c] = -INFINITY;
            } else {
#pragma unroll
              for (int c = 0; c < NQH; ++c) {
                const int cm = col_meta[c0 + c];
                if (!visible_cache(cm & 3, cm >> 2, kdr, 1)) s[c] = -INFINITY;
              }
            }
          }
        }
      }

      // ---- running max: raised only when a score exceeds it by more than 2^8
      // (with m = -inf any finite score does; masked scores, -inf, never do).
      // A segment's first tile always sets it, so that no column keeps the
      // previous segment's max.
      bool need = first;
#pragma unroll
      for (int c = 0; c < NQH; ++c) need |= fmaf(s[c], scale, -mrun[c]) > kThresh;
      const bool any = bar_any(2, kSmx, need);
      if (any) {
#pragma unroll
        for (int c = 0; c < NQH; ++c) {
          const float wm = warp_max(s[c]);
          if (lane == (c & 31)) wred[quarter * NQ + c0 + c] = wm * scale;
        }
        tc::named_bar_sync(1, kSmx);
        if (st < NQ) {
          const float mo = m_run[st];
          const float tm = fmaxf(fmaxf(wred[st], wred[NQ + st]), fmaxf(wred[2 * NQ + st], wred[3 * NQ + st]));
          const bool first_col = first || !(mo > -INFINITY);
          const float mcur = first_col ? -INFINITY : mo;
          const float mn = (tm > mcur + kThresh) ? tm : mcur;
          alpha[st] = (mcur == -INFINITY) ? 0.f : exp2f(mcur - mn);
          m_run[st] = mn;
        }
        tc::named_bar_sync(1, kSmx);
#pragma unroll
        for (int c = 0; c < NQH; ++c) {
          mrun[c] = m_run[c0 + c];
          l[c] *= alpha[c0 + c];
        }
      }

      // ---- P buffer i&1 is free once PV(i-2) is done; rescaling O needs PV(i-1)
      if (i >= 2 && pv_waited < i - 2) {
        tc::mbar_wait(&pv_done[i & 1], (uint32_t)((i - 2) >> 1) & 1u, abort_flag, p.status);
        pv_waited = i - 2;
      }
      if (any && !first && i >= 1 && pv_waited < i - 1) {
        tc::mbar_wait(&pv_done[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u, abort_flag, p.status);
        pv_waited = i - 1;
      }
      tc::tc_fence_after();
      if (any && !first) {
        // rescale this thread's columns of the O^T accumulator (row kl)
        float o[16];
#pragma unroll
        for (int cc = 0; cc < NQH; cc += 16) {
          const int w = NQH - cc < 16 ? NQH - cc : 16;
          tmem_ld_chunk(t_oc + lane_off + c0 + cc, o, w);
          tc::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < w; ++c) o[c] *= alpha[c0 + cc + c];
          tmem_st_chunk(t_oc + lane_off + c0 + cc, o, w);
        }
        tc::tmem_wait_st();
      }
      // a side tile's key rows past the used slots may hold anything: zero them
      if (side_tile && !valid && half == 0) {
        tc::mbar_wait(&v_full[i % NV], (uint32_t)(i / NV) & 1u, abort_flag, p.status);
        uint8_t* vrow = v_ring + (i % NV) * L::kTileBytes + kl * 128;
#pragma unroll
        for (int x = 0; x < L::kBoxes; ++x)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<uint4*>(vrow + x * 16384 + q * 16) = make_uint4(0u, 0u, 0u, 0u);
      }

      // ---- P = 2^(s*scale - m) into row kl of the MN-major swizzled P^T tile
      {
        uint32_t pk[NQH / 2];
#pragma unroll
        for (int c = 0; c < NQH; c += 2) {
          // fmaxf turns the NaN of (-inf) - (-inf) into -inf, i.e. p = 0
          const float p0 = ex2_approx(fmaxf(fmaf(s[c], scale, -mrun[c]), -INFINITY));
          const float p1 = ex2_approx(fmaxf(fmaf(s[c + 1], scale, -mrun[c + 1]), -INFINITY));
          l[c] += p0;
          l[c + 1] += p1;
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
        constexpr uint32_t mask = L::kPRow / 16 - 1;  // swizzle span: row bytes
#pragma unroll
        for (int ch = 0; ch < NQH / 8; ++ch) {
          const uint32_t off = (uint32_t)(kl * L::kPRow + (c0 * 2) + ch * 16);
          const uint32_t sw = off ^ (((off >> 7) & mask) << 4);
          *reinterpret_cast<uint4*>(p_buf + (i & 1) * L::kPBufBytes + sw) =
              make_uint4(pk[ch * 4], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
        }
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&p_full[i & 1]);

      if (last) {
        // ---- segment done: l summed per column; (m, l) and the segment's
        // place are kept for its finish, two tiles on
#pragma unroll
        for (int c = 0; c < NQH; ++c) {
          float v = l[c];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == (c & 31)) wred[quarter * NQ + c0 + c] = v;
          // the next segment starts afresh: end the live ranges here
          l[c] = 0.f;
          mrun[c] = -INFINITY;
        }
        tc::named_bar_sync(1, kSmx);
        const int sl = seg & 1;
        if (st < NQ) {
          seg_m[sl * 64 + st] = m_run[st];
          seg_l[sl * 64 + st] = wred[st] + wred[NQ + st] + wred[2 * NQ + st] + wred[3 * NQ + st];
        }
        if (st == 0) {
          seg_info[sl * 3] = item;
          seg_info[sl * 3 + 1] = seg_t0;
          seg_info[sl * 3 + 2] = t;
        }
        if (sl) end1 = i; else end0 = i;
        ++n_done;
      }

      // ---- a finished segment writes its result once its last PV is two
      // tiles back, and at the latest at the end of the segment after it: the
      // segment two on reuses its O buffer from its first P.  (Kept at the end
      // of the tile: this code, placed ahead of the scores' wait, slowed each
      // range's first tile by some microseconds.)
      while (n_fin < n_done) {
        const int e = (n_fin & 1) ? end1 : end0;
        if (!(e <= i - 2 || (last && seg == n_fin + 1))) break;
        if (pv_waited < e) {
          tc::mbar_wait(&pv_done[e & 1], (uint32_t)(e >> 1) & 1u, abort_flag, p.status);
          pv_waited = e;
        }
        tc::tc_fence_after();
        finish(n_fin);
        ++n_fin;
      }
    }

    // ---- the segments not yet finished: the last one or two
    tc::named_bar_sync(1, kSmx);  // their (m, l) and places are in shared memory
    if (n_fin < n_done) {
      if (pv_waited < T - 1) {
        tc::mbar_wait(&pv_done[(T - 1) & 1], (uint32_t)((T - 1) >> 1) & 1u, abort_flag, p.status);
        pv_waited = T - 1;
      }
      tc::tc_fence_after();
    }
    if (clustered) {
      tc::named_bar_sync(3, kSmx + 32);  // releases the finisher to the cluster barriers
      // ---- cluster merge of the one segment.  The rings are idle (the last
      // PV is done), so this CTA's partial goes to the start of the K ring: O^T
      // as [dh row][NQ + 4] (the pad keeps 16-byte reads of rows at a 144- or
      // 272-byte stride off each other's banks), then m[NQ], l[NQ].
      constexpr int kP = NQ + 4;
      float* cpart = reinterpret_cast<float*>(k_ring);
#pragma unroll
      for (int cc = 0; cc < NQH; cc += 16) {
        const int w = NQH - cc < 16 ? NQH - cc : 16;
        float o[16];
        tmem_ld_chunk(tmem_o + lane_off + c0 + cc, o, w);
        tc::tmem_wait_ld();
        if (kl < DH) {
          float4* dst = reinterpret_cast<float4*>(cpart + kl * kP + c0 + cc);
#pragma unroll
          for (int v = 0; v < w / 4; ++v)
            dst[v] = make_float4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
        }
      }
      if (st < NQ) {
        cpart[DH * kP + st] = seg_m[st];
        cpart[DH * kP + NQ + st] = seg_l[st];
      }
      tc::cluster_sync();
      const int bh = item0 / p.n_qc, qc = item0 - bh * p.n_qc;
      const int b = bh / p.H, h = bh - b * p.H;
      const int cs = p.cs;
      const uint32_t cbase = tc::smem_u32(cpart);
      // This CTA merges its slice of dh rows.  A thread takes one row and 4
      // columns (consecutive threads: consecutive rows, so the output stores
      // coalesce) and loads (m, l, O) of those columns from up to 4 CTAs at
      // once, merging online: one round trip per 4 CTAs.
      const int r0 = (crank * DH) / cs, nr = ((crank + 1) * DH) / cs - r0;
      for (int idx = st; idx < nr * (NQ / 4); idx += kSmx) {
        const int row = r0 + idx % nr, c4 = (idx / nr) * 4;
        float M[4], Lsum[4], acc[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          M[e] = -INFINITY;
          Lsum[e] = 0.f;
          acc[e] = 0.f;
        }
        for (int g = 0; g < cs; g += 4) {
          float4 mv[4], lv[4], ov[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (g + j < cs) {
              const uint32_t a = tc::map_peer(cbase, (uint32_t)(g + j));
              mv[j] = tc::ld_peer_f32x4(a + (uint32_t)(DH * kP + c4) * 4u);
              lv[j] = tc::ld_peer_f32x4(a + (uint32_t)(DH * kP + NQ + c4) * 4u);
              ov[j] = tc::ld_peer_f32x4(a + (uint32_t)(row * kP + c4) * 4u);
            } else {
              mv[j] = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
              lv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
              ov[j] = lv[j];
            }
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float mj[4], lj[4], oj[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              mj[j] = e == 0 ? mv[j].x : e == 1 ? mv[j].y : e == 2 ? mv[j].z : mv[j].w;
              lj[j] = e == 0 ? lv[j].x : e == 1 ? lv[j].y : e == 2 ? lv[j].z : lv[j].w;
              oj[j] = e == 0 ? ov[j].x : e == 1 ? ov[j].y : e == 2 ? ov[j].z : ov[j].w;
            }
            const float mn = fmaxf(fmaxf(M[e], fmaxf(mj[0], mj[1])), fmaxf(mj[2], mj[3]));
            if (mn > -INFINITY) {
              const float sc = (M[e] == -INFINITY) ? 0.f : exp2f(M[e] - mn);
              Lsum[e] *= sc;
              acc[e] *= sc;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float w = (mj[j] == -INFINITY) ? 0.f : exp2f(mj[j] - mn);
                Lsum[e] = fmaf(w, lj[j], Lsum[e]);
                acc[e] = fmaf(w, oj[j], acc[e]);
              }
              M[e] = mn;
            }
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = qc * NQ + c4 + e;
          if (r < p.rows) {
            p.out[(((size_t)b * p.rows + r) * p.H + h) * DH + row] =
                __float2bfloat16_rn(Lsum[e] > 0.f ? acc[e] / Lsum[e] : 0.f);
            if (row == 0 && p.lse) p.lse[((size_t)b * p.rows + r) * p.H + h] = M[e] + log2f(Lsum[e]);
          }
        }
      }
      // no CTA leaves while another may still read its shared memory
      tc::cluster_sync();
    } else {
      while (n_fin < n_done) {
        finish(n_fin);
        ++n_fin;
      }
      // the finisher has taken the counts of this CTA's partial segments
      tc::named_bar_sync(3, kSmx + 32);
      for (int slot = 0; slot < 2; ++slot) {
        const int item = merge_item[slot];
        if (item < 0) continue;
        // ---- merge item `item`, whose contributors have all stored their
        // partials, in CTA order.  The loads of a batch are all issued before
        // any is used, so the merge costs a few L2 round trips, not a few per
        // contributor.
        //   (1) per column: M = max m_j, L = sum 2^(m_j - M) l_j (8 at a time)
        //   (2) O = sum (2^(m_j - M) / L) O_j, weights staged in shared memory
        __threadfence();
        const int bh = item / p.n_qc, qc = item - bh * p.n_qc;
        const int b = bh / p.H, h = bh - b * p.H;
        const long long iu0 = (long long)item * tpi;
        const int c_first = owner_of(iu0, p.total_units, G);
        const int c_last = owner_of(iu0 + tpi - 1, p.total_units, G);
        const int n_c = c_last - c_first + 1;
        // slot 0 when the item is the contributor's first, i.e. its range
        // starts inside the item: unit_lo(cb) >= iu0 <=> total * cb >= iu0 * G
        const long long lim0 = iu0 * (long long)G;
        auto part_of = [&](int cb) -> const float* {
          const int sl = (p.total_units * cb >= lim0) ? 0 : 1;
          return p.partials + ((size_t)cb * 2 + sl) * part_floats;
        };
        float* wts = reinterpret_cast<float*>(draft_pos);  // [8][NQ], free after the range
        float M = -INFINITY, Lsum = 0.f;
        float mv[8];
        if (st < NQ) {
          for (int g0 = 0; g0 < n_c; g0 += 8) {
            float lv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              mv[j] = -INFINITY;
              lv[j] = 0.f;
              if (g0 + j < n_c) {
                const float* pc = part_of(c_first + g0 + j);
                mv[j] = __ldcg(pc + (size_t)NQ * DH + st);
                lv[j] = __ldcg(pc + (size_t)NQ * DH + NQ + st);
              }
            }
            float mc = M;
#pragma unroll
            for (int j = 0; j < 8; ++j) mc = fmaxf(mc, mv[j]);
            if (mc > -INFINITY) {
              Lsum *= (M == -INFINITY) ? 0.f : exp2f(M - mc);
#pragma unroll
              for (int j = 0; j < 8; ++j) Lsum += (mv[j] == -INFINITY) ? 0.f : exp2f(mv[j] - mc) * lv[j];
              M = mc;
            }
          }
        }
        if (st < NQ && p.lse && qc * NQ + st < p.rows)
          p.lse[((size_t)b * p.rows + qc * NQ + st) * p.H + h] = M + log2f(Lsum);
        constexpr int kJ = NQH >= 24 ? 2 : 4;  // contributors per batch of O loads
        float acc[NQH];
#pragma unroll
        for (int c = 0; c < NQH; ++c) acc[c] = 0.f;
        for (int g0 = 0; g0 < n_c; g0 += 8) {
          if (st < NQ) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              float m = mv[j];
              if (n_c > 8) m = (g0 + j < n_c) ? __ldcg(part_of(c_first + g0 + j) + (size_t)NQ * DH + st) : -INFINITY;
              wts[j * NQ + st] = (m == -INFINITY || !(Lsum > 0.f)) ? 0.f : exp2f(m - M) / Lsum;
            }
          }
          tc::named_bar_sync(1, kSmx);
          if (kl < DH) {
            const int nj = min(8, n_c - g0);
            for (int j0 = 0; j0 < nj; j0 += kJ) {
              float4 ov[kJ][NQH / 4];
#pragma unroll
              for (int j = 0; j < kJ; ++j) {
                if (j0 + j < nj) {
                  const float4* src = reinterpret_cast<const float4*>(part_of(c_first + g0 + j0 + j) + (size_t)kl * NQ + c0);
#pragma unroll
                  for (int v = 0; v < NQH / 4; ++v) ov[j][v] = __ldcg(src + v);
                } else {
#pragma unroll
                  for (int v = 0; v < NQH / 4; ++v) ov[j][v] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
              }
#pragma unroll
              for (int j = 0; j < kJ; ++j) {
                const float* wj = wts + (j0 + j) * NQ + c0;
#pragma unroll
                for (int v = 0; v < NQH / 4; ++v) {
                  // weights past nj are stale but multiply zeros
                  const float w0 = (j0 + j < nj) ? wj[4 * v] : 0.f;
                  const float w1 = (j0 + j < nj) ? wj[4 * v + 1] : 0.f;
                  const float w2 = (j0 + j < nj) ? wj[4 * v + 2] : 0.f;
                  const float w3 = (j0 + j < nj) ? wj[4 * v + 3] : 0.f;
                  acc[4 * v] = fmaf(w0, ov[j][v].x, acc[4 * v]);
                  acc[4 * v + 1] = fmaf(w1, ov[j][v].y, acc[4 * v + 1]);
                  acc[4 * v + 2] = fmaf(w2, ov[j][v].z, acc[4 * v + 2]);
                  acc[4 * v + 3] = fmaf(w3, ov[j][v].w, acc[4 * v + 3]);
                }
              }
            }
          }
          tc::named_bar_sync(1, kSmx);
        }
        if (kl < DH) {
#pragma unroll
          for (int c = 0; c < NQH; ++c) {
            const int r = qc * NQ + c0 + c;
            if (r < p.rows)
              p.out[(((size_t)b * p.rows + r) * p.H + h) * DH + kl] = __float2bfloat16_rn(acc[c]);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ finisher
    // For each partial segment of this CTA's range, in order: wait until the
    // softmax warps have issued its stores, make them visible device-wide,
    // then count this contributor in.  The last of an item's contributors
    // merges it; the softmax warps do that after the range.
    if (!clustered) {
      if (lane == 0) {
        merge_item[0] = -1;
        merge_item[1] = -1;
        const int item_a = unit_div(u0, tpi), item_z = unit_div(u1 - 1, tpi);
        for (int slot = 0; slot < 2; ++slot) {
          const int item = slot == 0 ? item_a : item_z;
          if (slot == 1 && item_z == item_a) break;
          const long long iu0 = (long long)item * tpi;
          if (u0 <= iu0 && u1 >= iu0 + tpi) continue;  // whole: the softmax warps write it
          // polled with a pause between tests, so that this warp takes no issue
          // slots from the softmax warps of its SM sub-partition meanwhile
          bool ready = false;
          IdleClock clk;
          while (!(ready = tc::mbar_test(&fin_full[slot], 0u))) {
            __nanosleep(256);
            if (!clk.idle(abort_flag, p.status)) break;
          }
          if (!ready) break;
          __threadfence();
          const int c_first = owner_of(iu0, p.total_units, G);
          const int c_last = owner_of(iu0 + tpi - 1, p.total_units, G);
          const unsigned prev = atomicAdd(&p.item_cnt[item], 1u);
          if (prev == (unsigned)(c_last - c_first)) {
            p.item_cnt[item] = 0u;  // reset for the next call
            merge_item[slot] = item;
          }
        }
      }
      __syncwarp();
      tc::named_bar_sync(3, kSmx + 32);
    }
  }

  // the softmax warps meet the two cluster barriers of the merge; the other
  // warps, done with their loops, meet them here (the finisher once the merge
  // begins: it waits on a CTA barrier, not a cluster one, meanwhile)
  if (clustered && (warp < 2 || warp == Threads<NQ>::kFinisher)) {
    if (warp == Threads<NQ>::kFinisher) tc::named_bar_sync(3, kSmx + 32);
    tc::cluster_sync();
    tc::cluster_sync();
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
  int NQ, n_qc, nct, nst, tpi, nk, nv, grid;  // rings; stream-K grid
  int cs;                                      // cluster size wanted (0: none)
  bool whole_items;                            // many items: one CTA per item, no merges
  long long items, total_units;
  size_t smem_bytes, partial_bytes, counter_bytes;
};

constexpr size_t kSmemBudget = 227 * 1024;

AttnPlan plan(int B, int N, int H, int dh, int rows, int S_max, int verify, int num_sms) {
  AttnPlan q{};
  q.NQ = rows <= 16 ? 16 : (rows <= 32 ? 32 : (rows <= 48 ? 48 : 64));
  q.n_qc = (rows + q.NQ - 1) / q.NQ;
  q.nct = (N + kKT - 1) / kKT;
  q.nst = (verify && S_max > 0) ? (S_max + kKT - 1) / kKT : 0;
  q.tpi = q.nct + q.nst;
  q.items = (long long)B * H * q.n_qc;
  q.total_units = q.items * q.tpi;
  q.grid = (int)(q.total_units < num_sms ? q.total_units : num_sms);
  // few items: a cluster of cs CTAs per item, merging through shared memory
  q.cs = 0;
  if (q.items * 2 <= num_sms) {
    int cs = (int)(num_sms / q.items);
    cs = cs > 8 ? 8 : cs;
    cs = cs > q.tpi ? q.tpi : cs;
    if (cs >= 2) q.cs = cs;
  }
  const size_t boxes = dh / 64;
  const size_t tile = boxes * 16384;
  const size_t qbytes = boxes * q.NQ * 128;
  const size_t nqp = q.NQ == 48 ? 64 : q.NQ;  // P's padded columns
  const size_t pbytes = 2 * (((size_t)kKT * nqp * 2 + 1023) / 1024 * 1024);
  // misc: barriers, softmax scratch and the finished segments' (m, l), then the
  // verify tables (or, without them, the [8][NQ] merge weights)
  const size_t misc = kMiscTables + (verify ? 3 * kMaxRows * 4 + kDraftTab * 2 : 8 * 64 * 4);
  // K and V tiles share what shared memory is left.  A V tile is held from its
  // load until its PV is done, longer than a K tile, so V gets the odd one.
  const size_t fixed = 1024 + qbytes + pbytes + misc;
  int tiles = (int)((kSmemBudget - fixed) / tile);
  if (tiles > 16) tiles = 16;
  q.nv = (tiles + 1) / 2;
  q.nk = tiles - q.nv;
  if (q.nv > 8) q.nv = 8;
  q.smem_bytes = fixed + (size_t)(q.nk + q.nv) * tile;
  // Items beyond the clusters' reach, in at most two waves: one CTA per whole
  // item has no item boundary inside a CTA's range and no merge, but every
  // wave pays a cold start.  Taken when that makespan is no longer than
  // stream-K's share plus one start, its end merge and two boundaries.  With
  // more waves the starts add up and persistent stream-K, which pipelines its
  // loads across item boundaries, wins (measured: 2048 items, 649 -> 705 us).
  q.whole_items = false;
  if (q.cs == 0 && q.items * 2 > num_sms) {
    const long long waves = (q.items + num_sms - 1) / num_sms;
    const double whole = (double)waves * (q.tpi + kStartTiles);
    const double sk = (double)q.total_units / num_sms + kStartTiles + kMergeTiles + 2 * kBoundaryTiles;
    q.whole_items = waves <= 2 && whole <= sk;
  }
  q.partial_bytes = align_up((size_t)q.grid * 2 * ((size_t)q.NQ * dh + 2 * q.NQ) * sizeof(float), 256);
  q.counter_bytes = align_up((size_t)q.items * sizeof(unsigned), 256);
  return q;
}

// How many clusters of cs CTAs of this kernel can be resident at once (cached).
template <int NQ, int DH, bool VERIFY>
int max_clusters(int cs, size_t smem_bytes) {
  static int cache[9] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
  if (cache[cs] == 0) {
    cudaLaunchConfig_t c = {};
    c.gridDim = dim3(cs * 16);
    c.blockDim = dim3(Threads<NQ>::kAll);
    c.dynamicSmemBytes = smem_bytes;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    c.attrs = at;
    c.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, attn_tc_kernel<NQ, DH, VERIFY>, &c) != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
    cache[cs] = n > 0 ? n : -1;
  }
  return cache[cs];
}

// The work split a launch of this plan takes (kSplit*), after the kernel's
// shared-memory limit is raised; *cs_out gets the cluster size (0 without).
// Cluster mode only when every item's cluster fits in one wave.
template <int NQ, int DH, bool VERIFY>
cudaError_t resolve_split(const AttnPlan& q, int* mode, int* cs_out) {
  auto kern = attn_tc_kernel<NQ, DH, VERIFY>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)q.smem_bytes);
  if (e != cudaSuccess) return e;
  int cs = q.cs;
  while (cs >= 2 && max_clusters<NQ, DH, VERIFY>(cs, q.smem_bytes) < q.items) --cs;
  if (cs >= 2) {
    *mode = kSplitClusters;
    *cs_out = cs;
  } else {
    *mode = q.whole_items ? kSplitWholeItems : kSplitStreamK;
    *cs_out = 0;
  }
  return cudaSuccess;
}

template <int NQ, int DH, bool VERIFY>
cudaError_t launch_t(const AttnArgs& a, const AttnPlan& q, AttnTcParams prm, const CUtensorMap* maps,
                     cudaStream_t stream) {
  auto kern = attn_tc_kernel<NQ, DH, VERIFY>;
  int mode = 0, cs = 0;
  cudaError_t e = resolve_split<NQ, DH, VERIFY>(q, &mode, &cs);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(Threads<NQ>::kAll);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (mode == kSplitClusters) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cs;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
    cfg.gridDim = dim3((unsigned)(q.items * cs));
    prm.cs = cs;
  } else if (mode == kSplitWholeItems) {
    // grid = items: the unit split gives every CTA exactly one whole item
    cfg.gridDim = dim3((unsigned)q.items);
    prm.cs = 0;
  } else {
    cfg.gridDim = dim3(q.grid);
    prm.cs = 0;
  }
  cfg.dynamicSmemBytes = q.smem_bytes;
  prm.nk = q.nk;
  prm.nv = q.nv;
  e = cudaLaunchKernelEx(&cfg, kern, maps[0], maps[1], maps[2], maps[3], maps[4], prm);
  count_launches(1);
  return e;
}

}  // namespace

size_t attn_tc_workspace_bytes(int B, int N, int H, int dh, int rows, int S_max, int verify,
                               int num_sms) {
  if (B * rows <= 0) return 256;
  const AttnPlan q = plan(B, N, H, dh, rows, S_max, verify, num_sms);
  return q.partial_bytes + q.counter_bytes;
}

int attn_tc_split(int B, int N, int H, int dh, int rows, int S_max, int verify, int* cs) {
  *cs = 0;
  if (B * rows <= 0 || (verify && rows > kMaxRows)) return -1;
  const AttnPlan q = plan(B, N, H, dh, rows, S_max, verify, device_sm_count());
  int mode = -1;
  cudaError_t e = cudaErrorInvalidValue;
#define FDLLM_ATTN_SPLIT(NQv, DHv)                                                           \
  if (q.NQ == NQv && dh == DHv)                                                             \
    e = verify ? resolve_split<NQv, DHv, true>(q, &mode, cs)                                \
               : resolve_split<NQv, DHv, false>(q, &mode, cs);
  FDLLM_ATTN_SPLIT(16, 64)
  FDLLM_ATTN_SPLIT(32, 64)
  FDLLM_ATTN_SPLIT(48, 64)
  FDLLM_ATTN_SPLIT(64, 64)
  FDLLM_ATTN_SPLIT(16, 128)
  FDLLM_ATTN_SPLIT(32, 128)
  FDLLM_ATTN_SPLIT(48, 128)
  FDLLM_ATTN_SPLIT(64, 128)
#undef FDLLM_ATTN_SPLIT
  return e == cudaSuccess ? mode : -1;
}

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t stream) {
  if (a.B * a.rows_per_seq == 0) return cudaSuccess;
  if (a.verify && a.rows_per_seq > kMaxRows) return cudaErrorInvalidValue;
  const AttnPlan q = plan(a.B, a.N, a.H, a.dh, a.rows_per_seq, a.S_max, a.verify, device_sm_count());
  if (q.nk < 2 || q.nv < 2) return cudaErrorInvalidValue;
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
  prm.total_units = q.total_units;
  prm.qk_scale = kLog2e / sqrtf((float)dh);
  prm.pos = a.pos; prm.view = a.view; prm.rank = a.rank;
  prm.k_cache = static_cast<const __nv_bfloat16*>(a.k_cache);
  prm.v_cache = static_cast<const __nv_bfloat16*>(a.v_cache);
  prm.out = static_cast<__nv_bfloat16*>(a.out);
  prm.lse = a.lse;
  prm.status = a.status;
  prm.partials = static_cast<float*>(a.ws);
  prm.item_cnt = reinterpret_cast<unsigned*>(static_cast<char*>(a.ws) + q.partial_bytes);

#define FDLLM_ATTN_CASE(NQv, DHv)                                                           \
  if (q.NQ == NQv && dh == DHv)                                                            \
    return a.verify ? launch_t<NQv, DHv, true>(a, q, prm, maps, stream)                    \
                    : launch_t<NQv, DHv, false>(a, q, prm, maps, stream);
  FDLLM_ATTN_CASE(16, 64)
  FDLLM_ATTN_CASE(32, 64)
  FDLLM_ATTN_CASE(48, 64)
  FDLLM_ATTN_CASE(64, 64)
  FDLLM_ATTN_CASE(16, 128)
  FDLLM_ATTN_CASE(32, 128)
  FDLLM_ATTN_CASE(48, 128)
  FDLLM_ATTN_CASE(64, 128)
#undef FDLLM_ATTN_CASE
  return cudaErrorInvalidValue;
}

}  // namespace fdllm
