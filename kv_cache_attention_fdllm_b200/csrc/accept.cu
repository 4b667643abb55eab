// Top-1 / confidence / epsilon split / gamma prefix acceptance over logits rows.
//
// Flash-dLLM review, "Flash-Verify" (sec. 2.3) and "How It Works" (Step 1):
// confidence c_i = max_v q_i(v); D_t = {i : c_i >= eps}; verification accepts
// the S_t rows in decoding order while the mask-view prediction equals the
// draft and its confidence is >= gamma, stopping at the first mismatch.
//
// Design (HBM-bound scan of B*R*V fp32 logits):
//   grid = rows x splits.  Each CTA streams one contiguous span of one row with
//   128-bit evict-first loads and keeps, per thread, an online (max, sum of
//   exp(l - max), first argmax).  The CTA merges its threads in a fixed tree,
//   writes its partial, and the last CTA of the row (atomic counter) merges the
//   row's partials in split order, so the result does not depend on timing.
//   The last row of a sequence to finish applies the prefix rule.  No CTA
//   waits on another: every dependency is resolved by whoever arrives last.
#include <float.h>
#include <limits.h>

#include "common.cuh"
#include "kernels.h"

namespace fdllm {

namespace {

constexpr int kAcceptThreads = 256;
constexpr int kAcceptUnroll = 4;
constexpr float kLog2e = 1.4426950408889634f;

struct MaxSum {
  float m;   // running max
  float l;   // sum of exp(x - m)
  int idx;   // lowest index attaining m
};

__device__ __forceinline__ float scale_to(float m_old, float m_new) {
  return (m_old == -INFINITY) ? 0.f : exp2f((m_old - m_new) * kLog2e);
}

__device__ __forceinline__ MaxSum merge(const MaxSum& a, const MaxSum& b) {
  MaxSum r;
  r.m = fmaxf(a.m, b.m);
  r.l = a.l * scale_to(a.m, r.m) + b.l * scale_to(b.m, r.m);
  if (a.m == b.m)
    r.idx = min(a.idx, b.idx);
  else
    r.idx = (a.m > b.m) ? a.idx : b.idx;
  return r;
}

// Fold one value at index i into a thread's state (indices visited in
// increasing order by each thread).
__device__ __forceinline__ void fold1(MaxSum& s, float x, int i) {
  if (x > s.m) {
    s.l = s.l * scale_to(s.m, x) + 1.f;
    s.m = x;
    s.idx = i;
  } else if (x > -INFINITY) {  // a -inf logit adds nothing (and s.m is finite here)
    s.l += exp2f((x - s.m) * kLog2e);
  }
}

__global__ void __launch_bounds__(kAcceptThreads)
accept_kernel(int R, int V, int splits, int span, const float* __restrict__ logits,
              const int8_t* __restrict__ kind, const int32_t* __restrict__ ref_tok,
              const int32_t* __restrict__ rank, float eps, float gamma, int32_t* __restrict__ top1,
              float* __restrict__ conf, uint8_t* __restrict__ flags,
              int32_t* __restrict__ n_accept, AcceptPartial* __restrict__ parts,
              unsigned* __restrict__ row_cnt, unsigned* __restrict__ seq_cnt) {
  const int row = blockIdx.x;
  const int split = blockIdx.y;
  const int tid = threadIdx.x;
  const int s0 = split * span;
  const int s1 = min(V, s0 + span);
  const float* p = logits + (size_t)row * (size_t)V;

  MaxSum st{-INFINITY, 0.f, INT_MAX};
  // scalar head up to a 16-byte boundary, vector body, scalar tail
  const size_t off0 = (size_t)row * (size_t)V + (size_t)s0;
  int a0 = s0 + (int)((4 - (off0 & 3)) & 3);
  if (a0 > s1) a0 = s1;
  const int a1 = a0 + ((s1 - a0) & ~3);
  if (tid < a0 - s0) fold1(st, p[s0 + tid], s0 + tid);

  const int stride = kAcceptThreads * 4;
  for (int base = a0 + tid * 4; base < a1; base += stride * kAcceptUnroll) {
    float4 v[kAcceptUnroll];
#pragma unroll
    for (int u = 0; u < kAcceptUnroll; ++u) {
      const int i = base + u * stride;
      if (i < a1)
        v[u] = __ldcs(reinterpret_cast<const float4*>(p + i));
      else
        v[u] = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    }
    float cm = -INFINITY;
#pragma unroll
    for (int u = 0; u < kAcceptUnroll; ++u)
      cm = fmaxf(cm, fmaxf(fmaxf(v[u].x, v[u].y), fmaxf(v[u].z, v[u].w)));
    if (cm > st.m) {
      // the first index of the chunk that holds the new max
      int ci = INT_MAX;
#pragma unroll
      for (int u = kAcceptUnroll - 1; u >= 0; --u) {
        const int i = base + u * stride;
        if (v[u].w == cm) ci = i + 3;
        if (v[u].z == cm) ci = i + 2;
        if (v[u].y == cm) ci = i + 1;
        if (v[u].x == cm) ci = i;
      }
      st.l *= scale_to(st.m, cm);
      st.m = cm;
      st.idx = ci;
    }
    if (st.m > -INFINITY) {  // else this thread has seen nothing but -inf so far
      const float ms = st.m * kLog2e;
      float acc = 0.f;
#pragma unroll
      for (int u = 0; u < kAcceptUnroll; ++u) {
        acc += exp2f(fmaf(v[u].x, kLog2e, -ms)) + exp2f(fmaf(v[u].y, kLog2e, -ms)) +
               exp2f(fmaf(v[u].z, kLog2e, -ms)) + exp2f(fmaf(v[u].w, kLog2e, -ms));
      }
      st.l += acc;
    }
  }
  if (a1 + tid < s1) fold1(st, p[a1 + tid], a1 + tid);

  // CTA merge: warp butterfly, then warp 0 over the warps in order
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    MaxSum other;
    other.m = __shfl_xor_sync(0xffffffffu, st.m, o);
    other.l = __shfl_xor_sync(0xffffffffu, st.l, o);
    other.idx = __shfl_xor_sync(0xffffffffu, st.idx, o);
    st = merge(st, other);
  }
  __shared__ MaxSum warp_part[kAcceptThreads / 32];
  __shared__ int s_last_row, s_last_seq;
  const int warp = tid >> 5, lane = tid & 31;
  if (lane == 0) warp_part[warp] = st;
  __syncthreads();
  if (tid == 0) {
    MaxSum c = warp_part[0];
    for (int w = 1; w < kAcceptThreads / 32; ++w) c = merge(c, warp_part[w]);
    if (splits > 1) {
      parts[(size_t)row * splits + split] = AcceptPartial{c.m, c.l, c.idx, 0};
      __threadfence();
      const unsigned prev = atomicAdd(&row_cnt[row], 1u);
      s_last_row = (prev == (unsigned)splits - 1u);
      if (s_last_row) {
        __threadfence();
        const volatile AcceptPartial* vp = parts + (size_t)row * splits;
        MaxSum t{vp[0].m, vp[0].l, vp[0].idx};
        for (int s = 1; s < splits; ++s) t = merge(t, MaxSum{vp[s].m, vp[s].l, vp[s].idx});
        c = t;
        row_cnt[row] = 0u;  // leave the counter zeroed for the next call
      }
    } else {
      s_last_row = 1;
    }
    if (s_last_row) {
      const float cf = 1.f / c.l;  // the max contributes exp(0) = 1 to l
      const int k = kind[row];
      uint8_t f = 0;
      if (k == 1 && cf >= eps) f |= FDLLM_FLAG_COMMIT;
      if (k == 2 && c.idx == ref_tok[row] && cf >= gamma) f |= FDLLM_FLAG_PASS;
      top1[row] = c.idx;
      conf[row] = cf;
      flags[row] = f;
      __threadfence();
      const int b = row / R;
      const unsigned prev = atomicAdd(&seq_cnt[b], 1u);
      s_last_seq = (prev == (unsigned)R - 1u);
    } else {
      s_last_seq = 0;
    }
  }
  __syncthreads();
  if (!s_last_seq) return;

  // Last row of sequence b: the prefix rule over its kind-2 rows.
  __threadfence();
  const int b = row / R;
  const int r0 = b * R;
  const volatile uint8_t* vf = flags + r0;
  int ff = INT_MAX;  // smallest rank of a failing kind-2 row
  for (int r = tid; r < R; r += kAcceptThreads)
    if (kind[r0 + r] == 2 && !(vf[r] & FDLLM_FLAG_PASS)) ff = min(ff, rank[r0 + r]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ff = min(ff, __shfl_xor_sync(0xffffffffu, ff, o));
  __shared__ int warp_ff[kAcceptThreads / 32];
  __shared__ int warp_cnt[kAcceptThreads / 32];
  if (lane == 0) warp_ff[warp] = ff;
  __syncthreads();
  ff = warp_ff[0];
  for (int w = 1; w < kAcceptThreads / 32; ++w) ff = min(ff, warp_ff[w]);
  int cnt = 0;
  for (int r = tid; r < R; r += kAcceptThreads) {
    if (kind[r0 + r] == 2 && rank[r0 + r] < ff) {
      flags[r0 + r] = vf[r] | FDLLM_FLAG_ACCEPT;
      ++cnt;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) warp_cnt[warp] = cnt;
  __syncthreads();
  if (tid == 0) {
    int total = 0;
    for (int w = 0; w < kAcceptThreads / 32; ++w) total += warp_cnt[w];
    n_accept[b] = total;
    seq_cnt[b] = 0u;
  }
}

}  // namespace

AcceptLayout accept_layout(int B, int R, int V, int num_sms) {
  AcceptLayout L{};
  const long long rows = (long long)B * R;
  // one wave of resident CTAs (8 per SM at 256 threads), at least 2048
  // elements per CTA, at most one split per row when the rows fill the GPU
  const int resident = num_sms * 8;
  int sp = (int)(resident / (rows > 0 ? rows : 1));
  const int max_s = (V + 2047) / 2048;
  if (sp > max_s) sp = max_s;
  if (sp < 1) sp = 1;
  L.splits = sp;
  L.parts_bytes = align_up((size_t)rows * sp * sizeof(AcceptPartial), 256);
  L.row_cnt_bytes = align_up((size_t)rows * sizeof(unsigned), 256);
  L.seq_cnt_bytes = align_up((size_t)(B > 0 ? B : 1) * sizeof(unsigned), 256);
  return L;
}

cudaError_t launch_accept(const AcceptArgs& a, const AcceptLayout& L, cudaStream_t stream) {
  const int rows = a.B * a.R;
  if (rows == 0) return cudaSuccess;
  int span = (a.V + L.splits - 1) / L.splits;
  span = (span + 3) & ~3;
  dim3 grid(rows, L.splits);
  accept_kernel<<<grid, kAcceptThreads, 0, stream>>>(
      a.R, a.V, L.splits, span, a.logits, a.kind, a.ref_tok, a.rank, a.eps, a.gamma, a.top1,
      a.conf, a.flags, a.n_accept, a.parts, a.row_cnt, a.seq_cnt);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace fdllm
