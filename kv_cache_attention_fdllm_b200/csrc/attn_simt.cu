// Full-cache attention on the CUDA cores (fp32 storage path).
//
// Flash-dLLM review, "How It Works", Step 1: Draft: after the new k, v are
// written, every query attends over the whole bidirectional cache.  With the
// verify metadata it applies the Flash-Verify view rule ("Flash-Verify",
// sec. 2.3): draft and mask views share positions, each hidden from the other.
//
// One CTA (4 warps) per (sequence, head, group of 4 query rows).  Warps take
// keys round-robin; the lanes of a warp split the head dimension, so each key
// row is one coalesced load.  Each warp keeps an online softmax per query; the
// four warps are merged at the end.
#include "common.cuh"
#include "kernels.h"

namespace fdllm {

namespace {

constexpr int kQG = 4;
constexpr int kNW = 4;
constexpr float kLog2e = 1.4426950408889634f;

template <typename T, int EPL>
__device__ __forceinline__ void load_row(const T* p, float* v) {
#pragma unroll
  for (int e = 0; e < EPL; ++e) v[e] = Store<T>::ld(p + e);
}

template <typename T, int EPL>
__global__ void __launch_bounds__(128) attn_simt(AttnArgs a) {
  extern __shared__ int smeta[];  // verify: dpos[R], drank[R], srank[R]
  __shared__ float sm_m[kNW][kQG], sm_l[kNW][kQG];
  __shared__ float sm_acc[kNW][kQG][EPL * 32];
  __shared__ int s_ndraft, s_nside;
  const int dh = EPL * 32;
  const int b = blockIdx.x / a.H, h = blockIdx.x % a.H;
  const int r0 = blockIdx.y * kQG;
  const int rows = a.rows_per_seq;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float qscale = kLog2e / sqrtf((float)dh);

  int* dpos = smeta;
  int* drank = smeta + rows;
  int* srank = smeta + 2 * rows;
  if (a.verify && threadIdx.x == 0) {
    int nd = 0, ns = 0;
    for (int r = 0; r < rows; ++r) {
      const int vw = a.view[b * rows + r];
      if (vw == 1) {
        dpos[nd] = a.pos[b * rows + r];
        drank[nd++] = a.rank[b * rows + r];
      } else if (vw == 2) {
        srank[ns++] = a.rank[b * rows + r];
      }
    }
    s_ndraft = nd;
    s_nside = ns < a.S_max ? ns : a.S_max;
  }
  __syncthreads();

  float q[kQG][EPL];
  bool qvalid[kQG];
  int qview[kQG], qrank[kQG];
#pragma unroll
  for (int g = 0; g < kQG; ++g) {
    const int r = r0 + g;
    qvalid[g] = r < rows;
    qview[g] = 0;
    qrank[g] = 0;
    if (qvalid[g]) {
      const T* qp = static_cast<const T*>(a.q) + (((size_t)b * rows + r) * a.H + h) * dh + lane * EPL;
      load_row<T, EPL>(qp, q[g]);
#pragma unroll
      for (int e = 0; e < EPL; ++e) q[g][e] *= qscale;
      if (a.verify) {
        qview[g] = a.view[b * rows + r];
        qrank[g] = a.rank[b * rows + r];
      }
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) q[g][e] = 0.f;
    }
  }

  float m[kQG], l[kQG], acc[kQG][EPL];
#pragma unroll
  for (int g = 0; g < kQG; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[g][e] = 0.f;
  }

  const int n_draft = a.verify ? s_ndraft : 0;
  const int n_side = a.verify ? s_nside : 0;
  const int n_keys = a.N + n_side;
  const T* Kc = static_cast<const T*>(a.k_cache) + ((size_t)b * a.H + h) * a.N * dh;
  const T* Vc = static_cast<const T*>(a.v_cache) + ((size_t)b * a.H + h) * a.N * dh;
  const T* Ks = a.verify ? static_cast<const T*>(a.k_side) + ((size_t)b * a.H + h) * a.S_max * dh : nullptr;
  const T* Vs = a.verify ? static_cast<const T*>(a.v_side) + ((size_t)b * a.H + h) * a.S_max * dh : nullptr;

  for (int j = warp; j < n_keys; j += kNW) {
    const bool side = j >= a.N;
    const int js = j - a.N;
    float k[EPL];
    load_row<T, EPL>((side ? Ks + (size_t)js * dh : Kc + (size_t)j * dh) + lane * EPL, k);
    float s[kQG];
#pragma unroll
    for (int g = 0; g < kQG; ++g) {
      float t = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) t = fmaf(q[g][e], k[e], t);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      s[g] = t;
    }
    int kdr = -1;
    if (!side)
      for (int t = 0; t < n_draft; ++t)
        if (dpos[t] == j) kdr = drank[t];
    bool vis[kQG];
    bool any = false;
#pragma unroll
    for (int g = 0; g < kQG; ++g) {
      bool v = qvalid[g];
      if (v && a.verify)
        v = side ? visible_side(qview[g], qrank[g], srank[js], a.causal_cross)
                 : visible_cache(qview[g], qrank[g], kdr, a.causal_cross);
      vis[g] = v;
      any |= v;
    }
    if (!any) continue;
    float v[EPL];
    load_row<T, EPL>((side ? Vs + (size_t)js * dh : Vc + (size_t)j * dh) + lane * EPL, v);
#pragma unroll
    for (int g = 0; g < kQG; ++g) {
      if (!vis[g]) continue;
      const float mn = fmaxf(m[g], s[g]);
      const float sc = (m[g] == -INFINITY) ? 0.f : exp2f(m[g] - mn);
      const float p = exp2f(s[g] - mn);
      l[g] = l[g] * sc + p;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[g][e] = fmaf(p, v[e], acc[g][e] * sc);
      m[g] = mn;
    }
  }

#pragma unroll
  for (int g = 0; g < kQG; ++g) {
    if (lane == 0) {
      sm_m[warp][g] = m[g];
      sm_l[warp][g] = l[g];
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) sm_acc[warp][g][lane * EPL + e] = acc[g][e];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kQG * dh; i += blockDim.x) {
    const int g = i / dh, d = i % dh;
    const int r = r0 + g;
    if (r >= rows) continue;
    float M = -INFINITY;
    for (int w = 0; w < kNW; ++w) M = fmaxf(M, sm_m[w][g]);
    float num = 0.f, den = 0.f;
    for (int w = 0; w < kNW; ++w) {
      const float sc = (sm_m[w][g] == -INFINITY) ? 0.f : exp2f(sm_m[w][g] - M);
      num += sm_acc[w][g][d] * sc;
      den += sm_l[w][g] * sc;
    }
    T* o = static_cast<T*>(a.out) + ((size_t)b * rows + r) * a.H * dh + h * dh + d;
    Store<T>::st(o, num / den);
    if (d == 0 && a.lse) a.lse[((size_t)b * rows + r) * a.H + h] = M + log2f(den);
  }
}

template <typename T>
cudaError_t launch_typed(const AttnArgs& a, cudaStream_t stream) {
  dim3 grid(a.B * a.H, (a.rows_per_seq + kQG - 1) / kQG);
  const size_t smem = a.verify ? (size_t)3 * a.rows_per_seq * sizeof(int) : 0;
  if (a.dh == 64)
    attn_simt<T, 2><<<grid, 128, smem, stream>>>(a);
  else
    attn_simt<T, 4><<<grid, 128, smem, stream>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t stream) {
  if (a.B * a.rows_per_seq == 0) return cudaSuccess;
  return a.dtype == FDLLM_F32 ? launch_typed<float>(a, stream)
                              : launch_typed<__nv_bfloat16>(a, stream);
}

}  // namespace fdllm
