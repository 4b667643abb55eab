// QKV projection + RoPE + cache scatter on the CUDA cores (fp32 storage path).
//
// Flash-dLLM review, "How It Works", Step 1: Draft (Alg. 1): the step reads only
// the hidden rows x[Q], builds q, k, v from them and writes k, v into the cache at
// exactly the slots of Q.  Two kernels:
//   proj_gemm_simt   Y[m, f] = sum_d x_row(m)[d] * W[f, d]  (fp32 accumulation)
//   rope_scatter     rotates the q and k heads of each row (pairs j, j + dh/2)
//                    and writes q -> q_out, k, v -> cache (or side slots).
#include "common.cuh"
#include "kernels.h"

namespace fdllm {

namespace {

constexpr int kTF = 64;  // features per tile
constexpr int kTM = 32;  // rows per tile
constexpr int kTK = 32;  // reduction chunk

// Row m of the projection input, or nullptr when its index is out of range.
template <typename T>
__device__ __forceinline__ const T* proj_row(const ProjArgs& a, int m) {
  const T* x = static_cast<const T*>(a.x);
  const int j = a.idx[m];
  if (a.verify) return x + (size_t)m * a.D;
  if (j < 0 || j >= a.N) return nullptr;
  if (a.packed) return x + (size_t)m * a.D;
  const int b = m / a.rows_per_seq;
  return x + ((size_t)b * a.N + j) * a.D;
}

template <typename T>
__global__ void __launch_bounds__(256) proj_gemm_simt(ProjArgs a, int M, float* __restrict__ Y) {
  __shared__ float Ws[kTK][kTF + 1];
  __shared__ float Xs[kTK][kTM + 1];
  __shared__ const T* rows[kTM];
  const int F = 3 * a.H * a.dh;
  const int f0 = blockIdx.x * kTF;
  const int m0 = blockIdx.y * kTM;
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  if (tid < kTM) rows[tid] = (m0 + tid < M) ? proj_row<T>(a, m0 + tid) : nullptr;
  __syncthreads();
  const T* W = static_cast<const T*>(a.w);
  float acc[4][2] = {};
  for (int k0 = 0; k0 < a.D; k0 += kTK) {
    for (int e = tid; e < kTF * kTK; e += 256) {
      const int f = e / kTK, k = e % kTK;
      const int gf = f0 + f, gk = k0 + k;
      Ws[k][f] = (gf < F && gk < a.D) ? Store<T>::ld(W + (size_t)gf * a.D + gk) : 0.f;
    }
    for (int e = tid; e < kTM * kTK; e += 256) {
      const int r = e / kTK, k = e % kTK;
      const T* row = rows[r];
      const int gk = k0 + k;
      Xs[k][r] = (row && gk < a.D) ? Store<T>::ld(row + gk) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kTK; ++k) {
      float w[4], x[2];
#pragma unroll
      for (int i = 0; i < 4; ++i) w[i] = Ws[k][tx * 4 + i];
#pragma unroll
      for (int j = 0; j < 2; ++j) x[j] = Xs[k][ty * 2 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) acc[i][j] = fmaf(w[i], x[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int f = f0 + tx * 4 + i, m = m0 + ty * 2 + j;
      if (f < F && m < M) Y[(size_t)m * F + f] = acc[i][j];
    }
}

// One CTA per projection row: rotate and write q, k, v of every head.
template <typename T>
__global__ void __launch_bounds__(128) rope_scatter_simt(ProjArgs a, const float* __restrict__ Y) {
  const int m = blockIdx.x;
  const int b = m / a.rows_per_seq;
  const int E = a.H * a.dh;
  const int half = a.dh / 2;
  const float* y = Y + (size_t)m * 3 * E;
  __shared__ int s_pos, s_dst_side, s_slot;
  if (threadIdx.x == 0) {
    const int p = a.idx[m];
    int side = 0, slot = p;
    bool ok = (p >= 0 && p < a.N);
    if (a.verify && a.view[m] == 2) {
      side = 1;
      slot = 0;
      const int r0 = b * a.rows_per_seq;
      for (int r = r0; r < m; ++r) slot += (a.view[r] == 2);
      if (slot >= a.S_max) ok = false;
    }
    if (!ok) set_status(a.status, FDLLM_ERR_BAD_INDEX);
    s_pos = ok ? p : -1;
    s_dst_side = side;
    s_slot = slot;
  }
  __syncthreads();
  const int pos = s_pos;
  T* qo = static_cast<T*>(a.q_out) + (size_t)m * E;
  T* kc = static_cast<T*>(s_dst_side ? a.k_side : a.k_cache);
  T* vc = static_cast<T*>(s_dst_side ? a.v_side : a.v_cache);
  const int n_slots = s_dst_side ? a.S_max : a.N;
  for (int e = threadIdx.x; e < a.H * half; e += blockDim.x) {
    const int h = e / half, j = e % half;
    float c = 1.f, s = 0.f;
    if (pos >= 0) rope_cos_sin(pos, rope_inv_freq(j, a.dh, a.log2_base), &c, &s);
    const int o1 = h * a.dh + j, o2 = o1 + half;
    // q
    {
      const float x1 = y[o1], x2 = y[o2];
      Store<T>::st(qo + o1, pos >= 0 ? x1 * c - x2 * s : 0.f);
      Store<T>::st(qo + o2, pos >= 0 ? x1 * s + x2 * c : 0.f);
    }
    if (pos < 0) continue;
    const size_t dst = (((size_t)b * a.H + h) * n_slots + s_slot) * a.dh;
    {
      const float x1 = y[E + o1], x2 = y[E + o2];
      Store<T>::st(kc + dst + j, x1 * c - x2 * s);
      Store<T>::st(kc + dst + j + half, x1 * s + x2 * c);
    }
    Store<T>::st(vc + dst + j, y[2 * E + o1]);
    Store<T>::st(vc + dst + j + half, y[2 * E + o2]);
  }
}

}  // namespace

size_t proj_simt_workspace_bytes(int M, int H, int dh) {
  return align_up((size_t)M * 3 * H * dh * sizeof(float), 256);
}

cudaError_t launch_proj_simt(const ProjArgs& a, cudaStream_t stream) {
  const int M = a.B * a.rows_per_seq;
  if (M == 0) return cudaSuccess;
  const int F = 3 * a.H * a.dh;
  float* Y = static_cast<float*>(a.ws);
  dim3 g1((F + kTF - 1) / kTF, (M + kTM - 1) / kTM);
  if (a.dtype == FDLLM_F32) {
    proj_gemm_simt<float><<<g1, 256, 0, stream>>>(a, M, Y);
    rope_scatter_simt<float><<<M, 128, 0, stream>>>(a, Y);
  } else {
    proj_gemm_simt<__nv_bfloat16><<<g1, 256, 0, stream>>>(a, M, Y);
    rope_scatter_simt<__nv_bfloat16><<<M, 128, 0, stream>>>(a, Y);
  }
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace fdllm
