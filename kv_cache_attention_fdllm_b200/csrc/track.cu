// Tracked-set selection for the next step.
//
// Flash-dLLM review, "How It Works", Step 1: Cache selection: the next tracked
// set T is the beta_t decoded positions the masked queries attend to most, the
// positions decoded in this step ranked with the earlier ones.  The attention
// mass of slot j is
//   a[b, j] = sum over masked-query rows i and heads h of p_ij,
//   p_ij = 2^(s_ij - lse_i),  s_ij = q_ih . K_hj * log2(e) / sqrt(dh),
// the draft pass's own probabilities: lse (per row and head, log2 units) is
// what the attention kernels leave in the workspace, q the staged queries.
//
//   track_mass     grid (key tiles of 128, H, B), one thread per slot: the
//                  slot's K row in registers, the masked rows' q in shared
//                  memory 32 at a time; writes the per-head mass.
//   track_select   one CTA per sequence: sums the heads in order, keys each
//                  candidate slot by (mass bits, inverted slot) - unique, so
//                  the order is total and the result exact - finds the
//                  beta_t-th largest key by an 8-bit radix select, gathers the
//                  keys at or above it and sorts them (bitonic) into T.
#include "common.cuh"
#include "kernels.h"

namespace fdllm {

namespace {

constexpr int kSlots = 128;      // slots per CTA of the mass kernel
constexpr int kRowsChunk = 32;   // masked rows staged per pass
constexpr int kSelThreads = 1024;
constexpr float kLog2eF = 1.4426950408889634f;

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T, int DH>
__global__ void __launch_bounds__(kSlots) track_mass_kernel(TrackArgs a) {
  __shared__ float qs[kRowsChunk][DH];
  __shared__ float ls[kRowsChunk];
  const int b = blockIdx.z, h = blockIdx.y;
  const int j = blockIdx.x * kSlots + threadIdx.x;
  const float scale = kLog2eF / sqrtf((float)DH);
  const T* q = static_cast<const T*>(a.q);
  float k[DH];
  if (j < a.N) {
    const T* kr = static_cast<const T*>(a.k_cache) + (((size_t)b * a.H + h) * a.N + j) * DH;
#pragma unroll
    for (int d = 0; d < DH; ++d) k[d] = to_f<T>(kr[d]);
  }
  float acc = 0.f;
  for (int base = 0; base < a.nq; base += kRowsChunk) {
    __syncthreads();
    for (int i = threadIdx.x; i < kRowsChunk * DH; i += kSlots) {
      const int rr = base + i / DH, d = i % DH;
      const bool use = rr < a.nq && a.q_masked[(size_t)b * a.nq + rr] != 0;
      qs[i / DH][d] = use ? to_f<T>(q[(((size_t)b * a.nq + rr) * a.H + h) * DH + d]) * scale : 0.f;
    }
    if (threadIdx.x < kRowsChunk) {
      const int rr = base + threadIdx.x;
      const bool use = rr < a.nq && a.q_masked[(size_t)b * a.nq + rr] != 0;
      ls[threadIdx.x] = use ? a.lse[((size_t)b * a.nq + rr) * a.H + h] : INFINITY;
    }
    __syncthreads();
    if (j < a.N) {
      for (int i = 0; i < kRowsChunk; ++i) {
        if (ls[i] == INFINITY) continue;  // not a masked row (uniform over the CTA)
        float s = 0.f;
#pragma unroll
        for (int d = 0; d < DH; ++d) s = fmaf(qs[i][d], k[d], s);
        acc += exp2f(s - ls[i]);
      }
    }
  }
  if (j < a.N) a.mass_h[((size_t)b * a.H + h) * a.N + j] = acc;
}

__device__ __forceinline__ unsigned long long slot_key(float m, int j) {
  // m >= 0: its bits order like the value; the low word prefers the lower slot
  return ((unsigned long long)__float_as_uint(m) << 32) | (unsigned long long)(0xFFFFFFFFu - (unsigned)j);
}

__global__ void __launch_bounds__(kSelThreads) track_select_kernel(TrackArgs a) {
  __shared__ unsigned hist[256];
  __shared__ unsigned long long list[kMaxBetaT];
  __shared__ unsigned long long s_prefix;
  __shared__ unsigned s_rank, s_cnt, s_ncand;
  const int b = blockIdx.x, tid = threadIdx.x;
  const int N = a.N;
  float* mass = a.mass + (size_t)b * N;
  const int8_t* cand = a.candidate + (size_t)b * N;

  // head sum in a fixed order (deterministic), candidates counted
  if (tid == 0) s_ncand = 0u;
  __syncthreads();
  unsigned nc = 0;
  for (int j = tid; j < N; j += kSelThreads) {
    float s = 0.f;
    for (int h = 0; h < a.H; ++h) s += a.mass_h[((size_t)b * a.H + h) * N + j];
    mass[j] = s;
    nc += cand[j] != 0;
  }
  atomicAdd(&s_ncand, nc);
  __syncthreads();
  const unsigned k_eff = s_ncand < (unsigned)a.beta_t ? s_ncand : (unsigned)a.beta_t;

  // radix select of the k_eff-th largest candidate key, 8 bits at a time
  if (tid == 0) {
    s_prefix = 0ull;
    s_rank = k_eff;
  }
  unsigned long long mask = 0ull;
  for (int shift = 56; shift >= 0 && k_eff > 0; shift -= 8) {
    for (int d = tid; d < 256; d += kSelThreads) hist[d] = 0u;
    __syncthreads();
    const unsigned long long prefix = s_prefix;
    for (int j = tid; j < N; j += kSelThreads) {
      if (cand[j] == 0) continue;
      const unsigned long long key = slot_key(mass[j], j);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255ull], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      unsigned cum = 0u, need = s_rank;
      for (int d = 255; d >= 0; --d) {
        if (cum + hist[d] >= need) {
          s_prefix = prefix | ((unsigned long long)d << shift);
          s_rank = need - cum;
          break;
        }
        cum += hist[d];
      }
    }
    mask |= 255ull << shift;
    __syncthreads();
  }

  // the k_eff keys at or above the threshold (keys are unique), then sort them
  if (tid == 0) s_cnt = 0u;
  __syncthreads();
  const unsigned long long thr = s_prefix;
  if (k_eff > 0) {
    for (int j = tid; j < N; j += kSelThreads) {
      if (cand[j] == 0) continue;
      const unsigned long long key = slot_key(mass[j], j);
      if (key >= thr) {
        const unsigned at = atomicAdd(&s_cnt, 1u);
        if (at < (unsigned)kMaxBetaT) list[at] = key;
      }
    }
  }
  __syncthreads();
  unsigned n2 = 1;
  while (n2 < k_eff) n2 <<= 1;
  for (unsigned i = k_eff + tid; i < n2; i += kSelThreads) list[i] = 0ull;
  __syncthreads();
  // bitonic sort, descending
  for (unsigned size = 2; size <= n2; size <<= 1) {
    for (unsigned stride = size >> 1; stride > 0; stride >>= 1) {
      for (unsigned i = tid; i < n2; i += kSelThreads) {
        const unsigned p = i ^ stride;
        if (p > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long x = list[i], y = list[p];
          if (desc ? (x < y) : (x > y)) {
            list[i] = y;
            list[p] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int t = tid; t < a.beta_t; t += kSelThreads)
    a.track[(size_t)b * a.beta_t + t] =
        (unsigned)t < k_eff ? (int32_t)(0xFFFFFFFFu - (unsigned)(list[t] & 0xFFFFFFFFull)) : -1;
}

template <typename T>
cudaError_t launch_mass(const TrackArgs& a, cudaStream_t stream) {
  const dim3 grid((unsigned)((a.N + kSlots - 1) / kSlots), (unsigned)a.H, (unsigned)a.B);
  if (a.dh == 64)
    track_mass_kernel<T, 64><<<grid, kSlots, 0, stream>>>(a);
  else
    track_mass_kernel<T, 128><<<grid, kSlots, 0, stream>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

size_t track_workspace_bytes(int B, int N, int H) {
  return align_up((size_t)B * H * N * sizeof(float), 256) + align_up((size_t)B * N * sizeof(float), 256);
}

cudaError_t launch_track(const TrackArgs& a, cudaStream_t stream) {
  if (a.B == 0) return cudaSuccess;
  cudaError_t e = a.dtype == FDLLM_F32 ? launch_mass<float>(a, stream) : launch_mass<__nv_bfloat16>(a, stream);
  if (e != cudaSuccess) return e;
  track_select_kernel<<<a.B, kSelThreads, 0, stream>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace fdllm
