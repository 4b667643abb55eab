// C ABI of the fused KV-cache step: argument checks, workspace layout, launches.
// The operations are defined in include/fdllm.h.
#include <math.h>
#include <string.h>

#include <atomic>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "kernels.h"

using namespace fdllm;

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr int kMaxVerifyRows = 512;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// An NVTX range around each entry point, so that a profiler's timeline shows
// which call launched which kernels (a no-op when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

size_t elt_size(int dtype) { return dtype == FDLLM_F32 ? 4 : 2; }

fdllm_status check_shape(int B, int N, int D, int H, int dh, int rows, int dtype) {
  if (B < 0 || N < 1 || D < 1 || H < 1 || rows < 0) return FDLLM_ERR_INVALID_ARG;
  if (dtype != FDLLM_F32 && dtype != FDLLM_BF16) return FDLLM_ERR_UNSUPPORTED;
  if (dh != 64 && dh != 128) return FDLLM_ERR_UNSUPPORTED;
  if (dtype == FDLLM_BF16 && D % 64 != 0) return FDLLM_ERR_UNSUPPORTED;
  if (dtype == FDLLM_F32 && D % 4 != 0) return FDLLM_ERR_UNSUPPORTED;
  if ((long long)B * N > (1ll << 31) || (long long)3 * H * dh > (1 << 20))
    return FDLLM_ERR_UNSUPPORTED;
  return FDLLM_OK;
}

// Workspace layout shared by a full step, its two stage calls and the
// tracked-set selection that follows a fused step:
//   [header 256 B | q staging | lse | selection scratch (fused step only) |
//    attention scratch | projection scratch]
// Everything before the projection region is independent of D, so a stage
// attention call or a selection call finds it at the same offsets whatever D
// the full step was sized for.
struct Layout {
  size_t q_off, lse_off, track_off, attn_off, proj_off, total;
  size_t track_bytes, proj_bytes, attn_bytes;
};

Layout step_layout(int B, int N, int D, int H, int dh, int rows, int S_max, int verify,
                   int dtype) {
  const int sms = device_sm_count();
  Layout L;
  L.q_off = kWsHeaderBytes;
  const size_t q_bytes = align_up((size_t)B * rows * H * dh * elt_size(dtype), 256);
  L.lse_off = L.q_off + q_bytes;
  L.track_off = L.lse_off + align_up((size_t)B * rows * H * sizeof(float), 256);
  L.track_bytes = verify ? 0 : align_up(track_workspace_bytes(B, N, H), 256);
  L.attn_off = L.track_off + L.track_bytes;
  L.attn_bytes =
      align_up(attn_workspace_bytes(B, N, H, dh, rows, S_max, verify, dtype, sms), 256);
  L.proj_off = L.attn_off + L.attn_bytes;
  L.proj_bytes = align_up(proj_workspace_bytes(B * rows, D, H, dh, dtype, sms), 256);
  L.total = L.proj_off + L.proj_bytes;
  return L;
}

fdllm_status check_ws(void* ws, size_t bytes, size_t need) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || bytes < need)
    return FDLLM_ERR_WORKSPACE;
  return FDLLM_OK;
}

fdllm_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FDLLM_OK : FDLLM_ERR_CUDA; }

char* ws_at(void* ws, size_t off) { return static_cast<char*>(ws) + off; }

fdllm_status run_proj(int B, int N, int D, int H, int dh, int rows, int S_max, int verify,
                      int dtype, const void* x, const int32_t* idx, const int8_t* view,
                      const void* w, float rope_base, void* k_cache, void* v_cache,
                      void* k_side, void* v_side, void* q_out, void* ws, const Layout& L,
                      cudaStream_t stream, int packed = 0) {
  ProjArgs a{};
  a.B = B; a.N = N; a.D = D; a.H = H; a.dh = dh; a.rows_per_seq = rows; a.S_max = S_max;
  a.verify = verify; a.dtype = dtype; a.packed = verify ? 1 : packed;
  a.x = x; a.idx = idx; a.view = view; a.w = w;
  a.log2_base = log2((double)rope_base);
  a.k_cache = k_cache; a.v_cache = v_cache; a.k_side = k_side; a.v_side = v_side;
  a.q_out = q_out;
  a.status = reinterpret_cast<int*>(ws);
  a.ws = ws_at(ws, L.proj_off);
  a.ws_bytes = L.proj_bytes;
  return from_cuda(launch_proj(a, stream));
}

fdllm_status run_attn(int B, int N, int H, int dh, int rows, int S_max, int verify, int causal,
                      int dtype, const void* q, const int32_t* pos, const int8_t* view,
                      const int32_t* rank, const void* k_cache, const void* v_cache,
                      const void* k_side, const void* v_side, void* out, void* ws,
                      const Layout& L, cudaStream_t stream) {
  AttnArgs a{};
  a.B = B; a.N = N; a.H = H; a.dh = dh; a.rows_per_seq = rows; a.S_max = S_max;
  a.verify = verify; a.causal_cross = causal; a.dtype = dtype;
  a.q = q; a.k_cache = k_cache; a.v_cache = v_cache; a.k_side = k_side; a.v_side = v_side;
  a.pos = pos; a.view = view; a.rank = rank; a.out = out;
  a.lse = reinterpret_cast<float*>(ws_at(ws, L.lse_off));
  a.status = reinterpret_cast<int*>(ws);
  a.ws = ws_at(ws, L.attn_off);
  a.ws_bytes = L.attn_bytes;
  return from_cuda(launch_attn(a, stream));
}

bool all_aligned(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (!p || !aligned16(p)) return false;
  return true;
}

fdllm_status check_verify_extra(int R, int S_max, int causal) {
  if (R > kMaxVerifyRows) return FDLLM_ERR_UNSUPPORTED;
  if (S_max < 0 || (causal != 0 && causal != 1)) return FDLLM_ERR_INVALID_ARG;
  return FDLLM_OK;
}

}  // namespace

namespace fdllm {
static std::atomic<unsigned long long> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}
}  // namespace fdllm

extern "C" {

int fdllm_version(void) { return kVersion; }

uint64_t fdllm_launch_count(void) { return (uint64_t)g_launches.load(std::memory_order_relaxed); }

const char* fdllm_status_string(fdllm_status s) {
  switch (s) {
    case FDLLM_OK: return "ok";
    case FDLLM_ERR_INVALID_ARG: return "invalid argument";
    case FDLLM_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case FDLLM_ERR_CUDA: return "CUDA error";
    case FDLLM_ERR_BAD_INDEX: return "index out of range";
    case FDLLM_ERR_TIMEOUT: return "bounded wait ran out on the device";
    case FDLLM_ERR_WORKSPACE: return "workspace too small or misaligned";
  }
  return "unknown status";
}

size_t fdllm_fused_step_workspace_bytes(int B, int N, int D, int H, int dh, int nq, int dtype) {
  if (check_shape(B, N, D, H, dh, nq, dtype) != FDLLM_OK) return 0;
  return step_layout(B, N, D, H, dh, nq, 0, 0, dtype).total;
}

size_t fdllm_verify_step_workspace_bytes(int B, int N, int D, int H, int dh, int R, int S_max,
                                         int dtype) {
  if (check_shape(B, N, D, H, dh, R, dtype) != FDLLM_OK) return 0;
  if (check_verify_extra(R, S_max, 0) != FDLLM_OK) return 0;
  return step_layout(B, N, D, H, dh, R, S_max, 1, dtype).total;
}

size_t fdllm_accept_workspace_bytes(int B, int R, int V) {
  if (B < 0 || R < 0 || V < 1) return 0;
  return kWsHeaderBytes + accept_layout(B, R, V, device_sm_count()).total();
}

fdllm_status fdllm_qkv_rope_scatter(int B, int N, int D, int H, int dh, int nq, int dtype,
                                    const void* x, const int32_t* q_idx, const void* w_qkv,
                                    float rope_base, void* k_cache, void* v_cache, void* q_out,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("fdllm_qkv_rope_scatter");
  fdllm_status st = check_shape(B, N, D, H, dh, nq, dtype);
  if (st != FDLLM_OK) return st;
  if (!(rope_base > 0.f)) return FDLLM_ERR_INVALID_ARG;
  const Layout L = step_layout(B, N, D, H, dh, nq, 0, 0, dtype);
  if ((st = check_ws(workspace, workspace_bytes, L.total)) != FDLLM_OK) return st;
  if (B * nq == 0) return FDLLM_OK;
  if (!all_aligned({x, q_idx, w_qkv, k_cache, v_cache, q_out})) return FDLLM_ERR_INVALID_ARG;
  return run_proj(B, N, D, H, dh, nq, 0, 0, dtype, x, q_idx, nullptr, w_qkv, rope_base, k_cache,
                  v_cache, nullptr, nullptr, q_out, workspace, L,
                  static_cast<cudaStream_t>(stream));
}

fdllm_status fdllm_attend(int B, int N, int H, int dh, int nq, int dtype, const void* q,
                          const void* k_cache, const void* v_cache, void* out, void* workspace,
                          size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("fdllm_attend");
  fdllm_status st = check_shape(B, N, 64, H, dh, nq, dtype);
  if (st != FDLLM_OK) return st;
  // the attention region does not depend on D
  const Layout L = step_layout(B, N, 64, H, dh, nq, 0, 0, dtype);
  if ((st = check_ws(workspace, workspace_bytes, L.attn_off + L.attn_bytes)) != FDLLM_OK)
    return st;
  if (B * nq == 0) return FDLLM_OK;
  if (!all_aligned({q, k_cache, v_cache, out})) return FDLLM_ERR_INVALID_ARG;
  return run_attn(B, N, H, dh, nq, 0, 0, 0, dtype, q, nullptr, nullptr, nullptr, k_cache,
                  v_cache, nullptr, nullptr, out, workspace, L,
                  static_cast<cudaStream_t>(stream));
}

fdllm_status fdllm_fused_step(int B, int N, int D, int H, int dh, int nq, int dtype,
                              const void* x, const int32_t* q_idx, const void* w_qkv,
                              float rope_base, void* k_cache, void* v_cache, void* out,
                              void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("fdllm_fused_step");
  fdllm_status st = check_shape(B, N, D, H, dh, nq, dtype);
  if (st != FDLLM_OK) return st;
  if (!(rope_base > 0.f)) return FDLLM_ERR_INVALID_ARG;
  const Layout L = step_layout(B, N, D, H, dh, nq, 0, 0, dtype);
  if ((st = check_ws(workspace, workspace_bytes, L.total)) != FDLLM_OK) return st;
  if (B * nq == 0) return FDLLM_OK;
  if (!all_aligned({x, q_idx, w_qkv, k_cache, v_cache, out})) return FDLLM_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* q = ws_at(workspace, L.q_off);
  st = run_proj(B, N, D, H, dh, nq, 0, 0, dtype, x, q_idx, nullptr, w_qkv, rope_base, k_cache,
                v_cache, nullptr, nullptr, q, workspace, L, s);
  if (st != FDLLM_OK) return st;
  return run_attn(B, N, H, dh, nq, 0, 0, 0, dtype, q, nullptr, nullptr, nullptr, k_cache,
                  v_cache, nullptr, nullptr, out, workspace, L, s);
}

fdllm_status fdllm_fused_step_rows(int B, int N, int D, int H, int dh, int nq, int dtype,
                                   const void* x_rows, const int32_t* q_idx, const void* w_qkv,
                                   float rope_base, void* k_cache, void* v_cache, void* out,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("fdllm_fused_step_rows");
  fdllm_status st = check_shape(B, N, D, H, dh, nq, dtype);
  if (st != FDLLM_OK) return st;
  if (!(rope_base > 0.f)) return FDLLM_ERR_INVALID_ARG;
  const Layout L = step_layout(B, N, D, H, dh, nq, 0, 0, dtype);
  if ((st = check_ws(workspace, workspace_bytes, L.total)) != FDLLM_OK) return st;
  if (B * nq == 0) return FDLLM_OK;
  if (!all_aligned({x_rows, q_idx, w_qkv, k_cache, v_cache, out})) return FDLLM_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* q = ws_at(workspace, L.q_off);
  st = run_proj(B, N, D, H, dh, nq, 0, 0, dtype, x_rows, q_idx, nullptr, w_qkv, rope_base,
                k_cache, v_cache, nullptr, nullptr, q, workspace, L, s, /*packed=*/1);
  if (st != FDLLM_OK) return st;
  return run_attn(B, N, H, dh, nq, 0, 0, 0, dtype, q, nullptr, nullptr, nullptr, k_cache,
                  v_cache, nullptr, nullptr, out, workspace, L, s);
}

fdllm_status fdllm_verify_qkv_rope_scatter(int B, int N, int D, int H, int dh, int R, int S_max,
                                           int dtype, const void* x_rows, const int32_t* pos,
                                           const int8_t* view, const void* w_qkv,
                                           float rope_base, void* k_cache, void* v_cache,
                                           void* k_side, void* v_side, void* q_out,
                                           void* workspace, size_t workspace_bytes,
                                           void* stream) {
  NvtxRange nvtx_range("fdllm_verify_qkv_rope_scatter");
  fdllm_status st = check_shape(B, N, D, H, dh, R, dtype);
  if (st != FDLLM_OK) return st;
  if ((st = check_verify_extra(R, S_max, 0)) != FDLLM_OK) return st;
  if (!(rope_base > 0.f)) return FDLLM_ERR_INVALID_ARG;
  const Layout L = step_layout(B, N, D, H, dh, R, S_max, 1, dtype);
  if ((st = check_ws(workspace, workspace_bytes, L.total)) != FDLLM_OK) return st;
  if (B * R == 0) return FDLLM_OK;
  if (!all_aligned({x_rows, pos, view, w_qkv, k_cache, v_cache, q_out}))
    return FDLLM_ERR_INVALID_ARG;
  if (S_max > 0 && !all_aligned({k_side, v_side})) return FDLLM_ERR_INVALID_ARG;
  return run_proj(B, N, D, H, dh, R, S_max, 1, dtype, x_rows, pos, view, w_qkv, rope_base,
                  k_cache, v_cache, k_side, v_side, q_out, workspace, L,
                  static_cast<cudaStream_t>(stream));
}

fdllm_status fdllm_verify_attend(int B, int N, int H, int dh, int R, int S_max, int dtype,
                                 const void* q, const int32_t* pos, const int8_t* view,
                                 const int32_t* rank, const void* k_cache, const void* v_cache,
                                 const void* k_side, const void* v_side, void* out,
                                 int causal_cross, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  NvtxRange nvtx_range("fdllm_verify_attend");
  fdllm_status st = check_shape(B, N, 64, H, dh, R, dtype);
  if (st != FDLLM_OK) return st;
  if ((st = check_verify_extra(R, S_max, causal_cross)) != FDLLM_OK) return st;
  const Layout L = step_layout(B, N, 64, H, dh, R, S_max, 1, dtype);
  if ((st = check_ws(workspace, workspace_bytes, L.attn_off + L.attn_bytes)) != FDLLM_OK)
    return st;
  if (B * R == 0) return FDLLM_OK;
  if (!all_aligned({q, pos, view, rank, k_cache, v_cache, out})) return FDLLM_ERR_INVALID_ARG;
  if (S_max > 0 && !all_aligned({k_side, v_side})) return FDLLM_ERR_INVALID_ARG;
  return run_attn(B, N, H, dh, R, S_max, 1, causal_cross, dtype, q, pos, view, rank, k_cache,
                  v_cache, k_side, v_side, out, workspace, L, static_cast<cudaStream_t>(stream));
}

fdllm_status fdllm_verify_step(int B, int N, int D, int H, int dh, int R, int S_max, int dtype,
                               const void* x_rows, const int32_t* pos, const int8_t* view,
                               const int32_t* rank, const void* w_qkv, float rope_base,
                               void* k_cache, void* v_cache, void* k_side, void* v_side,
                               void* out, int causal_cross, void* workspace,
                               size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("fdllm_verify_step");
  fdllm_status st = check_shape(B, N, D, H, dh, R, dtype);
  if (st != FDLLM_OK) return st;
  if ((st = check_verify_extra(R, S_max, causal_cross)) != FDLLM_OK) return st;
  if (!(rope_base > 0.f)) return FDLLM_ERR_INVALID_ARG;
  const Layout L = step_layout(B, N, D, H, dh, R, S_max, 1, dtype);
  if ((st = check_ws(workspace, workspace_bytes, L.total)) != FDLLM_OK) return st;
  if (B * R == 0) return FDLLM_OK;
  if (!all_aligned({x_rows, pos, view, rank, w_qkv, k_cache, v_cache, out}))
    return FDLLM_ERR_INVALID_ARG;
  if (S_max > 0 && !all_aligned({k_side, v_side})) return FDLLM_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* q = ws_at(workspace, L.q_off);
  st = run_proj(B, N, D, H, dh, R, S_max, 1, dtype, x_rows, pos, view, w_qkv, rope_base, k_cache,
                v_cache, k_side, v_side, q, workspace, L, s);
  if (st != FDLLM_OK) return st;
  return run_attn(B, N, H, dh, R, S_max, 1, causal_cross, dtype, q, pos, view, rank, k_cache,
                  v_cache, k_side, v_side, out, workspace, L, s);
}

fdllm_status fdllm_accept(int B, int R, int V, const float* logits, const int8_t* kind,
                          const int32_t* ref_tok, const int32_t* rank, float eps, float gamma,
                          int32_t* top1, float* conf, uint8_t* flags, int32_t* n_accept,
                          void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("fdllm_accept");
  if (B < 0 || R < 0 || V < 1) return FDLLM_ERR_INVALID_ARG;
  if ((long long)B * R > (1ll << 31) - 1 || (long long)B * R * V > (1ll << 40))
    return FDLLM_ERR_UNSUPPORTED;
  fdllm_status st = check_ws(workspace, workspace_bytes, fdllm_accept_workspace_bytes(B, R, V));
  if (st != FDLLM_OK) return st;
  if (B * R == 0) return FDLLM_OK;
  if (!all_aligned({logits, kind, top1, conf, flags, n_accept})) return FDLLM_ERR_INVALID_ARG;
  if ((ref_tok && !aligned16(ref_tok)) || (rank && !aligned16(rank)))
    return FDLLM_ERR_INVALID_ARG;
  // kind-2 rows need ref_tok and rank; the kernel reads them only for such rows
  const AcceptLayout AL = accept_layout(B, R, V, device_sm_count());
  AcceptArgs a{};
  a.B = B; a.R = R; a.V = V;
  a.logits = logits; a.kind = kind; a.ref_tok = ref_tok; a.rank = rank;
  a.eps = eps; a.gamma = gamma;
  a.top1 = top1; a.conf = conf; a.flags = flags; a.n_accept = n_accept;
  size_t off = kWsHeaderBytes;
  a.parts = reinterpret_cast<AcceptPartial*>(ws_at(workspace, off));
  off += AL.parts_bytes;
  a.row_cnt = reinterpret_cast<unsigned*>(ws_at(workspace, off));
  off += AL.row_cnt_bytes;
  a.seq_cnt = reinterpret_cast<unsigned*>(ws_at(workspace, off));
  return from_cuda(launch_accept(a, AL, static_cast<cudaStream_t>(stream)));
}

fdllm_status fdllm_track_select(int B, int N, int H, int dh, int nq, int dtype,
                                const int8_t* q_masked, const int8_t* candidate,
                                const void* k_cache, int beta_t, int32_t* track, float* mass,
                                void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("fdllm_track_select");
  fdllm_status st = check_shape(B, N, 64, H, dh, nq, dtype);
  if (st != FDLLM_OK) return st;
  if (beta_t < 1 || beta_t > kMaxBetaT) return FDLLM_ERR_UNSUPPORTED;
  // the regions it reads and uses sit before the D-dependent projection region
  const Layout L = step_layout(B, N, 64, H, dh, nq, 0, 0, dtype);
  if ((st = check_ws(workspace, workspace_bytes, L.track_off + L.track_bytes)) != FDLLM_OK)
    return st;
  if (B == 0) return FDLLM_OK;
  if (!all_aligned({q_masked, candidate, k_cache, track})) return FDLLM_ERR_INVALID_ARG;
  if (mass && !aligned16(mass)) return FDLLM_ERR_INVALID_ARG;
  TrackArgs a{};
  a.B = B; a.N = N; a.H = H; a.dh = dh; a.nq = nq; a.dtype = dtype; a.beta_t = beta_t;
  a.q = ws_at(workspace, L.q_off);
  a.lse = reinterpret_cast<const float*>(ws_at(workspace, L.lse_off));
  a.q_masked = q_masked; a.candidate = candidate; a.k_cache = k_cache; a.track = track;
  a.mass_h = reinterpret_cast<float*>(ws_at(workspace, L.track_off));
  a.mass = mass ? mass
                : reinterpret_cast<float*>(ws_at(
                      workspace, L.track_off + align_up((size_t)B * H * N * sizeof(float), 256)));
  return from_cuda(launch_track(a, static_cast<cudaStream_t>(stream)));
}

int fdllm_attention_split(int B, int N, int H, int dh, int rows, int S_max, int verify,
                          int* cluster_size) {
  int cs = 0;
  int mode = -1;
  if (check_shape(B, N, 64, H, dh, rows, FDLLM_BF16) == FDLLM_OK && (verify == 0 || verify == 1) &&
      S_max >= 0 && !(verify && rows > kMaxVerifyRows))
    mode = attn_tc_split(B, N, H, dh, rows, verify ? S_max : 0, verify, &cs);
  if (cluster_size) *cluster_size = mode == 3 ? cs : 0;
  return mode;
}

fdllm_status fdllm_bounded_wait_selftest(uint64_t limit_ns, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  if (limit_ns < 1000 || limit_ns > kWaitLimitNs) return FDLLM_ERR_INVALID_ARG;
  fdllm_status st = check_ws(workspace, workspace_bytes, kWsHeaderBytes + 32);
  if (st != FDLLM_OK) return st;
  return from_cuda(launch_bounded_wait_selftest(
      reinterpret_cast<int*>(workspace), limit_ns,
      reinterpret_cast<unsigned long long*>(ws_at(workspace, kWsHeaderBytes)),
      static_cast<cudaStream_t>(stream)));
}

fdllm_status fdllm_get_status(void* workspace, void* stream) {
  if (!workspace) return FDLLM_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return FDLLM_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return FDLLM_ERR_CUDA;
  if (v != 0 && cudaMemset(workspace, 0, sizeof(int)) != cudaSuccess) return FDLLM_ERR_CUDA;
  return static_cast<fdllm_status>(v);
}

}  // extern "C"
