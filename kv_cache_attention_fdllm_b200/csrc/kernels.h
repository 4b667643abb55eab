// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace fdllm {

// ----------------------------------------------------------------- acceptance
struct AcceptPartial {
  float m;
  float l;
  int idx;
  int pad;
};

struct AcceptArgs {
  int B, R, V;
  const float* logits;
  const int8_t* kind;
  const int32_t* ref_tok;
  const int32_t* rank;
  float eps, gamma;
  int32_t* top1;
  float* conf;
  uint8_t* flags;
  int32_t* n_accept;
  AcceptPartial* parts;  // layout.parts_bytes
  unsigned* row_cnt;     // [B*R], zero between calls
  unsigned* seq_cnt;     // [B], zero between calls
};

// How the acceptance scan is split (grid rows x splits, each CTA one span of
// one row), and the scratch it needs.
struct AcceptLayout {
  int splits;
  size_t parts_bytes, row_cnt_bytes, seq_cnt_bytes;
  size_t total() const { return parts_bytes + row_cnt_bytes + seq_cnt_bytes; }
};
AcceptLayout accept_layout(int B, int R, int V, int num_sms);
cudaError_t launch_accept(const AcceptArgs& a, const AcceptLayout& L, cudaStream_t stream);

// ----------------------------------------------------------------- projection
// Rows of the projection: token m of sequence b = m / rows_per_seq.
//   fused  (verify == 0): RoPE position and cache slot q_idx[m]; the input row
//                         is x row (b, q_idx[m]), or row m when packed.
//   verify (verify == 1): x_rows row m (always packed); position pos[m]; view[m]
//                         chooses the destination (0/1: cache slot pos[m]; 2: side slot).
struct ProjArgs {
  int B, N, D, H, dh, rows_per_seq, S_max, verify, dtype;
  int packed;              // x holds the rows themselves, [B, rows, D]
  const void* x;           // gathered: [B, N, D]; packed: [B, rows, D]
  const int32_t* idx;      // fused: q_idx [B, nq]; verify: pos [B, R]
  const int8_t* view;      // verify only
  const void* w;           // [3E, D]
  double log2_base;
  void* k_cache;
  void* v_cache;
  void* k_side;
  void* v_side;
  void* q_out;             // [B, rows, H, dh]
  int* status;
  void* ws;                // kernel scratch
  size_t ws_bytes;
};

size_t proj_workspace_bytes(int M, int D, int H, int dh, int dtype, int num_sms);
cudaError_t launch_proj(const ProjArgs& a, cudaStream_t stream);

// ----------------------------------------------------------------- attention
struct AttnArgs {
  int B, N, H, dh, rows_per_seq, S_max, verify, causal_cross, dtype;
  const void* q;           // [B, rows, H, dh]
  const void* k_cache;
  const void* v_cache;
  const void* k_side;
  const void* v_side;
  const int32_t* pos;      // verify only
  const int8_t* view;      // verify only
  const int32_t* rank;     // verify only
  void* out;               // [B, rows, H*dh]
  float* lse;              // [B, rows, H]: log2 of the softmax denominator of the
                           // scaled scores s * log2(e) / sqrt(dh); may be null
  int* status;
  void* ws;
  size_t ws_bytes;
};

size_t attn_workspace_bytes(int B, int N, int H, int dh, int rows_per_seq, int S_max, int verify,
                            int dtype, int num_sms);
cudaError_t launch_attn(const AttnArgs& a, cudaStream_t stream);

// ----------------------------------------------------------------- tracked-set selection
constexpr int kMaxBetaT = FDLLM_MAX_BETA_T;

struct TrackArgs {
  int B, N, H, dh, nq, dtype, beta_t;
  const void* q;            // [B, nq, H, dh], staged by the step
  const float* lse;         // [B, nq, H], left by the step's attention
  const int8_t* q_masked;   // [B, nq]: 1 = masked-query row
  const int8_t* candidate;  // [B, N]: 1 = decoded slot
  const void* k_cache;      // [B, H, N, dh]
  int32_t* track;           // [B, beta_t]
  float* mass;              // [B, N]
  float* mass_h;            // [B, H, N] scratch
};

size_t track_workspace_bytes(int B, int N, int H);
cudaError_t launch_track(const TrackArgs& a, cudaStream_t stream);

// ----------------------------------------------------------------- kernel families
size_t proj_simt_workspace_bytes(int M, int H, int dh);
size_t proj_tc_workspace_bytes(int M, int D, int H, int dh, int num_sms);
cudaError_t launch_proj_tc(const ProjArgs& a, cudaStream_t stream);
// bf16 projections of at least kPairMinRows rows run on CTA pairs.  Below it W
// is the whole cost and the single-CTA kernel spreads it over every SM, where
// the pairs' whole tiles leave SMs idle.
constexpr int kPairMinRows = 128;
size_t proj_pair_workspace_bytes(int M, int D, int H, int dh, int num_sms);
cudaError_t launch_proj_pair(const ProjArgs& a, cudaStream_t stream);
// packs x[Q] (rows b, q_idx[m] of x) into xq [M, D] for the fused step
cudaError_t launch_proj_prep(const ProjArgs& a, __nv_bfloat16* xq, cudaStream_t stream);
cudaError_t launch_proj_simt(const ProjArgs& a, cudaStream_t stream);
cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t stream);
size_t attn_tc_workspace_bytes(int B, int N, int H, int dh, int rows, int S_max, int verify,
                               int num_sms);
cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t stream);
// The work split launch_attn_tc takes for these shapes on the current device:
// 1 persistent stream-K, 2 one CTA per whole item, 3 clusters of *cs CTAs per
// item; -1 for shapes it does not run.
int attn_tc_split(int B, int N, int H, int dh, int rows, int S_max, int verify, int* cs);

// ----------------------------------------------------------------- diagnostics
// result[0..3]: first wait completed (0/1), its ns; second wait completed, its ns
cudaError_t launch_bounded_wait_selftest(int* status, uint64_t limit_ns,
                                         unsigned long long* result, cudaStream_t stream);

// ----------------------------------------------------------------- helpers
int device_sm_count();
void count_launches(int n);
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace fdllm
