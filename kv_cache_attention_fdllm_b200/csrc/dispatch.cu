// Chooses the kernel family for each stage and sizes its scratch.
#include "common.cuh"
#include "kernels.h"

namespace fdllm {

size_t proj_workspace_bytes(int M, int D, int H, int dh, int dtype, int num_sms) {
  if (dtype == FDLLM_BF16) {
    // a workspace sized for more rows serves fewer: the larger of the two layouts
    const size_t tc = proj_tc_workspace_bytes(M < kPairMinRows ? M : kPairMinRows - 1, D, H, dh,
                                              num_sms);
    const size_t pair = M >= kPairMinRows ? proj_pair_workspace_bytes(M, D, H, dh, num_sms) : 0;
    return tc > pair ? tc : pair;
  }
  return proj_simt_workspace_bytes(M, H, dh);
}

cudaError_t launch_proj(const ProjArgs& a, cudaStream_t stream) {
  if (a.dtype == FDLLM_BF16) {
    if (a.B * a.rows_per_seq >= kPairMinRows) return launch_proj_pair(a, stream);
    return launch_proj_tc(a, stream);
  }
  return launch_proj_simt(a, stream);
}

size_t attn_workspace_bytes(int B, int N, int H, int dh, int rows_per_seq, int S_max, int verify,
                            int dtype, int num_sms) {
  if (dtype == FDLLM_BF16)
    return attn_tc_workspace_bytes(B, N, H, dh, rows_per_seq, S_max, verify, num_sms);
  return 0;
}

cudaError_t launch_attn(const AttnArgs& a, cudaStream_t stream) {
  if (a.dtype == FDLLM_BF16) return launch_attn_tc(a, stream);
  return launch_attn_simt(a, stream);
}

}  // namespace fdllm
