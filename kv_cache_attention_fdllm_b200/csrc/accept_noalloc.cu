// fdllm_accept_noalloc: the acceptance reduction without a caller workspace.
//
// Some host programs cannot allocate device memory at the point where they
// call this library: a plugin that an inference server hands only its input
// and output buffers, a runtime that reserved all device memory up front for
// its own pool, or a latency-critical loop where a cudaMalloc would
// synchronise the device.  For them this entry point keeps the reduction's
// scratch (per-split partials and the last-arriver counters) in a fixed
// device array compiled into the library, so the call allocates nothing.
//
// The array is file-scope and static: every GPU that loads the library holds
// it until the process exits.  Host code only sees a host-side stand-in under
// its name, so the device address is looked up with cudaGetSymbolAddress, with
// the device current, once per device and context (the first call there), and
// that address is what the kernel receives.  The lookup is keyed on the
// current context's unique id: after a cudaDeviceReset, or with another
// context current on the same device, the module is loaded anew at another
// address, and the next call looks it up again.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = FDLLM_ACCEPT_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_accept_scratch[kScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct DriverFns {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

const DriverFns& driver_fns() {
  static DriverFns f;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  return f;
}

// Unique id of the calling thread's current context, 0 when there is none yet.
unsigned long long current_context_id() {
  const DriverFns& f = driver_fns();
  if (!f.get_current || !f.get_id) return 0;
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  return f.get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

struct ScratchAddr {
  unsigned long long ctx_id;  // context the address belongs to (0: none cached)
  void* ptr;
};

std::mutex g_scratch_mu;
ScratchAddr g_scratch[kMaxDevices];  // device address of g_accept_scratch, per device

// Device address of the scratch array in the current context (set-up on the
// first call on each device and context).
fdllm_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FDLLM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FDLLM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long id = current_context_id();
  if (id == 0 || g_scratch[dev].ctx_id != id || !g_scratch[dev].ptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_accept_scratch);
    if (e != cudaSuccess || p == nullptr) return FDLLM_ERR_CUDA;
    // the lookup made the device's primary context current if none was
    g_scratch[dev].ctx_id = current_context_id();
    g_scratch[dev].ptr = p;
  }
  *out = g_scratch[dev].ptr;
  return FDLLM_OK;
}

bool is_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" fdllm_status fdllm_accept_noalloc(int B, int R, int V, const float* logits,
                                             const int8_t* kind, const int32_t* ref_tok,
                                             const int32_t* rank, float eps, float gamma,
                                             int32_t* top1, float* conf, uint8_t* flags,
                                             int32_t* n_accept, void* stream) {
  using namespace fdllm;
  if (B < 0 || R < 0 || V < 1) return FDLLM_ERR_INVALID_ARG;
  if ((long long)B * R > (1ll << 31) - 1 || (long long)B * R * V > (1ll << 40))
    return FDLLM_ERR_UNSUPPORTED;
  const int rows = B * R;
  const AcceptLayout AL = accept_layout(B, R, V, device_sm_count());
  // scratch layout: [partials | per-row counters | per-sequence counters]
  if (AL.total() > kScratchBytes) return FDLLM_ERR_UNSUPPORTED;
  if (rows == 0) return FDLLM_OK;
  if (!logits || !kind || !top1 || !conf || !flags || !n_accept) return FDLLM_ERR_INVALID_ARG;
  if (!is_aligned16(logits) || !is_aligned16(kind) || !is_aligned16(top1) ||
      !is_aligned16(conf) || !is_aligned16(flags) || !is_aligned16(n_accept))
    return FDLLM_ERR_INVALID_ARG;
  if ((ref_tok && !is_aligned16(ref_tok)) || (rank && !is_aligned16(rank)))
    return FDLLM_ERR_INVALID_ARG;

  void* base = nullptr;
  fdllm_status st = scratch_address(&base);
  if (st != FDLLM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* p = static_cast<char*>(base);
  // the counters must start at zero; the array keeps whatever the last call left
  if (cudaMemsetAsync(p + AL.parts_bytes, 0, AL.row_cnt_bytes + AL.seq_cnt_bytes,
                      s) != cudaSuccess)
    return FDLLM_ERR_CUDA;

  AcceptArgs a{};
  a.B = B; a.R = R; a.V = V;
  a.logits = logits; a.kind = kind; a.ref_tok = ref_tok; a.rank = rank;
  a.eps = eps; a.gamma = gamma;
  a.top1 = top1; a.conf = conf; a.flags = flags; a.n_accept = n_accept;
  a.parts = reinterpret_cast<AcceptPartial*>(p);
  a.row_cnt = reinterpret_cast<unsigned*>(p + AL.parts_bytes);
  a.seq_cnt = reinterpret_cast<unsigned*>(p + AL.parts_bytes + AL.row_cnt_bytes);
  return launch_accept(a, AL, s) == cudaSuccess ? FDLLM_OK : FDLLM_ERR_CUDA;
}
