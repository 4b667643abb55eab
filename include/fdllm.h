/*
 * fdllm.h - C ABI of the Flash-dLLM fused KV-cache step on NVIDIA B200 (sm_100a).
 *
 * What the calls compute.  Passages are cited by page title and section:
 *   [review]  "Flash-dLLM: IO-Aware KV Caching and Parallel Decoding for Fast,
 *             Memory-Efficient Diffusion LLMs" (jaehun.me review of arXiv 2609.26796)
 *   [summary] "Flash-dLLM: IO-Aware KV Caching and Parallel Decoding for Fast
 *             Diffusion LLMs" (alanhou.org summary), "Core Mechanism"
 *
 *   fdllm_fused_step   one step of the IO-aware fused KV-cache kernel
 *                      ([review] "How It Works", Step 1: Draft, Alg. 1): read only
 *                      the hidden rows x[Q], build q,k,v, rotate q,k (RoPE) at their
 *                      cache slots, write k,v into the cache at exactly Q, then
 *                      attend every query over the whole (bidirectional) cache.
 *   fdllm_verify_step  the Flash-Verify pass ([review] "Flash-Verify", sec. 2.3,
 *                      Fig. 2; "How It Works", Step 1: Verification): rows
 *                      [T_v | draft view of S | mask view of S]; the two views share
 *                      positions (RoPE) while each is hidden from the other.
 *   fdllm_accept       per-row top-1 and confidence, the epsilon split D_t / S_t
 *                      and the gamma prefix acceptance up to the first mismatch
 *                      ([review] "Flash-Verify", sec. 2.3 and the worked example).
 *   fdllm_track_select the tracked set of the next step: the decoded slots the
 *                      masked queries attend to most ([review] "How It Works",
 *                      Step 1: Cache selection).
 *
 * Conventions shared by every call
 *   - Every pointer argument is a DEVICE pointer owned by the caller, unless
 *     stated otherwise; the library allocates no device memory and keeps no
 *     per-call state between calls.  `stream` is a cudaStream_t (NULL = legacy
 *     default stream).  Calls are asynchronous on `stream`.
 *   - Kernels launch on the calling thread's current CUDA device; every pointer
 *     and `stream` must belong to that device.
 *   - The return value reports host-side validation and launch errors only.
 *     Errors the GPU detects (an index out of range, a bounded wait that ran
 *     out) are recorded in a status word inside `workspace`; read them with
 *     fdllm_get_status after the work has run.
 *   - Layouts are dense, row-major, with the last dimension contiguous:
 *       x        [B, N, D]        hidden states of every cache slot (only the
 *                                 rows at Q are read)
 *       x_rows   [B, R, D]        packed verify rows
 *       w_qkv    [3*H*dh, D]      rows: the q block, then k, then v; head-major
 *                                 inside each block (no bias)
 *       k_cache,
 *       v_cache  [B, H, N, dh]    the flat preallocated cache of one layer
 *       k_side,
 *       v_side   [B, H, S_max, dh] mask-view keys/values of a verify pass
 *       q        [B, nq, H, dh]   rotated queries (stage calls only)
 *       out      [B, nq, H*dh]    attention output, in the storage dtype
 *   - dtype: FDLLM_BF16 (bf16 storage, fp32 accumulation, tensor cores) or
 *     FDLLM_F32 (fp32 storage and arithmetic).  Supported: dh in {64, 128};
 *     D a multiple of 64 (bf16) or of 4 (fp32); every pointer 16-byte aligned.
 *     Anything else returns FDLLM_ERR_UNSUPPORTED or FDLLM_ERR_INVALID_ARG.
 *   - RoPE (the pages fix only that the views share position embeddings): pairs
 *     (j, j+dh/2) are turned by pos * rope_base^(-2j/dh), pos = the cache slot.
 *     Attention scale is 1/sqrt(dh).
 *   - workspace: device scratch of at least the size the matching
 *     *_workspace_bytes function returns, 256-byte aligned, ZERO-FILLED before
 *     its first use.  Every call leaves its counters at zero again, so one
 *     zeroed workspace serves any number of later calls on ONE stream.  Calls
 *     that overlap on the GPU must not share a workspace.  After an
 *     FDLLM_ERR_TIMEOUT, zero the workspace again before reusing it.
 */
#ifndef FDLLM_H_
#define FDLLM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FDLLM_OK = 0,
  FDLLM_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer */
  FDLLM_ERR_UNSUPPORTED = 2,   /* shape or dtype outside the supported set */
  FDLLM_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
  FDLLM_ERR_BAD_INDEX = 4,     /* device: a position outside [0, N) or a side slot beyond S_max */
  FDLLM_ERR_TIMEOUT = 5,       /* device: a bounded wait inside a kernel ran out */
  FDLLM_ERR_WORKSPACE = 6      /* workspace too small or misaligned */
} fdllm_status;

typedef enum { FDLLM_F32 = 0, FDLLM_BF16 = 1 } fdllm_dtype;

/* fdllm_accept flag bits (one byte per row). */
#define FDLLM_FLAG_COMMIT 1u /* kind 1 row with confidence >= eps: joins D_t */
#define FDLLM_FLAG_ACCEPT 2u /* kind 2 row accepted by the gamma prefix rule */
#define FDLLM_FLAG_PASS 4u   /* kind 2 row whose own test passed */

/* Library version, major*10000 + minor*100 + patch. */
int fdllm_version(void);

/* Human-readable name of a status code (static storage). */
const char* fdllm_status_string(fdllm_status s);

/* Workspace sizes in bytes for the three operations and their stage calls.
 * They depend on the shapes and on the current device's SM count.  Return 0
 * for unsupported arguments. */
size_t fdllm_fused_step_workspace_bytes(int B, int N, int D, int H, int dh, int nq, int dtype);
size_t fdllm_verify_step_workspace_bytes(int B, int N, int D, int H, int dh, int R, int S_max,
                                         int dtype);
size_t fdllm_accept_workspace_bytes(int B, int R, int V);

/* One fused KV-cache step ([review] "How It Works", Step 1: Draft, Alg. 1).
 *   q_idx [B, nq] int32: the query set Q = T u M^{beta_m} of each sequence
 *   ([review] "Flash-Verify": Q_t = T_t u M_t^{beta_m}); slots within [0, N),
 *   distinct within a row, any order.  An index outside [0, N) sets
 *   FDLLM_ERR_BAD_INDEX in the status word and that row is skipped (nothing is
 *   written for it).  A repeated index also sets FDLLM_ERR_BAD_INDEX (both rows
 *   write the same slot; which write lands is undefined); bf16 only, the fp32
 *   path does not check.
 *   k_cache / v_cache are read and written in place: only the slots in Q
 *   change.  x must not alias any buffer the call writes.
 *   out [B, nq, H*dh]: row i is the attention output of query q_idx[b, i]. */
fdllm_status fdllm_fused_step(int B, int N, int D, int H, int dh, int nq, int dtype,
                              const void* x, const int32_t* q_idx, const void* w_qkv,
                              float rope_base, void* k_cache, void* v_cache, void* out,
                              void* workspace, size_t workspace_bytes, void* stream);

/* fdllm_fused_step for a caller that holds only the rows the step reads: x_rows
 * [B, nq, D], row i of sequence b being the hidden state of slot q_idx[b, i]
 * (what a layer of the same decode step produces, since only the rows of Q are
 * recomputed).  Everything else, the workspace and the results are those of
 * fdllm_fused_step; both give the same bits.  A repeated or out-of-range index
 * sets FDLLM_ERR_BAD_INDEX (repeats: bf16 only). */
fdllm_status fdllm_fused_step_rows(int B, int N, int D, int H, int dh, int nq, int dtype,
                                   const void* x_rows, const int32_t* q_idx, const void* w_qkv,
                                   float rope_base, void* k_cache, void* v_cache, void* out,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* Stage 1 of fdllm_fused_step: gather x[Q], project, rotate, write k,v into the
 * cache and the rotated queries into q_out [B, nq, H, dh] (storage dtype). */
fdllm_status fdllm_qkv_rope_scatter(int B, int N, int D, int H, int dh, int nq, int dtype,
                                    const void* x, const int32_t* q_idx, const void* w_qkv,
                                    float rope_base, void* k_cache, void* v_cache, void* q_out,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* Stage 2 of fdllm_fused_step: out = softmax(q K^T / sqrt(dh)) V over all N
 * slots of each sequence's cache, q [B, nq, H, dh].  The workspace is the one
 * sized by fdllm_fused_step_workspace_bytes. */
fdllm_status fdllm_attend(int B, int N, int H, int dh, int nq, int dtype, const void* q,
                          const void* k_cache, const void* v_cache, void* out, void* workspace,
                          size_t workspace_bytes, void* stream);

/* One Flash-Verify pass ([review] "Flash-Verify", sec. 2.3, Fig. 2).
 *   x_rows [B, R, D]; pos, rank [B, R] int32; view [B, R] int8:
 *     view 0 = tracked row (T_v), 1 = draft view of an S position,
 *     2 = mask view of an S position (its draft twin has the same pos).
 *   Rows of view 0 and 1 write their k,v into the cache at pos; rows of view 2
 *   write theirs into side slots 0, 1, ... in row order (at most S_max of them),
 *   so the cache never holds mask-view keys.  Visibility:
 *     view 0/1 rows: every cache slot, no side slot;
 *     view 2 rows, causal_cross = 0 (the two views mutually hidden, the default):
 *       every cache slot except the draft-view positions, and every side slot;
 *     view 2 rows, causal_cross = 1 (reading of [review] Appx. C, Remark 1):
 *       the draft key at a position of smaller rank and the mask key at a
 *       position of equal or larger rank.
 *   rank is the decoding order of S (shared by the two views); ignored for
 *   view 0.  Positions must be distinct among view 0/1 rows. */
fdllm_status fdllm_verify_step(int B, int N, int D, int H, int dh, int R, int S_max, int dtype,
                               const void* x_rows, const int32_t* pos, const int8_t* view,
                               const int32_t* rank, const void* w_qkv, float rope_base,
                               void* k_cache, void* v_cache, void* k_side, void* v_side,
                               void* out, int causal_cross, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Stage 1 of fdllm_verify_step (projection, RoPE, cache and side writes). */
fdllm_status fdllm_verify_qkv_rope_scatter(int B, int N, int D, int H, int dh, int R, int S_max,
                                           int dtype, const void* x_rows, const int32_t* pos,
                                           const int8_t* view, const void* w_qkv,
                                           float rope_base, void* k_cache, void* v_cache,
                                           void* k_side, void* v_side, void* q_out,
                                           void* workspace, size_t workspace_bytes,
                                           void* stream);

/* Stage 2 of fdllm_verify_step (view-masked attention), q [B, R, H, dh]. */
fdllm_status fdllm_verify_attend(int B, int N, int H, int dh, int R, int S_max, int dtype,
                                 const void* q, const int32_t* pos, const int8_t* view,
                                 const int32_t* rank, const void* k_cache, const void* v_cache,
                                 const void* k_side, const void* v_side, void* out,
                                 int causal_cross, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* Top-1, confidence, epsilon split and gamma prefix acceptance
 * ([review] "Flash-Verify", sec. 2.3; "How It Works", Step 1).
 *   logits [B, R, V] fp32; kind, ref_tok, rank [B, R]:
 *     kind 0: top-1 and confidence only;
 *     kind 1: draft-pass masked row: FDLLM_FLAG_COMMIT iff conf >= eps;
 *     kind 2: mask-view row: FDLLM_FLAG_PASS iff top1 == ref_tok (the draft
 *             token) and conf >= gamma; rows are taken in ascending rank and
 *             accepted up to the first that does not pass (FDLLM_FLAG_ACCEPT).
 *   top1 [B, R] int32: the lowest index of the largest logit;
 *   conf [B, R] fp32: the largest softmax probability, 1 / sum_v exp(l_v - max);
 *   flags [B, R] uint8; n_accept [B] int32: number of accepted kind-2 rows.
 *   ref_tok / rank may be NULL when no row is of kind 2. */
fdllm_status fdllm_accept(int B, int R, int V, const float* logits, const int8_t* kind,
                          const int32_t* ref_tok, const int32_t* rank, float eps, float gamma,
                          int32_t* top1, float* conf, uint8_t* flags, int32_t* n_accept,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Size of the device array that fdllm_accept_noalloc uses as its scratch. */
#define FDLLM_ACCEPT_NOALLOC_SCRATCH_BYTES (4u << 20)

/* fdllm_accept without a workspace.  The paper has no counterpart: this entry
 * point exists for callers that cannot allocate device memory where they call
 * the library, e.g. a plugin that its host hands only the input and output
 * buffers, a runtime that reserved all device memory for its own pool up front,
 * or a latency-critical loop where a cudaMalloc would synchronise the device.
 *   Arguments and results are those of fdllm_accept (same kernel, same rows),
 *   minus the workspace.  The call allocates nothing (no cudaMalloc, no
 *   cudaFree, no allocating library routine).  Its scratch is a device array of
 *   FDLLM_ACCEPT_NOALLOC_SCRATCH_BYTES compiled into the library: every GPU that
 *   loads the library holds it until the process exits.  A call needs at most
 *   align256(16*(B*R + 8*SMs)) + align256(4*B*R) + align256(4*B) bytes of it
 *   (the row partials of the scan, then per-row and per-sequence counters);
 *   B*R <= 131072 always fits on GPUs of up to 256 SMs, and a call that does not
 *   fit returns FDLLM_ERR_UNSUPPORTED without launching anything.
 *   Every call on a device shares the one array, which keeps the last call's
 *   contents; each call first clears (cudaMemsetAsync on `stream`) the counters
 *   that must start at zero.  Calls that overlap on the GPU (on different
 *   streams, or from several threads) race on the array: order them.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.  The address is kept per device and per
 *   context: a call made after cudaDeviceReset (or a primary-context reset),
 *   or with another context current, looks it up again, since the array then
 *   lives at a new address; the array's contents do not survive a reset. */
fdllm_status fdllm_accept_noalloc(int B, int R, int V, const float* logits, const int8_t* kind,
                                  const int32_t* ref_tok, const int32_t* rank, float eps,
                                  float gamma, int32_t* top1, float* conf, uint8_t* flags,
                                  int32_t* n_accept, void* stream);

/* Largest tracked-set size fdllm_track_select accepts. */
#define FDLLM_MAX_BETA_T 1024

/* The tracked set of the next step ([review] "How It Works", Step 1: Cache
 * selection): the beta_t decoded cache slots that the step's masked queries
 * attend to most.
 *   Call it after fdllm_fused_step (or fdllm_qkv_rope_scatter followed by
 *   fdllm_attend) on the SAME workspace, with the same B, N, H, dh, nq, dtype,
 *   and before that workspace is used again: it reads the rotated queries and
 *   the per-row softmax normalisers the step left there.  k_cache is the cache
 *   as that step left it.
 *   Attention mass: a[b, j] = sum over the rows i of Q with q_masked[b, i] != 0
 *   (the masked queries M^{beta_m}) and over the heads h of the step's softmax
 *   probability p_ihj (taken over all N slots).
 *   q_masked   int8 [B, nq]    1 = masked-query row, 0 = tracked row
 *   candidate  int8 [B, N]     1 = decoded slot (the slots decoded in this
 *                              step included: they are ranked with the rest)
 *   beta_t     1..FDLLM_MAX_BETA_T
 *   track      int32 [B, beta_t] out: the candidates with the largest mass,
 *              mass descending, equal mass to the lower slot; -1 past the
 *              number of candidates
 *   mass       float [B, N] out, may be NULL: a[b, j] for every slot
 *   Deterministic: the heads are summed in order and the selection is exact
 *   on the fp32 masses.  Returns FDLLM_ERR_UNSUPPORTED for beta_t out of range;
 *   FDLLM_ERR_WORKSPACE when the workspace is smaller than the fused step's. */
fdllm_status fdllm_track_select(int B, int N, int H, int dh, int nq, int dtype,
                                const int8_t* q_masked, const int8_t* candidate,
                                const void* k_cache, int beta_t, int32_t* track, float* mass,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Diagnostic: how the bf16 attention of a step with these shapes spreads its
 * work over the current device's SMs (the choice depends only on the shapes and
 * the device).  rows = nq (fused step) or R (verify pass, verify = 1).
 *   1  persistent stream-K: one CTA per SM, each an equal contiguous range of
 *      (item, 128-key tile) units; an item split between CTAs is merged by its
 *      last contributor;
 *   2  one CTA per whole (sequence, head, query chunk) item, no merge;
 *   3  a thread-block cluster per item, merged through distributed shared
 *      memory; *cluster_size (host pointer, may be NULL) gets its CTA count.
 *  -1  shapes the bf16 attention does not run.
 * Launches nothing and allocates nothing. */
int fdllm_attention_split(int B, int N, int H, int dh, int rows, int S_max, int verify,
                          int* cluster_size);

/* Diagnostic: runs the bounded wait that every kernel of this library uses on
 * its mbarriers, against an mbarrier that nothing completes, so that its
 * timeout path can be checked without a fault or a hang.  One CTA: one thread
 * waits with limit_ns (1 us .. 2 s, the kernels' own limit; else
 * FDLLM_ERR_INVALID_ARG) and must give up, recording FDLLM_ERR_TIMEOUT in the
 * status word; a second thread then waits on the same barrier and must return
 * at once, as every later wait of a kernel does after a timeout.
 *   workspace: >= 288 bytes, 256-byte aligned, status word zero.  Results at
 *   byte 256, four uint64: first wait completed (0/1), its duration in ns,
 *   second wait completed (0/1), its duration in ns.
 * Read the status with fdllm_get_status; zero the workspace before reusing it. */
fdllm_status fdllm_bounded_wait_selftest(uint64_t limit_ns, void* workspace,
                                         size_t workspace_bytes, void* stream);

/* Number of kernels this library has launched in this process (a diagnostic
 * counter, incremented on the host at every launch; never reset). */
uint64_t fdllm_launch_count(void);

/* Synchronises `stream`, returns the device status word of `workspace`
 * (FDLLM_OK when no error was recorded) and clears it. */
fdllm_status fdllm_get_status(void* workspace, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FDLLM_H_ */
