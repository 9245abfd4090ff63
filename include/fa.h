/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library.
 *
 * The library computes exact scaled-dot-product attention FlashAttention-style:
 *
 *   O = softmax(scale * Q K^T) V                        (forward)
 *   dQ, dK, dV = gradients of sum(dO * O)               (backward)
 *
 * Sources for the operations (page title, then section):
 *   - "FlashAttention为什么更快更省显存" (hi-bin.com lesson 16), opening formula:
 *     Attention(Q,K,V) = softmax(QK^T / sqrt(d_k)) V; section 把整张表改为分块计算:
 *     a Q block stays on chip while K/V blocks stream past; section
 *     反向传播为什么还要重算: the backward recomputes scores from Q, K, V and a
 *     few saved statistics.
 *   - "从零实现 FlashAttention-2：分块在线 Softmax", section 在线 softmax：重缩放恒等式:
 *     running max m and sum l per row, the output accumulator rescaled by
 *     exp(m_old - m_new), final O = O_final / l_final; section 反向传播：重算，
 *     而不是存储: the backward keeps only Q, K, V, O and per-row statistics;
 *     section 提示: the causal mask hides keys whose position is greater than
 *     the query's, applied inside the tile loop.
 *   - "FlashAttention 为什么能节省显存并提速,是否改变注意力结果?" (mianstack.com
 *     q-0277), section 难点在于分块后softmax如何归一: the (m, l, u) merge rule.
 *
 * Layout (all calls): Q, K, V, O, dO, dQ, dK, dV are bf16 tensors of shape
 * [B, H, N, d], row-major and contiguous (d innermost).  LSE is fp32 [B, H, N]:
 * the natural-log logsumexp of each row of scale * Q K^T over its unmasked
 * keys.  Query and key sequence lengths are equal (N).  d must be 64 or 128.
 * Causal masking keeps key j for query i iff j <= i.
 *
 * Ownership: the caller owns every buffer (device memory) and the stream.  The
 * library allocates no device memory at call time and never synchronises
 * except inside fa_check_device_error and fa_timing_end.  Calls are
 * asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 * stream).  Concurrent calls on different streams must use distinct output
 * and workspace buffers.
 *
 * Library-owned device state (static device arrays, part of the loaded
 * library, never allocated per call): the error word; the work counters of
 * the persistent kernels (16384 slots of 16 bytes: each launch takes the next
 * slot of a per-device sequence, the first CTA to ask for work in a launch
 * starts the slot's count afresh and the last CTA to finish clears it, so
 * concurrent launches and replays of a captured CUDA graph each count their
 * own work); and the scratch of fa_bwd_noalloc.
 *
 * Errors: arguments are checked before anything is launched; a failing check
 * returns its code and launches nothing.  A launch failure returns
 * FA_ERR_CUDA.  Every wait inside the kernels is bounded: a wait that runs out
 * makes the kernel record the fact in a device error word and return early;
 * fa_check_device_error reports it as FA_ERR_DEVICE_TIMEOUT.
 */
#ifndef EXACT_ATTENTION_B200_FA_H
#define EXACT_ATTENTION_B200_FA_H

#include <stddef.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_NULL = 1,            /* a required pointer is NULL                      */
  FA_ERR_SHAPE = 2,           /* B, H or N < 1, or a size overflows              */
  FA_ERR_UNSUPPORTED_D = 3,   /* d is not 64 or 128                              */
  FA_ERR_ALIGN = 4,           /* a tensor pointer is not 16-byte aligned         */
  FA_ERR_SCALE = 5,           /* scale is NaN or infinite                        */
  FA_ERR_WORKSPACE = 6,       /* workspace NULL or smaller than required         */
  FA_ERR_CUDA = 7,            /* a CUDA runtime call or launch failed            */
  FA_ERR_DEVICE_TIMEOUT = 8,  /* a kernel gave up on a bounded wait              */
  FA_ERR_STATE = 9            /* timing calls out of order                       */
} fa_status;

/*
 * Forward pass.
 *   q, k, v : bf16 [B, H, N, d] device pointers, 16-byte aligned, read only.
 *   o       : bf16 [B, H, N, d] output, 16-byte aligned.
 *   lse     : fp32 [B, H, N] output (natural log of the row sum of
 *             exp(scale * q_i . k_j) over unmasked keys j).
 *   causal  : 0 = every key, nonzero = keys j <= i only.
 *   scale   : any finite float (the usual value is 1/sqrt(d)).
 * Deterministic: the same inputs give bitwise the same outputs (each pair of
 * 128-row Q tiles is computed by one CTA in a fixed order, whichever CTA it
 * lands on).  One persistent CTA per SM takes the (head, Q-tile pair) work
 * items longest first from a per-launch counter.
 */
FA_API fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int N, int d, int causal, float scale, void* stream);

/*
 * Split-KV forward (page "FlashAttention 为什么能节省显存并提速,是否改变注意力结果?",
 * section 难点在于分块后softmax如何归一: per-block statistics are brought to a
 * common max and merged).  The key tiles are divided into num_splits
 * contiguous ranges; one launch computes, for every Q tile and range, the
 * normalised partial output and its logsumexp into the workspace, and a
 * second launch merges the ranges: M = max_s LSE_s, w_s = exp(LSE_s - M),
 * O = sum_s w_s O_s / sum_s w_s, LSE = M + ln sum_s w_s.  Same arguments,
 * layouts and results as fa_fwd (up to rounding), plus:
 *   num_splits : 1..64; ranges past the causal diagonal are skipped.  Useful
 *                when B * H * ceil(N / 256) CTAs would not fill the GPU.
 *   workspace  : device scratch of fa_fwd_splitkv_workspace_size bytes,
 *                16-byte aligned, contents on entry irrelevant.
 * Returns FA_ERR_SHAPE for num_splits out of range.
 */
FA_API size_t fa_fwd_splitkv_workspace_size(int B, int H, int N, int d, int num_splits);
FA_API fa_status fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int H, int N, int d, int causal, float scale,
                                int num_splits, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * Bytes of device workspace fa_bwd needs: an fp32 dQ accumulator of
 * B*H*Np*d floats (internal tile layout) plus two fp32 per-row vectors
 * [B, H, Np] (D = rowsum(dO * O) and the log2-domain LSE), with Np = N
 * rounded up to a multiple of 128.
 * Returns 0 if the arguments are invalid.
 */
FA_API size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward pass (recomputes the score tiles; no N x N tensor is stored).
 *   q, k, v, o, dout : bf16 [B, H, N, d] device pointers (o from fa_fwd).
 *   lse              : fp32 [B, H, N] from fa_fwd with the same causal/scale.
 *   dq, dk, dv       : bf16 [B, H, N, d] outputs.
 *   workspace        : device scratch of at least fa_bwd_workspace_size bytes,
 *                      16-byte aligned; its contents on entry do not matter.
 * dK and dV are written by exactly one CTA per 128-key tile (no atomics); dQ
 * is summed in fp32 with atomic adds, so it is not bitwise reproducible from
 * run to run (the rounding order of the adds varies).
 */
FA_API fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o,
                 const float* lse, const void* dout,
                 void* dq, void* dk, void* dv,
                 void* workspace, size_t workspace_bytes,
                 int B, int H, int N, int d, int causal, float scale, void* stream);

/*
 * Deterministic backward: same arguments, workspace size, preconditions and
 * results as fa_bwd, but dQ is bitwise reproducible from run to run.
 *
 * Same recompute backward ("从零实现 FlashAttention-2：分块在线 Softmax",
 * section 反向传播：重算，而不是存储), with the work split in two passes so that
 * no output is summed by atomics: a key-tile-owned pass writes dK and dV
 * exactly as fa_bwd does, and a query-tile-owned pass recomputes the score
 * and dP tiles of each 128-row query tile against every key tile it sees,
 * summing dQ = scale * sum_j dS_j K_j in one fixed order in on-chip
 * accumulators and writing it once.  Costs one extra recompute of S and dP
 * (7 instead of 5 tile GEMMs per tile pair).  Only the two fp32 row vectors
 * of the workspace are used.
 */
FA_API fa_status fa_bwd_deterministic(const void* q, const void* k, const void* v,
                                      const void* o, const float* lse, const void* dout,
                                      void* dq, void* dk, void* dv,
                                      void* workspace, size_t workspace_bytes,
                                      int B, int H, int N, int d, int causal, float scale,
                                      void* stream);

/*
 * Backward pass that allocates nothing.  (The pages have no counterpart to
 * this entry point: it exists only for callers that cannot allocate.)
 *
 * Same arguments and results as fa_bwd, minus the workspace: the scratch the
 * backward needs lives in one fixed array of FA_BWD_NOALLOC_SCRATCH_BYTES
 * bytes of device memory that is part of this library, so the call itself
 * never calls cudaMalloc or any other allocating routine.  Meant for callers
 * that may not allocate device memory on the call path: code running under a
 * host framework that owns all device memory through its own pool (a direct
 * allocation would bypass it or fail), and latency-critical loops that must
 * not allocate or free after start-up because cudaFree can synchronise the
 * device.
 *
 * Limits and caveats:
 *   - A problem needing more than FA_BWD_NOALLOC_SCRATCH_BYTES of scratch
 *     (the size fa_bwd_workspace_size reports) is rejected with
 *     FA_ERR_WORKSPACE before anything is launched.
 *   - Every GPU that loads this library holds the array (32 MiB) until the
 *     process exits.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls on a device share the one array.  Calls whose kernels overlap
 *     on the GPU (different streams, no ordering between them) race on it;
 *     order them, e.g. by issuing them on one stream.  Each call rewrites
 *     every part of the array it reads, so leftovers of an earlier call never
 *     leak into its result.
 *   - The looked-up address is kept for the life of the process.  Do not go
 *     on using the library on a device after cudaDeviceReset (or any other
 *     teardown of its primary context) once a call has run there: the kept
 *     address, like the library's other per-device settings, would belong to
 *     the destroyed context.
 */
#define FA_BWD_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
FA_API fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dout,
                                void* dq, void* dk, void* dv,
                                int B, int H, int N, int d, int causal, float scale,
                                void* stream);

/*
 * Forward in the FlashAttention-1 loop order, for measurement (a loop-order
 * ablation): same arguments, preconditions and results as fa_fwd, up to
 * rounding, plus a workspace.
 *
 * Page "从零实现 FlashAttention-2：分块在线 Softmax", section 从 FlashAttention-1
 * 到 FlashAttention-2: the first version loops over key/value tiles outside
 * and query tiles inside; the second swaps the loops (fa_fwd) and also
 * parallelises over the sequence.  Here one CTA per (batch, head) loads each
 * K/V tile once and, for every query tile that sees it, reads Q_i and the
 * running row statistics m_i, l_i and output O_i (fp32, in the workspace) from
 * global memory, merges the tile's contribution with the page-3 rule
 * ("FlashAttention 为什么能节省显存并提速,是否改变注意力结果?", section
 * 难点在于分块后softmax如何归一) and writes them back; bf16 O and LSE are
 * written after the last key tile.  It is slower than fa_fwd by design: the
 * extra reads and writes of O_i per (i, j) step and the B*H-CTA grid are what
 * it measures.
 *
 *   workspace : device scratch of at least fa_fwd_kv_outer_workspace_size
 *               bytes (fp32 O of B*H*Np*d floats, then m and l of B*H*Np
 *               floats each, Np = N rounded up to 128), 16-byte aligned; its
 *               contents on entry do not matter.
 * Returns the same codes as fa_fwd, and FA_ERR_WORKSPACE for a missing or
 * short workspace.
 */
FA_API size_t fa_fwd_kv_outer_workspace_size(int B, int H, int N, int d);
FA_API fa_status fa_fwd_kv_outer(const void* q, const void* k, const void* v, void* o,
                                 float* lse, int B, int H, int N, int d, int causal,
                                 float scale, void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * Synchronises `stream`, then reads and clears the device error word of the
 * current device.  Returns FA_OK, FA_ERR_DEVICE_TIMEOUT (a bounded wait ran
 * out; *detail, if non-NULL, receives which one) or FA_ERR_CUDA.
 */
FA_API fa_status fa_check_device_error(void* stream, unsigned int* detail);

/*
 * Self-test of the device-side wait limit (the pages have no counterpart: it
 * checks this library's failure detection).  Launches one 32-thread kernel on
 * `stream` that waits on a barrier no thread ever arrives on, with a limit of
 * `limit_ms` milliseconds (1..2000).  The wait gives up, records the fact in
 * the device error word and the kernel returns, so the next
 * fa_check_device_error reports FA_ERR_DEVICE_TIMEOUT (detail bit 1 << 15)
 * and the context stays usable.  Returns FA_ERR_SHAPE for a limit out of
 * range, FA_ERR_CUDA if the launch fails.
 */
FA_API fa_status fa_selftest_watchdog(unsigned int limit_ms, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
FA_API const char* fa_status_string(fa_status s);

/* Kernel identifiers for the timing calls below. */
typedef enum {
  FA_KERNEL_FWD = 0,       /* forward kernel                         */
  FA_KERNEL_BWD_PRE = 1,   /* backward: D = rowsum(dO*O), clears dQ  */
  FA_KERNEL_BWD_MAIN = 2,  /* backward: per-KV-tile main kernel      */
  FA_KERNEL_BWD_DQ = 3,    /* backward: dQ fp32 -> bf16 (fa_bwd), or the
                              dQ pass (fa_bwd_deterministic)         */
  FA_KERNEL_FWD_COMBINE = 4, /* split-KV forward: merge of the splits */
  FA_KERNEL_FWD_KV_OUTER = 5, /* forward in the KV-outer loop order    */
  FA_KERNEL_COUNT = 6
} fa_kernel_id;

/*
 * Measurement support.  Between fa_timing_begin and fa_timing_end every kernel
 * this library launches is bracketed by CUDA events recorded on the stream it
 * is launched on.  fa_timing_end synchronises those events and writes, per
 * fa_kernel_id, the summed milliseconds and the launch count into the caller's
 * arrays of FA_KERNEL_COUNT entries (either may be NULL).  Off by default;
 * at most 65536 launches are recorded per session.  Not thread-safe with
 * respect to concurrent fa_timing_* calls.
 */
FA_API fa_status fa_timing_begin(void);
FA_API fa_status fa_timing_end(float* ms_per_kernel, int* launches_per_kernel);

/* Library version, major*10000 + minor*100 + patch. */
FA_API int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_ATTENTION_B200_FA_H */
