/*
 * kda.h -- C ABI of libkda_b200.so, the B200 (sm_100a) Kimi Delta Attention
 * recurrence.
 *
 * The operation (daiw.net "Kimi Delta Attention", section "KDA 的更新式"), per
 * sequence and head, with S in R^{d_k x d_v}:
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = d_k^{-1/2} S_t^T q_t
 *
 * alpha_t in (0,1]^{d_k} is one decay per key channel (section
 * "一、Diag(alpha_t)：通道级遗忘"), passed as log_alpha = log(alpha_t) <= 0;
 * beta_t is a scalar write strength (section "二、I - beta k k^T：delta 规则").
 * The step order -- forget per channel, predict on the decayed state, correct,
 * write, read with d_k^{-1/2} -- is the one in news.bugfactory.tech/news/3610
 * (KDA paragraph), which also names the two modes exposed here: a chunkwise
 * mode for training and long prefill, and a token-by-token recurrent mode for
 * decoding.  Keys and queries are used as given (the library does not
 * normalise them).
 *
 * Conventions shared by every call:
 *  - All tensor pointers are DEVICE pointers to contiguous row-major tensors,
 *    16-byte aligned, owned by the caller.  The library allocates nothing and
 *    never synchronises the stream (except kda_workspace_status).
 *  - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *    stream.  All work is enqueued asynchronously on it.
 *  - Supported head sizes: d_k, d_v in {64, 128}.
 *  - q, k, v and o have the element type `dtype` (fp32 or bf16); log_alpha,
 *    beta and every state tensor are fp32.
 *  - On any status other than KDA_OK nothing was enqueued, except for
 *    KDA_ERR_CUDA (a launch failed) -- kda_last_error() has the message.
 *  - Calls are thread-safe; the last-error message is per host thread.
 */
#ifndef KDA_B200_KDA_H
#define KDA_B200_KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, B != 1 with cu_seqlens */
    KDA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d_k = 96) */
    KDA_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    KDA_ERR_TIMEOUT = 4,       /* device status: a bounded wait inside a kernel gave up */
    KDA_ERR_WORKSPACE = 5,     /* workspace missing, too small or misaligned */
    KDA_ERR_BAD_SEQLENS = 6,   /* device status: cu_seqlens not 0 .. T non-decreasing */
    KDA_ERR_RANGE = 7          /* device status: a bf16-path intermediate left the fp16 range */
} kda_status;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

/*
 * Shape of the decay gate.  KDA_GATE_CHANNEL is Kimi Delta Attention: one
 * log-decay per key channel, log_alpha [.., H, dk] (daiw.net "Kimi Delta
 * Attention", section "一、Diag(alpha_t)：通道级遗忘").  KDA_GATE_HEAD is Gated
 * DeltaNet: one scalar log-decay per token and head, log_alpha [.., H], applied
 * to the whole state before the prediction (news.bugfactory.tech/news/3610,
 * Gated DeltaNet paragraph).  KDA_GATE_NONE is DeltaNet: no decay (alpha = 1,
 * log_alpha unused, may be NULL) (same page, DeltaNet paragraph).  The three
 * are the same recurrence with log_alpha broadcast to [.., H, dk].
 */
typedef enum { KDA_GATE_CHANNEL = 0, KDA_GATE_HEAD = 1, KDA_GATE_NONE = 2 } kda_gate;

/*
 * Bytes of device workspace kda_chunk_fwd needs for these sizes.  `varlen` is
 * non-zero when cu_seqlens will be passed (then B must be 1 and num_seqs is
 * the number of packed sequences); otherwise num_seqs is ignored (= B).
 * Returns 0 for invalid sizes.
 */
size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv,
                                    int num_seqs, int varlen, kda_dtype dtype);

/*
 * Chunkwise forward over whole sequences ("chunkwise" mode, news.bugfactory.tech
 * /news/3610, KDA paragraph; chunks of 64 tokens as in the chunk-wise parallel
 * scheme on the kongchang.com page, section "硬件效率的优化策略").  Inside a
 * chunk the tokens are combined with matrix products (the WY/UT form of the
 * product of transitions D_t - beta_t D_t k_t k_t^T); between chunks the state
 * is carried.  The result equals the token-by-token recurrence above up to
 * rounding.
 *
 *  q, k        [B, T, H, dk]   dtype
 *  v           [B, T, H, dv]   dtype
 *  log_alpha   [B, T, H, dk]   fp32, <= 0 (finite)
 *  beta        [B, T, H]       fp32
 *  initial_state [N, H, dk, dv] fp32, or NULL for zeros
 *  cu_seqlens  [N + 1] int32 device array, or NULL.  With it, B must be 1 and
 *              the T tokens hold N = num_seqs packed sequences,
 *              cu_seqlens[0] = 0 <= ... <= cu_seqlens[N] = T (empty sequences
 *              allowed).  Without it, N = B sequences of T tokens each.
 *              The device checks the array; a bad one sets KDA_ERR_BAD_SEQLENS
 *              in the workspace status and leaves o / final_state unwritten.
 *  o           [B, T, H, dv]   dtype, written
 *  final_state [N, H, dk, dv]  fp32, written, or NULL.  May alias
 *              initial_state exactly (each state is read before it is written).
 *  workspace   device scratch of at least kda_chunk_fwd_workspace_size(...)
 *              bytes (bf16 inputs: or at least
 *              kda_chunk_fwd_fused_workspace_size(...), which runs the fused
 *              pass, see kda_chunk_fwd_plan), 256-byte aligned; its contents
 *              on entry do not matter.  Calls that share one workspace must be
 *              ordered on one stream.
 *
 * Numerics: every product runs on the tensor cores with fp32 accumulation.
 * bf16 inputs use fp16 operands (tf32 where a factor can leave the fp16
 * range); fp32 inputs use split tf32 (each operand as a tf32 high part plus an
 * fp32 remainder, three products), about 2e-6 max-relative error against the
 * fp64 recurrence on the documented workloads.
 */
kda_status kda_chunk_fwd(const void* q, const void* k, const void* v,
                         const float* log_alpha, const float* beta,
                         const float* initial_state, const int32_t* cu_seqlens,
                         int B, int T, int H, int dk, int dv, int num_seqs,
                         kda_dtype dtype, void* o, float* final_state,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * One decoding step for B sequences ("fused recurrent" mode,
 * news.bugfactory.tech/news/3610, KDA paragraph): each (sequence, head) state
 * is read once, updated by one token and written back in place.
 *
 *  q, k        [B, H, dk]  dtype       v [B, H, dv] dtype
 *  log_alpha   [B, H, dk]  fp32        beta [B, H] fp32
 *  state_inout [B, H, dk, dv] fp32, updated in place
 *  o           [B, H, dv]  dtype, written (must not alias the state)
 */
kda_status kda_recurrent_step(const void* q, const void* k, const void* v,
                              const float* log_alpha, const float* beta,
                              float* state_inout, int B, int H, int dk, int dv,
                              kda_dtype dtype, void* o, void* stream);

/*
 * The two forms of the bf16 chunk forward.  Both compute the same result up
 * to rounding.
 *  - split (two kernels): all (chunk, head) items in parallel, two CTAs per
 *    SM, their intermediates through the workspace; then the chunk-to-chunk
 *    recurrence, one CTA per (sequence, head, value slice).  Needs
 *    kda_chunk_fwd_workspace_size bytes (about 74 KB per chunk and head at
 *    d_k = d_v = 128).
 *  - fused (one pass): one CTA per (sequence, head) pair carries the state
 *    through the pair's chunks and keeps each chunk's intermediates on chip
 *    (no intermediate traffic to memory); one CTA per SM.  Needs only
 *    kda_chunk_fwd_fused_workspace_size bytes (header, chunk table, pair
 *    order).  Slower than the split form on B200 at the shapes measured (its
 *    intra-chunk phases cannot overlap a second CTA's), so it runs only when
 *    the workspace passed to kda_chunk_fwd is too small for the split form,
 *    or when forced.
 * The environment variable KDA_CHUNK_PATH=fused or =split (read at every call)
 * forces one form for bf16 inputs; fp32 inputs always take the split form.
 *
 * kda_chunk_fwd_plan returns 1 if kda_chunk_fwd with a workspace of
 * `workspace_bytes` runs the fused pass, 0 for the split form, -1 for invalid
 * sizes or a workspace too small for either.  Other arguments as
 * kda_chunk_fwd_workspace_size.  kda_chunk_fwd_fused_workspace_size returns
 * the fused pass's workspace bytes (0 for fp32 inputs or invalid sizes).
 */
int kda_chunk_fwd_plan(int B, int T, int H, int dk, int dv, int num_seqs, int varlen,
                       kda_dtype dtype, size_t workspace_bytes);
size_t kda_chunk_fwd_fused_workspace_size(int B, int T, int H, int dk, int dv,
                                          int num_seqs, int varlen, kda_dtype dtype);

/*
 * Waits for `stream`, then reads the device status that the last
 * kda_chunk_fwd or kda_chunk_bwd on this workspace left: KDA_OK, KDA_ERR_BAD_SEQLENS,
 * KDA_ERR_TIMEOUT or KDA_ERR_RANGE (or KDA_ERR_CUDA if the copy fails).
 * KDA_ERR_RANGE means a value-side quantity (|v|, the state, the per-token
 * errors u) exceeded 65000 in magnitude: the bf16 path keeps its chunk
 * intermediates in fp16, so such inputs need the fp32 path.  This is the only
 * call that synchronises.
 */
kda_status kda_workspace_status(const void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * kda_chunk_fwd with the gate shape chosen by `gate` (see kda_gate): log_alpha
 * is [B, T, H, dk] for KDA_GATE_CHANNEL (16-byte aligned), [B, T, H] for
 * KDA_GATE_HEAD, and unused for KDA_GATE_NONE.  Everything else as kda_chunk_fwd;
 * the workspace size does not depend on the gate.
 */
kda_status kda_chunk_fwd_gated(const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta,
                               const float* initial_state, const int32_t* cu_seqlens,
                               int B, int T, int H, int dk, int dv, int num_seqs,
                               kda_dtype dtype, kda_gate gate, void* o, float* final_state,
                               void* workspace, size_t workspace_bytes, void* stream);

/*
 * kda_recurrent_step with the gate shape chosen by `gate`: log_alpha is
 * [B, H, dk] for KDA_GATE_CHANNEL, [B, H] for KDA_GATE_HEAD, unused for
 * KDA_GATE_NONE.
 */
kda_status kda_recurrent_step_gated(const void* q, const void* k, const void* v,
                                    const float* log_alpha, const float* beta,
                                    float* state_inout, int B, int H, int dk, int dv,
                                    kda_dtype dtype, kda_gate gate, void* o, void* stream);

/*
 * kda_chunk_fwd without a caller-provided workspace.  The method itself has
 * no counterpart to this call; it exists for callers that cannot allocate device
 * memory -- a plugin whose host framework owns all device memory and forbids
 * other allocations, a latency-critical loop that cannot afford cudaMalloc's
 * implicit synchronisation, or a tool with a fixed memory budget.
 *
 * The scratch space comes from one fixed array of KDA_STATIC_WORKSPACE_BYTES
 * in the library's device image, present on every GPU that loads the library
 * until the process exits.  Arguments and results are those of kda_chunk_fwd
 * minus the workspace.  Sizes whose workspace (kda_chunk_fwd_workspace_size)
 * exceeds KDA_STATIC_WORKSPACE_BYTES are rejected with KDA_ERR_WORKSPACE and
 * nothing is launched.  Nothing is allocated: no cudaMalloc or cudaFree.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  The address is cached with the device's CUDA
 * context; a call that finds another context current (after cudaDeviceReset,
 * say) looks it up again.  Every call uses the same array, so calls that
 * overlap on one GPU (e.g. on two streams) race; order them on one stream.
 * kda_workspace_status cannot read this workspace (use kda_chunk_fwd when the
 * device status is needed).
 */
#define KDA_STATIC_WORKSPACE_BYTES (64u << 20)
kda_status kda_chunk_fwd_static(const void* q, const void* k, const void* v,
                                const float* log_alpha, const float* beta,
                                const float* initial_state, const int32_t* cu_seqlens,
                                int B, int T, int H, int dk, int dv, int num_seqs,
                                kda_dtype dtype, void* o, float* final_state, void* stream);

/*
 * Bytes of device workspace kda_chunk_bwd needs for these sizes (arguments as
 * kda_chunk_fwd_workspace_size).  Returns 0 for invalid sizes.
 */
size_t kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv,
                                    int num_seqs, int varlen, kda_dtype dtype);

/*
 * Gradients of the chunkwise forward (the chunkwise mode is the training mode
 * of news.bugfactory.tech/news/3610, KDA paragraph).  For the loss
 *     L = sum <d_o, o> + sum <d_final_state, final_state>
 * of the kda_chunk_fwd call with the same inputs, it writes dL/dq, dL/dk,
 * dL/dv, dL/dlog_alpha, dL/dbeta and dL/dinitial_state.  The forward
 * quantities are recomputed from the inputs (no forward output is needed).
 * fp32 inputs: every product in fp32 on CUDA cores (max-relative error 1e-4
 * against an fp64 reference).  bf16 inputs: the products on the tensor cores
 * with fp16 operands (tf32 for the split-factor products) and fp32
 * accumulation (relative L2 error 5e-3); chunks whose decay is too strong for
 * the split factors on CUDA cores in fp32.  As in the forward, a bf16-path
 * value beyond the fp16 range sets KDA_ERR_RANGE in the workspace status.
 *
 *  q, k, v, log_alpha, beta, initial_state, cu_seqlens, sizes, dtype:
 *              as kda_chunk_fwd (per-channel gate)
 *  d_o         [B, T, H, dv]   dtype, cotangent of o
 *  d_final_state [N, H, dk, dv] fp32, cotangent of the final state, or NULL
 *              for zeros
 *  dq, dk      [B, T, H, dk]   dtype, written
 *  dv          [B, T, H, dv]   dtype, written
 *  dlog_alpha  [B, T, H, dk]   fp32, written
 *  dbeta       [B, T, H]       fp32, written
 *  d_initial_state [N, H, dk, dv] fp32, written, or NULL (not computed)
 *  workspace   device scratch of at least kda_chunk_bwd_workspace_size(...)
 *              bytes, 256-byte aligned; kda_workspace_status reads its status.
 * Outputs must not alias inputs.  Nothing is allocated or synchronised.
 */
kda_status kda_chunk_bwd(const void* q, const void* k, const void* v,
                         const float* log_alpha, const float* beta,
                         const float* initial_state, const int32_t* cu_seqlens,
                         const void* d_o, const float* d_final_state,
                         int B, int T, int H, int dk, int dv, int num_seqs,
                         kda_dtype dtype, void* dq, void* dk_out, void* dv_out,
                         float* dlog_alpha, float* dbeta, float* d_initial_state,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * kda_chunk_bwd with the gate shape chosen by `gate` (see kda_gate): log_alpha
 * and dlog_alpha are [B, T, H, dk] for KDA_GATE_CHANNEL, [B, T, H] for
 * KDA_GATE_HEAD (the cotangent of a per-head log-decay is the sum over the key
 * channels it decays), and unused (may be NULL) for KDA_GATE_NONE.  Everything
 * else as kda_chunk_bwd; the workspace size does not depend on the gate.
 */
kda_status kda_chunk_bwd_gated(const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta,
                               const float* initial_state, const int32_t* cu_seqlens,
                               const void* d_o, const float* d_final_state,
                               int B, int T, int H, int dk, int dv, int num_seqs,
                               kda_dtype dtype, kda_gate gate, void* dq, void* dk_out,
                               void* dv_out, float* dlog_alpha, float* dbeta,
                               float* d_initial_state, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * Training forward: kda_chunk_fwd_gated (same arguments and outputs) that
 * also keeps, in `workspace`, everything kda_chunk_bwd would otherwise
 * recompute from the inputs: the chunk table, the per-chunk records, T =
 * (I + A)^-1 (for bf16 inputs with the K~ and V tiles, M and the strong-decay
 * flags) and the state entering every chunk.  `workspace` must have at least
 * kda_chunk_bwd_workspace_size(...) bytes (256-byte aligned); pass it, with
 * the same inputs and sizes, to kda_chunk_bwd_saved.  It always runs the
 * two-kernel form (never the fused pass; KDA_CHUNK_PATH does not apply), with
 * the kernels that also write what the backward reads.  The chunkwise mode is
 * the training mode of news.bugfactory.tech/news/3610 (KDA paragraph).
 */
kda_status kda_chunk_fwd_save(const void* q, const void* k, const void* v,
                              const float* log_alpha, const float* beta,
                              const float* initial_state, const int32_t* cu_seqlens,
                              int B, int T, int H, int dk, int dv, int num_seqs,
                              kda_dtype dtype, kda_gate gate, void* o, float* final_state,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * kda_chunk_bwd_gated after kda_chunk_fwd_save: the same arguments, but the
 * forward is not recomputed.  `workspace` must be the one kda_chunk_fwd_save
 * filled for exactly these inputs and sizes, unchanged since; its contents are
 * not checked (a different workspace gives wrong gradients, not an error).
 * Its status word keeps what the forward recorded (kda_workspace_status).
 */
kda_status kda_chunk_bwd_saved(const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta,
                               const float* initial_state, const int32_t* cu_seqlens,
                               const void* d_o, const float* d_final_state,
                               int B, int T, int H, int dk, int dv, int num_seqs,
                               kda_dtype dtype, kda_gate gate, void* dq, void* dk_out,
                               void* dv_out, float* dlog_alpha, float* dbeta,
                               float* d_initial_state, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * Measurement hook for benchmarks.  When `events` is non-NULL, each later
 * kda_chunk_fwd on this host thread records the caller-created CUDA events
 * (cudaEvent_t passed as void*) on its stream at the stage boundaries:
 * events[0] before the first kernel, events[1] after the chunk-table/status
 * kernel, events[2] after the intra-chunk stage (the whole fused pass, when
 * kda_chunk_fwd_plan says 1), events[3] after the inter-chunk stage (empty
 * for the fused pass).  With `count` >= 7, each later kda_chunk_bwd records
 * events[0] before its first kernel and events[1..6] after the chunk-table,
 * forward intra-chunk, forward inter-chunk, reversed inter-chunk, tensor-core
 * product kernels (bf16 inputs: every chunk without strong decay is finished
 * there; an empty stage for fp32) and the CUDA-core per-chunk gradient kernel.
 * `count` must be >= 4 (only the first 7 are used).  Pass
 * NULL to stop.  Recording an event costs a few microseconds of stream time
 * and changes no result.
 */
kda_status kda_set_stage_events(void* const* events, int count);

/*
 * Test hook for the failure path (no counterpart in the pages).  Arms the next
 * kda_chunk_fwd with bf16 inputs and the per-channel gate on this host thread
 * (one call only): its intra-chunk kernel leaves out one asynchronous copy
 * (the log-decay tile of the third work item of its first CTA, or of that
 * CTA's last item if it has fewer) and caps each of its waits at
 * `wait_cycles` SM clock cycles.  The wait on the missing copy
 * gives up, the kernel records KDA_ERR_TIMEOUT in the workspace status
 * (kda_workspace_status) and returns; that call's outputs are not meaningful.
 * Nothing faults or hangs, and later calls run normally.  0 disarms.
 */
kda_status kda_debug_drop_copy(long long wait_cycles);

/* Message of the last failing call on this host thread ("" if none). */
const char* kda_last_error(void);

/* Library version string, e.g. "kda-b200 0.1.0 sm_100a". */
const char* kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_B200_KDA_H */
