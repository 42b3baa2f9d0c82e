/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention operator.
 *
 * KDA is a gated delta-rule linear attention with a per-channel diagonal
 * forget gate.  Per sequence and head it keeps a dk x dv state S and, for each
 * token t, computes
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = scale * S_t^T q_t,        alpha_t = exp(log_alpha_t) in (0, 1]^dk
 *
 * Sources: "Kimi Linear ... 深度解读报告" (zako-mio knowledge base), section 2.3
 * (the three parts of the update) and section 3.1 (the chunkwise algorithm:
 * a = b = k DPLR specialisation, WY representation, UT transform, forward-
 * substitution triangular inverse); zhaixingw.cn ai-news/151, section
 * "KDA：把遗忘门从一个数变成一串数" (the Gated DeltaNet update whose scalar gate
 * KDA replaces by a dk-vector; the fixed-size dk x dv state).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor is a plain pointer to DEVICE memory, row-major and
 *    contiguous, with 16-byte aligned base addresses.  Host pointers are
 *    rejected (KDA_ERR_INVALID_ARG); there is no CPU fallback.
 *  - The caller owns every buffer, including the device workspace that some
 *    kernels need: kda_chunk_fwd_workspace_bytes() and
 *    kda_chunk_bwd_workspace_bytes() give its size for a call, and the call
 *    takes it as (workspace, workspace_bytes).  No entry point allocates
 *    device memory (kda_chunk_fwd_noalloc below uses a fixed array of the
 *    library's module instead of a workspace).
 *  - Calls are asynchronous: kernels are enqueued on `stream` and the call
 *    returns.  Launch failures return KDA_ERR_CUDA.  Faults during execution
 *    surface at the caller's next synchronisation.  A kernel whose internal
 *    wait runs out of time records it; kda_device_error() reports it.
 *  - Supported sizes: dk = dv = 128, chunk = 64.  Anything else returns
 *    KDA_ERR_UNSUPPORTED.  dtype is the type of q, k, v and out; log_alpha,
 *    beta and states are always fp32.
 *  - No C++ exception crosses this interface.
 */
#ifndef KDA_B200_KDA_H_
#define KDA_B200_KDA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,  /* null/host/misaligned pointer, bad size     */
    KDA_ERR_UNSUPPORTED = 2,  /* valid request this build does not support   */
    KDA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed        */
    KDA_ERR_TIMEOUT = 4       /* a kernel's bounded internal wait ran out    */
} kda_status;

typedef enum {
    KDA_DTYPE_F32 = 0,
    KDA_DTYPE_BF16 = 1
} kda_dtype;

/* Options of the _ex entry points (a bit set). */
enum {
    /* Fused L2Norm of q and k ("深度解读报告" 3.2: the layer normalises q and
     * k before the recurrence): every [dk] row of q and of k is first divided
     * by max(||row||_2, 1e-6), in fp32 inside the kernels, so the caller may
     * pass un-normalised q and k. */
    KDA_FLAG_L2NORM_QK = 1,
    /* Output epilogue ("深度解读报告" 3.2, the output side: head-wise RMSNorm
     * and a data-dependent sigmoid output gate): every [dv] row o of out
     * becomes o / sqrt(mean(o^2) + out_eps) * out_weight * sigmoid(g), with
     * g the matching row of out_gate (the gate's pre-activations, dtype,
     * shaped like out) and out_weight [dv] fp32; out_eps > 0. */
    KDA_FLAG_OUT_NORM_GATE = 2,
    /* Raw gate ("深度解读报告" 3.2: the gate comes from a low-rank projection
     * of the token; no activation is printed, and the logistic sigmoid is the
     * one taken): `log_alpha` holds the gate's pre-activations z (fp32, any
     * finite value) and the kernels use log alpha = log sigmoid(z) =
     * -softplus(-z).  The per-chunk precondition applies to log sigmoid(z). */
    KDA_FLAG_RAW_GATE = 4
};

/*
 * kda_chunk_fwd -- chunked prefill over whole sequences.
 *
 * Computes the recurrence above for every token of every sequence, chunk by
 * chunk (chunk = 64 tokens): inside a chunk the per-channel log-decay is
 * prefix-summed, the decayed strictly-lower beta*K*K^T matrix is inverted by
 * forward substitution, the WY tiles W, U' are formed, the state is carried
 * across chunks sequentially and the output is Q*S plus the masked
 * intra-chunk attention ("深度解读报告" 3.1).
 *
 *   q, k       [B, T, H, dk]  dtype
 *   v          [B, T, H, dv]  dtype
 *   log_alpha  [B, T, H, dk]  fp32, finite, <= 0 (log of the forget gate).
 *              Precondition: within any chunk the per-channel sum is > -80.
 *   beta       [B, T, H]      fp32
 *   initial_state [N, H, dk, dv] fp32, or NULL for zeros.
 *   cu_seqlens [N + 1] int32 on the device, or NULL.  With it, B must be 1
 *              and sequence n is tokens [cu_seqlens[n], cu_seqlens[n+1]) of
 *              the T-token stream; cu_seqlens[0] = 0, non-decreasing,
 *              cu_seqlens[N] = T (the library cannot check device contents
 *              without a copy; a violating array gives undefined results).
 *              Without it N must equal B.  Chunks restart at every sequence
 *              start; a zero-length sequence passes its state through.
 *   scale      output scale (callers normally pass dk^-0.5).
 *   chunk      must be 64.
 *   out        [B, T, H, dv]  dtype.  Must not alias any input.
 *   final_state [N, H, dk, dv] fp32, or NULL to skip it.  May be the same
 *              pointer as initial_state (each state is read before written).
 *   B, T, H, dk, dv, N   sizes; T = 0 or N = 0 is a valid empty call.
 *   dtype      KDA_DTYPE_BF16 (tensor-core path: bf16 operands, fp32 state
 *              and accumulation) or KDA_DTYPE_F32 (fp32 FFMA path).
 *   workspace, workspace_bytes
 *              caller-owned device scratch of at least
 *              kda_chunk_fwd_workspace_bytes(B, T, H, N, dtype) bytes, 256-byte
 *              aligned, overlapping no tensor argument; NULL and 0 when that
 *              is 0.  Too small, misaligned or overlapping: KDA_ERR_INVALID_ARG.
 *              Its contents need not be initialised and are undefined after
 *              the call; calls whose executions overlap in time need
 *              separate workspaces.
 *   stream     CUDA stream the kernels are enqueued on.
 */
kda_status kda_chunk_fwd(const void* q, const void* k, const void* v,
                         const float* log_alpha, const float* beta,
                         const float* initial_state, const int32_t* cu_seqlens,
                         float scale, int chunk,
                         void* out, float* final_state,
                         int B, int T, int H, int dk, int dv, int N,
                         kda_dtype dtype, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream);

/*
 * kda_chunk_fwd_workspace_bytes -- bytes of device workspace a
 * kda_chunk_fwd / kda_chunk_fwd_ex call with these sizes and dtype needs on
 * the current device under the current kda_set_prefill_kernel setting (a
 * pure function of those: call it again after changing the setting or the
 * device).  0 when the kernel the call selects needs none, and for sizes the
 * call would reject.  The bf16 prefill for few (sequence, head) chains hands
 * each chunk's operand tiles from the CTAs that prepare them to the CTA that
 * carries the state through a ring in this workspace (133,120 bytes per
 * preparing CTA and cluster); a segmented run adds 3 x 64 KiB per segment
 * and chain for the segments' transitions and states; the
 * one-CTA-per-chain and fp32 kernels need none.
 */
size_t kda_chunk_fwd_workspace_bytes(int B, int T, int H, int N, kda_dtype dtype);

/*
 * kda_chunk_fwd_ex -- kda_chunk_fwd with options: `flags` is a set of
 * KDA_FLAG_* bits (0 gives exactly kda_chunk_fwd).  Unknown bits return
 * KDA_ERR_UNSUPPORTED.  out_gate [B, T, H, dv] (dtype, must not alias out),
 * out_weight [dv] fp32 and out_eps are read only with
 * KDA_FLAG_OUT_NORM_GATE (pass NULL, NULL, 0 otherwise); final_state is
 * never affected by it.  Every other argument as for kda_chunk_fwd.
 */
kda_status kda_chunk_fwd_ex(const void* q, const void* k, const void* v,
                            const float* log_alpha, const float* beta,
                            const float* initial_state, const int32_t* cu_seqlens,
                            float scale, int chunk,
                            void* out, float* final_state,
                            int B, int T, int H, int dk, int dv, int N,
                            kda_dtype dtype, unsigned flags, const void* out_gate,
                            const float* out_weight, float out_eps,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * kda_recurrent_step -- one batched decode step, state updated in place.
 *
 * For each request n and head h, applies the recurrence to one token:
 * S <- (I - beta k k^T) Diag(exp log_alpha) S + beta k v^T and
 * o = scale * S^T q, reading and writing the fp32 state once
 * (zhaixingw.cn ai-news/151: the fixed-size per-request state that replaces
 * the KV cache).
 *
 *   q, k       [N, H, dk]  dtype
 *   v          [N, H, dv]  dtype
 *   log_alpha  [N, H, dk]  fp32, finite, <= 0
 *   beta       [N, H]      fp32
 *   state      [N, H, dk, dv] fp32, read and written in place; nothing else
 *              may alias it.
 *   out        [N, H, dv]  dtype
 *   N = 0 is a valid empty call.
 */
kda_status kda_recurrent_step(const void* q, const void* k, const void* v,
                              const float* log_alpha, const float* beta,
                              float* state, void* out,
                              int N, int H, int dk, int dv, float scale,
                              kda_dtype dtype, cudaStream_t stream);

/*
 * kda_recurrent_step_ex -- kda_recurrent_step with options (KDA_FLAG_* bits;
 * 0 gives exactly kda_recurrent_step; unknown bits: KDA_ERR_UNSUPPORTED).
 * out_gate [N, H, dv] (dtype), out_weight [dv] fp32 and out_eps as for
 * kda_chunk_fwd_ex; the state update does not depend on them.
 */
kda_status kda_recurrent_step_ex(const void* q, const void* k, const void* v,
                                 const float* log_alpha, const float* beta,
                                 float* state, void* out,
                                 int N, int H, int dk, int dv, float scale,
                                 kda_dtype dtype, unsigned flags, const void* out_gate,
                                 const float* out_weight, float out_eps, cudaStream_t stream);

/*
 * kda_chunk_debug_stages -- stage-by-stage view of the bf16 tensor-core
 * prefill, for testing.  Runs the same kernel as kda_chunk_fwd (bf16) on ONE
 * chunk of one sequence of one head (B = N = H = 1, 1 <= T <= 64, dk = dv =
 * 128) and, besides out [T, dv] and final_state [dk, dv], writes the chunk's
 * intermediates ("深度解读报告" 3.1: the decayed K K^T / Q K^T matrices, the
 * forward-substitution inverse, the WY tiles, the state update) as fp32,
 * row-major, into `stages` (device, kda_chunk_debug_stage_floats() floats):
 *
 *   offset        shape      content (C = 64 rows, rows >= T are padding)
 *   0             128 x 64   [Kt Kh^T ; Qt Kh^T], before masking and beta
 *   8192          64 x 64    T = (I + A)^-1 Diag(beta) (before bf16 rounding)
 *   12288         128 x 64   W^T,   W = T Kt
 *   20480         128 x 64   U'^T,  U' = T V
 *   28672         128 x 64   (Qt S0)^T
 *   36864         128 x 64   U^T,   U = U' - W S0
 *   45056         128 x 128  (Kh^T U)^T
 *   61440         128 x 64   O^T,   O = Qt S0 + P U
 *   69632         128 x 128  S'^T,  the exit state, transposed
 *
 * with Kt = K e^G, Kh = K e^-G, Qt = scale Q e^G and G the per-channel
 * prefix sum of log_alpha.  Pointer rules are those of kda_chunk_fwd;
 * initial_state may be NULL (zeros).
 */
kda_status kda_chunk_debug_stages(const void* q, const void* k, const void* v,
                                  const float* log_alpha, const float* beta,
                                  const float* initial_state, float scale, int T,
                                  void* out, float* final_state, float* stages,
                                  cudaStream_t stream);

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd for callers that must not allocate
 * device memory during the call (e.g. an engine that reserves nearly all of
 * HBM for its state caches up front and runs each step at a fixed
 * footprint).  The pages describe no such call: it is an interface of this
 * library only, computing exactly what kda_chunk_fwd computes.
 *
 * Arguments, layouts and results as for kda_chunk_fwd without its workspace
 * arguments, with dtype KDA_DTYPE_BF16 only (anything else:
 * KDA_ERR_UNSUPPORTED).  It always runs
 * the one-cluster-per-chain kernel, whose hand-off ring (133,120 bytes per
 * prep CTA and (sequence, head) chain, 1-3 prep CTAs per chain) lives in a
 * fixed 16 MiB device array of the library instead of pool memory: N * H
 * must be at most 126 (one prep CTA per chain fits), else the call returns
 * KDA_ERR_UNSUPPORTED before touching any pointer.  Nothing in the array
 * needs to start at zero (every ring slot is written before it is read).
 * Every call shares that array: calls whose executions overlap in time, on
 * different streams or from different host threads, race on it and give
 * wrong results; serialise them.  Its results equal kda_chunk_fwd's with
 * kda_set_prefill_kernel(2) bit for bit.
 *
 * The array, like the kernels' code, is device memory that the CUDA driver
 * creates when it loads this library's module on a device.  Under CUDA's
 * default lazy module loading that happens on the first call on each device
 * (the call's set-up looks up the array's address and the kernel's cluster
 * residency), so the first call may fail with KDA_ERR_CUDA if the caller has
 * already reserved nearly all device memory.  Make one call per device
 * before reserving memory (the results of that call can be discarded), or
 * run with CUDA_MODULE_LOADING=EAGER so the module loads with the context.
 * Later calls allocate nothing.
 */
kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                 const float* log_alpha, const float* beta,
                                 const float* initial_state, const int32_t* cu_seqlens,
                                 float scale, int chunk,
                                 void* out, float* final_state,
                                 int B, int T, int H, int dk, int dv, int N,
                                 kda_dtype dtype, cudaStream_t stream);

/*
 * kda_chunk_transition -- the state transition of every (sequence, head): the
 * dk x dk matrix M with which kda_chunk_fwd's final state from any initial
 * state S0 is M S0 + B, B its final state from a zero initial state.  The
 * recurrence is affine in the state ("深度解读报告" 2.3: each token applies
 * (I - beta k k^T) Diag(alpha) and adds beta k v^T), so M is the product of
 * the tokens' (I - beta_t k_t k_t^T) Diag(alpha_t) factors, computed here as
 * the chunked recurrence from S = I with v = 0.  Splitting a long sequence
 * across devices uses it: each device computes M and B of its token range,
 * the pairs are exchanged, and every device chains the entry state of its
 * range with kda_state_affine before running kda_chunk_fwd on it.
 *
 *   q, k, log_alpha, beta, cu_seqlens, B, T, H, N as for kda_chunk_fwd (q is
 *              read only with KDA_FLAG_L2NORM_QK set, and then not used);
 *   flags      KDA_FLAG_L2NORM_QK and KDA_FLAG_RAW_GATE as for
 *              kda_chunk_fwd_ex (others: KDA_ERR_UNSUPPORTED);
 *   transition [N, H, dk, dk] fp32, written; must not overlap an input.
 *   dk must be 128; dtype KDA_DTYPE_BF16 only (bf16 operands, fp32
 *   accumulation, like the bf16 prefill).  workspace as for kda_chunk_fwd,
 *   sized by kda_chunk_transition_workspace_bytes().
 */
kda_status kda_chunk_transition(const void* q, const void* k, const float* log_alpha,
                                const float* beta, const int32_t* cu_seqlens, float* transition,
                                int B, int T, int H, int dk, int N, kda_dtype dtype,
                                unsigned flags, void* workspace, size_t workspace_bytes,
                                cudaStream_t stream);

/* Bytes of workspace a kda_chunk_transition call of these sizes needs. */
size_t kda_chunk_transition_workspace_bytes(int B, int T, int H, int N, kda_dtype dtype);

/*
 * kda_state_affine -- S_out = M S_in + B for N x H fp32 states in fp32
 * (M [N, H, dk, dk], B, S_in, S_out [N, H, dk, dv], dk = dv = 128): one step
 * of chaining the entry states of consecutive token ranges (see
 * kda_chunk_transition).  S_out may be the same pointer as B; it must not
 * overlap M or S_in.
 */
kda_status kda_state_affine(const float* M, const float* B, const float* S_in, float* S_out,
                            int N, int H, int dk, int dv, cudaStream_t stream);

/*
 * kda_chunk_bwd -- backward pass of kda_chunk_fwd (without its L2Norm and
 * output-gate options), for training with the operator: the pages train the
 * layer end to end ("深度解读报告" 3.4); the gradients follow from the chunk
 * form of "深度解读报告" 3.1 by reverse-mode differentiation.
 *
 * Given the forward call's inputs (same meaning, layout, dtype and sizes as
 * for kda_chunk_fwd, device pointers) and the adjoints
 *   d_out          [B,T,H,dv] in dtype: dLoss/d out,
 *   d_final_state  [N,H,dk,dv] fp32 or NULL (zero): dLoss/d final_state,
 * it writes, all fp32 device arrays owned by the caller:
 *   grad_q, grad_k   [B,T,H,dk]   grad_v     [B,T,H,dv]
 *   grad_log_alpha   [B,T,H,dk]   grad_beta  [B,T,H]
 *   grad_initial_state [N,H,dk,dv] or NULL (not computed).
 * The outputs must not overlap one another or any input.  Every step runs on
 * the FFMA pipes in fp32 from the exact input values: a forward recompute
 * keeping the entry state of every chunk, a reverse pass over each
 * sequence's chunks carrying the state adjoint, and a pass over all chunks
 * at once for the rest.  The caller-owned workspace (workspace_bytes at
 * least kda_chunk_bwd_workspace_bytes(B, T, H, N, cu_seqlens != NULL,
 * dtype), 256-byte aligned, overlapping no tensor argument) holds the entry
 * state and the exit-state adjoint of every chunk and head (2 x 64 KiB) and
 * the adjoint of U (512 B per token and head).  Errors as for
 * kda_chunk_fwd; dk = dv = 128 and chunk = 64 only.
 */
kda_status kda_chunk_bwd(const void* q, const void* k, const void* v,
                         const float* log_alpha, const float* beta,
                         const float* initial_state, const int32_t* cu_seqlens,
                         const void* d_out, const float* d_final_state,
                         float scale, int chunk,
                         float* grad_q, float* grad_k, float* grad_v, float* grad_log_alpha,
                         float* grad_beta, float* grad_initial_state,
                         int B, int T, int H, int dk, int dv, int N,
                         kda_dtype dtype, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream);

/*
 * kda_chunk_bwd_workspace_bytes -- bytes of device workspace a kda_chunk_bwd
 * call with these sizes needs; `packed` is nonzero when the call passes
 * cu_seqlens.  0 for sizes the call would reject.
 */
size_t kda_chunk_bwd_workspace_bytes(int B, int T, int H, int N, int packed, kda_dtype dtype);

/*
 * kda_set_prefill_kernel -- which kernel the bf16 kda_chunk_fwd uses, for
 * tuning and testing; process-wide, set it while no kda_chunk_fwd call is
 * being made on another thread (and query the workspace size after it).
 *   0  automatic (default): one thread-block cluster per (sequence, head)
 *      chain when the chains are few enough that each gets two or more SMs
 *      (a chain CTA and 1-3 CTAs that prepare its chunks' operand tiles, see
 *      "深度解读报告" 3.1 for the split between per-chunk and carried work),
 *      segmented (below) when the chains are so few that it is estimated to
 *      be faster still, else one CTA per chain;
 *   1  always one CTA per chain;
 *   2  always one cluster per chain;
 *   3  always segmented: each sequence is cut into G segments of whole
 *      chunks.  The recurrence is affine in the state, so a segment maps its
 *      entry state to S_out = M S_in + B, M its dk x dk state transition (the
 *      segment run from the identity with v = 0) and B its exit state from a
 *      zero state.  A first pass of clusters runs segment 0 in full and M, B
 *      of segments 1 .. G-2 at once; a small fp32 pass chains the entry
 *      states S_in(g + 1) = M_g S_in(g) + B_g; a second pass runs segments
 *      1 .. G-1 from their entry states, so the sequential chain is about
 *      2/G of the sequence long instead of all of it.
 * All compute the same operator; results may differ in rounding only by the
 * order of fp32 accumulations inside a tensor-core product (and, segmented,
 * by the bf16 operands of the transition runs).
 * Returns KDA_ERR_INVALID_ARG for any other value.
 */
kda_status kda_set_prefill_kernel(int kind);

/*
 * kda_set_prefill_segments -- the segment count G of runs forced segmented
 * (kda_set_prefill_kernel(3)); 0 (default) chooses it by the cost model.
 * Process-wide, like kda_set_prefill_kernel.  KDA_ERR_INVALID_ARG unless 0
 * or 2 .. 4096.
 */
kda_status kda_set_prefill_segments(int segments);

/*
 * kda_set_prefill_dual -- layout of a segmented run's first pass, for tuning
 * and testing (process-wide, like kda_set_prefill_kernel): 0 (default) the
 * one the cost model prefers; 1 the zero-start and transition runs of a
 * segment in separate clusters; 2 both in one cluster whose two chain CTAs
 * share its prep CTAs (needs G >= 3).  KDA_ERR_INVALID_ARG for other values.
 */
kda_status kda_set_prefill_dual(int mode);

/*
 * kda_prefill_kernel_choice -- the kernel a bf16 kda_chunk_fwd call of these
 * sizes would use on the current device under the current setting: 1 (one
 * CTA per chain), 2 (one cluster per chain) or 3 (segmented); -1 for invalid
 * sizes.
 */
int kda_prefill_kernel_choice(int B, int T, int H, int N);

/*
 * kda_prefill_segments -- the segment count G such a call would use (1 when
 * it is not segmented); -1 for invalid sizes.
 */
int kda_prefill_segments(int B, int T, int H, int N);

/*
 * kda_selftest_wait_timeout -- test hook for the failure path of the
 * kernels' bounded waits; the pages have no counterpart.  Enqueues on
 * `stream` one CTA that waits, with the same wait routine as the
 * tensor-core kernels but a limit of `limit_us` microseconds (1 .. 10^6), on
 * an mbarrier that nothing arrives on.  The wait runs out, the kernel records
 * the timeout in the device error word and returns; the next
 * kda_device_error(stream) reports KDA_ERR_TIMEOUT (and clears it).  Nothing
 * faults and the context stays usable.  KDA_ERR_INVALID_ARG for a limit out
 * of range.
 */
kda_status kda_selftest_wait_timeout(int limit_us, cudaStream_t stream);

/* Number of floats kda_chunk_debug_stages writes to `stages`. */
int kda_chunk_debug_stage_floats(void);

/* Static, NUL-terminated description of a status code. */
const char* kda_status_string(kda_status status);

/*
 * kda_device_error -- synchronises `stream`, then reads and clears the
 * library's device-side error word on the current device.  Returns KDA_OK if
 * no kernel recorded an error since the last call, KDA_ERR_TIMEOUT if a
 * bounded internal wait ran out, KDA_ERR_CUDA if the synchronisation failed.
 */
kda_status kda_device_error(cudaStream_t stream);

/* Library version: major * 10000 + minor * 100 + patch. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_B200_KDA_H_ */
