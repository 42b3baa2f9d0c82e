// Internal launcher interface between the C ABI (api.cu) and the kernels.
// Arguments have already been validated by the caller; launchers only pick a
// launch configuration and enqueue on `stream`.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/kda.h"

namespace kda {

// Sizes the kernels are specialised for.
constexpr int kDk = 128;
constexpr int kDv = 128;
constexpr int kChunk = 64;

// Error-word bits written by kernels (read and cleared by kda_device_error).
constexpr unsigned kErrTimeout = 1u;

struct ChunkArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* log_alpha;
    const float* beta;
    const float* initial_state;
    const int32_t* cu_seqlens;  // nullptr: sequence n is batch row n
    void* out;
    float* final_state;
    float scale;
    int B, T, H, N;
    unsigned* err;              // device error word
    int l2norm = 0;             // L2-normalise the q and k rows first (KDA_FLAG_L2NORM_QK)
    int raw_gate = 0;           // log_alpha holds gate pre-activations (KDA_FLAG_RAW_GATE)
    void* workspace = nullptr;  // caller-owned device scratch (256-byte aligned)
    size_t workspace_bytes = 0;
};

struct DecodeArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* log_alpha;
    const float* beta;
    float* state;
    void* out;
    float scale;
    int N, H;
    unsigned* err;
    int l2norm = 0;             // L2-normalise the q and k rows first (KDA_FLAG_L2NORM_QK)
    int raw_gate = 0;           // log_alpha holds gate pre-activations (KDA_FLAG_RAW_GATE)
    const void* out_gate = nullptr;     // output RMSNorm + sigmoid gate (KDA_FLAG_OUT_NORM_GATE)
    const float* out_weight = nullptr;
    float out_eps = 0.f;
};

cudaError_t launch_decode(const DecodeArgs& a, kda_dtype dtype, cudaStream_t stream);
cudaError_t launch_chunk_simt(const ChunkArgs& a, kda_dtype dtype, cudaStream_t stream);
cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t stream);
// How a bf16 prefill runs (by the chain count, the sequence length and the
// device's SMs, unless set_prefill_kernel forced a kind):
//   kind 1  one CTA per (sequence, head) chain;
//   kind 2  one thread-block cluster per chain: a chain CTA and P (1..3)
//           CTAs that prepare its chunks' operand tiles, handed over through
//           a ring in the caller's workspace;
//   kind 3  segmented: every sequence cut into G segments; a first pass of
//           clusters (P1 prep CTAs) runs segment 0 and the state transition
//           and zero-start exit state of segments 1 .. G-2, a prefix pass
//           chains the segments' entry states, a second pass (P3) runs
//           segments 1 .. G-1.
struct PrefillPlan {
    int kind = 1;
    int P = 0;
    int G = 0, P1 = 0, P3 = 0;
    bool dual = false;         // kind 3: first pass with two chain CTAs per cluster
    size_t ring_bytes = 0;     // workspace: ring, then
    size_t seg_bytes = 0;      //   the segment states
};
PrefillPlan plan_prefill(const ChunkArgs& a);
cudaError_t launch_chunk_split(const ChunkArgs& a, const PrefillPlan& plan, cudaStream_t stream);
size_t split_ring_bytes(long long chains, int prep);
// The state transition M [N][H][dk][dk] of every (sequence, head): the cluster
// kernel from the identity with v = 0 and no outputs (bf16 operands), its
// ring in a.workspace (transition_workspace_bytes(a) bytes).
size_t transition_workspace_bytes(const ChunkArgs& a);
cudaError_t launch_chunk_transition(const ChunkArgs& a, float* transition, cudaStream_t stream);
// `units` [dk][dk] identity matrices.
cudaError_t launch_identity_states(float* M, long long units, cudaStream_t stream);
// S_out = M S_in + B for `chains` fp32 [dk][dv] states (M [dk][dk] each).
cudaError_t launch_state_affine(const float* M, const float* B, const float* S_in, float* S_out,
                                long long chains, cudaStream_t stream);
// Prep CTAs per cluster of a kind-2 plan, else 0.
int split_prep_ctas(const ChunkArgs& a);
// 0 automatic, 1 one CTA per chain, 2 one cluster per chain, 3 segmented.
void set_prefill_kernel(int kind);
// Segments of a forced segmented run (0: by the cost model).
void set_prefill_segments(int segments);
// First pass of a segmented run: 0 the cheaper layout, 1 separate clusters for
// the zero-start and transition runs, 2 one cluster with two chain CTAs.
void set_prefill_dual(int mode);
// The cluster kernel with its hand-off ring in a fixed 16 MiB device array of
// the library (no allocation): for kda_chunk_fwd_noalloc.
bool noalloc_ring_fits(long long chains);
cudaError_t launch_chunk_split_noalloc(const ChunkArgs& a, cudaStream_t stream);
// Same kernel, instantiated to dump the first chunk's intermediates of the
// first (sequence, head) into `stages` (chunk_tc_debug_floats() floats).
cudaError_t launch_chunk_tc_debug(const ChunkArgs& a, float* stages, cudaStream_t stream);
int chunk_tc_debug_floats();
// In place on out [rows][dv]: head-wise RMSNorm and the sigmoid output gate.
cudaError_t launch_out_norm_gate(void* out, const void* gate, const float* weight, float eps,
                                 long long rows, kda_dtype dtype, cudaStream_t stream);
// One CTA whose bounded mbarrier wait has nothing to wait for: it runs out
// after limit_ns and records kErrTimeout in *err.
cudaError_t launch_wait_selftest(unsigned* err, unsigned long long limit_ns, cudaStream_t stream);

}  // namespace kda
