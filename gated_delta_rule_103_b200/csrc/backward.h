// Backward pass of the chunked KDA operator: what the FFMA chunk kernel (which
// keeps the entry state of every chunk for it) and the backward kernels share.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"
#include "kda_internal.h"

namespace kda {

// First chunk slot of sequence n in the [slot][H][dk][dv] checkpoint arrays:
// the chunks of the sequences before it, ceil(len / 64) each.
__device__ __forceinline__ long long chunk_slot_offset(const int32_t* cu_seqlens, int T, int n)
{
    if (!cu_seqlens) return (long long)n * ((T + kChunk - 1) / kChunk);
    long long off = 0;
    for (int m = 0; m < n; ++m) off += (cu_seqlens[m + 1] - cu_seqlens[m] + kChunk - 1) / kChunk;
    return off;
}

// Upper bound on the number of chunk slots of B x T tokens in N sequences.
inline long long chunk_slots_bound(int B, int T, int N, bool varlen)
{
    const long long per = (T + kChunk - 1) / kChunk;
    return varlen ? per + N : (long long)B * per;
}

struct BwdArgs {
    ChunkArgs fwd;                 // the forward call's inputs (out, final_state unused)
    const void* d_out;             // [B,T,H,dv], the forward's dtype
    const float* d_final_state;    // [N,H,dk,dv] or nullptr (zero adjoint)
    float* dq;                     // [B,T,H,dk]
    float* dk;                     // [B,T,H,dk]
    float* dv;                     // [B,T,H,dv]
    float* dlog_alpha;             // [B,T,H,dk]
    float* dbeta;                  // [B,T,H]
    float* d_initial_state;        // [N,H,dk,dv] or nullptr
};

// The FFMA forward with the entry state of every chunk stored to `states`
// ([slot][H][dk][dv] fp32; nullptr: not stored).
cudaError_t launch_chunk_simt_states(const ChunkArgs& a, float* states, kda_dtype dtype,
                                     cudaStream_t stream);

// Layout of the backward pass's workspace: the entry state of every chunk
// slot and head, then the exit-state adjoints (state_bytes each), then dU
// [tokens][H][dv] fp32; each part 256-byte aligned.
struct BwdWorkspace {
    long long slots = 0;
    size_t state_bytes = 0;
    size_t du_bytes = 0;
    size_t total = 0;
};
BwdWorkspace bwd_workspace_layout(int B, int T, int H, int N, bool varlen);

// Forward recompute of the chunk states, then the reverse chain over the
// chunks and the per-chunk gradients, in the caller's workspace
// (a.fwd.workspace, bwd_workspace_layout(...).total bytes).
cudaError_t launch_chunk_bwd(const BwdArgs& a, kda_dtype dtype, cudaStream_t stream);

}  // namespace kda
