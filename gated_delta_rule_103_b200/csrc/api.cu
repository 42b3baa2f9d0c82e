// C ABI of the KDA library: argument validation, dispatch to the kernels, the
// device error word and status strings.  See include/kda.h for the contract.
#include <cstdint>
#include <cstring>

#include "backward.h"
#include "kda_internal.h"

namespace {

// Error word written by kernels whose bounded waits run out.  One copy per
// device (a __device__ variable is instantiated on every device that loads
// the module).
__device__ unsigned g_kda_error_word = 0u;

constexpr int kMaxDevices = 64;
unsigned* g_err_ptr[kMaxDevices] = {};

// Device address of the error word on the current device (looked up once).
unsigned* error_word_ptr()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    if (!g_err_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_kda_error_word) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<unsigned*>(p);
    }
    return g_err_ptr[dev];
}

// A pointer the kernels may dereference: device (or managed) memory of the
// current device, 16-byte aligned.
bool device_ptr_ok(const void* p)
{
    if (!p) return false;
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return false;
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
        cudaGetLastError();  // clear the sticky-free error state
        return false;
    }
    if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged) return false;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    return attr.type == cudaMemoryTypeManaged || attr.device == dev;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb)
{
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

size_t elem_size(kda_dtype d) { return d == KDA_DTYPE_BF16 ? 2 : 4; }

struct Region {
    const void* p;
    size_t n;
};

// The caller's workspace for a call that needs `need` bytes: device memory of
// the current device, 256-byte aligned, large enough, overlapping none of the
// call's tensors.  A call that needs none ignores it.
bool workspace_ok(const void* ws, size_t ws_bytes, size_t need, const Region* r, int nr)
{
    if (need == 0) return true;
    if (!ws || ws_bytes < need || reinterpret_cast<uintptr_t>(ws) % 256 != 0) return false;
    if (!device_ptr_ok(ws)) return false;
    for (int i = 0; i < nr; ++i)
        if (overlaps(ws, need, r[i].p, r[i].n)) return false;
    return true;
}

// Device workspace of a bf16 prefill: the cluster kernel's hand-off ring
// (and the segment states of a segmented run), or nothing for the one-CTA
// kernel.
size_t fwd_workspace(const kda::ChunkArgs& a, kda_dtype dtype)
{
    if (dtype != KDA_DTYPE_BF16) return 0;
    const kda::PrefillPlan pl = kda::plan_prefill(a);
    return pl.kind == 1 ? 0 : pl.ring_bytes + pl.seg_bytes;
}

}  // namespace

extern "C" {

const char* kda_status_string(kda_status s)
{
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: invalid argument";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: unsupported size, chunk or dtype";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA call or kernel launch failed";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a kernel's bounded wait ran out";
    }
    return "KDA_ERR_UNKNOWN";
}

int kda_version(void) { return 1 * 10000 + 0 * 100 + 0; }

kda_status kda_device_error(cudaStream_t stream)
{
    if (cudaStreamSynchronize(stream) != cudaSuccess) return KDA_ERR_CUDA;
    unsigned word = 0;
    if (cudaMemcpyFromSymbol(&word, g_kda_error_word, sizeof(word)) != cudaSuccess)
        return KDA_ERR_CUDA;
    if (word) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_kda_error_word, &zero, sizeof(zero)) != cudaSuccess)
            return KDA_ERR_CUDA;
    }
    return (word & kda::kErrTimeout) ? KDA_ERR_TIMEOUT : KDA_OK;
}

kda_status kda_chunk_fwd_ex(const void* q, const void* k, const void* v,
                            const float* log_alpha, const float* beta,
                            const float* initial_state, const int32_t* cu_seqlens,
                            float scale, int chunk,
                            void* out, float* final_state,
                            int B, int T, int H, int dk, int dv, int N,
                            kda_dtype dtype, unsigned flags, const void* out_gate,
                            const float* out_weight, float out_eps,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream)
{
    if (flags & ~(unsigned)(KDA_FLAG_L2NORM_QK | KDA_FLAG_OUT_NORM_GATE | KDA_FLAG_RAW_GATE))
        return KDA_ERR_UNSUPPORTED;
    const bool norm_gate = (flags & KDA_FLAG_OUT_NORM_GATE) != 0;
    if (norm_gate && !(out_eps > 0.f && out_eps < 1e30f)) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || H <= 0 || N < 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (dk != kda::kDk || dv != kda::kDv || chunk != kda::kChunk) return KDA_ERR_UNSUPPORTED;
    if (cu_seqlens) {
        if (B != 1) return KDA_ERR_INVALID_ARG;
    } else if (N != B) {
        return KDA_ERR_INVALID_ARG;
    }
    if (!(scale == scale)) return KDA_ERR_INVALID_ARG;  // NaN
    const size_t tokens = (size_t)B * (size_t)T;
    if (tokens * (size_t)H > (size_t)INT32_MAX * 64) return KDA_ERR_UNSUPPORTED;
    const size_t units = (size_t)N * (size_t)H;
    if (units > (size_t)INT32_MAX / 4) return KDA_ERR_UNSUPPORTED;

    const size_t es = elem_size(dtype);
    const size_t n_qk = tokens * H * dk, n_v = tokens * H * dv, n_b = tokens * H;
    const size_t n_s = units * dk * dv;
    if (tokens > 0) {
        if (!device_ptr_ok(q) || !device_ptr_ok(k) || !device_ptr_ok(v) ||
            !device_ptr_ok(log_alpha) || !device_ptr_ok(beta) || !device_ptr_ok(out))
            return KDA_ERR_INVALID_ARG;
    } else if (units == 0) {
        return KDA_OK;
    }
    if (cu_seqlens && !device_ptr_ok(cu_seqlens)) return KDA_ERR_INVALID_ARG;
    if (initial_state && !device_ptr_ok(initial_state)) return KDA_ERR_INVALID_ARG;
    if (final_state && !device_ptr_ok(final_state)) return KDA_ERR_INVALID_ARG;
    if (norm_gate && tokens > 0 &&
        (!device_ptr_ok(out_gate) || !device_ptr_ok(out_weight) ||
         overlaps(out, n_v * es, out_gate, n_v * es) || overlaps(out, n_v * es, out_weight, (size_t)dv * 4)))
        return KDA_ERR_INVALID_ARG;
    // out must not alias any input; final_state may only equal initial_state.
    const size_t out_bytes = n_v * es;
    if (overlaps(out, out_bytes, q, n_qk * es) || overlaps(out, out_bytes, k, n_qk * es) ||
        overlaps(out, out_bytes, v, n_v * es) || overlaps(out, out_bytes, log_alpha, n_qk * 4) ||
        overlaps(out, out_bytes, beta, n_b * 4) ||
        overlaps(out, out_bytes, initial_state, n_s * 4) ||
        overlaps(out, out_bytes, final_state, n_s * 4))
        return KDA_ERR_INVALID_ARG;
    if (final_state && final_state != initial_state &&
        overlaps(final_state, n_s * 4, initial_state, n_s * 4))
        return KDA_ERR_INVALID_ARG;
    if (final_state &&
        (overlaps(final_state, n_s * 4, q, n_qk * es) || overlaps(final_state, n_s * 4, k, n_qk * es) ||
         overlaps(final_state, n_s * 4, v, n_v * es) ||
         overlaps(final_state, n_s * 4, log_alpha, n_qk * 4) ||
         overlaps(final_state, n_s * 4, beta, n_b * 4)))
        return KDA_ERR_INVALID_ARG;

    unsigned* err = error_word_ptr();
    if (!err) return KDA_ERR_CUDA;
    kda::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.initial_state = initial_state; a.cu_seqlens = cu_seqlens;
    a.out = out; a.final_state = final_state; a.scale = scale;
    a.B = B; a.T = T; a.H = H; a.N = N; a.err = err;
    a.l2norm = (flags & KDA_FLAG_L2NORM_QK) ? 1 : 0;
    a.raw_gate = (flags & KDA_FLAG_RAW_GATE) ? 1 : 0;
    {
        const Region r[10] = {{q, n_qk * es}, {k, n_qk * es}, {v, n_v * es}, {log_alpha, n_qk * 4},
                              {beta, n_b * 4}, {initial_state, n_s * 4}, {final_state, n_s * 4},
                              {out, out_bytes}, {norm_gate ? out_gate : nullptr, n_v * es},
                              {norm_gate ? out_weight : nullptr, (size_t)dv * 4}};
        if (!workspace_ok(workspace, workspace_bytes, fwd_workspace(a, dtype), r, 10))
            return KDA_ERR_INVALID_ARG;
    }
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    cudaError_t e;
    if (dtype == KDA_DTYPE_BF16) {
        // Few chains: clusters (segmented for very few); otherwise one CTA per chain.
        const kda::PrefillPlan pl = kda::plan_prefill(a);
        e = pl.kind == 1 ? kda::launch_chunk_tc(a, stream) : kda::launch_chunk_split(a, pl, stream);
    } else {
        e = kda::launch_chunk_simt(a, dtype, stream);
    }
    if (e == cudaSuccess && norm_gate)
        e = kda::launch_out_norm_gate(out, out_gate, out_weight, out_eps, (long long)tokens * H, dtype,
                                      stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                 const float* log_alpha, const float* beta,
                                 const float* initial_state, const int32_t* cu_seqlens,
                                 float scale, int chunk,
                                 void* out, float* final_state,
                                 int B, int T, int H, int dk, int dv, int N,
                                 kda_dtype dtype, cudaStream_t stream)
{
    // For callers that may not allocate device memory during the call (see
    // kda.h): the same checks as kda_chunk_fwd, then the cluster kernel on
    // the library's fixed ring array.  Nothing here allocates.
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || H <= 0 || N < 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_DTYPE_BF16) return KDA_ERR_UNSUPPORTED;
    if (dk != kda::kDk || dv != kda::kDv || chunk != kda::kChunk) return KDA_ERR_UNSUPPORTED;
    if (cu_seqlens) {
        if (B != 1) return KDA_ERR_INVALID_ARG;
    } else if (N != B) {
        return KDA_ERR_INVALID_ARG;
    }
    if (!(scale == scale)) return KDA_ERR_INVALID_ARG;
    const size_t tokens = (size_t)B * (size_t)T;
    const size_t units = (size_t)N * (size_t)H;
    if (tokens * (size_t)H > (size_t)INT32_MAX * 64) return KDA_ERR_UNSUPPORTED;
    if (!kda::noalloc_ring_fits((long long)units)) return KDA_ERR_UNSUPPORTED;

    const size_t es = 2;
    const size_t n_qk = tokens * H * dk, n_v = tokens * H * dv, n_b = tokens * H;
    const size_t n_s = units * dk * dv;
    if (tokens > 0) {
        if (!device_ptr_ok(q) || !device_ptr_ok(k) || !device_ptr_ok(v) ||
            !device_ptr_ok(log_alpha) || !device_ptr_ok(beta) || !device_ptr_ok(out))
            return KDA_ERR_INVALID_ARG;
    } else if (units == 0) {
        return KDA_OK;
    }
    if (cu_seqlens && !device_ptr_ok(cu_seqlens)) return KDA_ERR_INVALID_ARG;
    if (initial_state && !device_ptr_ok(initial_state)) return KDA_ERR_INVALID_ARG;
    if (final_state && !device_ptr_ok(final_state)) return KDA_ERR_INVALID_ARG;
    const size_t out_bytes = n_v * es;
    if (overlaps(out, out_bytes, q, n_qk * es) || overlaps(out, out_bytes, k, n_qk * es) ||
        overlaps(out, out_bytes, v, n_v * es) || overlaps(out, out_bytes, log_alpha, n_qk * 4) ||
        overlaps(out, out_bytes, beta, n_b * 4) ||
        overlaps(out, out_bytes, initial_state, n_s * 4) ||
        overlaps(out, out_bytes, final_state, n_s * 4))
        return KDA_ERR_INVALID_ARG;
    if (final_state && final_state != initial_state &&
        overlaps(final_state, n_s * 4, initial_state, n_s * 4))
        return KDA_ERR_INVALID_ARG;
    if (final_state &&
        (overlaps(final_state, n_s * 4, q, n_qk * es) || overlaps(final_state, n_s * 4, k, n_qk * es) ||
         overlaps(final_state, n_s * 4, v, n_v * es) ||
         overlaps(final_state, n_s * 4, log_alpha, n_qk * 4) ||
         overlaps(final_state, n_s * 4, beta, n_b * 4)))
        return KDA_ERR_INVALID_ARG;

    unsigned* err = error_word_ptr();
    if (!err) return KDA_ERR_CUDA;
    kda::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.initial_state = initial_state; a.cu_seqlens = cu_seqlens;
    a.out = out; a.final_state = final_state; a.scale = scale;
    a.B = B; a.T = T; a.H = H; a.N = N; a.err = err;
    // no tokens: only the states pass through (the FFMA kernel, no ring)
    const cudaError_t e = tokens == 0 ? kda::launch_chunk_simt(a, dtype, stream)
                                      : kda::launch_chunk_split_noalloc(a, stream);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

size_t kda_chunk_transition_workspace_bytes(int B, int T, int H, int N, kda_dtype dtype)
{
    if (dtype != KDA_DTYPE_BF16 || B < 0 || T < 0 || H <= 0 || N < 0) return 0;
    kda::ChunkArgs a = {};
    a.B = B; a.T = T; a.H = H; a.N = N;
    return kda::transition_workspace_bytes(a);
}

kda_status kda_chunk_transition(const void* q, const void* k, const float* log_alpha,
                                const float* beta, const int32_t* cu_seqlens, float* transition,
                                int B, int T, int H, int dk, int N, kda_dtype dtype,
                                unsigned flags, void* workspace, size_t workspace_bytes,
                                cudaStream_t stream)
{
    if (flags & ~(unsigned)(KDA_FLAG_L2NORM_QK | KDA_FLAG_RAW_GATE)) return KDA_ERR_UNSUPPORTED;
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || H <= 0 || N < 0 || dk <= 0) return KDA_ERR_INVALID_ARG;
    if (dk != kda::kDk || dtype != KDA_DTYPE_BF16) return KDA_ERR_UNSUPPORTED;
    if (cu_seqlens) {
        if (B != 1) return KDA_ERR_INVALID_ARG;
    } else if (N != B) {
        return KDA_ERR_INVALID_ARG;
    }
    const size_t tokens = (size_t)B * (size_t)T;
    if (tokens * (size_t)H > (size_t)INT32_MAX * 64) return KDA_ERR_UNSUPPORTED;
    const size_t units = (size_t)N * (size_t)H;
    if (units > (size_t)INT32_MAX / 4) return KDA_ERR_UNSUPPORTED;
    if (units == 0) return KDA_OK;
    const size_t n_qk = tokens * H * dk, n_b = tokens * H, n_m = units * dk * dk;
    if (!device_ptr_ok(transition)) return KDA_ERR_INVALID_ARG;
    if (tokens > 0 && (!device_ptr_ok(k) || !device_ptr_ok(log_alpha) || !device_ptr_ok(beta) ||
                       ((flags & KDA_FLAG_L2NORM_QK) && !device_ptr_ok(q))))
        return KDA_ERR_INVALID_ARG;
    if (cu_seqlens && !device_ptr_ok(cu_seqlens)) return KDA_ERR_INVALID_ARG;
    if (overlaps(transition, n_m * 4, q, n_qk * 2) || overlaps(transition, n_m * 4, k, n_qk * 2) ||
        overlaps(transition, n_m * 4, log_alpha, n_qk * 4) || overlaps(transition, n_m * 4, beta, n_b * 4))
        return KDA_ERR_INVALID_ARG;
    unsigned* err = error_word_ptr();
    if (!err) return KDA_ERR_CUDA;
    kda::ChunkArgs a;
    // q only matters for its tensor map (and the L2Norm, which does not change M)
    a.q = q ? q : k; a.k = k; a.v = nullptr; a.log_alpha = log_alpha; a.beta = beta;
    a.initial_state = nullptr; a.cu_seqlens = cu_seqlens;
    a.out = nullptr; a.final_state = nullptr; a.scale = 1.f;
    a.B = B; a.T = T; a.H = H; a.N = N; a.err = err;
    a.l2norm = (flags & KDA_FLAG_L2NORM_QK) ? 1 : 0;
    a.raw_gate = (flags & KDA_FLAG_RAW_GATE) ? 1 : 0;
    if (tokens == 0) {
        // empty sequences: M = I
        return kda::launch_identity_states(transition, (long long)units, stream) == cudaSuccess
                   ? KDA_OK : KDA_ERR_CUDA;
    }
    {
        const Region r[4] = {{q, n_qk * 2}, {k, n_qk * 2}, {log_alpha, n_qk * 4}, {beta, n_b * 4}};
        const Region r2[1] = {{transition, n_m * 4}};
        const size_t need = kda::transition_workspace_bytes(a);
        if (!workspace_ok(workspace, workspace_bytes, need, r, 4) ||
            !workspace_ok(workspace, workspace_bytes, need, r2, 1))
            return KDA_ERR_INVALID_ARG;
    }
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    return kda::launch_chunk_transition(a, transition, stream) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_state_affine(const float* M, const float* B, const float* S_in, float* S_out,
                            int N, int H, int dk, int dv, cudaStream_t stream)
{
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (dk != kda::kDk || dv != kda::kDv) return KDA_ERR_UNSUPPORTED;
    const size_t units = (size_t)N * (size_t)H;
    if (units == 0) return KDA_OK;
    if (units > (size_t)INT32_MAX) return KDA_ERR_UNSUPPORTED;
    if (!device_ptr_ok(M) || !device_ptr_ok(B) || !device_ptr_ok(S_in) || !device_ptr_ok(S_out))
        return KDA_ERR_INVALID_ARG;
    const size_t n_s = units * dk * dv * 4, n_m = units * dk * dk * 4;
    if (overlaps(S_out, n_s, M, n_m) || overlaps(S_out, n_s, S_in, n_s) ||
        (S_out != B && overlaps(S_out, n_s, B, n_s)))
        return KDA_ERR_INVALID_ARG;
    return kda::launch_state_affine(M, B, S_in, S_out, (long long)units, stream) == cudaSuccess
               ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_selftest_wait_timeout(int limit_us, cudaStream_t stream)
{
    if (limit_us < 1 || limit_us > 1000000) return KDA_ERR_INVALID_ARG;
    unsigned* err = error_word_ptr();
    if (!err) return KDA_ERR_CUDA;
    return kda::launch_wait_selftest(err, 1000ull * (unsigned long long)limit_us, stream) == cudaSuccess
               ? KDA_OK : KDA_ERR_CUDA;
}

size_t kda_chunk_fwd_workspace_bytes(int B, int T, int H, int N, kda_dtype dtype)
{
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return 0;
    if (B < 0 || T < 0 || H <= 0 || N < 0) return 0;
    kda::ChunkArgs a = {};
    a.B = B; a.T = T; a.H = H; a.N = N;
    return fwd_workspace(a, dtype);
}

size_t kda_chunk_bwd_workspace_bytes(int B, int T, int H, int N, int packed, kda_dtype dtype)
{
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return 0;
    if (B < 0 || T < 0 || H <= 0 || N < 0) return 0;
    if ((long long)N * H == 0) return 0;
    return kda::bwd_workspace_layout(B, T, H, N, packed != 0).total;
}

int kda_prefill_kernel_choice(int B, int T, int H, int N)
{
    if (B < 0 || T < 0 || H <= 0 || N < 0) return -1;
    kda::ChunkArgs a = {};
    a.B = B; a.T = T; a.H = H; a.N = N;
    return kda::plan_prefill(a).kind;
}

int kda_prefill_segments(int B, int T, int H, int N)
{
    if (B < 0 || T < 0 || H <= 0 || N < 0) return -1;
    kda::ChunkArgs a = {};
    a.B = B; a.T = T; a.H = H; a.N = N;
    const kda::PrefillPlan pl = kda::plan_prefill(a);
    return pl.kind == 3 ? pl.G : 1;
}

kda_status kda_set_prefill_dual(int mode)
{
    if (mode < 0 || mode > 2) return KDA_ERR_INVALID_ARG;
    kda::set_prefill_dual(mode);
    return KDA_OK;
}

kda_status kda_set_prefill_segments(int segments)
{
    if (segments != 0 && (segments < 2 || segments > 4096)) return KDA_ERR_INVALID_ARG;
    kda::set_prefill_segments(segments);
    return KDA_OK;
}

kda_status kda_chunk_fwd(const void* q, const void* k, const void* v,
                         const float* log_alpha, const float* beta,
                         const float* initial_state, const int32_t* cu_seqlens,
                         float scale, int chunk,
                         void* out, float* final_state,
                         int B, int T, int H, int dk, int dv, int N,
                         kda_dtype dtype, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream)
{
    return kda_chunk_fwd_ex(q, k, v, log_alpha, beta, initial_state, cu_seqlens, scale, chunk,
                            out, final_state, B, T, H, dk, dv, N, dtype, 0u, nullptr, nullptr, 0.f,
                            workspace, workspace_bytes, stream);
}

kda_status kda_chunk_bwd(const void* q, const void* k, const void* v,
                         const float* log_alpha, const float* beta,
                         const float* initial_state, const int32_t* cu_seqlens,
                         const void* d_out, const float* d_final_state,
                         float scale, int chunk,
                         float* grad_q, float* grad_k, float* grad_v, float* grad_log_alpha,
                         float* grad_beta, float* grad_initial_state,
                         int B, int T, int H, int dk, int dv, int N,
                         kda_dtype dtype, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream)
{
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || H <= 0 || N < 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (dk != kda::kDk || dv != kda::kDv || chunk != kda::kChunk) return KDA_ERR_UNSUPPORTED;
    if (cu_seqlens) {
        if (B != 1) return KDA_ERR_INVALID_ARG;
    } else if (N != B) {
        return KDA_ERR_INVALID_ARG;
    }
    if (!(scale == scale)) return KDA_ERR_INVALID_ARG;  // NaN
    const size_t tokens = (size_t)B * (size_t)T;
    if (tokens * (size_t)H > (size_t)INT32_MAX * 64) return KDA_ERR_UNSUPPORTED;
    const size_t units = (size_t)N * (size_t)H;
    if (units > (size_t)INT32_MAX / 4) return KDA_ERR_UNSUPPORTED;
    if ((long long)kda::chunk_slots_bound(B, T, N, cu_seqlens != nullptr) * H > (long long)INT32_MAX)
        return KDA_ERR_UNSUPPORTED;

    const size_t es = elem_size(dtype);
    const size_t n_qk = tokens * H * dk, n_v = tokens * H * dv, n_b = tokens * H;
    const size_t n_s = units * dk * dv;
    if (tokens > 0) {
        if (!device_ptr_ok(q) || !device_ptr_ok(k) || !device_ptr_ok(v) ||
            !device_ptr_ok(log_alpha) || !device_ptr_ok(beta) || !device_ptr_ok(d_out) ||
            !device_ptr_ok(grad_q) || !device_ptr_ok(grad_k) || !device_ptr_ok(grad_v) ||
            !device_ptr_ok(grad_log_alpha) || !device_ptr_ok(grad_beta))
            return KDA_ERR_INVALID_ARG;
    } else if (units == 0) {
        return KDA_OK;
    }
    if (cu_seqlens && !device_ptr_ok(cu_seqlens)) return KDA_ERR_INVALID_ARG;
    if (initial_state && !device_ptr_ok(initial_state)) return KDA_ERR_INVALID_ARG;
    if (d_final_state && !device_ptr_ok(d_final_state)) return KDA_ERR_INVALID_ARG;
    if (grad_initial_state && !device_ptr_ok(grad_initial_state)) return KDA_ERR_INVALID_ARG;
    // no output may overlap another output or an input
    const void* outs[6] = {grad_q, grad_k, grad_v, grad_log_alpha, grad_beta, grad_initial_state};
    const size_t out_n[6] = {n_qk * 4, n_qk * 4, n_v * 4, n_qk * 4, n_b * 4, n_s * 4};
    const void* ins[8] = {q, k, v, log_alpha, beta, initial_state, d_out, d_final_state};
    const size_t in_n[8] = {n_qk * es, n_qk * es, n_v * es, n_qk * 4, n_b * 4, n_s * 4, n_v * es, n_s * 4};
    for (int i = 0; i < 6; ++i) {
        if (!outs[i] || out_n[i] == 0) continue;
        for (int j = 0; j < 8; ++j)
            if (overlaps(outs[i], out_n[i], ins[j], in_n[j])) return KDA_ERR_INVALID_ARG;
        for (int j = i + 1; j < 6; ++j)
            if (overlaps(outs[i], out_n[i], outs[j], out_n[j])) return KDA_ERR_INVALID_ARG;
    }
    {
        Region r[14];
        for (int i = 0; i < 6; ++i) r[i] = {outs[i], out_n[i]};
        for (int j = 0; j < 8; ++j) r[6 + j] = {ins[j], in_n[j]};
        const size_t need = kda::bwd_workspace_layout(B, T, H, N, cu_seqlens != nullptr).total;
        if (!workspace_ok(workspace, workspace_bytes, need, r, 14)) return KDA_ERR_INVALID_ARG;
    }

    unsigned* err = error_word_ptr();
    if (!err) return KDA_ERR_CUDA;
    kda::BwdArgs b;
    kda::ChunkArgs& a = b.fwd;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.initial_state = initial_state; a.cu_seqlens = cu_seqlens;
    a.out = nullptr; a.final_state = nullptr; a.scale = scale;
    a.B = B; a.T = T; a.H = H; a.N = N; a.err = err;
    b.d_out = d_out; b.d_final_state = d_final_state;
    b.dq = grad_q; b.dk = grad_k; b.dv = grad_v; b.dlog_alpha = grad_log_alpha;
    b.dbeta = grad_beta; b.d_initial_state = grad_initial_state;
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    return kda::launch_chunk_bwd(b, dtype, stream) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_set_prefill_kernel(int kind)
{
    if (kind < 0 || kind > 3) return KDA_ERR_INVALID_ARG;
    kda::set_prefill_kernel(kind);
    return KDA_OK;
}

int kda_chunk_debug_stage_floats(void) { return kda::chunk_tc_debug_floats(); }

kda_status kda_chunk_debug_stages(const void* q, const void* k, const void* v,
                                  const float* log_alpha, const float* beta,
                                  const float* initial_state, float scale, int T,
                                  void* out, float* final_state, float* stages,
                                  cudaStream_t stream)
{
    if (T < 1 || T > kda::kChunk) return KDA_ERR_UNSUPPORTED;
    if (!(scale == scale)) return KDA_ERR_INVALID_ARG;
    if (!device_ptr_ok(q) || !device_ptr_ok(k) || !device_ptr_ok(v) ||
        !device_ptr_ok(log_alpha) || !device_ptr_ok(beta) || !device_ptr_ok(out) ||
        !device_ptr_ok(final_state) || !device_ptr_ok(stages))
        return KDA_ERR_INVALID_ARG;
    if (initial_state && !device_ptr_ok(initial_state)) return KDA_ERR_INVALID_ARG;
    const size_t sb = (size_t)kda::chunk_tc_debug_floats() * 4;
    if (overlaps(stages, sb, q, (size_t)T * 256) || overlaps(stages, sb, k, (size_t)T * 256) ||
        overlaps(stages, sb, v, (size_t)T * 256) || overlaps(stages, sb, out, (size_t)T * 256) ||
        overlaps(stages, sb, final_state, 65536) || overlaps(out, (size_t)T * 256, q, (size_t)T * 256) ||
        overlaps(out, (size_t)T * 256, k, (size_t)T * 256) || overlaps(out, (size_t)T * 256, v, (size_t)T * 256))
        return KDA_ERR_INVALID_ARG;
    unsigned* err = error_word_ptr();
    if (!err) return KDA_ERR_CUDA;
    kda::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.initial_state = initial_state; a.cu_seqlens = nullptr;
    a.out = out; a.final_state = final_state; a.scale = scale;
    a.B = 1; a.T = T; a.H = 1; a.N = 1; a.err = err;
    return kda::launch_chunk_tc_debug(a, stages, stream) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_recurrent_step_ex(const void* q, const void* k, const void* v,
                                 const float* log_alpha, const float* beta,
                                 float* state, void* out,
                                 int N, int H, int dk, int dv, float scale,
                                 kda_dtype dtype, unsigned flags, const void* out_gate,
                                 const float* out_weight, float out_eps, cudaStream_t stream)
{
    if (flags & ~(unsigned)(KDA_FLAG_L2NORM_QK | KDA_FLAG_OUT_NORM_GATE | KDA_FLAG_RAW_GATE))
        return KDA_ERR_UNSUPPORTED;
    const bool norm_gate = (flags & KDA_FLAG_OUT_NORM_GATE) != 0;
    if (norm_gate && !(out_eps > 0.f && out_eps < 1e30f)) return KDA_ERR_INVALID_ARG;
    if (dtype != KDA_DTYPE_F32 && dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARG;
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return KDA_ERR_INVALID_ARG;
    if (dk != kda::kDk || dv != kda::kDv) return KDA_ERR_UNSUPPORTED;
    if (!(scale == scale)) return KDA_ERR_INVALID_ARG;
    const size_t units = (size_t)N * (size_t)H;
    if (units == 0) return KDA_OK;
    if (units > (size_t)INT32_MAX) return KDA_ERR_UNSUPPORTED;
    if (!device_ptr_ok(q) || !device_ptr_ok(k) || !device_ptr_ok(v) ||
        !device_ptr_ok(log_alpha) || !device_ptr_ok(beta) || !device_ptr_ok(state) ||
        !device_ptr_ok(out))
        return KDA_ERR_INVALID_ARG;
    const size_t es = elem_size(dtype);
    const size_t n_s = units * dk * dv * 4, n_o = units * dv * es;
    if (overlaps(state, n_s, q, units * dk * es) || overlaps(state, n_s, k, units * dk * es) ||
        overlaps(state, n_s, v, units * dv * es) || overlaps(state, n_s, log_alpha, units * dk * 4) ||
        overlaps(state, n_s, beta, units * 4) || overlaps(state, n_s, out, n_o) ||
        overlaps(out, n_o, q, units * dk * es) || overlaps(out, n_o, k, units * dk * es) ||
        overlaps(out, n_o, v, units * dv * es) || overlaps(out, n_o, log_alpha, units * dk * 4) ||
        overlaps(out, n_o, beta, units * 4))
        return KDA_ERR_INVALID_ARG;
    if (norm_gate && (!device_ptr_ok(out_gate) || !device_ptr_ok(out_weight) ||
                      overlaps(out, n_o, out_gate, n_o) || overlaps(state, n_s, out_gate, n_o) ||
                      overlaps(out, n_o, out_weight, (size_t)dv * 4)))
        return KDA_ERR_INVALID_ARG;
    unsigned* err = error_word_ptr();
    if (!err) return KDA_ERR_CUDA;
    kda::DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.log_alpha = log_alpha; a.beta = beta;
    a.state = state; a.out = out; a.scale = scale; a.N = N; a.H = H; a.err = err;
    a.l2norm = (flags & KDA_FLAG_L2NORM_QK) ? 1 : 0;
    a.raw_gate = (flags & KDA_FLAG_RAW_GATE) ? 1 : 0;
    if (norm_gate) {
        a.out_gate = out_gate;
        a.out_weight = out_weight;
        a.out_eps = out_eps;
    }
    return kda::launch_decode(a, dtype, stream) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_recurrent_step(const void* q, const void* k, const void* v,
                              const float* log_alpha, const float* beta,
                              float* state, void* out,
                              int N, int H, int dk, int dv, float scale,
                              kda_dtype dtype, cudaStream_t stream)
{
    return kda_recurrent_step_ex(q, k, v, log_alpha, beta, state, out, N, H, dk, dv, scale,
                                 dtype, 0u, nullptr, nullptr, 0.f, stream);
}

}  // extern "C"
