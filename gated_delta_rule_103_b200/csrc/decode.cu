// Batched KDA decode step: one token per (request, head), fp32 state updated
// in place with a single read and a single write of each state element.
//
// Per (n, h) with S in R^{128 x 128} (row c = key channel, column j = value):
//   S_bar = Diag(exp g) S                       (per-channel forget gate)
//   u     = beta (v - S_bar^T k)                (erase coefficient along k)
//   S'    = S_bar + k u^T      = (I - beta k k^T) S_bar + beta k v^T
//   o     = scale S'^T q       = scale (S_bar^T q + (q.k) u)
// (zhaixingw.cn ai-news/151, the gated delta update with a per-channel gate;
//  "深度解读报告" 2.3.)
//
// Memory-bound: 64 KiB read + 64 KiB written per head.  One CTA of 256
// threads per head.  Thread (warp w, lane l) owns columns 4l..4l+3 of rows
// w, w+8, ..., w+120: each warp reads and writes whole 512-byte rows with
// 16-byte vector accesses (streaming cache hints: the state is touched once).
#include <cuda_bf16.h>

#include "gate.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerThread = kDk / kWarps;  // 16

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 2)
kda_decode_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const float* __restrict__ log_alpha, const float* __restrict__ beta,
                  float* __restrict__ state, T* __restrict__ out, float scale, int l2norm,
                  int raw_gate, const T* __restrict__ out_gate, const float* __restrict__ out_weight,
                  float out_eps)
{
    const int nh = blockIdx.x;  // n * H + h
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float* S = state + (size_t)nh * kDk * kDv;

    // Issue every state load first so that 64 KiB per CTA are in flight.
    float4 s[kRowsPerThread];
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i)
        s[i] = __ldcs(reinterpret_cast<const float4*>(S + (size_t)(warp + kWarps * i) * kDv) + lane);

    __shared__ float sk[kDk], sq[kDk], sa[kDk];
    __shared__ float4 red_k[kWarps][kDv / 4], red_q[kWarps][kDv / 4];
    __shared__ float su[kDv];
    if (tid < kDk) {
        sk[tid] = to_f32(k[(size_t)nh * kDk + tid]);
        sq[tid] = to_f32(q[(size_t)nh * kDk + tid]);
        const float g = log_alpha[(size_t)nh * kDk + tid];
        sa[tid] = expf(raw_gate ? log_sigmoid(g) : g);
    }
    __syncthreads();
    if (l2norm) {
        // fused L2Norm of k (warp 0) and q (warp 1): x / max(||x||_2, 1e-6)
        __shared__ float inv_norm[2];
        if (warp < 2) {
            const float* x = warp == 0 ? sk : sq;
            float ss = 0.f;
#pragma unroll
            for (int c = lane; c < kDk; c += 32) ss = fmaf(x[c], x[c], ss);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            if (lane == 0) inv_norm[warp] = 1.f / fmaxf(sqrtf(ss), 1e-6f);
        }
        __syncthreads();
        if (tid < kDk) {
            sk[tid] *= inv_norm[0];
            sq[tid] *= inv_norm[1];
        }
        __syncthreads();
    }

    // q . k, reduced redundantly by every warp (4 products per lane).
    float qk = 0.f;
#pragma unroll
    for (int c = lane; c < kDk; c += 32) qk = fmaf(sq[c], sk[c], qk);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) qk += __shfl_xor_sync(0xffffffffu, qk, off);

    // Decay rows, and partial sums of S_bar^T k and S_bar^T q over this
    // thread's 16 rows.
    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
        const int r = warp + kWarps * i;
        const float a = sa[r], kr = sk[r], qr = sq[r];
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        pk.x = fmaf(s[i].x, kr, pk.x); pk.y = fmaf(s[i].y, kr, pk.y);
        pk.z = fmaf(s[i].z, kr, pk.z); pk.w = fmaf(s[i].w, kr, pk.w);
        pq.x = fmaf(s[i].x, qr, pq.x); pq.y = fmaf(s[i].y, qr, pq.y);
        pq.z = fmaf(s[i].z, qr, pq.z); pq.w = fmaf(s[i].w, qr, pq.w);
    }
    red_k[warp][lane] = pk;
    red_q[warp][lane] = pq;
    __syncthreads();

    float o = 0.f;
    if (tid < kDv) {
        const int j = tid;
        const float* rk = reinterpret_cast<const float*>(red_k);
        const float* rq = reinterpret_cast<const float*>(red_q);
        float pred = 0.f, oq = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            pred += rk[w * kDv + j];
            oq += rq[w * kDv + j];
        }
        const float u = beta[nh] * (to_f32(v[(size_t)nh * kDv + j]) - pred);
        su[j] = u;
        o = scale * fmaf(qk, u, oq);
    }
    if (out_gate) {
        // output epilogue: head-wise RMSNorm of the row and the sigmoid gate
        __shared__ float red_o[kDv / 32];
        float ss = o * o;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (tid < kDv && lane == 0) red_o[warp] = ss;
        __syncthreads();
        if (tid < kDv) {
            float tot = 0.f;
#pragma unroll
            for (int w = 0; w < kDv / 32; ++w) tot += red_o[w];
            const float g = to_f32(out_gate[(size_t)nh * kDv + tid]);
            o = o * rsqrtf(tot * (1.f / kDv) + out_eps) * out_weight[tid] / (1.f + __expf(-g));
        }
    }
    if (tid < kDv) out[(size_t)nh * kDv + tid] = from_f32<T>(o);
    __syncthreads();

    const float4 u4 = reinterpret_cast<const float4*>(su)[lane];
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
        const int r = warp + kWarps * i;
        const float kr = sk[r];
        float4 x = s[i];
        x.x = fmaf(kr, u4.x, x.x); x.y = fmaf(kr, u4.y, x.y);
        x.z = fmaf(kr, u4.z, x.z); x.w = fmaf(kr, u4.w, x.w);
        __stcs(reinterpret_cast<float4*>(S + (size_t)r * kDv) + lane, x);
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, kda_dtype dtype, cudaStream_t stream)
{
    const long long units = (long long)a.N * a.H;
    if (units == 0) return cudaSuccess;
    const dim3 grid((unsigned)units), block(kThreads);
    if (dtype == KDA_DTYPE_BF16) {
        kda_decode_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>(
            (const __nv_bfloat16*)a.q, (const __nv_bfloat16*)a.k, (const __nv_bfloat16*)a.v,
            a.log_alpha, a.beta, a.state, (__nv_bfloat16*)a.out, a.scale, a.l2norm, a.raw_gate,
            (const __nv_bfloat16*)a.out_gate, a.out_weight, a.out_eps);
    } else {
        kda_decode_kernel<float><<<grid, block, 0, stream>>>(
            (const float*)a.q, (const float*)a.k, (const float*)a.v,
            a.log_alpha, a.beta, a.state, (float*)a.out, a.scale, a.l2norm, a.raw_gate,
            (const float*)a.out_gate, a.out_weight, a.out_eps);
    }
    return cudaGetLastError();
}

}  // namespace kda
