// Output epilogue of a KDA layer, applied in place to the operator's output:
// head-wise RMSNorm and a sigmoid output gate ("深度解读报告" 3.2, the output
// side: head-wise RMSNorm + a data-dependent sigmoid output gate).  For each
// (token, head) row o of dv values, with gate pre-activations g (same shape
// as o) and a weight w [dv]:
//
//     o' = o / sqrt(mean(o^2) + eps) * w * sigmoid(g)
//
// Memory-bound: one warp per row, 4 values per lane; the row's mean square
// is a 5-step warp reduction.
#include <cuda_bf16.h>

#include "kda_internal.h"
#include "out_gate.cuh"

namespace kda {
namespace {

constexpr int kWarpsPerBlock = 8;

__device__ __forceinline__ void load4(const float* p, float (&x)[4])
{
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&x)[4])
{
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}
__device__ __forceinline__ void store4(float* p, const float (&x)[4])
{
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, const float (&x)[4])
{
    const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
    const __nv_bfloat162 b = __floats2bfloat162_rn(x[2], x[3]);
    uint2 v;
    v.x = *reinterpret_cast<const uint32_t*>(&a);
    v.y = *reinterpret_cast<const uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = v;
}

template <typename T>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
kda_out_norm_gate_kernel(T* __restrict__ out, const T* __restrict__ gate,
                         const float* __restrict__ weight, float eps, long long rows)
{
    const int lane = threadIdx.x & 31;
    float w[4];
    load4(weight + 4 * lane, w);
    const long long warps = (long long)gridDim.x * kWarpsPerBlock;
    for (long long r = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5); r < rows; r += warps) {
        T* o = out + r * kDv + 4 * lane;
        float x[4], g[4];
        load4(o, x);
        load4(gate + r * kDv + 4 * lane, g);
        out_norm_gate_row(x, g, w, eps);
        store4(o, x);
    }
}

}  // namespace

cudaError_t launch_out_norm_gate(void* out, const void* gate, const float* weight, float eps,
                                 long long rows, kda_dtype dtype, cudaStream_t stream)
{
    if (rows <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long want = (rows + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const unsigned blocks = (unsigned)(want < (long long)sms * 16 ? want : (long long)sms * 16);
    if (dtype == KDA_DTYPE_BF16)
        kda_out_norm_gate_kernel<__nv_bfloat16><<<blocks, kWarpsPerBlock * 32, 0, stream>>>(
            static_cast<__nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(gate), weight, eps, rows);
    else
        kda_out_norm_gate_kernel<float><<<blocks, kWarpsPerBlock * 32, 0, stream>>>(
            static_cast<float*>(out), static_cast<const float*>(gate), weight, eps, rows);
    return cudaGetLastError();
}

}  // namespace kda
