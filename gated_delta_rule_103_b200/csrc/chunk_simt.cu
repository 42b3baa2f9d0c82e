// KDA chunked prefill, fp32 FFMA path (used for fp32 inputs).
//
// Chunkwise algorithm of "深度解读报告" 3.1 (a = b = k DPLR specialisation,
// WY representation, UT transform, forward substitution), for a chunk of L
// tokens with entry state S0 and G_r = sum_{i<=r} g_i (per channel):
//
//   Kt = K e^G, Kh = K e^-G, Qt = scale Q e^G, Gamma = e^{G_L}
//   A  = strict_lower(Diag(beta) Kt Kh^T)          P = lower_incl(Qt Kh^T)
//   T  = (I + A)^-1 Diag(beta)                     (forward substitution)
//   U  = T (V - Kt S0)                             (= U' - W S0, W = T Kt, U' = T V)
//   O  = Qt S0 + P U
//   S  = Diag(Gamma) (S0 + Kh^T U)                 (= Diag(Gamma) S0 + Kend^T U)
//
// One CTA of 256 threads per (sequence, head, half of dv); it walks the
// sequence's chunks in order and keeps every tile of the chunk and the fp32
// state slice in shared memory.  This path favours plainness over speed: the
// bf16 path runs on the tensor cores.  The backward pass runs it with
// `states` set, to keep the entry state of every chunk, and `out` null.
#include <cuda_bf16.h>

#include "backward.h"
#include "gate.cuh"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kC = kChunk;          // 64
constexpr int kDvb = kDv / 2;       // value columns per CTA
constexpr int kLdK = kDk + 4;       // padded row pitch of the [64][128] tiles
constexpr int kLdS = kDvb + 4;      // padded row pitch of the 64-wide tiles

struct Smem {
    float Kt[kC][kLdK];
    float Kh[kC][kLdK];
    float Qt[kC][kLdK];
    float V[kC][kLdS];      // V, then X = V - Kt S0 in place
    float Am[kC][kLdS];     // A, then U
    float Tm[kC][kLdS];
    float Pm[kC][kLdS];
    float S[kDk][kLdS];     // fp32 state slice [channel][value column]
    float gamma[kDk];
    float beta[kC];
};

template <typename T> __device__ __forceinline__ float ld_f32(const T* p);
template <> __device__ __forceinline__ float ld_f32<float>(const float* p) { return *p; }
template <> __device__ __forceinline__ float ld_f32<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ void st_f32(T* p, float x);
template <> __device__ __forceinline__ void st_f32<float>(float* p, float x) { *p = x; }
template <> __device__ __forceinline__ void st_f32<__nv_bfloat16>(__nv_bfloat16* p, float x) {
    *p = __float2bfloat16_rn(x);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
kda_chunk_simt_kernel(ChunkArgs a, float* __restrict__ states)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
    const T* __restrict__ q = static_cast<const T*>(a.q);
    const T* __restrict__ k = static_cast<const T*>(a.k);
    const T* __restrict__ v = static_cast<const T*>(a.v);
    T* __restrict__ out = static_cast<T*>(a.out);

    const int jb = blockIdx.x & 1;
    const int nh = blockIdx.x >> 1;
    const int n = nh / a.H, h = nh % a.H;
    const int H = a.H;
    const int tid = threadIdx.x;
    long long t_begin, t_end;
    if (a.cu_seqlens) {
        t_begin = a.cu_seqlens[n];
        t_end = a.cu_seqlens[n + 1];
    } else {
        t_begin = (long long)n * a.T;
        t_end = t_begin + a.T;
    }
    const int j0 = jb * kDvb;
    const long long slot0 = states ? chunk_slot_offset(a.cu_seqlens, a.T, n) : 0;

    // Entry state slice.
    for (int e = tid; e < kDk * kDvb; e += kThreads) {
        const int c = e / kDvb, j = e % kDvb;
        sm.S[c][j] = a.initial_state
            ? a.initial_state[((size_t)nh * kDk + c) * kDv + j0 + j] : 0.f;
    }

    // Thread tiling of the 64 x 64 products: 4 x 4 outputs per thread.
    const int tr = (tid >> 4) * 4;   // row block
    const int tc = (tid & 15) * 4;   // column block

    for (long long t0 = t_begin; t0 < t_end; t0 += kC) {
        const int L = (t_end - t0) < kC ? (int)(t_end - t0) : kC;
        __syncthreads();  // previous chunk fully consumed
        if (states) {
            // entry state of this chunk: [slot][H][dk][dv]
            float* st = states + ((size_t)(slot0 + (t0 - t_begin) / kC) * H + h) * kDk * kDv + j0;
            for (int e = tid; e < kDk * kDvb; e += kThreads) {
                const int c = e / kDvb, j = e % kDvb;
                st[(size_t)c * kDv + j] = sm.S[c][j];
            }
        }

        // 1. Stage k -> Kt, q -> Qt, g -> Kh, v -> V, beta (zero rows >= L).
        for (int e = tid; e < kC * kDk; e += kThreads) {
            const int r = e / kDk, c = e % kDk;
            const size_t gi = ((size_t)(t0 + r) * H + h) * kDk + c;
            const bool ok = r < L;
            sm.Kt[r][c] = ok ? ld_f32(k + gi) : 0.f;
            sm.Qt[r][c] = ok ? ld_f32(q + gi) : 0.f;
            sm.Kh[r][c] = ok ? (a.raw_gate ? log_sigmoid(a.log_alpha[gi]) : a.log_alpha[gi]) : 0.f;
        }
        for (int e = tid; e < kC * kDvb; e += kThreads) {
            const int r = e / kDvb, j = e % kDvb;
            sm.V[r][j] = r < L ? ld_f32(v + ((size_t)(t0 + r) * H + h) * kDv + j0 + j) : 0.f;
        }
        if (tid < kC) sm.beta[tid] = tid < L ? a.beta[(size_t)(t0 + tid) * H + h] : 0.f;
        __syncthreads();
        if (a.l2norm) {
            // fused L2Norm: every k and q row divided by max(||row||_2, 1e-6);
            // warp w normalises rows w, w + 8, ..., 4 channels per lane
            const int w = tid >> 5, ln = tid & 31;
            for (int r = w; r < kC; r += kThreads / 32) {
                float sk = 0.f, sq = 0.f;
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float kv = sm.Kt[r][ln + 32 * x], qv = sm.Qt[r][ln + 32 * x];
                    sk = fmaf(kv, kv, sk);
                    sq = fmaf(qv, qv, sq);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    sk += __shfl_xor_sync(0xffffffffu, sk, off);
                    sq += __shfl_xor_sync(0xffffffffu, sq, off);
                }
                const float ik = 1.f / fmaxf(sqrtf(sk), 1e-6f), iq = 1.f / fmaxf(sqrtf(sq), 1e-6f);
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    sm.Kt[r][ln + 32 * x] *= ik;
                    sm.Qt[r][ln + 32 * x] *= iq;
                }
            }
            __syncthreads();
        }

        // 2. Per-channel prefix sum of the log-decay, then the decayed tiles.
        if (tid < kDk) {
            const int c = tid;
            float G = 0.f;
            for (int r = 0; r < kC; ++r) {
                G += sm.Kh[r][c];
                sm.Kh[r][c] = G;
            }
            sm.gamma[c] = expf(G);  // rows >= L add 0, so this is e^{G_L}
            for (int r = 0; r < kC; ++r) {
                const float Gr = sm.Kh[r][c];
                const float e = expf(Gr), ei = expf(-Gr);
                const float kk = sm.Kt[r][c];
                sm.Kt[r][c] = kk * e;
                sm.Kh[r][c] = kk * ei;
                sm.Qt[r][c] = a.scale * sm.Qt[r][c] * e;
            }
        }
        __syncthreads();

        // 3. A = strict_lower(Diag(beta) Kt Kh^T), P = lower_incl(Qt Kh^T).
        {
            float accA[4][4] = {}, accP[4][4] = {};
            for (int c = 0; c < kDk; c += 4) {
                float4 kt[4], qt[4], kh[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    kt[x] = *reinterpret_cast<const float4*>(&sm.Kt[tr + x][c]);
                    qt[x] = *reinterpret_cast<const float4*>(&sm.Qt[tr + x][c]);
                    kh[x] = *reinterpret_cast<const float4*>(&sm.Kh[(tid & 15) + 16 * x][c]);
                }
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        accA[x][y] += kt[x].x * kh[y].x + kt[x].y * kh[y].y
                                    + kt[x].z * kh[y].z + kt[x].w * kh[y].w;
                        accP[x][y] += qt[x].x * kh[y].x + qt[x].y * kh[y].y
                                    + qt[x].z * kh[y].z + qt[x].w * kh[y].w;
                    }
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    const int r = tr + x, i = (tid & 15) + 16 * y;
                    sm.Am[r][i] = i < r ? sm.beta[r] * accA[x][y] : 0.f;
                    sm.Pm[r][i] = i <= r ? accP[x][y] : 0.f;
                }
        }
        __syncthreads();

        // 4. T = (I + A)^-1 Diag(beta) by forward substitution, one column
        //    per thread: T_rm = beta_r [r == m] - sum_{i<r} A_ri T_im.
        if (tid < kC) {
            const int m = tid;
            for (int r = 0; r < kC; ++r) {
                float acc = (r == m) ? sm.beta[r] : 0.f;
                for (int i = m; i < r; ++i) acc -= sm.Am[r][i] * sm.Tm[i][m];
                sm.Tm[r][m] = acc;
            }
        }

        // 5. O1 = Qt S0 (kept in registers) and X = V - Kt S0 (in place).
        float o1[4][4] = {}, ks[4][4] = {};
        for (int c = 0; c < kDk; ++c) {
            const float4 s4 = *reinterpret_cast<const float4*>(&sm.S[c][tc]);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const float qv = sm.Qt[tr + x][c], kv = sm.Kt[tr + x][c];
                o1[x][0] += qv * s4.x; o1[x][1] += qv * s4.y;
                o1[x][2] += qv * s4.z; o1[x][3] += qv * s4.w;
                ks[x][0] += kv * s4.x; ks[x][1] += kv * s4.y;
                ks[x][2] += kv * s4.z; ks[x][3] += kv * s4.w;
            }
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) sm.V[tr + x][tc + y] -= ks[x][y];
        __syncthreads();

        // 6. U = T X (written over A, which the substitution no longer needs).
        {
            float acc[4][4] = {};
            for (int i = 0; i < kC; ++i) {
                const float4 x4 = *reinterpret_cast<const float4*>(&sm.V[i][tc]);
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float tv = sm.Tm[tr + x][i];
                    acc[x][0] += tv * x4.x; acc[x][1] += tv * x4.y;
                    acc[x][2] += tv * x4.z; acc[x][3] += tv * x4.w;
                }
            }
            // A was last read by the substitution, before the barrier above.
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) sm.Am[tr + x][tc + y] = acc[x][y];
        }
        __syncthreads();

        // 7a. O = O1 + P U for the valid rows.
        {
            for (int i = 0; i < kC; ++i) {
                const float4 u4 = *reinterpret_cast<const float4*>(&sm.Am[i][tc]);
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float pv = sm.Pm[tr + x][i];
                    o1[x][0] += pv * u4.x; o1[x][1] += pv * u4.y;
                    o1[x][2] += pv * u4.z; o1[x][3] += pv * u4.w;
                }
            }
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int r = tr + x;
                if (r < L && out) {
                    T* o = out + ((size_t)(t0 + r) * H + h) * kDv + j0 + tc;
#pragma unroll
                    for (int y = 0; y < 4; ++y) st_f32(o + y, o1[x][y]);
                }
            }
        }
        // 7b. S = Diag(Gamma) (S0 + Kh^T U): 128 x 64 outputs, 8 x 4 per thread.
        {
            const int cr = (tid >> 4) * 8, cj = (tid & 15) * 4;
            float acc[8][4];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const float4 s4 = *reinterpret_cast<const float4*>(&sm.S[cr + x][cj]);
                acc[x][0] = s4.x; acc[x][1] = s4.y; acc[x][2] = s4.z; acc[x][3] = s4.w;
            }
            for (int r = 0; r < kC; ++r) {
                const float4 u4 = *reinterpret_cast<const float4*>(&sm.Am[r][cj]);
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const float kv = sm.Kh[r][cr + x];
                    acc[x][0] += kv * u4.x; acc[x][1] += kv * u4.y;
                    acc[x][2] += kv * u4.z; acc[x][3] += kv * u4.w;
                }
            }
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const float gm = sm.gamma[cr + x];
                float4 s4;
                s4.x = gm * acc[x][0]; s4.y = gm * acc[x][1];
                s4.z = gm * acc[x][2]; s4.w = gm * acc[x][3];
                *reinterpret_cast<float4*>(&sm.S[cr + x][cj]) = s4;
            }
        }
    }
    __syncthreads();
    if (a.final_state) {
        for (int e = tid; e < kDk * kDvb; e += kThreads) {
            const int c = e / kDvb, j = e % kDvb;
            a.final_state[((size_t)nh * kDk + c) * kDv + j0 + j] = sm.S[c][j];
        }
    }
}

}  // namespace

cudaError_t launch_chunk_simt_states(const ChunkArgs& a, float* states, kda_dtype dtype,
                                     cudaStream_t stream)
{
    const long long units = (long long)a.N * a.H;
    if (units == 0) return cudaSuccess;
    const size_t smem = sizeof(Smem);
    const dim3 grid((unsigned)(units * 2)), block(kThreads);
    cudaError_t e;
    if (dtype == KDA_DTYPE_BF16) {
        e = cudaFuncSetAttribute(kda_chunk_simt_kernel<__nv_bfloat16>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kda_chunk_simt_kernel<__nv_bfloat16><<<grid, block, smem, stream>>>(a, states);
    } else {
        e = cudaFuncSetAttribute(kda_chunk_simt_kernel<float>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kda_chunk_simt_kernel<float><<<grid, block, smem, stream>>>(a, states);
    }
    return cudaGetLastError();
}

cudaError_t launch_chunk_simt(const ChunkArgs& a, kda_dtype dtype, cudaStream_t stream)
{
    return launch_chunk_simt_states(a, nullptr, dtype, stream);
}

}  // namespace kda
