// KDA backward pass on the FFMA pipes (fp32 throughout).
//
// Training differentiates the operator ("深度解读报告" 3.4: the layer is
// pre-trained, fine-tuned and trained by RL end to end).  With the chunk form of the forward ("深度解读报告" 3.1) for a
// chunk of L tokens with entry state S0 (Qt carries the scale):
//
//   Kt = K e^G, Kh = K e^-G, Qt = scale Q e^G, Gamma = e^{G_L}
//   A = strict_lower(Diag(beta) Kt Kh^T), M = (I + A)^-1, T = M Diag(beta)
//   P = lower_incl(Qt Kh^T),  R = V - Kt S0,  U = T R
//   O = Qt S0 + P U,          S' = Diag(Gamma) (S0 + Kh^T U)
//
// the adjoints, given dO and dS' (the adjoint of the chunk's exit state):
//
//   Z   = Diag(Gamma) dS'            dU  = P^T dO + Kh Z
//   dR  = T^T dU  (= dV)             dS0 = Z + Qt^T dO - Kt^T dR
//   dT  = dU R^T                     dP  = lower_incl(dO U^T)
//   dM  = dT Diag(beta)              dA  = strict_lower(-M^T dM M^T)
//   dbeta_i = sum_r dT_ri M_ri + sum_k dA_ik (Kt Kh^T)_ik
//   dQt = dO S0^T + dP Kh
//   dKt = -dR S0^T + Diag(beta) dA Kh
//   dKh = U Z^T + (Diag(beta) dA)^T Kt + dP^T Qt
//   dGamma_c = sum_j dS'_cj (S0 + Kh^T U)_cj
//
// and through the decay factors: dq = scale e^G dQt, dk = e^G dKt + e^-G dKh,
// dG = dQt Qt + dKt Kt - dKh Kh (+ dGamma Gamma on the chunk's last row), and
// dlog_alpha is the reverse prefix sum of dG over the chunk's rows.
//
// Three launches:
//   1. the FFMA forward keeps the entry state S0 of every chunk;
//   2. kda_bwd_chain_kernel, one CTA per (sequence, head, half of dv), walks
//      the chunks backwards carrying dS: it writes dS' of every chunk, dU and
//      dV (the only dS-dependent quantities the rest needs);
//   3. kda_bwd_chunk_kernel, one CTA per (chunk, head), all chunks at once:
//      everything else, 16 value columns at a time.
// This path favours plainness over speed.
#include <cuda_bf16.h>

#include "backward.h"
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kC = kChunk;          // 64
constexpr int kDvb = kDv / 2;       // value columns per chain CTA
constexpr int kLdK = kDk + 4;       // padded pitch of the [64][128] tiles
constexpr int kLdS = kDvb + 4;      // padded pitch of the 64-wide tiles
constexpr int kJb = 16;             // value columns per block of the chunk kernel
// The gate prefix sum maps two threads to each channel (tid >> 1) and the
// forward-substitution solves map four threads to each column (tid >> 2):
// both cover their index range exactly only at this block size.
static_assert(kThreads == 2 * kDk && kThreads == 4 * kC,
              "thread-to-channel and thread-to-column maps assume 256 threads");

template <typename T> __device__ __forceinline__ float ld_f32(const T* p);
template <> __device__ __forceinline__ float ld_f32<float>(const float* p) { return *p; }
template <> __device__ __forceinline__ float ld_f32<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
}

struct SeqRange {
    long long t_begin, t_end;
};

__device__ __forceinline__ SeqRange seq_range(const ChunkArgs& a, int n)
{
    SeqRange s;
    if (a.cu_seqlens) {
        s.t_begin = a.cu_seqlens[n];
        s.t_end = a.cu_seqlens[n + 1];
    } else {
        s.t_begin = (long long)n * a.T;
        s.t_end = s.t_begin + a.T;
    }
    return s;
}

// k -> Kt, q -> Qt (scaled), g -> Kh as the decayed tiles, beta, Gamma, for the
// chunk of L valid rows starting at token t0 (rows >= L are zero).  The tiles
// have pitch kLdK.
template <typename T>
__device__ void stage_decayed(const ChunkArgs& a, long long t0, int L, int h,
                              float (*Kt)[kLdK], float (*Kh)[kLdK], float (*Qt)[kLdK],
                              float* beta, float* gamma)
{
    const int tid = threadIdx.x, H = a.H;
    const T* q = static_cast<const T*>(a.q);
    const T* k = static_cast<const T*>(a.k);
    for (int e = tid; e < kC * kDk; e += kThreads) {
        const int r = e / kDk, c = e % kDk;
        const size_t gi = ((size_t)(t0 + r) * H + h) * kDk + c;
        const bool ok = r < L;
        Kt[r][c] = ok ? ld_f32(k + gi) : 0.f;
        Qt[r][c] = ok ? ld_f32(q + gi) : 0.f;
        Kh[r][c] = ok ? a.log_alpha[gi] : 0.f;
    }
    if (tid < kC) beta[tid] = tid < L ? a.beta[(size_t)(t0 + tid) * H + h] : 0.f;
    __syncthreads();
    {
        // two threads (neighbouring lanes) per channel, 32 rows each: local
        // prefix sums, then the second half adds the first half's total
        const int c = tid >> 1, half = tid & 1, ra = 32 * half;
        float G = 0.f;
        for (int r = ra; r < ra + 32; ++r) {
            G += Kh[r][c];
            Kh[r][c] = G;
        }
        const float other = __shfl_xor_sync(0xffffffffu, G, 1);
        const float off = half ? other : 0.f;
        if (half) gamma[c] = expf(other + G);   // rows >= L add 0: e^{G_L}
        for (int r = ra; r < ra + 32; ++r) {
            const float Gr = Kh[r][c] + off;
            const float e = expf(Gr), ei = expf(-Gr);
            const float kk = Kt[r][c];
            Kt[r][c] = kk * e;
            Kh[r][c] = kk * ei;
            Qt[r][c] = a.scale * Qt[r][c] * e;
        }
    }
    __syncthreads();
}

// ============================================================ reverse chain

struct ChainSmem {
    float Kt[kC][kLdK];
    float Kh[kC][kLdK];
    float Qt[kC][kLdK];
    float dO[kC][kLdS];     // dO, this CTA's value columns
    float Am[kC][kLdS];     // A, then dU
    float Tm[kC][kLdS];     // T = (I + A)^-1 Diag(beta)
    float Pm[kC][kLdS];     // P, then dR
    float dS[kDk][kLdS];    // adjoint of the state slice
    float gamma[kDk];
    float beta[kC];
};

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
kda_bwd_chain_kernel(BwdArgs b, float* __restrict__ dse, float* __restrict__ dU_out)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    ChainSmem& sm = *reinterpret_cast<ChainSmem*>(smem_raw);
    const ChunkArgs& a = b.fwd;
    const T* __restrict__ dout = static_cast<const T*>(b.d_out);
    const int jb = blockIdx.x & 1;
    const int nh = blockIdx.x >> 1;
    const int n = nh / a.H, h = nh % a.H;
    const int H = a.H;
    const int tid = threadIdx.x;
    const SeqRange sr = seq_range(a, n);
    const int j0 = jb * kDvb;
    const long long slot0 = chunk_slot_offset(a.cu_seqlens, a.T, n);
    const int n_chunks = (int)((sr.t_end - sr.t_begin + kC - 1) / kC);

    for (int e = tid; e < kDk * kDvb; e += kThreads) {
        const int c = e / kDvb, j = e % kDvb;
        sm.dS[c][j] = b.d_final_state ? b.d_final_state[((size_t)nh * kDk + c) * kDv + j0 + j] : 0.f;
    }
    const int tr = (tid >> 4) * 4, tc = (tid & 15) * 4;   // 64 x 64 tiling

    for (int ci = n_chunks - 1; ci >= 0; --ci) {
        const long long t0 = sr.t_begin + (long long)ci * kC;
        const int L = (sr.t_end - t0) < kC ? (int)(sr.t_end - t0) : kC;
        __syncthreads();   // the previous (later) chunk is done with every tile
        for (int e = tid; e < kC * kDvb; e += kThreads) {
            const int r = e / kDvb, j = e % kDvb;
            sm.dO[r][j] = r < L ? ld_f32(dout + ((size_t)(t0 + r) * H + h) * kDv + j0 + j) : 0.f;
        }
        stage_decayed<T>(a, t0, L, h, sm.Kt, sm.Kh, sm.Qt, sm.beta, sm.gamma);

        // A = strict_lower(Diag(beta) Kt Kh^T), P = lower_incl(Qt Kh^T)
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
        // T by forward substitution: four neighbouring lanes per column,
        // each summing every fourth term; then dS' of this chunk is kept for
        // the chunk kernel
        {
            const int m = tid >> 2, sub = tid & 3;
            for (int r = 0; r < kC; ++r) {
                float part = 0.f;
                for (int i = m + sub; i < r; i += 4) part += sm.Am[r][i] * sm.Tm[i][m];
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                part += __shfl_xor_sync(0xffffffffu, part, 2);
                if (sub == 0) sm.Tm[r][m] = ((r == m) ? sm.beta[r] : 0.f) - part;
                __syncwarp();
            }
        }
        {
            float* st = dse + ((size_t)(slot0 + ci) * H + h) * kDk * kDv + j0;
            for (int e = tid; e < kDk * kDvb; e += kThreads) {
                const int c = e / kDvb, j = e % kDvb;
                st[(size_t)c * kDv + j] = sm.dS[c][j];
            }
        }
        __syncthreads();
        // dU = P^T dO + Kh Z, Z = Diag(Gamma) dS'  (over A, which is dead)
        {
            float acc[4][4] = {};
            for (int i = 0; i < kC; ++i) {
                const float4 d4 = *reinterpret_cast<const float4*>(&sm.dO[i][tc]);
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float pv = sm.Pm[i][tr + x];
                    acc[x][0] += pv * d4.x; acc[x][1] += pv * d4.y;
                    acc[x][2] += pv * d4.z; acc[x][3] += pv * d4.w;
                }
            }
            for (int c = 0; c < kDk; ++c) {
                const float gm = sm.gamma[c];
                const float4 s4 = *reinterpret_cast<const float4*>(&sm.dS[c][tc]);
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float kv = sm.Kh[tr + x][c] * gm;
                    acc[x][0] += kv * s4.x; acc[x][1] += kv * s4.y;
                    acc[x][2] += kv * s4.z; acc[x][3] += kv * s4.w;
                }
            }
            __syncthreads();   // the substitution read A; every thread read P, dS
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int r = tr + x;
#pragma unroll
                for (int y = 0; y < 4; ++y) sm.Am[r][tc + y] = acc[x][y];
                if (r < L) {
                    float* o = dU_out + ((size_t)(t0 + r) * H + h) * kDv + j0 + tc;
                    *reinterpret_cast<float4*>(o) = make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
                }
            }
        }
        __syncthreads();
        // dR = T^T dU (= dV), over P
        {
            float acc[4][4] = {};
            for (int r = 0; r < kC; ++r) {
                const float4 u4 = *reinterpret_cast<const float4*>(&sm.Am[r][tc]);
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float tv = sm.Tm[r][tr + x];
                    acc[x][0] += tv * u4.x; acc[x][1] += tv * u4.y;
                    acc[x][2] += tv * u4.z; acc[x][3] += tv * u4.w;
                }
            }
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int i = tr + x;
#pragma unroll
                for (int y = 0; y < 4; ++y) sm.Pm[i][tc + y] = acc[x][y];
                if (i < L) {
                    float* o = b.dv + ((size_t)(t0 + i) * H + h) * kDv + j0 + tc;
                    *reinterpret_cast<float4*>(o) = make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
                }
            }
        }
        __syncthreads();
        // dS0 = Diag(Gamma) dS' + Qt^T dO - Kt^T dR: 128 x 64, 8 x 4 per thread
        {
            const int cr = (tid >> 4) * 8, cj = (tid & 15) * 4;
            float acc[8][4];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const float gm = sm.gamma[cr + x];
                const float4 s4 = *reinterpret_cast<const float4*>(&sm.dS[cr + x][cj]);
                acc[x][0] = gm * s4.x; acc[x][1] = gm * s4.y; acc[x][2] = gm * s4.z; acc[x][3] = gm * s4.w;
            }
            for (int r = 0; r < kC; ++r) {
                const float4 d4 = *reinterpret_cast<const float4*>(&sm.dO[r][cj]);
                const float4 e4 = *reinterpret_cast<const float4*>(&sm.Pm[r][cj]);
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const float qv = sm.Qt[r][cr + x], kv = sm.Kt[r][cr + x];
                    acc[x][0] += qv * d4.x - kv * e4.x; acc[x][1] += qv * d4.y - kv * e4.y;
                    acc[x][2] += qv * d4.z - kv * e4.z; acc[x][3] += qv * d4.w - kv * e4.w;
                }
            }
#pragma unroll
            for (int x = 0; x < 8; ++x)
                *reinterpret_cast<float4*>(&sm.dS[cr + x][cj]) =
                    make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
        }
    }
    __syncthreads();
    if (b.d_initial_state) {
        for (int e = tid; e < kDk * kDvb; e += kThreads) {
            const int c = e / kDvb, j = e % kDvb;
            b.d_initial_state[((size_t)nh * kDk + c) * kDv + j0 + j] = sm.dS[c][j];
        }
    }
}

// ============================================================ per chunk
//
// Thread tilings, chosen so that the threads of a warp read consecutive
// shared-memory words (or one word) in every product: a 64 x 64 output is
// rows tr..tr+3 by columns ti + 16y, a 64 x 128 output rows r0..r0+3 by
// columns cc + 16y; S0 and dS' blocks are stored transposed ([j][channel]);
// the 64-wide tiles have an odd pitch.

constexpr int kLdT = kC + 1;        // pitch of the 64 x 64 tiles
constexpr int kLdC = kJb + 1;       // pitch of the [64][16] column blocks

struct ChunkSmem {
    float Kt[kC][kLdK];
    float Kh[kC][kLdK];
    float Qt[kC][kLdK];
    float Mm[kC][kLdT];     // M = (I + A)^-1
    float Ar[kC][kLdT];     // strict_lower(Kt Kh^T), without beta
    float Xs[kC][kLdT];     // dT, then dM, then dA, then Diag(beta) dA
    float Ys[kC][kLdT];     // dP
    union {
        struct {            // one block of kJb value columns
            float St[kJb][kLdK];    // S0, transposed
            float Dt[kJb][kLdK];    // dS', transposed
            float Rb[kC][kLdC];     // V, then R = V - Kt S0
            float Ub[kC][kLdC];     // U = T R
            float dUb[kC][kLdC];
            float dOb[kC][kLdC];
            float dRb[kC][kLdC];
        } blk;
        float X[kC][kLdT];          // dM M^T
        float G[kC][kDk];           // G, then dG
    } u;
    float gamma[kDk];
    float dgamma[kDk];
    float dgam2[2][kDk];
    float beta[kC];
    float dbeta[kC];
};

template <typename T>
__global__ void __launch_bounds__(kThreads, 1)
kda_bwd_chunk_kernel(BwdArgs b, const float* __restrict__ states, const float* __restrict__ dse,
                     const float* __restrict__ dU_in)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    ChunkSmem& sm = *reinterpret_cast<ChunkSmem*>(smem_raw);
    const ChunkArgs& a = b.fwd;
    const T* __restrict__ v = static_cast<const T*>(a.v);
    const T* __restrict__ dout = static_cast<const T*>(b.d_out);
    const int H = a.H;
    const long long slot = blockIdx.x / H;
    const int h = blockIdx.x % H;
    const int tid = threadIdx.x;

    // the (sequence, chunk) this slot holds; slots past the last chunk exit
    int n = -1;
    long long ci = 0;
    if (a.cu_seqlens) {
        long long off = 0;
        for (int m = 0; m < a.N; ++m) {
            const long long nc = (a.cu_seqlens[m + 1] - a.cu_seqlens[m] + kC - 1) / kC;
            if (slot < off + nc) { n = m; ci = slot - off; break; }
            off += nc;
        }
    } else {
        const long long per = (a.T + kC - 1) / kC;
        if (per > 0 && slot / per < a.N) { n = (int)(slot / per); ci = slot % per; }
    }
    if (n < 0) return;
    const SeqRange sr = seq_range(a, n);
    const long long t0 = sr.t_begin + ci * kC;
    const int L = (sr.t_end - t0) < kC ? (int)(sr.t_end - t0) : kC;
    const float* S0 = states + ((size_t)slot * H + h) * kDk * kDv;
    const float* dS1 = dse + ((size_t)slot * H + h) * kDk * kDv;

    stage_decayed<T>(a, t0, L, h, sm.Kt, sm.Kh, sm.Qt, sm.beta, sm.gamma);

    const int tr = (tid >> 4) * 4, ti = tid & 15;     // 64 x 64: rows tr.., columns ti + 16y
    const int r0 = tr, cc = ti;                        // 64 x 128: rows r0.., columns cc + 16y
    const int ar = tid >> 2, jj = tid & 3;             // 64 x 16: row ar, columns jj + 4y
    const int gc = tid & (kDk - 1), gh = tid >> 7;     // dGamma: channel gc, columns gh + 2y

    // Ar = strict_lower(Kt Kh^T)
    {
        float acc[4][4] = {};
        for (int c = 0; c < kDk; c += 4) {
            float4 kt[4], kh[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                kt[x] = *reinterpret_cast<const float4*>(&sm.Kt[tr + x][c]);
                kh[x] = *reinterpret_cast<const float4*>(&sm.Kh[ti + 16 * x][c]);
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y)
                    acc[x][y] += kt[x].x * kh[y].x + kt[x].y * kh[y].y
                               + kt[x].z * kh[y].z + kt[x].w * kh[y].w;
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) {
                const int r = tr + x, i = ti + 16 * y;
                sm.Ar[r][i] = i < r ? acc[x][y] : 0.f;
            }
    }
    __syncthreads();
    // M = (I + A)^-1 by forward substitution, A_ri = beta_r Ar_ri: four
    // neighbouring lanes per column, each summing every fourth term
    {
        const int m = tid >> 2, sub = tid & 3;
        for (int r = 0; r < kC; ++r) {
            float part = 0.f;
            for (int i = m + sub; i < r; i += 4) part += sm.Ar[r][i] * sm.Mm[i][m];
            part += __shfl_xor_sync(0xffffffffu, part, 1);
            part += __shfl_xor_sync(0xffffffffu, part, 2);
            if (sub == 0) sm.Mm[r][m] = ((r == m) ? 1.f : 0.f) - sm.beta[r] * part;
            __syncwarp();
        }
    }
    __syncthreads();

    float dQt[4][8] = {}, dKt[4][8] = {}, dKh[4][8] = {};
    float dT[4][4] = {}, dP[4][4] = {};
    float gam[8];
#pragma unroll
    for (int y = 0; y < 8; ++y) gam[y] = sm.gamma[cc + 16 * y];
    float dgam = 0.f;

    for (int j0 = 0; j0 < kDv; j0 += kJb) {
        // load the block (S0 and dS' transposed)
        for (int e = tid; e < kDk * kJb; e += kThreads) {
            const int c = e / kJb, j = e % kJb;
            sm.u.blk.St[j][c] = S0[(size_t)c * kDv + j0 + j];
            sm.u.blk.Dt[j][c] = dS1[(size_t)c * kDv + j0 + j];
        }
        for (int e = tid; e < kC * kJb; e += kThreads) {
            const int r = e / kJb, j = e % kJb;
            const bool ok = r < L;
            const size_t gi = ((size_t)(t0 + r) * H + h) * kDv + j0 + j;
            sm.u.blk.Rb[r][j] = ok ? ld_f32(v + gi) : 0.f;
            sm.u.blk.dUb[r][j] = ok ? dU_in[gi] : 0.f;
            sm.u.blk.dOb[r][j] = ok ? ld_f32(dout + gi) : 0.f;
            sm.u.blk.dRb[r][j] = ok ? b.dv[gi] : 0.f;
        }
        __syncthreads();
        // R = V - Kt S0 (in place; each thread its own 4 outputs)
        {
            float acc[4] = {};
            for (int c = 0; c < kDk; c += 4) {
                const float4 k4 = *reinterpret_cast<const float4*>(&sm.Kt[ar][c]);
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    const float4 s4 = *reinterpret_cast<const float4*>(&sm.u.blk.St[jj + 4 * y][c]);
                    acc[y] += k4.x * s4.x + k4.y * s4.y + k4.z * s4.z + k4.w * s4.w;
                }
            }
#pragma unroll
            for (int y = 0; y < 4; ++y) sm.u.blk.Rb[ar][jj + 4 * y] -= acc[y];
        }
        __syncthreads();
        // U = T R = M Diag(beta) R
        {
            float acc[4] = {};
            for (int i = 0; i < kC; ++i) {
                const float tv = sm.Mm[ar][i] * sm.beta[i];
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[y] += tv * sm.u.blk.Rb[i][jj + 4 * y];
            }
#pragma unroll
            for (int y = 0; y < 4; ++y) sm.u.blk.Ub[ar][jj + 4 * y] = acc[y];
        }
        __syncthreads();
        // sums over this block's value columns
        for (int j = 0; j < kJb; ++j) {
            float du[4], dov[4], rv[4], uv[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                du[x] = sm.u.blk.dUb[tr + x][j];
                dov[x] = sm.u.blk.dOb[tr + x][j];
                rv[x] = sm.u.blk.Rb[ti + 16 * x][j];
                uv[x] = sm.u.blk.Ub[ti + 16 * x][j];
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    dT[x][y] += du[x] * rv[y];      // dT = dU R^T
                    dP[x][y] += dov[x] * uv[y];     // dP = dO U^T (masked below)
                }
            float dor[4], drr[4], ur[4], sc[8], zc[8];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                dor[x] = sm.u.blk.dOb[r0 + x][j];
                drr[x] = sm.u.blk.dRb[r0 + x][j];
                ur[x] = sm.u.blk.Ub[r0 + x][j];
            }
#pragma unroll
            for (int y = 0; y < 8; ++y) {
                sc[y] = sm.u.blk.St[j][cc + 16 * y];
                zc[y] = gam[y] * sm.u.blk.Dt[j][cc + 16 * y];
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 8; ++y) {
                    dQt[x][y] += dor[x] * sc[y];    // dO S0^T
                    dKt[x][y] -= drr[x] * sc[y];    // -dR S0^T
                    dKh[x][y] += ur[x] * zc[y];     // U Z^T
                }
        }
        // dGamma_c += sum_j dS'_cj (S0 + Kh^T U)_cj: channel gc, columns gh + 2y
        {
            float y8[8];
#pragma unroll
            for (int y = 0; y < 8; ++y) y8[y] = sm.u.blk.St[gh + 2 * y][gc];
            for (int r = 0; r < kC; ++r) {
                const float kv = sm.Kh[r][gc];
#pragma unroll
                for (int y = 0; y < 8; ++y) y8[y] += kv * sm.u.blk.Ub[r][gh + 2 * y];
            }
#pragma unroll
            for (int y = 0; y < 8; ++y) dgam += sm.u.blk.Dt[gh + 2 * y][gc] * y8[y];
        }
        __syncthreads();   // the block buffers are refilled next
    }
    sm.dgam2[gh][gc] = dgam;

    // dT and dP to shared memory; dP masked to the lower triangle
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const int r = tr + x, i = ti + 16 * y;
            sm.Xs[r][i] = dT[x][y];
            sm.Ys[r][i] = i <= r ? dP[x][y] : 0.f;
        }
    __syncthreads();
    // dbeta_i (first part) = sum_r dT_ri M_ri; dGamma from its two halves
    if (tid < kC) {
        const int i = tid;
        float acc = 0.f;
        for (int r = 0; r < kC; ++r) acc += sm.Xs[r][i] * sm.Mm[r][i];
        sm.dbeta[i] = acc;
    }
    if (tid < kDk) sm.dgamma[tid] = sm.dgam2[0][tid] + sm.dgam2[1][tid];
    __syncthreads();
    // dM = dT Diag(beta)
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) sm.Xs[tr + x][ti + 16 * y] *= sm.beta[ti + 16 * y];
    __syncthreads();
    // X = dM M^T
    {
        float acc[4][4] = {};
        for (int m = 0; m < kC; ++m) {
            float dm[4], mm[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                dm[x] = sm.Xs[tr + x][m];
                mm[x] = sm.Mm[ti + 16 * x][m];
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] += dm[x] * mm[y];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) sm.u.X[tr + x][ti + 16 * y] = acc[x][y];
    }
    __syncthreads();
    // dA = strict_lower(-M^T X), over dM
    {
        float acc[4][4] = {};
        for (int m = 0; m < kC; ++m) {
            float mt[4], xv[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                mt[x] = sm.Mm[m][tr + x];
                xv[x] = sm.u.X[m][ti + 16 * x];
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] -= mt[x] * xv[y];
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) {
                const int r = tr + x, i = ti + 16 * y;
                sm.Xs[r][i] = i < r ? acc[x][y] : 0.f;
            }
    }
    __syncthreads();
    // dbeta_r (second part) = sum_i dA_ri Ar_ri
    if (tid < kC) {
        const int r = tid;
        float acc = 0.f;
        for (int i = 0; i < r; ++i) acc += sm.Xs[r][i] * sm.Ar[r][i];
        sm.dbeta[r] += acc;
    }
    __syncthreads();
    // dB = Diag(beta) dA
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) sm.Xs[tr + x][ti + 16 * y] *= sm.beta[tr + x];
    __syncthreads();
    // dQt += dP Kh; dKt += dB Kh; dKh += dB^T Kt + dP^T Qt
    for (int i = 0; i < kC; ++i) {
        float dpr[4], dbr[4], dbc[4], dpc[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            dpr[x] = sm.Ys[r0 + x][i];
            dbr[x] = sm.Xs[r0 + x][i];
            dbc[x] = sm.Xs[i][r0 + x];
            dpc[x] = sm.Ys[i][r0 + x];
        }
#pragma unroll
        for (int y = 0; y < 8; ++y) {
            const float kh = sm.Kh[i][cc + 16 * y], kt = sm.Kt[i][cc + 16 * y],
                        qt = sm.Qt[i][cc + 16 * y];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                dQt[x][y] += dpr[x] * kh;
                dKt[x][y] += dbr[x] * kh;
                dKh[x][y] += dbc[x] * kt + dpc[x] * qt;
            }
        }
    }
    // G again (the per-channel prefix sum of the chunk's log-decay)
    if (tid < kDk) {
        const int c = tid;
        float G = 0.f;
        for (int r = 0; r < kC; ++r) {
            G += r < L ? a.log_alpha[((size_t)(t0 + r) * H + h) * kDk + c] : 0.f;
            sm.u.G[r][c] = G;
        }
    }
    __syncthreads();
    // dq, dk; dG over G
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        const int r = r0 + x;
        const size_t gi = ((size_t)(t0 + r) * H + h) * kDk;
#pragma unroll
        for (int y = 0; y < 8; ++y) {
            const int c = cc + 16 * y;
            const float G = sm.u.G[r][c];
            const float e = expf(G), ei = expf(-G);
            if (r < L) {
                b.dq[gi + c] = a.scale * e * dQt[x][y];
                b.dk[gi + c] = e * dKt[x][y] + ei * dKh[x][y];
            }
            sm.u.G[r][c] = dQt[x][y] * sm.Qt[r][c] + dKt[x][y] * sm.Kt[r][c] - dKh[x][y] * sm.Kh[r][c];
        }
    }
    __syncthreads();
    // dlog_alpha: reverse prefix sum of dG over the valid rows, with
    // dGamma Gamma on the last one (Gamma = e^{G_{L-1}})
    if (tid < kDk) {
        const int c = tid;
        float acc = sm.dgamma[c] * sm.gamma[c];
        for (int r = L - 1; r >= 0; --r) {
            acc += sm.u.G[r][c];
            b.dlog_alpha[((size_t)(t0 + r) * H + h) * kDk + c] = acc;
        }
    }
    if (tid < L) b.dbeta[(size_t)(t0 + tid) * H + h] = sm.dbeta[tid];
}

template <typename T>
cudaError_t launch_bwd_kernels(const BwdArgs& b, float* dse, float* du, const float* states,
                               long long slots, cudaStream_t stream)
{
    const ChunkArgs& a = b.fwd;
    cudaError_t e = cudaFuncSetAttribute(kda_bwd_chain_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(ChainSmem));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kda_bwd_chunk_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sizeof(ChunkSmem));
    if (e != cudaSuccess) return e;
    const long long units = (long long)a.N * a.H;
    kda_bwd_chain_kernel<T><<<(unsigned)(units * 2), kThreads, sizeof(ChainSmem), stream>>>(b, dse, du);
    e = cudaGetLastError();
    if (e != cudaSuccess || slots == 0) return e;
    kda_bwd_chunk_kernel<T><<<(unsigned)(slots * a.H), kThreads, sizeof(ChunkSmem), stream>>>(
        b, states, dse, du);
    return cudaGetLastError();
}

}  // namespace

namespace {
size_t round256(size_t n) { return (n + 255) & ~(size_t)255; }
}  // namespace

BwdWorkspace bwd_workspace_layout(int B, int T, int H, int N, bool varlen)
{
    BwdWorkspace w;
    w.slots = chunk_slots_bound(B, T, N, varlen);
    w.state_bytes = round256((size_t)w.slots * H * kDk * kDv * sizeof(float));
    w.du_bytes = round256((size_t)B * T * H * kDv * sizeof(float));
    w.total = 2 * w.state_bytes + w.du_bytes;
    return w;
}

cudaError_t launch_chunk_bwd(const BwdArgs& b, kda_dtype dtype, cudaStream_t stream)
{
    const ChunkArgs& a = b.fwd;
    const long long units = (long long)a.N * a.H;
    if (units == 0) return cudaSuccess;
    // the caller's workspace: chunk entry states, exit-state adjoints, dU
    const BwdWorkspace w = bwd_workspace_layout(a.B, a.T, a.H, a.N, a.cu_seqlens != nullptr);
    if (w.total > 0 && (!a.workspace || a.workspace_bytes < w.total ||
                        reinterpret_cast<uintptr_t>(a.workspace) % 256 != 0))
        return cudaErrorInvalidValue;
    unsigned char* ws = static_cast<unsigned char*>(a.workspace);
    float* states = w.state_bytes ? reinterpret_cast<float*>(ws) : nullptr;
    float* dse = w.state_bytes ? reinterpret_cast<float*>(ws + w.state_bytes) : nullptr;
    float* du = w.du_bytes ? reinterpret_cast<float*>(ws + 2 * w.state_bytes) : nullptr;
    ChunkArgs f = a;
    f.out = nullptr;
    f.final_state = nullptr;
    f.l2norm = 0;
    cudaError_t e = launch_chunk_simt_states(f, states, dtype, stream);
    if (e != cudaSuccess) return e;
    return dtype == KDA_DTYPE_BF16
               ? launch_bwd_kernels<__nv_bfloat16>(b, dse, du, states, w.slots, stream)
               : launch_bwd_kernels<float>(b, dse, du, states, w.slots, stream);
}

}  // namespace kda
