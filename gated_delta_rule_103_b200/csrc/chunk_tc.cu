// KDA chunked prefill on the sm_100a tensor cores (bf16 q/k/v, fp32 gate,
// fp32 state and accumulation).
//
// The chunkwise algorithm of "深度解读报告" 3.1: binding both low-rank DPLR
// vectors to k leaves two C x C matrices per chunk (decayed K K^T and Q K^T);
// a WY representation with a UT transform, T = (I + A)^-1 Diag(beta) by
// forward substitution, turns the sequential rank-one updates into dense
// products.  For a chunk of L <= 64 tokens, entry state S (dk x dv) and
// G_r = sum_{i<=r} g_i (per channel):
//
//   Kt = K e^G, Kh = K e^-G, Qt = scale Q e^G, Gamma = e^{G_L}
//   [A; P] = [Kt; Qt] Kh^T       A: strictly lower, rows scaled by beta
//                                P: lower triangle incl. diagonal
//   T  = (I + A)^-1 Diag(beta)                       (forward substitution)
//   W  = T Kt,  U' = T V                             (WY / UT transform)
//   U  = U' - W S                                    (state-dependent)
//   O  = Qt S + P U
//   S' = Diag(Gamma) (S + Kh^T U)                    (= Diag(Gamma) S + Kend^T U)
//
// Layout of the work: one CTA (128 threads) per (sequence, head) walks the
// sequence's chunks in order.  Every product is a tcgen05.mma with M = 128
// and an fp32 accumulator in tensor memory, issued by one thread:
//   [A; P]   = [Kt; Qt] . Kh^T          M = 128 (two 64-row operands stacked)
//   W^T      = Kt^T . T^T               M = dk
//   U'^T     = V^T . T^T                M = dv
//   O^T      = S^T . Qt^T               M = dv
//   U^T     += S^T . (-W^T)             M = dv   (accumulates onto U'^T)
//   D^T      = U^T . Kh                 M = dv
//   O^T     += U^T . P^T                M = dv
// The state is held transposed (thread j owns row j of S^T in fp32 registers)
// and re-rounded to bf16 in shared memory as the A operand of the next chunk.
// q, k, v and g tiles arrive by TMA.  The per-channel cumsum and the decayed
// operand tiles are formed by all threads; the triangular solve runs on the
// CUDA cores.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_internal.h"
#include "sm100_ptx.cuh"

namespace kda {
namespace {

using namespace ptx;

constexpr int kThreads = 128;
constexpr int kC = kChunk;  // 64
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait

// Shared-memory map (byte offsets from a 1024-byte aligned base).  Operand
// tiles are 128B-swizzled; a "[R rows x 128]" bf16 tile is two 64-wide atoms
// of R x 128 bytes.
constexpr uint32_t OFF_Q   = 0;                       // q   [64 x 128] bf16, 16 KB
constexpr uint32_t OFF_K   = OFF_Q + 16384;           // k   [64 x 128] bf16, 16 KB
constexpr uint32_t OFF_V   = OFF_K + 16384;           // v   [64 x 128] bf16, 16 KB
constexpr uint32_t OFF_G   = OFF_V + 16384;           // g   [64 x 128] fp32 (plain), 32 KB
constexpr uint32_t OFF_KQ  = OFF_G + 32768;           // [Kt; Qt] [128 x 128] bf16, 32 KB
constexpr uint32_t OFF_KH  = OFF_KQ + 32768;          // Kh  [64 x 128] bf16, 16 KB
constexpr uint32_t OFF_TB  = OFF_KH + 16384;          // T   [64 x 64] bf16, 8 KB
constexpr uint32_t OFF_PB  = OFF_TB + 8192;           // P   [64 x 64] bf16, 8 KB
constexpr uint32_t OFF_WB  = OFF_PB + 8192;           // W^T as [dk rows x 64] bf16, 16 KB
constexpr uint32_t OFF_UB  = OFF_WB + 16384;          // U^T [dv rows x 64] bf16, 16 KB
                                                      //   (solve: A in fp32, [64][64],
                                                      //    16-byte groups XOR-swizzled by row)
constexpr uint32_t OFF_SB  = OFF_UB + 16384;          // S^T [dv rows x 128] bf16, 32 KB
constexpr uint32_t OFF_GAM = OFF_SB + 32768;          // Gamma [128] fp32
constexpr uint32_t OFF_BET = OFF_GAM + 512;           // beta [64] fp32
constexpr uint32_t OFF_TOT = OFF_BET + 256;           // per-warp g totals [4][128] fp32
constexpr uint32_t OFF_BAR = OFF_TOT + 2048;          // mbarriers (8 B each)
constexpr uint32_t OFF_TMEM = OFF_BAR + 64;           // TMEM base address
constexpr uint32_t OFF_FLAG = OFF_TMEM + 16;
constexpr uint32_t kSmemBytes = OFF_FLAG + 16 + 1024; // + alignment slack

// Tensor-memory columns (512 allocated; 128 lanes each).
constexpr uint32_t TM_AP = 0;     // [A; P]   128 x 64
constexpr uint32_t TM_W  = 64;    // W^T      128 x 64
constexpr uint32_t TM_U  = 128;   // U'^T/U^T 128 x 64
constexpr uint32_t TM_O  = 192;   // O^T      128 x 64
constexpr uint32_t TM_D  = 256;   // D^T      128 x 128
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kBytesQKG = 16384 + 16384 + 32768;
constexpr uint32_t kBytesV = 16384;

struct TcParams {
    const float* beta;
    const float* initial_state;
    const int32_t* cu_seqlens;
    __nv_bfloat16* out;
    float* final_state;
    unsigned* err;
    float* dbg;     // stage dump of chunk 0 of CTA 0 (debug instantiation only)
    float scale;
    int T, H;
};

// Stage-dump layout (fp32, row-major), written by the debug instantiation
// for the first chunk of the first (sequence, head):
constexpr int DBG_AP = 0;                    // [A_raw; P_raw] 128 x 64 (unmasked)
constexpr int DBG_T  = DBG_AP + 128 * 64;    // T 64 x 64 (before bf16 rounding)
constexpr int DBG_WT = DBG_T + 64 * 64;      // W^T 128 x 64
constexpr int DBG_UP = DBG_WT + 128 * 64;    // U'^T 128 x 64
constexpr int DBG_O1 = DBG_UP + 128 * 64;    // (Qt S)^T 128 x 64
constexpr int DBG_UT = DBG_O1 + 128 * 64;    // U^T 128 x 64
constexpr int DBG_DT = DBG_UT + 128 * 64;    // (Kh^T U)^T 128 x 128
constexpr int DBG_OT = DBG_DT + 128 * 128;   // O^T 128 x 64
constexpr int DBG_ST = DBG_OT + 128 * 64;    // S'^T 128 x 128
constexpr int DBG_FLOATS = DBG_ST + 128 * 128;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                 :: "r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void st_shared_v2(uint32_t addr, uint32_t a, uint32_t b)
{
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" :: "r"(addr), "r"(a), "r"(b) : "memory");
}

__device__ __forceinline__ uint2 ld_shared_v2(uint32_t addr)
{
    uint2 r;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr) : "memory");
    return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Writes 64 fp32 values as one 128-byte swizzled bf16 row (row index `row`
// of a tile whose atom starts at `atom_base`).
__device__ __forceinline__ void store_row64_bf16(uint32_t atom_base, int row, const float* v)
{
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        const uint32_t addr = atom_base + row * 128 + (((ch ^ (row & 7)) & 7) << 4);
        st_shared_v4(addr, pack_bf16x2(v[8 * ch + 0], v[8 * ch + 1]),
                     pack_bf16x2(v[8 * ch + 2], v[8 * ch + 3]),
                     pack_bf16x2(v[8 * ch + 4], v[8 * ch + 5]),
                     pack_bf16x2(v[8 * ch + 6], v[8 * ch + 7]));
    }
}

template <bool kDebug>
__global__ void __launch_bounds__(kThreads, 1)
kda_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_g,
                    const TcParams p)
{
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* const sbase = smem_raw + (base - raw);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nh = blockIdx.x;
    const int n = nh / p.H, h = nh % p.H;
    long long t_begin, t_end;
    if (p.cu_seqlens) {
        t_begin = p.cu_seqlens[n];
        t_end = p.cu_seqlens[n + 1];
    } else {
        t_begin = (long long)n * p.T;
        t_end = t_begin + p.T;
    }
    const int n_chunks = (int)((t_end - t_begin + kC - 1) / kC);

    float* const gam_s = reinterpret_cast<float*>(sbase + OFF_GAM);
    float* const beta_s = reinterpret_cast<float*>(sbase + OFF_BET);
    float* const tot_s = reinterpret_cast<float*>(sbase + OFF_TOT);
    float* const g_s = reinterpret_cast<float*>(sbase + OFF_G);
    float* const a_s = reinterpret_cast<float*>(sbase + OFF_UB);   // A (fp32) during the solve
    volatile int* const flag_s = reinterpret_cast<volatile int*>(sbase + OFF_FLAG);
    const uint32_t bar_qkg = base + OFF_BAR;
    const uint32_t bar_v = base + OFF_BAR + 8;
    const uint32_t bar_mma = base + OFF_BAR + 16;

    if (tid == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        prefetch_tensormap(&tm_g);
        mbar_init(bar_qkg, 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        *flag_s = 0;
    }
    if (warp == 0) {
        tmem_alloc(base + OFF_TMEM, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sbase + OFF_TMEM);
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;   // this warp's TMEM lanes

    auto issue_qkg = [&](long long t0) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar_qkg, kBytesQKG);
        const int row = (int)t0;
        tma_load_3d(base + OFF_Q, &tm_q, bar_qkg, 0, h, row);
        tma_load_3d(base + OFF_Q + 8192, &tm_q, bar_qkg, 64, h, row);
        tma_load_3d(base + OFF_K, &tm_k, bar_qkg, 0, h, row);
        tma_load_3d(base + OFF_K + 8192, &tm_k, bar_qkg, 64, h, row);
        tma_load_3d(base + OFF_G, &tm_g, bar_qkg, 0, h, row);
    };
    auto issue_v = [&](long long t0) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar_v, kBytesV);
        const int row = (int)t0;
        tma_load_3d(base + OFF_V, &tm_v, bar_v, 0, h, row);
        tma_load_3d(base + OFF_V + 8192, &tm_v, bar_v, 64, h, row);
    };

    // Entry state: thread j holds row j of S^T (column j of S) in fp32.
    const int j = tid;
    float S[128];
    if (p.initial_state) {
        const float* s0 = p.initial_state + (size_t)nh * kDk * kDv;
#pragma unroll
        for (int c = 0; c < 128; ++c) S[c] = s0[c * kDv + j];
    } else {
#pragma unroll
        for (int c = 0; c < 128; ++c) S[c] = 0.f;
    }
    store_row64_bf16(base + OFF_SB, j, S);
    store_row64_bf16(base + OFF_SB + 16384, j, S + 64);

    if (tid == 0 && n_chunks > 0) {
        issue_qkg(t_begin);
        issue_v(t_begin);
    }

    // Instruction descriptors.
    constexpr uint32_t ID_AP = idesc_bf16(128, 64, false, false, false);
    constexpr uint32_t ID_W  = idesc_bf16(128, 64, true, false, false);   // Kt^T (MN) . T^T
    constexpr uint32_t ID_O1 = idesc_bf16(128, 64, false, false, false);
    constexpr uint32_t ID_C1 = idesc_bf16(128, 64, false, true, true);    // S^T . (-W^T) (MN)
    constexpr uint32_t ID_C2 = idesc_bf16(128, 128, false, true, false);  // U^T . Kh (MN)

    uint32_t ph_qkg = 0, ph_v = 0, ph_mma = 0;
    bool failed = false;

    // All threads wait on an mbarrier; a run-out wait anywhere aborts the CTA.
    auto wait_all = [&](uint32_t bar, uint32_t& phase) -> bool {
        const bool ok = mbar_wait_bounded(bar, phase, kWaitLimitNs);
        phase ^= 1u;
        const int any_fail = __syncthreads_or(ok ? 0 : 1);
        tc_fence_after_sync();
        return any_fail == 0;
    };

    for (int ci = 0; ci < n_chunks; ++ci) {
        const long long t0 = t_begin + (long long)ci * kC;
        const int L = (int)((t_end - t0) < kC ? (t_end - t0) : kC);
        const bool has_next = ci + 1 < n_chunks;

        if (tid < kC) beta_s[tid] = tid < L ? p.beta[(size_t)(t0 + tid) * p.H + h] : 0.f;
        if (!wait_all(bar_qkg, ph_qkg)) { failed = true; break; }

        // ---- per-channel cumsum of g and the decayed operand tiles ----------
        // Thread (warp w, lane l): rows 16w..16w+15, channels 4l..4l+3.
        {
            const int r0 = warp * 16, c0 = lane * 4;
            float gl[16][4];
            float run[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = r0 + i;
                float4 g4 = *reinterpret_cast<const float4*>(g_s + r * 128 + c0);
                if (r >= L) g4 = make_float4(0.f, 0.f, 0.f, 0.f);
                run[0] += g4.x; run[1] += g4.y; run[2] += g4.z; run[3] += g4.w;
                gl[i][0] = run[0]; gl[i][1] = run[1]; gl[i][2] = run[2]; gl[i][3] = run[3];
            }
            *reinterpret_cast<float4*>(tot_s + warp * 128 + c0) =
                make_float4(run[0], run[1], run[2], run[3]);
            __syncthreads();
            float off[4] = {0.f, 0.f, 0.f, 0.f};
            for (int w = 0; w < warp; ++w) {
                const float4 t4 = *reinterpret_cast<const float4*>(tot_s + w * 128 + c0);
                off[0] += t4.x; off[1] += t4.y; off[2] += t4.z; off[3] += t4.w;
            }
            if (warp == 3) {
                // G over the whole chunk (rows >= L contribute 0): Gamma = e^{G_L}.
                *reinterpret_cast<float4*>(gam_s + c0) =
                    make_float4(expf(off[0] + gl[15][0]), expf(off[1] + gl[15][1]),
                                expf(off[2] + gl[15][2]), expf(off[3] + gl[15][3]));
            }
            const int atom = c0 >> 6, cc = c0 & 63;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = r0 + i;
                const uint32_t o_row = atom * 8192 + r * 128 + ((((cc >> 3) ^ (r & 7)) << 4) | ((cc & 7) << 1));
                const uint2 kw = ld_shared_v2(base + OFF_K + o_row);
                const uint2 qw = ld_shared_v2(base + OFF_Q + o_row);
                float kt[4], kh[4], qt[4];
                const float kv[4] = {bf16_lo(kw.x), bf16_hi(kw.x), bf16_lo(kw.y), bf16_hi(kw.y)};
                const float qv[4] = {bf16_lo(qw.x), bf16_hi(qw.x), bf16_lo(qw.y), bf16_hi(qw.y)};
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float G = off[x] + gl[i][x];
                    const float e = expf(G), ei = expf(-G);
                    const bool ok = r < L;
                    kt[x] = ok ? kv[x] * e : 0.f;
                    kh[x] = ok ? kv[x] * ei : 0.f;
                    qt[x] = ok ? p.scale * qv[x] * e : 0.f;
                }
                const uint32_t o_kq = atom * 16384 + r * 128 + ((((cc >> 3) ^ (r & 7)) << 4) | ((cc & 7) << 1));
                const uint32_t o_q2 = atom * 16384 + (r + 64) * 128 + ((((cc >> 3) ^ (r & 7)) << 4) | ((cc & 7) << 1));
                st_shared_v2(base + OFF_KQ + o_kq, pack_bf16x2(kt[0], kt[1]), pack_bf16x2(kt[2], kt[3]));
                st_shared_v2(base + OFF_KQ + o_q2, pack_bf16x2(qt[0], qt[1]), pack_bf16x2(qt[2], qt[3]));
                st_shared_v2(base + OFF_KH + o_row, pack_bf16x2(kh[0], kh[1]), pack_bf16x2(kh[2], kh[3]));
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        if (tid == 0) {
            tc_fence_after_sync();
            if (has_next) issue_qkg(t0 + kC);   // q, k, g of this chunk are consumed
            // [A; P] = [Kt; Qt] . Kh^T   (M=128, N=64, K=128)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
                const uint32_t koff_b = (kk >> 2) * 8192 + (kk & 3) * 32;
                mma_bf16_ss(tmem + TM_AP, sw128_desc(base + OFF_KQ + koff, 16),
                            sw128_desc(base + OFF_KH + koff_b, 16), ID_AP, kk > 0);
            }
            mma_commit(bar_mma);
        }
        if (!wait_all(bar_mma, ph_mma)) { failed = true; break; }

        // ---- A rows (lanes 0-63) to fp32 smem; P rows (lanes 64-127) to bf16 --
        {
            float x[64];
            tmem_ld32(tmem + TM_AP + lane_base, *reinterpret_cast<float(*)[32]>(x));
            tmem_ld32(tmem + TM_AP + lane_base + 32, *reinterpret_cast<float(*)[32]>(x + 32));
            tmem_ld_wait();
            if (kDebug && ci == 0 && blockIdx.x == 0)
                for (int i = 0; i < 64; ++i) p.dbg[DBG_AP + tid * 64 + i] = x[i];
            if (tid < 64) {
                const int r = tid;
                const float b = beta_s[r];
#pragma unroll
                for (int i = 0; i < 64; i += 4) {
                    float4 v4;
                    v4.x = (i + 0 < r) ? b * x[i + 0] : 0.f;
                    v4.y = (i + 1 < r) ? b * x[i + 1] : 0.f;
                    v4.z = (i + 2 < r) ? b * x[i + 2] : 0.f;
                    v4.w = (i + 3 < r) ? b * x[i + 3] : 0.f;
                    // 16-byte group i/4 of row r stored at group (i/4) ^ (r & 7)
                    *reinterpret_cast<float4*>(a_s + r * 64 + ((((i >> 2) ^ (r & 7))) << 2)) = v4;
                }
            } else {
                const int r = tid - 64;
#pragma unroll
                for (int i = 0; i < 64; ++i) x[i] = (i <= r) ? x[i] : 0.f;
                store_row64_bf16(base + OFF_PB, r, x);
            }
        }
        __syncthreads();

        // ---- forward substitution: T = (I + A)^-1 Diag(beta) ----------------
        // Thread m < 64 owns column m: T_rm = beta_r [r == m] - sum_{i<r} A_ri T_im,
        // and writes it as bf16 into the K-major T tile (row r, K index m).
        if (tid < kC) {
            const int m = tid;
            float tcol[64];
#pragma unroll
            for (int r = 0; r < 64; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < r; i += 4) {
                    const float4 a4 = *reinterpret_cast<const float4*>(
                        a_s + r * 64 + ((((i >> 2) ^ (r & 7))) << 2));
                    acc = fmaf(a4.x, tcol[i], acc);
                    if (i + 1 < r) acc = fmaf(a4.y, tcol[i + 1], acc);
                    if (i + 2 < r) acc = fmaf(a4.z, tcol[i + 2], acc);
                    if (i + 3 < r) acc = fmaf(a4.w, tcol[i + 3], acc);
                }
                tcol[r] = ((r == m) ? beta_s[r] : 0.f) - acc;
            }
            if (kDebug && ci == 0 && blockIdx.x == 0)
                for (int r = 0; r < 64; ++r) p.dbg[DBG_T + r * 64 + m] = tcol[r];
            unsigned short* tb = reinterpret_cast<unsigned short*>(sbase + OFF_TB);
#pragma unroll
            for (int r = 0; r < 64; ++r) {
                const uint32_t off = r * 128 + ((((m >> 3) ^ (r & 7)) << 4) | ((m & 7) << 1));
                tb[off >> 1] = __bfloat16_as_ushort(__float2bfloat16_rn(tcol[r]));
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        if (tid == 0) {
            tc_fence_after_sync();
            const bool v_ok = mbar_wait_bounded(bar_v, ph_v, kWaitLimitNs);
            if (!v_ok) *flag_s = 1;
            // W^T = Kt^T . T^T   (A = Kt as MN-major: K rows = tokens, M = channels)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + TM_W, sw128_desc(base + OFF_KQ + kk * 2048, 16384),
                            sw128_desc(base + OFF_TB + kk * 32, 16), ID_W, kk > 0);
            // U'^T = V^T . T^T
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + TM_U, sw128_desc(base + OFF_V + kk * 2048, 8192),
                            sw128_desc(base + OFF_TB + kk * 32, 16), ID_W, kk > 0);
            // O^T = S^T . Qt^T   (B = Qt rows 64..127 of the [Kt; Qt] tile, K-major)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_bf16_ss(tmem + TM_O, sw128_desc(base + OFF_SB + koff, 16),
                            sw128_desc(base + OFF_KQ + 8192 + koff, 16), ID_O1, kk > 0);
            }
            mma_commit(bar_mma);
        }
        ph_v ^= 1u;
        if (!wait_all(bar_mma, ph_mma) || *flag_s) { failed = true; break; }

        // ---- W^T rows (lane = channel c) to the MN-major B operand ----------
        {
            float x[64];
            tmem_ld32(tmem + TM_W + lane_base, *reinterpret_cast<float(*)[32]>(x));
            tmem_ld32(tmem + TM_W + lane_base + 32, *reinterpret_cast<float(*)[32]>(x + 32));
            tmem_ld_wait();
            store_row64_bf16(base + OFF_WB, tid, x);
            if (kDebug && ci == 0 && blockIdx.x == 0) {
                for (int i = 0; i < 64; ++i) p.dbg[DBG_WT + tid * 64 + i] = x[i];
                tmem_ld32(tmem + TM_U + lane_base, *reinterpret_cast<float(*)[32]>(x));
                tmem_ld32(tmem + TM_U + lane_base + 32, *reinterpret_cast<float(*)[32]>(x + 32));
                tmem_ld_wait();
                for (int i = 0; i < 64; ++i) p.dbg[DBG_UP + tid * 64 + i] = x[i];
                tmem_ld32(tmem + TM_O + lane_base, *reinterpret_cast<float(*)[32]>(x));
                tmem_ld32(tmem + TM_O + lane_base + 32, *reinterpret_cast<float(*)[32]>(x + 32));
                tmem_ld_wait();
                for (int i = 0; i < 64; ++i) p.dbg[DBG_O1 + tid * 64 + i] = x[i];
            }
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        if (tid == 0) {
            tc_fence_after_sync();
            if (has_next) issue_v(t0 + kC);   // v of this chunk is consumed
            // U^T = U'^T - S^T . W^T   (B = W^T as MN-major: K rows = channels)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16_ss(tmem + TM_U, sw128_desc(base + OFF_SB + (kk >> 2) * 16384 + (kk & 3) * 32, 16),
                            sw128_desc(base + OFF_WB + kk * 2048, 8192), ID_C1, 1);
            mma_commit(bar_mma);
        }
        if (!wait_all(bar_mma, ph_mma)) { failed = true; break; }

        // ---- U^T rows (lane = value column j) to the K-major A operand ------
        {
            float x[64];
            tmem_ld32(tmem + TM_U + lane_base, *reinterpret_cast<float(*)[32]>(x));
            tmem_ld32(tmem + TM_U + lane_base + 32, *reinterpret_cast<float(*)[32]>(x + 32));
            tmem_ld_wait();
            store_row64_bf16(base + OFF_UB, tid, x);
            if (kDebug && ci == 0 && blockIdx.x == 0)
                for (int i = 0; i < 64; ++i) p.dbg[DBG_UT + tid * 64 + i] = x[i];
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();

        if (tid == 0) {
            tc_fence_after_sync();
            // D^T = U^T . Kh   (B = Kh as MN-major: K rows = tokens, N = channels)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + TM_D, sw128_desc(base + OFF_UB + kk * 32, 16),
                            sw128_desc(base + OFF_KH + kk * 2048, 8192), ID_C2, kk > 0);
            // O^T += U^T . P^T
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + TM_O, sw128_desc(base + OFF_UB + kk * 32, 16),
                            sw128_desc(base + OFF_PB + kk * 32, 16), ID_O1, 1);
            mma_commit(bar_mma);
        }
        if (!wait_all(bar_mma, ph_mma)) { failed = true; break; }

        // ---- state update S^T_j = Gamma . (S^T_j + D^T_j); output O^T_j -----
        {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                float d[32];
                tmem_ld32(tmem + TM_D + lane_base + q4 * 32, d);
                tmem_ld_wait();
                if (kDebug && ci == 0 && blockIdx.x == 0)
                    for (int c = 0; c < 32; ++c) p.dbg[DBG_DT + tid * 128 + q4 * 32 + c] = d[c];
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    S[q4 * 32 + c] = gam_s[q4 * 32 + c] * (S[q4 * 32 + c] + d[c]);
            }
            store_row64_bf16(base + OFF_SB, j, S);
            store_row64_bf16(base + OFF_SB + 16384, j, S + 64);
            float o[64];
            tmem_ld32(tmem + TM_O + lane_base, *reinterpret_cast<float(*)[32]>(o));
            tmem_ld32(tmem + TM_O + lane_base + 32, *reinterpret_cast<float(*)[32]>(o + 32));
            tmem_ld_wait();
            if (kDebug && ci == 0 && blockIdx.x == 0) {
                for (int i = 0; i < 64; ++i) p.dbg[DBG_OT + tid * 64 + i] = o[i];
                for (int c = 0; c < 128; ++c) p.dbg[DBG_ST + tid * 128 + c] = S[c];
            }
            __nv_bfloat16* op = p.out + ((size_t)t0 * p.H + h) * kDv + j;
#pragma unroll
            for (int r = 0; r < 64; ++r)
                if (r < L) op[(size_t)r * p.H * kDv] = __float2bfloat16_rn(o[r]);
        }
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncthreads();
    }

    if (failed) {
        if (tid == 0) {
            atomicOr(p.err, kErrTimeout);
            // Let copies and products still in flight land before the CTA's
            // shared and tensor memory are released (bounded).
            mbar_wait_bounded(bar_qkg, ph_qkg, kWaitLimitNs);
            mbar_wait_bounded(bar_v, ph_v, kWaitLimitNs);
            mbar_wait_bounded(bar_mma, ph_mma, kWaitLimitNs);
        }
    } else if (p.final_state) {
        float* fs = p.final_state + (size_t)nh * kDk * kDv;
#pragma unroll
        for (int c = 0; c < 128; ++c) fs[c * kDv + j] = S[c];
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 3-D view [tokens][H][d] of a [B*T, H, d] tensor; box {box_d, 1, 64}.
bool make_map(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int esize, int d,
              long long tokens, int H, int box_d, CUtensorMapSwizzle sw)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)tokens};
    const cuuint64_t strides[2] = {(cuuint64_t)d * esize, (cuuint64_t)d * esize * H};
    const cuuint32_t box[3] = {(cuuint32_t)box_d, 1u, (cuuint32_t)kC};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

static cudaError_t launch_tc(const ChunkArgs& a, float* dbg, cudaStream_t stream)
{
    const long long units = (long long)a.N * a.H;
    if (units == 0) return cudaSuccess;
    const long long tokens = (long long)a.B * a.T;
    if (tokens > 0x7fffffffLL) return cudaErrorInvalidValue;
    // No tokens: nothing to load, only states to pass through.
    if (tokens == 0) return launch_chunk_simt(a, KDA_DTYPE_BF16, stream);
    CUtensorMap tq, tk, tv, tg;
    if (!make_map(&tq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDk, tokens, a.H, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDk, tokens, a.H, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDv, tokens, a.H, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tg, a.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, kDk, tokens, a.H, 128,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    TcParams p;
    p.beta = a.beta;
    p.initial_state = a.initial_state;
    p.cu_seqlens = a.cu_seqlens;
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.final_state = a.final_state;
    p.err = a.err;
    p.dbg = dbg;
    p.scale = a.scale;
    p.T = a.T;
    p.H = a.H;
    if (dbg) {
        cudaError_t e = cudaFuncSetAttribute(kda_chunk_tc_kernel<true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        kda_chunk_tc_kernel<true><<<(unsigned)units, kThreads, kSmemBytes, stream>>>(tq, tk, tv, tg, p);
    } else {
        cudaError_t e = cudaFuncSetAttribute(kda_chunk_tc_kernel<false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        kda_chunk_tc_kernel<false><<<(unsigned)units, kThreads, kSmemBytes, stream>>>(tq, tk, tv, tg, p);
    }
    return cudaGetLastError();
}

cudaError_t launch_chunk_tc(const ChunkArgs& a, cudaStream_t stream)
{
    return launch_tc(a, nullptr, stream);
}

cudaError_t launch_chunk_tc_debug(const ChunkArgs& a, float* stages, cudaStream_t stream)
{
    if (!stages) return cudaErrorInvalidValue;
    return launch_tc(a, stages, stream);
}

int chunk_tc_debug_floats() { return DBG_FLOATS; }

}  // namespace kda
