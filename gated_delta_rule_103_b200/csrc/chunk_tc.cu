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
// One CTA per (sequence, head) walks the sequence's chunks in order, with
// two warpgroups that work on different chunks at the same time:
//
//   prep  (warps 0-3)  chunk c+1: per-channel cumsum and decayed operand
//                      tiles; [A; P] to fp32 / bf16; the triangular inverse
//                      (16x16 diagonal blocks by forward substitution, the
//                      off-diagonal blocks by warp-level tf32 mma.sync); T to a
//                      bf16 operand tile.  Its thread 0 issues the TMA loads of
//                      q, k and the gate, and the [A; P] product.
//   chain (warps 4-7)  chunk c: issues W^T = Kt^T T^T, U'^T = V^T T^T (and the
//                      TMA loads of v) once T is written, turns W^T into a
//                      bf16 operand; thread j owns row j of S^T in fp32
//                      registers; turns U^T into a bf16 operand, applies the
//                      state update and writes the output.  Its thread 0
//                      issues every product after [A; P].
//
// Products (all M = 128, fp32 accumulators in tensor memory):
//   [A; P]  = [Kt; Qt] . Kh^T          A, B from shared memory
//   W^T     = Kt^T . T^T, U'^T = V^T . T^T
//   O^T     = S^T . Qt^T               A = S^T (bf16) from tensor memory
//   U^T    += S^T . (-W^T)
//   D^T     = U^T . Kh                 A = U^T (bf16) from tensor memory
//   O^T    += U^T . P^T
// The per-chunk tiles the chain reads (Kt/Qt, Kh, P, Gamma) are double
// buffered so that prep can fill the next chunk's copy.  Every wait is
// bounded; a run-out wait aborts the CTA and sets the library's error word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "chunk_common.cuh"
#include "kda_internal.h"
#include "sm100_ptx.cuh"

namespace kda {
namespace {

using namespace ptx;
using namespace tc;

constexpr int kPrepWarps = 4;
constexpr int kChainWarps = 4;
constexpr int kThreads = (kPrepWarps + kChainWarps) * 32;   // 256
constexpr int kMaxRankedSeqs = 256;   // longest-first CTA order up to this many sequences

// Named hardware barriers (id 0 is __syncthreads).
constexpr int BAR_PREP = 1;
constexpr int BAR_CHAIN = 2;

// Shared-memory map (byte offsets from a 1024-byte aligned base).  Operand
// tiles are 128B-swizzled; a "[R rows x 128]" bf16 tile is two 64-wide atoms
// of R x 128 bytes.
constexpr uint32_t OFF_V    = 0;                  // v [64 x 128] bf16 (TMA)
constexpr uint32_t OFF_G    = OFF_V + 16384;      // g [64 x 128] fp32 plain rows (TMA)
constexpr uint32_t OFF_SCR  = OFF_G + 32768;      // A and X fp32 [64][64] (the solve)
constexpr uint32_t OFF_KQ   = OFF_SCR + 32768;    // 2 x [Kt; Qt] [128 x 128] bf16: k and
                                                  //   q land here by TMA (rows 0-63 and
                                                  //   64-127) and are rewritten in place
constexpr uint32_t OFF_KH   = OFF_KQ + 65536;     // 2 x Kh [64 x 128] bf16
constexpr uint32_t OFF_PB   = OFF_KH + 32768;     // 2 x P [64 x 64] bf16
constexpr uint32_t OFF_WB   = OFF_PB + 16384;     // W^T [dk rows x 64] bf16; between the
                                                  //   U^T product and the next W^T it
                                                  //   stages the output tile for TMA
constexpr uint32_t OFF_TB   = OFF_WB + 16384;     // T [64 x 64] bf16
constexpr uint32_t OFF_GAM  = OFF_TB + 8192;      // 3 x Gamma [128] fp32 (by chunk % 3)
constexpr uint32_t OFF_BET  = OFF_GAM + 1536;     // 2 x beta [64] fp32
constexpr uint32_t OFF_TOT  = OFF_BET + 512;      // per-warp g totals [4][128] fp32
constexpr uint32_t OFF_BAR  = OFF_TOT + 2048;    // mbarriers
constexpr uint32_t OFF_MISC = OFF_BAR + 8 * 16;   // TMEM base, abort flag
constexpr uint32_t kSmemBytes = OFF_MISC + 64 + 1024;

// mbarriers (one completion per chunk unless noted)
enum {
    B_QK_FULL0 = 0,  // TMA q, k landed in [Kt; Qt] buffer 0  (tx; every 2nd chunk)
    B_QK_FULL1,      // ... buffer 1
    B_V_FULL,        // TMA v landed                    (tx)
    B_G_FULL,        // TMA log_alpha landed            (tx)
    B_AP_FULL,       // [A; P] product done             (commit, prep)
    B_WU_FULL,       // W^T, U'^T products done         (commit, prep)
    B_T_READY,       // T operand written               (prep arrive)
    B_C1_FULL,       // U^T = U'^T - S^T W^T done       (commit, chain)
    B_C2_FULL,       // D^T done                        (commit, chain)
    B_O_FULL,        // O^T done                        (commit, chain)
    B_DRAIN_PREP,    // prep's products drained on abort  (commit)
    B_DRAIN_CHAIN,   // chain's products drained on abort (commit)
    B_DBG_O1,        // debug instantiation: O^T = S^T Qt^T done (commit)
    kNumBars
};

// Tensor-memory columns (512 allocated; 128 lanes each).
constexpr uint32_t TM_AP = 0;     // [A; P]     128 x 64
constexpr uint32_t TM_W  = 64;    // W^T        128 x 64
constexpr uint32_t TM_U  = 128;   // 2 x U'^T/U^T 128 x 64 (cols 0-31: U^T bf16)
constexpr uint32_t TM_O  = 256;   // O^T        128 x 64
constexpr uint32_t TM_D  = 320;   // D^T        128 x 128
constexpr uint32_t TM_S  = 448;   // S^T bf16 operand (two per column) 128 x 64
constexpr uint32_t kTmemCols = 512;

struct TcParams {
    const float* log_alpha;
    const float* beta;
    const float* initial_state;
    const int32_t* cu_seqlens;
    __nv_bfloat16* out;
    float* final_state;
    unsigned* err;
    float* dbg;     // stage dump of chunk 0 of CTA 0 (debug instantiation only)
    float scale;
    int T, H, N;
    int l2norm;     // L2-normalise the q and k rows first
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


// ------------------------------------------------------------------ kernel
// kL2: fused L2Norm of the q and k rows; kRaw: the gate tile holds
// pre-activations z, the decay is log sigmoid(z)
template <bool kDebug, bool kL2, bool kRaw>
__global__ void __launch_bounds__(kThreads, 1)
kda_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_g,
                    const __grid_constant__ CUtensorMap tm_o,
                    const TcParams p)
{
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* const sbase = smem_raw + (base - raw);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H;
    const int h = blockIdx.x % H;
    int n = blockIdx.x / H;
    if (p.cu_seqlens && p.N <= kMaxRankedSeqs) {
        // Packed sequences of different lengths: CTA k takes the sequence
        // whose length has rank k / H (longest first, ties by index), so that
        // the longest chains start in the first wave of CTAs.
        volatile int* pick = reinterpret_cast<volatile int*>(sbase + OFF_MISC + 16);
        const int q = (int)(blockIdx.x / H);
        for (int m = tid; m < p.N; m += kThreads) {
            const int lm = p.cu_seqlens[m + 1] - p.cu_seqlens[m];
            int rank = 0;
            for (int o = 0; o < p.N; ++o) {
                const int lo = p.cu_seqlens[o + 1] - p.cu_seqlens[o];
                rank += (lo > lm) || (lo == lm && o < m);
            }
            if (rank == q) *pick = m;
        }
        __syncthreads();
        n = *pick;
    }
    const int nh = n * H + h;
    long long t_begin, t_end;
    if (p.cu_seqlens) {
        t_begin = p.cu_seqlens[n];
        t_end = p.cu_seqlens[n + 1];
    } else {
        t_begin = (long long)n * p.T;
        t_end = t_begin + p.T;
    }
    const int n_chunks = (int)((t_end - t_begin + kC - 1) / kC);
    const bool dbg_cta = kDebug && blockIdx.x == 0;

    float* const gam_s = reinterpret_cast<float*>(sbase + OFF_GAM);
    float* const beta_s = reinterpret_cast<float*>(sbase + OFF_BET);
    float* const tot_s = reinterpret_cast<float*>(sbase + OFF_TOT);
    float* const a_s = reinterpret_cast<float*>(sbase + OFF_SCR);
    float* const x_s = reinterpret_cast<float*>(sbase + OFF_SCR + 16384);
    volatile uint32_t* const tmem_slot = reinterpret_cast<volatile uint32_t*>(sbase + OFF_MISC);
    volatile int* const abort_flag = reinterpret_cast<volatile int*>(sbase + OFF_MISC + 8);
    auto bar = [&](int i) -> uint32_t { return base + OFF_BAR + 8 * i; };

    // Instruction descriptors (bf16 x bf16 -> fp32, M = 128).
    constexpr uint32_t ID_AP = idesc_bf16(128, 64, false, false, false);
    constexpr uint32_t ID_W  = idesc_bf16(128, 64, true, false, false);   // MN-major A
    constexpr uint32_t ID_O  = idesc_bf16(128, 64, false, false, false);
    constexpr uint32_t ID_C1 = idesc_bf16(128, 64, false, true, true);    // -(MN-major B)
    constexpr uint32_t ID_C2 = idesc_bf16(128, 128, false, true, false);  // MN-major B

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), 1);
        fence_mbar_init();
        *abort_flag = 0;
    }
    if (warp == 0) {
        tmem_alloc(base + OFF_MISC, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    // q and k of chunk c land in the [Kt; Qt] buffer of parity c & 1: k in
    // rows 0-63, q in rows 64-127 (one 8 KB box per 64-channel atom).  The
    // chunks 0 and 1 are loaded at the start by prep, chunk c + 2 by the chain
    // once its update of chunk c has released the buffer.
    auto issue_qk = [&](long long tc, int bb) {
        const int row = (int)tc;
        const uint32_t dst = base + OFF_KQ + bb * 32768;
        const uint32_t fb = bar(B_QK_FULL0 + bb);
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(fb, 32768);
        tma_load_3d(dst + 0, &tm_k, fb, 0, h, row);
        tma_load_3d(dst + 16384, &tm_k, fb, 64, h, row);
        tma_load_3d(dst + 8192, &tm_q, fb, 0, h, row);
        tma_load_3d(dst + 16384 + 8192, &tm_q, fb, 64, h, row);
    };

    if (warp < kPrepWarps) {
        // ================================================================ prep
        const int pw = warp;
        const int c0 = lane * 4;                 // channels c0..c0+3
        const uint32_t lane_base = (uint32_t)(pw * 32) << 16;
        const float* g_s = reinterpret_cast<const float*>(sbase + OFF_G);
        int n_g = 0;                             // TMA loads of g issued (thread 0)
        auto issue_g = [&](long long tc) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(bar(B_G_FULL), 32768);
            tma_load_3d(base + OFF_G, &tm_g, bar(B_G_FULL), 0, h, (int)tc);
            ++n_g;
        };
        if (tid == 0 && n_chunks > 0) {
            prefetch_tensormap(&tm_q);
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_g);
            issue_g(t_begin);
            issue_qk(t_begin, 0);
            if (n_chunks > 1) issue_qk(t_begin + kC, 1);
        }
        float beta_reg = (n_chunks > 0 && tid < kC && t_begin + tid < t_end)
                             ? __ldg(p.beta + (size_t)(t_begin + tid) * H + h) : 0.f;
        // Byte offsets of this thread's 4 channels in a 128B-swizzled bf16 row,
        // by row phase (row & 7); rows 16*pw .. 16*pw + 15 of atom c0 / 64.
        const uint32_t cq = (uint32_t)((c0 & 63) >> 3), cb = (uint32_t)((c0 & 7) << 1);
        auto swz = [&](int i) -> uint32_t { return ((cq ^ (uint32_t)(i & 7)) << 4) | cb; };
        const uint32_t in_off = (c0 >> 6) * 8192 + pw * 2048;    // q, k tiles (64 rows)
        const uint32_t kq_off = (c0 >> 6) * 16384 + pw * 2048;   // [Kt; Qt] (128 rows)

        for (int ci = 0; ci < n_chunks; ++ci) {
            const int b = ci & 1;
            const long long t0 = t_begin + (long long)ci * kC;
            const int L = (int)((t_end - t0) < kC ? (t_end - t0) : kC);
            const bool has_next = ci + 1 < n_chunks;
            const uint32_t kq = base + OFF_KQ + b * 32768;
            const uint32_t kh = base + OFF_KH + b * 16384;
            const uint32_t pb = base + OFF_PB + b * 8192;

            // q, k of this chunk in [Kt; Qt] buffer b (issued once the chain
            // released the buffer, so Kh, P and Gamma of parity b are free too)
            bool ok = wait_bar(bar(B_QK_FULL0 + b), (ci >> 1) & 1, abort_flag, p.err);
            ok = ok && wait_bar(bar(B_G_FULL), ci & 1, abort_flag, p.err);
            if (named_barrier_or(BAR_PREP, 128, !ok)) break;
            if (tid < kC) beta_s[b * 64 + tid] = beta_reg;
            if (has_next) {
                const long long tn = t0 + kC;
                beta_reg = (tid < kC && tn + tid < t_end) ? __ldg(p.beta + (size_t)(tn + tid) * H + h)
                                                          : 0.f;
            }
            if (L < kC) {
                // Last, partial chunk: rows >= L of the loaded tiles belong to the
                // next sequence (or lie past the tensor); zero them so that every
                // derived tile and the gate sum see exact zeros there.
                float4* gz = reinterpret_cast<float4*>(sbase + OFF_G);
                uint4* kqz = reinterpret_cast<uint4*>(sbase + OFF_KQ + b * 32768);
                for (int e = tid; e < (kC - L) * 32; e += 128) {
                    const int r = L + e / 32, u = e % 32;   // g row: 32 x 16 B
                    gz[r * 32 + u] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                for (int e = tid; e < (kC - L) * 16; e += 128) {
                    const int r = L + e / 16, u = e % 16;   // k row r, q row r + 64: 2 atoms x 8 x 16 B
                    const int off = (u >> 3) * 1024 + r * 8 + (u & 7);
                    kqz[off] = make_uint4(0u, 0u, 0u, 0u);
                    kqz[off + 512] = make_uint4(0u, 0u, 0u, 0u);
                }
                named_barrier(BAR_PREP, 128);
            }

            // fused L2Norm: the inverse norms of this warp's 16 k rows and
            // 16 q rows (lanes 2i, 2i + 1 hold row i's); the decayed tiles
            // below take them as row factors of the decay factors, so k and q
            // are never rewritten
            float inv_k = 1.f, inv_q = 1.f;
            if constexpr (kL2) {
#pragma unroll 1
                for (int t = 0; t < 2; ++t) {
                    float ss[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        ss[i] = sq_sum4(ld_shared_v2(kq + kq_off + i * 128 + swz(i) + 8192 * t));
                    const float inv = rsqrtf(fmaxf(warp_sum16(ss, lane), 1e-12f));
                    if (t == 0) inv_k = inv; else inv_q = inv;
                }
            }
            // ---- per-channel cumsum of g (log2 units), decayed operand tiles ---
            // Kt = K e^G, Kh = K e^-G, Qt = scale Q e^G (with the L2Norm, the
            // rows of K and Q scaled by their inverse norms): bf16 x bf16 products
            // of the decay factors and the (bf16) k, q pairs, rounded to bf16
            // once more (the tiles are bf16 MMA operands either way)
            auto decayed_row = [&](int i, const float (&e)[4], const float (&ei)[4]) {
                const uint32_t o_in = in_off + i * 128 + swz(i);
                const uint32_t o_kq = kq_off + i * 128 + swz(i);
                const uint2 kw = ld_shared_v2(kq + o_kq);          // k, in place
                const uint2 qw = ld_shared_v2(kq + o_kq + 8192);   // q, in place
                float rk = 1.f, iq = p.scale;
                if constexpr (kL2) {
                    rk = __shfl_sync(0xffffffffu, inv_k, 2 * i);
                    iq *= __shfl_sync(0xffffffffu, inv_q, 2 * i);
                }
                const uint32_t e01 = pack_bf16x2(e[0] * rk, e[1] * rk), e23 = pack_bf16x2(e[2] * rk, e[3] * rk);
                const uint32_t i01 = pack_bf16x2(ei[0] * rk, ei[1] * rk), i23 = pack_bf16x2(ei[2] * rk, ei[3] * rk);
                const uint32_t s01 = pack_bf16x2(e[0] * iq, e[1] * iq);
                const uint32_t s23 = pack_bf16x2(e[2] * iq, e[3] * iq);
                st_shared_v2(kq + o_kq, bf16x2_mul(kw.x, e01), bf16x2_mul(kw.y, e23));
                st_shared_v2(kq + o_kq + 8192, bf16x2_mul(qw.x, s01), bf16x2_mul(qw.y, s23));
                st_shared_v2(kh + o_in, bf16x2_mul(kw.x, i01), bf16x2_mul(kw.y, i23));
            };
            if constexpr (kRaw) {
                // Gate pre-activations z: alpha = sigmoid(z), so 1/alpha =
                // 1 + e^-z, e^-G_r is the prefix product of 1/alpha over the
                // rows and e^G_r its reciprocal: one exponential and one
                // reciprocal per element, as many as the plain path takes.
                // 1/alpha goes back into the gate tile in place (each thread
                // its own rows and channels); rows past the chunk's end keep
                // 1/alpha = 1 (no decay).
                float4* const gw = reinterpret_cast<float4*>(sbase + OFF_G);
                float pa[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll 4
                for (int i = 0; i < 16; ++i) {
                    float4* const at = gw + (pw * 16 + i) * 32 + (c0 >> 2);
                    const float4 z = *at;
                    const bool valid = pw * 16 + i < L;
                    const float4 a = valid ? make_float4(1.f + ex2_approx(-kLog2e * z.x),
                                                         1.f + ex2_approx(-kLog2e * z.y),
                                                         1.f + ex2_approx(-kLog2e * z.z),
                                                         1.f + ex2_approx(-kLog2e * z.w))
                                           : make_float4(1.f, 1.f, 1.f, 1.f);
                    *at = a;
                    pa[0] *= a.x; pa[1] *= a.y; pa[2] *= a.z; pa[3] *= a.w;
                }
                *reinterpret_cast<float4*>(tot_s + pw * 128 + c0) = make_float4(pa[0], pa[1], pa[2], pa[3]);
                named_barrier(BAR_PREP, 128);
                // the product of 1/alpha over the rows of the warps before
                float ei[4] = {1.f, 1.f, 1.f, 1.f};
                for (int w = 0; w < pw; ++w) {
                    const float4 t4 = *reinterpret_cast<const float4*>(tot_s + w * 128 + c0);
                    ei[0] *= t4.x; ei[1] *= t4.y; ei[2] *= t4.z; ei[3] *= t4.w;
                }
                if (pw == 3)
                    *reinterpret_cast<float4*>(gam_s + (ci % 3) * 128 + c0) =
                        make_float4(__frcp_rn(ei[0] * pa[0]), __frcp_rn(ei[1] * pa[1]),
                                    __frcp_rn(ei[2] * pa[2]), __frcp_rn(ei[3] * pa[3]));
#pragma unroll 4
                for (int i = 0; i < 16; ++i) {
                    const float4 a = gw[(pw * 16 + i) * 32 + (c0 >> 2)];
                    ei[0] *= a.x; ei[1] *= a.y; ei[2] *= a.z; ei[3] *= a.w;
                    const float e[4] = {rcp_approx(ei[0]), rcp_approx(ei[1]), rcp_approx(ei[2]),
                                        rcp_approx(ei[3])};
                    decayed_row(i, e, ei);
                }
            } else {
                // per-channel cumsum of g (log2 units)
                float run[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                for (int i = 0; i < 16; ++i) {
                    const float4 gi = *reinterpret_cast<const float4*>(g_s + (pw * 16 + i) * 128 + c0);
                    run[0] += gi.x; run[1] += gi.y; run[2] += gi.z; run[3] += gi.w;
                }
                *reinterpret_cast<float4*>(tot_s + pw * 128 + c0) =
                    make_float4(run[0] * kLog2e, run[1] * kLog2e, run[2] * kLog2e, run[3] * kLog2e);
                named_barrier(BAR_PREP, 128);
                float G[4] = {0.f, 0.f, 0.f, 0.f};
                for (int w = 0; w < pw; ++w) {
                    const float4 t4 = *reinterpret_cast<const float4*>(tot_s + w * 128 + c0);
                    G[0] += t4.x; G[1] += t4.y; G[2] += t4.z; G[3] += t4.w;
                }
                if (pw == 3) {
                    // Gamma = e^{G_L} = 2^{G_L log2 e}
                    *reinterpret_cast<float4*>(gam_s + (ci % 3) * 128 + c0) =
                        make_float4(exp2f(fmaf(run[0], kLog2e, G[0])), exp2f(fmaf(run[1], kLog2e, G[1])),
                                    exp2f(fmaf(run[2], kLog2e, G[2])), exp2f(fmaf(run[3], kLog2e, G[3])));
                }
#pragma unroll 2
                for (int i = 0; i < 16; ++i) {
                    // rows reloaded: a rolled loop keeps the kernel's code small
                    const float4 gi = *reinterpret_cast<const float4*>(g_s + (pw * 16 + i) * 128 + c0);
                    G[0] = fmaf(gi.x, kLog2e, G[0]);
                    G[1] = fmaf(gi.y, kLog2e, G[1]);
                    G[2] = fmaf(gi.z, kLog2e, G[2]);
                    G[3] = fmaf(gi.w, kLog2e, G[3]);
                    float e[4], ei[4];
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        e[x] = ex2_approx(G[x]);
                        ei[x] = ex2_approx(-G[x]);
                    }
                    decayed_row(i, e, ei);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            named_barrier(BAR_PREP, 128);
            if (tid == 0) {
                tc_fence_after_sync();
                if (has_next) issue_g(t0 + kC);      // g of this chunk is consumed
                // [A; P] = [Kt; Qt] . Kh^T   (M = 128, N = 64, K = 128)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ss(tmem + TM_AP,
                                sw128_desc(kq + (kk >> 2) * 16384 + (kk & 3) * 32, 16),
                                sw128_desc(kh + (kk >> 2) * 8192 + (kk & 3) * 32, 16), ID_AP, kk > 0);
                mma_commit(bar(B_AP_FULL));
            }

            // ---- A rows (lanes 0-63) to fp32 scratch, P rows to bf16 ----------
            // A needs no mask: the inverse only reads its strictly lower part.
            ok = wait_bar(bar(B_AP_FULL), ci & 1, abort_flag, p.err);
            if (named_barrier_or(BAR_PREP, 128, !ok)) break;
            tc_fence_after_sync();
            {
                float x[64];
                tmem_ld32(tmem + TM_AP + lane_base, *reinterpret_cast<float(*)[32]>(x));
                tmem_ld32(tmem + TM_AP + lane_base + 32, *reinterpret_cast<float(*)[32]>(x + 32));
                tmem_ld_wait();
                if (dbg_cta && ci == 0)
                    for (int i = 0; i < 64; ++i) p.dbg[DBG_AP + tid * 64 + i] = x[i];
                if (tid < 64) {
                    const int r = tid;
                    const float bb = beta_s[b * 64 + r];
#pragma unroll
                    for (int i = 0; i < 64; i += 4)
                        *reinterpret_cast<float4*>(a_s + sidx(r, i)) =
                            make_float4(bb * x[i], bb * x[i + 1], bb * x[i + 2], bb * x[i + 3]);
                } else {
                    const int r = tid - 64;
#pragma unroll
                    for (int i = 0; i < 64; ++i) x[i] = (i <= r) ? x[i] : 0.f;
                    store_row64_bf16(pb, r, x);
                }
            }
            tc_fence_before_sync();
            named_barrier(BAR_PREP, 128);

            // ---- T = (I + A)^-1 Diag(beta) -----------------------------------
            invert_unit_lower<BAR_PREP>(a_s, x_s, tid, pw, lane);
            // the previous chunk's W^T, U'^T products still read the T tile
            ok = (ci == 0) || wait_bar(bar(B_WU_FULL), (ci - 1) & 1, abort_flag, p.err);
            if (named_barrier_or(BAR_PREP, 128, !ok)) break;
            {
                // Row r, columns 32*half..: the upper-right 32 x 32 quadrant of X
                // is never written (it is zero); the rest of X's upper triangle
                // holds exact zeros.
                const int r = tid >> 1, half = tid & 1;
                float v[32];
                if (r < 32 && half == 1) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0.f;
                } else {
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const int c = 32 * half + 4 * q4;
                        const float4 x4 = *reinterpret_cast<const float4*>(x_s + sidx(r, c));
                        const float4 b4 = *reinterpret_cast<const float4*>(beta_s + b * 64 + c);
                        v[4 * q4 + 0] = x4.x * b4.x;
                        v[4 * q4 + 1] = x4.y * b4.y;
                        v[4 * q4 + 2] = x4.z * b4.z;
                        v[4 * q4 + 3] = x4.w * b4.w;
                    }
                }
                if (dbg_cta && ci == 0)
                    for (int i = 0; i < 32; ++i) p.dbg[DBG_T + r * 64 + 32 * half + i] = v[i];
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    const int chunk = half * 4 + ch;
                    st_shared_v4(base + OFF_TB + r * 128 + (((chunk ^ (r & 7)) & 7) << 4),
                                 pack_bf16x2(v[8 * ch + 0], v[8 * ch + 1]),
                                 pack_bf16x2(v[8 * ch + 2], v[8 * ch + 3]),
                                 pack_bf16x2(v[8 * ch + 4], v[8 * ch + 5]),
                                 pack_bf16x2(v[8 * ch + 6], v[8 * ch + 7]));
                }
            }
            fence_proxy_async_smem();
            named_barrier(BAR_PREP, 128);
            if (tid == 0) mbar_arrive(bar(B_T_READY));
        }
        if (tid == 0 && *abort_flag) {
            // Drain this thread's products and copies before the CTA's shared
            // and tensor memory are released (bounded).
            mma_commit(bar(B_DRAIN_PREP));
            mbar_wait_bounded(bar(B_DRAIN_PREP), 0, kWaitLimitNs);
            // q, k of chunks 0 and 1 (later ones are the chain's)
            mbar_wait_bounded(bar(B_QK_FULL0), 0, kWaitLimitNs);
            if (n_chunks > 1) mbar_wait_bounded(bar(B_QK_FULL1), 0, kWaitLimitNs);
            if (n_g > 0) mbar_wait_bounded(bar(B_G_FULL), (n_g - 1) & 1, kWaitLimitNs);
        }
    } else {
        // ================================================================ chain
        const int j = tid - kPrepWarps * 32;          // value column / TMEM lane
        const int cw = warp - kPrepWarps;
        const uint32_t lane_base = (uint32_t)(cw * 32) << 16;
        float S[128];
        if (p.initial_state) {
            const float* s0 = p.initial_state + (size_t)nh * kDk * kDv;
#pragma unroll
            for (int c = 0; c < 128; ++c) S[c] = s0[c * kDv + j];
        } else {
#pragma unroll
            for (int c = 0; c < 128; ++c) S[c] = 0.f;
        }
        auto store_state_bf16 = [&]() {
            uint32_t w[32];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] = pack_bf16x2(S[64 * hh + 2 * i], S[64 * hh + 2 * i + 1]);
                tmem_st32(tmem + TM_S + lane_base + 32 * hh, w);
            }
            tmem_st_wait();
        };
        int n_v = 0;                                   // TMA loads of v issued (j == 0)
        int last_qk[2] = {-1, -1};                     // last chunk whose q, k it loaded
        auto issue_v = [&](long long tc) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(bar(B_V_FULL), 16384);
            tma_load_3d(base + OFF_V, &tm_v, bar(B_V_FULL), 0, h, (int)tc);
            tma_load_3d(base + OFF_V + 8192, &tm_v, bar(B_V_FULL), 64, h, (int)tc);
            ++n_v;
        };
        if (j == 0 && n_chunks > 0) {
            prefetch_tensormap(&tm_v);
            issue_v(t_begin);
        }
        store_state_bf16();
        tc_fence_before_sync();
        named_barrier(BAR_CHAIN, 128);
        bool failed = false;

        for (int ci = 0; ci < n_chunks; ++ci) {
            const int b = ci & 1;
            const long long t0 = t_begin + (long long)ci * kC;
            const int L = (int)((t_end - t0) < kC ? (t_end - t0) : kC);
            const uint32_t tu = tmem + TM_U + 64 * b + lane_base;

            const bool has_next = ci + 1 < n_chunks;
            const uint32_t kq = base + OFF_KQ + b * 32768;
            bool ok = wait_bar(bar(B_T_READY), ci & 1, abort_flag, p.err);
            if (named_barrier_or(BAR_CHAIN, 128, !ok)) { failed = true; break; }
            if (j == 0) {
                ok = wait_bar(bar(B_V_FULL), ci & 1, abort_flag, p.err);
                if (ok) {
                    tc_fence_after_sync();
                    // W^T = Kt^T . T^T   (A = Kt as MN-major: K rows = tokens)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ss(tmem + TM_W, sw128_desc(kq + kk * 2048, 16384),
                                    sw128_desc(base + OFF_TB + kk * 32, 16), ID_W, kk > 0);
                    // U'^T = V^T . T^T
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ss(tmem + TM_U + 64 * b, sw128_desc(base + OFF_V + kk * 2048, 8192),
                                    sw128_desc(base + OFF_TB + kk * 32, 16), ID_W, kk > 0);
                    mma_commit(bar(B_WU_FULL));
                }
            }
            ok = ok && wait_bar(bar(B_WU_FULL), ci & 1, abort_flag, p.err);
            if (j == 0) bulk_wait_group_read0();    // the last output store has read W^T's buffer
            if (named_barrier_or(BAR_CHAIN, 128, !ok)) { failed = true; break; }
            tc_fence_after_sync();
            if (j == 0 && has_next) issue_v(t0 + kC);   // v of this chunk is consumed
            // ---- W^T rows (lane = channel) to the MN-major B operand ---------
            {
                float x[64];
                tmem_ld32(tmem + TM_W + lane_base, *reinterpret_cast<float(*)[32]>(x));
                tmem_ld32(tmem + TM_W + lane_base + 32, *reinterpret_cast<float(*)[32]>(x + 32));
                tmem_ld_wait();
                store_row64_bf16(base + OFF_WB, j, x);
                if (dbg_cta && ci == 0) {
                    for (int i = 0; i < 64; ++i) p.dbg[DBG_WT + j * 64 + i] = x[i];
                    tmem_ld32(tmem + TM_U + lane_base, *reinterpret_cast<float(*)[32]>(x));
                    tmem_ld32(tmem + TM_U + lane_base + 32, *reinterpret_cast<float(*)[32]>(x + 32));
                    tmem_ld_wait();
                    for (int i = 0; i < 64; ++i) p.dbg[DBG_UP + j * 64 + i] = x[i];
                }
            }
            fence_proxy_async_smem();
            tc_fence_before_sync();
            named_barrier(BAR_CHAIN, 128);
            if (j == 0) {
                tc_fence_after_sync();
                // U^T = U'^T - S^T . W^T  (A = S^T bf16 in TMEM, B = W^T as
                // MN-major: K rows = channels)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tmem + TM_U + 64 * b, tmem + TM_S + kk * 8,
                                sw128_desc(base + OFF_WB + kk * 2048, 8192), ID_C1, 1);
                mma_commit(bar(B_C1_FULL));
            }
            ok = wait_bar(bar(B_C1_FULL), ci & 1, abort_flag, p.err);
            if (named_barrier_or(BAR_CHAIN, 128, !ok)) { failed = true; break; }
            tc_fence_after_sync();
            // ---- U^T row j to bf16, in place in tensor memory ----------------
            {
                float x[64];
                tmem_ld32(tu, *reinterpret_cast<float(*)[32]>(x));
                tmem_ld32(tu + 32, *reinterpret_cast<float(*)[32]>(x + 32));
                tmem_ld_wait();
                if (dbg_cta && ci == 0)
                    for (int i = 0; i < 64; ++i) p.dbg[DBG_UT + j * 64 + i] = x[i];
                uint32_t w[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) w[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
                tmem_st32(tu, w);
                tmem_st_wait();
            }
            tc_fence_before_sync();
            named_barrier(BAR_CHAIN, 128);
            if (j == 0) {
                tc_fence_after_sync();
                const uint32_t kh = base + OFF_KH + b * 16384;
                // D^T = U^T . Kh  (A = U^T bf16 in TMEM, B = Kh as MN-major)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ts(tmem + TM_D, tmem + TM_U + 64 * b + kk * 8,
                                sw128_desc(kh + kk * 2048, 8192), ID_C2, kk > 0);
                mma_commit(bar(B_C2_FULL));
                // O^T = S^T . Qt^T + U^T . P^T: needed only for the output
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tmem + TM_O, tmem + TM_S + kk * 8,
                                sw128_desc(kq + 8192 + (kk >> 2) * 16384 + (kk & 3) * 32, 16),
                                ID_O, kk > 0);
                if (dbg_cta) {
                    mma_commit(bar(B_DBG_O1));
                    mbar_wait_bounded(bar(B_DBG_O1), ci & 1, kWaitLimitNs);
                    tc_fence_after_sync();
                }
            }
            if (dbg_cta) {
                // debug: the S^T Qt^T part alone, before P U is added
                named_barrier(BAR_CHAIN, 128);
                tc_fence_after_sync();
                if (ci == 0) {
                    float o[64];
                    tmem_ld32(tmem + TM_O + lane_base, *reinterpret_cast<float(*)[32]>(o));
                    tmem_ld32(tmem + TM_O + lane_base + 32, *reinterpret_cast<float(*)[32]>(o + 32));
                    tmem_ld_wait();
                    for (int i = 0; i < 64; ++i) p.dbg[DBG_O1 + j * 64 + i] = o[i];
                }
                tc_fence_before_sync();
                named_barrier(BAR_CHAIN, 128);
            }
            if (j == 0) {
                tc_fence_after_sync();
                const uint32_t pb = base + OFF_PB + b * 8192;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ts(tmem + TM_O, tmem + TM_U + 64 * b + kk * 8,
                                sw128_desc(pb + kk * 32, 16), ID_O, 1);
                mma_commit(bar(B_O_FULL));
            }

            ok = wait_bar(bar(B_C2_FULL), ci & 1, abort_flag, p.err);
            if (named_barrier_or(BAR_CHAIN, 128, !ok)) { failed = true; break; }
            tc_fence_after_sync();

            // ---- S^T_j = Gamma (S^T_j + D^T_j); output O^T_j ------------------
            {
                const float* gm = gam_s + (ci % 3) * 128;
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    float d[32];
                    tmem_ld32(tmem + TM_D + lane_base + 32 * qq, d);
                    tmem_ld_wait();
                    if (dbg_cta && ci == 0)
                        for (int c = 0; c < 32; ++c) p.dbg[DBG_DT + j * 128 + 32 * qq + c] = d[c];
#pragma unroll
                    for (int c = 0; c < 32; c += 4) {
                        // packed f32x2: the scalar form's roundings, half the instructions
                        const float4 g4 = *reinterpret_cast<const float4*>(gm + 32 * qq + c);
                        add_mul_f32x2(S[32 * qq + c + 0], S[32 * qq + c + 1], d[c + 0], d[c + 1], g4.x, g4.y);
                        add_mul_f32x2(S[32 * qq + c + 2], S[32 * qq + c + 3], d[c + 2], d[c + 3], g4.z, g4.w);
                    }
                }
                if (dbg_cta && ci == 0)
                    for (int c = 0; c < 128; ++c) p.dbg[DBG_ST + j * 128 + c] = S[c];
            }
            // O^T is complete, and with it every product of this chunk: the old
            // S^T operand can be replaced, and [Kt; Qt], Kh, P of parity b are
            // free for the q, k of chunk ci + 2.
            ok = wait_bar(bar(B_O_FULL), ci & 1, abort_flag, p.err);
            if (named_barrier_or(BAR_CHAIN, 128, !ok)) { failed = true; break; }
            tc_fence_after_sync();
            if (j == 0 && ci + 2 < n_chunks) {
                issue_qk(t0 + 2 * kC, b);
                last_qk[b] = ci + 2;
            }
            {
                store_state_bf16();
                // Output row block O[0..63][j]: a full chunk goes through the
                // W^T buffer (two [64 rows x 64 cols] bf16 boxes) and a TMA
                // store; a partial last chunk is written directly, row by row,
                // so nothing lands past the sequence.
                __nv_bfloat16* op = p.out + ((size_t)t0 * H + h) * kDv + j;
                const size_t rs = (size_t)H * kDv;
                unsigned short* ost = reinterpret_cast<unsigned short*>(sbase + OFF_WB) +
                                      (j >> 6) * 4096 + (j & 63);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    float o[32];
                    tmem_ld32(tmem + TM_O + lane_base + 32 * hh, o);
                    tmem_ld_wait();
                    if (dbg_cta && ci == 0)
                        for (int i = 0; i < 32; ++i) p.dbg[DBG_OT + j * 64 + 32 * hh + i] = o[i];
                    if (L == kC) {
#pragma unroll
                        for (int r = 0; r < 32; ++r)
                            ost[(32 * hh + r) * 64] = __bfloat16_as_ushort(__float2bfloat16_rn(o[r]));
                    } else {
                        __nv_bfloat16* oph = op + (size_t)(32 * hh) * rs;
#pragma unroll
                        for (int r = 0; r < 32; ++r)
                            if (32 * hh + r < L) oph[r * rs] = __float2bfloat16_rn(o[r]);
                    }
                }
                fence_proxy_async_smem();
            }
            tc_fence_before_sync();
            named_barrier(BAR_CHAIN, 128);
            if (j == 0 && L == kC) {
                tma_store_3d(&tm_o, base + OFF_WB, 0, h, (int)t0);
                tma_store_3d(&tm_o, base + OFF_WB + 8192, 64, h, (int)t0);
                bulk_commit_group();
            }
        }
        if (j == 0) bulk_wait_group0();   // output stores complete before the CTA ends
        if (!failed && !*abort_flag && p.final_state) {
            float* fs = p.final_state + (size_t)nh * kDk * kDv;
#pragma unroll
            for (int c = 0; c < 128; ++c) fs[c * kDv + j] = S[c];
        }
        if (j == 0 && *abort_flag) {
            mma_commit(bar(B_DRAIN_CHAIN));
            mbar_wait_bounded(bar(B_DRAIN_CHAIN), 0, kWaitLimitNs);
            if (n_v > 0) mbar_wait_bounded(bar(B_V_FULL), (n_v - 1) & 1, kWaitLimitNs);
            for (int bb = 0; bb < 2; ++bb)
                if (last_qk[bb] >= 0)
                    mbar_wait_bounded(bar(B_QK_FULL0 + bb), (last_qk[bb] >> 1) & 1, kWaitLimitNs);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, kTmemCols);
    }
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
    CUtensorMap tq, tk, tv, tg, to;
    if (!make_map(&tq, a.q, kDk, tokens, a.H, false) || !make_map(&tk, a.k, kDk, tokens, a.H, false) ||
        !make_map(&tv, a.v, kDv, tokens, a.H, false) ||
        !make_map(&tg, a.log_alpha, kDk, tokens, a.H, true) ||
        !make_map(&to, a.out, kDv, tokens, a.H, false, false))
        return cudaErrorInvalidValue;
    TcParams p;
    p.log_alpha = a.log_alpha;
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
    p.N = a.N;
    p.l2norm = a.l2norm;
    // the debug instantiation runs without the options
    auto kern = dbg ? kda_chunk_tc_kernel<true, false, false>
              : a.raw_gate ? (p.l2norm ? kda_chunk_tc_kernel<false, true, true>
                                       : kda_chunk_tc_kernel<false, false, true>)
                           : (p.l2norm ? kda_chunk_tc_kernel<false, true, false>
                                       : kda_chunk_tc_kernel<false, false, false>);
    if (dbg) p.l2norm = 0;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)units, kThreads, kSmemBytes, stream>>>(tq, tk, tv, tg, to, p);
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
