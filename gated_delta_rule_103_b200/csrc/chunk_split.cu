// KDA chunked prefill for few (sequence, head) chains: one thread-block
// cluster per chain, so that a chain's per-chunk work spreads over several SMs.
//
// The chunk algebra is the one of the single-CTA kernel ("深度解读报告" 3.1,
// the DPLR specialisation with a = b = k, WY representation, UT transform):
//
//   Kt = K e^G, Kh = K e^-G, Qt = scale Q e^G, Gamma = e^{G_L}
//   [A; P] = [Kt; Qt] Kh^T,  T = (I + A)^-1 Diag(beta),  W = T Kt,  U' = T V
//   U = U' - W S,  O = Qt S + P U,  S' = Diag(Gamma) (S + Kh^T U)
//
// Everything up to W depends on the chunk's own inputs only; U, O and S'
// carry the state from chunk to chunk.  The cluster splits the two:
//
//   rank 0 (chain)     walks the chunks in order, thread (j, half) owning half
//                      of row j of S^T in fp32 registers:
//                        [U'^T | 0] = V^T T^T
//                        [U^T | S^T Qt^T] += S^T [-W; Qt]^T      (N = 128)
//                        D^T = U^T Kh,  O^T = S^T Qt^T + U^T P^T
//                        S'^T = (S^T + D^T) Diag(Gamma)
//                      Merging the products that share an operand cuts the
//                      number of tcgen05.mma issues, which cost about the same
//                      whatever their N; O^T stays in a double-buffered
//                      accumulator, so that a chunk's output is written while
//                      the next chunk's D^T is formed.  One warp only issues
//                      the products, so that the warps that convert and update
//                      never wait on an issue queue.
//   ranks 1..P (prep)  prep rank r takes chunks c = r - 1 (mod P): cumsum,
//                      decayed tiles, [A; P], the inverse, T, W; and hands the
//                      chain the chunk's bf16 operand tiles [-W; Qt], T,
//                      Kh, P and Gamma (64.5 KB).
//
// The hand-off goes through a small ring in the caller's workspace that
// stays in L2 (2 slots per prep CTA): a prep CTA writes a slot with bulk copies from its
// shared memory and signals the chain's mbarrier through distributed shared
// memory; the chain pulls the slot into its shared memory in two parts
// ([-W; Qt] and T, needed first; Kh, P and Gamma), each double-buffered,
// and signals the slot free.  The tiles keep their 128B-swizzled
// shared-memory images, so the chain feeds them to the tensor cores as they
// land.  v streams through a ring of three buffers, two chunks ahead.  Each CTA has 8 compute warps and
// one copy warp that issues the bulk copies and the signals; the chain CTA
// adds its issue warp.  Every wait is bounded; a run-out wait aborts the CTA
// and sets the library's error word, and the others then run out too.
//
// For very few chains the same kernel also runs segmented (see SplitParams):
// the recurrence is affine in the state, so a segment of whole chunks maps
// its entry state to M S_in + B.  One launch runs segment 0 and, for each
// middle segment, its zero-start exit state B (v as given) and its
// transition M (the chain from the identity with v = 0); a small fp32
// kernel chains the segments' entry states; a second launch reruns
// segments 1 .. G-1 from them with their outputs.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "chunk_common.cuh"
#include "kda_internal.h"
#include "sm100_ptx.cuh"

namespace kda {
namespace {

using namespace ptx;
using namespace tc;

constexpr int kComputeWarps = 8;
constexpr int kCompute = kComputeWarps * 32;       // 256
constexpr int kCopyWarp = kComputeWarps;           // bulk copies and signals
constexpr int kMmaWarp = kComputeWarps + 1;        // tensor-core issue (chain CTA)
constexpr int kThreadsS = kCompute + 64;
constexpr int kMaxPrep = 3;
constexpr int kMaxRankedSeqs = 256;                // longest-first order up to this many sequences

constexpr int BAR_ALL = 1;     // the 8 compute warps
constexpr int BAR_SOLVE = 2;   // prep group B, inside the inverse
constexpr int BAR_A = 3;       // prep group A (warps 0-3)
constexpr int BAR_B = 4;       // prep group B (warps 4-7)

// One hand-off slot: a chunk's operand tiles in their shared-memory images.
// Part A (needed first, by U'^T and the S^T products):
constexpr uint32_t SL_WQ  = 0;        // [-W; Qt] [128 tok][128 ch] bf16 K-major, two 16 KB
                                      //   channel atoms (rows 0-63 -W, rows 64-127 Qt)
constexpr uint32_t SL_TB  = 32768;    // T [64][64] bf16
constexpr uint32_t kPartA = 40960;
// Part B (offsets from its start at kPartA):
constexpr uint32_t SL_KP  = 0;        // Kh [64 tok][128 ch] bf16 MN-major, channel atoms at 0
                                      //   and 8 KB; P [i][j] bf16 K-major at 16 KB
constexpr uint32_t SL_GAM = 24576;    // Gamma [128] fp32
constexpr uint32_t kPartB = 25088;
constexpr uint32_t kSlotBytes = kPartA + kPartB;    // 66048
constexpr uint32_t kSlotStride = 66560;             // keeps every slot 1024-byte aligned
static_assert(kSlotBytes <= kSlotStride && kPartA % 1024 == 0, "slot layout");

// Chain CTA shared memory.
constexpr uint32_t kBStride = 25600;                   // part B buffers, 1024-byte aligned
constexpr uint32_t C_A   = 0;                          // 2 x part A
constexpr uint32_t C_B   = C_A + 2 * kPartA;           // 2 x part B
constexpr uint32_t C_V   = C_B + 2 * kBStride;         // 3 x v [64 x 128] bf16 (TMA)
constexpr uint32_t C_OST = C_V + 3 * 16384;            // output staging: 2 x [64 x 64] bf16
constexpr uint32_t C_GAM = C_OST + 16384;              // 2 x Gamma [128] fp32, out of part B
constexpr uint32_t C_END = C_GAM + 1024;

// Prep CTA shared memory.
constexpr uint32_t P_QK  = 0;                  // 2 x [Kt; Qt] [128 x 128] bf16: k, q land here by
                                               //   TMA, become Kt, Qt in place, then -W over Kt
constexpr uint32_t P_TB  = P_QK + 65536;       // 2 x T
constexpr uint32_t P_GS  = P_TB + 16384;       // 2 x g [64 x 128] fp32 (TMA), then A, X of the inverse
constexpr uint32_t P_KP  = P_GS + 65536;       // 2 x [Kh | P] (24 KB each)
constexpr uint32_t P_GAM = P_KP + 49152;       // 2 x Gamma [128] fp32
constexpr uint32_t P_BET = P_GAM + 1024;       // 2 x beta [64] fp32
constexpr uint32_t P_TOT = P_BET + 512;        // per-warp g totals [4][128] fp32
constexpr uint32_t P_END = P_TOT + 2048;
// The W product reads 128 rows of A from a T buffer: rows 64-127 (unused
// lanes of its accumulator) are the 8 KB after the buffer.
static_assert(P_TB + 3 * 8192 <= P_END, "T buffers and the rows read after them");

constexpr uint32_t OFF_BAR  = (C_END > P_END ? C_END : P_END);
constexpr uint32_t OFF_MISC = OFF_BAR + 48 * 8;       // TMEM base +0, abort +8, pick +16
constexpr uint32_t kSmemBytesS = OFF_MISC + 64 + 1024;
static_assert(kSmemBytesS <= 232448, "shared memory");

// mbarriers.  Chain: one completion per chunk (or per use of a buffer).
enum {
    B_A_FULL0 = 0,     // part A of chunk c in buffer c & 1                  (tx)
    B_A_FULL1,
    B_B_FULL0,         // part B of chunk c in buffer c & 1                  (tx)
    B_B_FULL1,
    B_A_EMPTY0,        // U^T, S^T Qt^T of chunk c formed: part A free       (commit)
    B_A_EMPTY1,
    B_B_EMPTY0,        // D^T and O^T of chunk c formed: part B free         (commit)
    B_B_EMPTY1,
    B_V_FULL0,         // v of chunk c in buffer c % 3                       (tx)
    B_V_FULL1,
    B_V_FULL2,
    B_V_EMPTY0,        // U'^T of chunk c formed: v buffer free              (commit)
    B_V_EMPTY1,
    B_V_EMPTY2,
    B_C1_FULL,         // [U^T | S^T Qt^T]                                    (commit)
    B_C2_FULL,         // D^T                                                 (commit)
    B_O_FULL0,         // O^T of chunk c in D1 buffer c & 1 (one barrier per
    B_O_FULL1,         //   buffer: the wait lags the commit by a chunk)      (commit)
    B_U_DONE,          // U^T in bf16 and Gamma copied (one arrive per compute warp)
    B_S_DONE0,         // S^T operand of the next chunk, channels 0-63 written (one
    B_S_DONE1,         //   per compute warp); channels 64-127
    B_DRAIN,           // products drained on abort                           (commit)
    B_FULLG0,          // hand-off slot s written (remote arrive by its prep CTA), 2P of them
    // prep
    B_QK_FULL0 = B_FULLG0 + 2 * kMaxPrep,   // k, q, g of local chunk m in buffers m & 1 (tx)
    B_QK_FULL1,
    B_AB_FULL0,        // group A's part of local chunk m done (buffer m & 1)   (arrive)
    B_AB_FULL1,
    B_AP_FULL,         // [A; P]                                              (commit)
    B_W_FULL,          // W                                                   (commit)
    B_READY,           // local chunk's tiles written                         (compute arrive)
    B_SENT0,           // local chunk's slot written and signalled            (copy arrive)
    B_SENT1,
    B_EMPTYG0,         // the chain holds a copy of local chunk m's slot      (remote arrive)
    B_EMPTYG1,
    B_DRAIN_B,         // group B's products drained on abort                 (commit)
    kNumBarsS
};
static_assert(kNumBarsS <= 48, "barrier space");

// Tensor-memory columns.  Chain (512 allocated):
constexpr uint32_t CT_D1 = 0;     // 2 x [U'^T -> U^T | O^T] 128 x 128; bf16 U^T in
                                  //   cols 0-15 and 32-47 once converted
constexpr uint32_t CT_D2 = 256;   // D^T 128 x 128
constexpr uint32_t CT_S  = 384;   // S^T bf16 operand 128 x 64
// Prep (128 allocated):
constexpr uint32_t PT_AP = 0;     // [A; P] 128 x 64
constexpr uint32_t PT_W  = 128;   // W in lanes 0-63 (lanes 64-127 unused), 128 x 128

struct SplitParams {
    const float* beta;
    const float* initial_state;
    const int32_t* cu_seqlens;
    __nv_bfloat16* out;
    float* final_state;
    unsigned* err;
    unsigned char* ring;   // 2 * P * kSlotStride bytes per cluster
    float scale;
    int T, H, N, P;
    int l2norm;            // L2-normalise the q and k rows first
    // Segmented runs: every sequence is cut into G segments of whole chunks
    // (segment g: chunks [g c, (g + 1) c), c = ceil(chunks / G)).
    //   phase 0  G = 1: cluster k runs chain k over the whole sequence.
    //   phase 1  cluster (task t, chain): t = 0 runs segment 0 with its
    //            outputs and stores its exit state S_in(1); t = 1 .. G-2 run
    //            segment t from a zero state without outputs, storing B_t;
    //            t = G-1 .. 2G-4 run segment g = t - G + 2 from the identity
    //            with v = 0, storing M_g (the segment's state transition:
    //            S_out = M_g S_in + B_g).
    //   phase 3  task t runs segment t + 1 from S_in(t + 1) with its outputs
    //            (the last segment writes final_state).
    //   phase 4  G = 1: cluster k runs chain k over the whole sequence from
    //            the identity with v = 0 and no outputs, writing the
    //            sequence's state transition M where final_state points.
    // S_in(g + 1) = M_g S_in(g) + B_g for g = 1 .. G-2 in between
    // (kda_segment_prefix_kernel).
    int G;
    int phase;
    float* seg;            // per chain [3][G][dk][dv] fp32: M_g, B_g, S_in(g)
    // Phase 1 with two chain CTAs per cluster (rank 0 and rank P + 1) that
    // share the prep CTAs' slots: task t = 0 runs segment 0 on rank 0 (rank
    // P + 1 idles); task t = 1 .. G-2 runs B_t on rank 0 and M_t on rank
    // P + 1 (every slot is released when both have copied it).
    int dual;
};

// Per-cluster role in a segmented run (see SplitParams).
struct Task {
    long long t_begin, t_end;   // the tokens this cluster's chain walks
    int nh;                     // chain: sequence * H + head
    int h;
    bool v_on;                  // false: v = 0 (a transition run)
    bool out_on;                // writes its output rows
    int init;                   // 0 zeros, 1 from init_ptr, 2 identity
    const float* init_ptr;      // [dk][dv] of the entry state
    float* fs_ptr;              // [dk][dv] of the exit state, or nullptr
};

__device__ __forceinline__ float* seg_slot(const SplitParams& p, int chain, int kind, int g)
{
    return p.seg + ((size_t)chain * 3 * p.G + (size_t)kind * p.G + g) * (kDk * kDv);
}

// Bounded wait without a sleep between polls (mbarrier.try_wait suspends the
// thread for a while by itself): for the waits on the chain's critical path,
// where a sleeping waiter adds its wake-up time to every chunk.
__device__ __forceinline__ bool wait_spin(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned* err)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(err, kErrTimeout);
            return false;
        }
    }
}

// Bounded wait for a phase that another CTA of the cluster completes.
static __device__ __noinline__ bool wait_bar_cluster_slow(uint32_t bar, uint32_t parity,
                                                   volatile int* abort_flag, unsigned* err)
{
    const uint64_t t0 = globaltimer();
    while (true) {
        __nanosleep(64);
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicOr(err, kErrTimeout);
            return false;
        }
    }
}

__device__ __forceinline__ bool wait_bar_cluster(uint32_t bar, uint32_t parity,
                                                 volatile int* abort_flag, unsigned* err)
{
    if (mbar_try_wait_cluster(bar, parity)) return true;
    return wait_bar_cluster_slow(bar, parity, abort_flag, err);
}

// kL2: fused L2Norm of the q and k rows; kRaw: the gate tile holds
// pre-activations z, the decay is log sigmoid(z)
template <bool kL2, bool kRaw>
__global__ void __launch_bounds__(kThreadsS, 1)
kda_chunk_split_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_g,
                       const __grid_constant__ CUtensorMap tm_o,
                       const SplitParams p)
{
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* const sbase = smem_raw + (base - raw);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int P = p.P;
    const uint32_t rank = cluster_ctarank();
    const int cl = (int)cluster_id_x();
    const int H = p.H;
    const int chains = p.N * H;
    const int chain = p.phase == 0 ? cl : cl % chains;
    const int task = p.phase == 0 ? 0 : cl / chains;
    const int h = chain % H;
    int n = chain / H;
    if (p.phase == 0 && p.cu_seqlens && p.N <= kMaxRankedSeqs) {
        // cluster k takes the sequence whose length has rank k / H (longest first)
        volatile int* pick = reinterpret_cast<volatile int*>(sbase + OFF_MISC + 16);
        const int q = cl / H;
        for (int m = tid; m < p.N; m += kThreadsS) {
            const int lm = p.cu_seqlens[m + 1] - p.cu_seqlens[m];
            int rk = 0;
            for (int o = 0; o < p.N; ++o) {
                const int lo = p.cu_seqlens[o + 1] - p.cu_seqlens[o];
                rk += (lo > lm) || (lo == lm && o < m);
            }
            if (rk == q) *pick = m;
        }
        __syncthreads();
        n = *pick;
    }
    const int nh = n * H + h;
    // the second chain CTA of a dual cluster, and whether this cluster's
    // slots have two consumers
    const bool chain_b = p.dual && (int)rank == P + 1;
    const bool dual_task = p.dual && task >= 1;
    Task tk;
    {
        long long s_begin, s_end;
        if (p.cu_seqlens) {
            s_begin = p.cu_seqlens[n];
            s_end = p.cu_seqlens[n + 1];
        } else {
            s_begin = (long long)n * p.T;
            s_end = s_begin + p.T;
        }
        tk.nh = nh;
        tk.h = h;
        tk.v_on = true;
        tk.out_on = true;
        tk.init = p.initial_state ? 1 : 0;
        tk.init_ptr = p.initial_state ? p.initial_state + (size_t)nh * kDk * kDv : nullptr;
        tk.fs_ptr = p.final_state ? p.final_state + (size_t)nh * kDk * kDv : nullptr;
        int g = 0;
        if (p.phase == 1 && p.dual) {
            g = task;
            if (task == 0 && chain_b) {
                tk.out_on = false;        // idle: nothing to walk, nothing to write
                tk.v_on = false;
                tk.fs_ptr = nullptr;
            } else if (task == 0) {
                tk.fs_ptr = seg_slot(p, nh, 2, 1);
            } else if (chain_b) {
                tk.out_on = false;
                tk.v_on = false;
                tk.init = 2;
                tk.fs_ptr = seg_slot(p, nh, 0, g);
            } else {
                tk.out_on = false;
                tk.init = 0;
                tk.fs_ptr = seg_slot(p, nh, 1, g);
            }
        } else if (p.phase == 1) {
            const int G = p.G;
            if (task == 0) {
                g = 0;
                tk.fs_ptr = seg_slot(p, nh, 2, 1);
            } else if (task <= G - 2) {
                g = task;
                tk.out_on = false;
                tk.init = 0;
                tk.fs_ptr = seg_slot(p, nh, 1, g);
            } else {
                g = task - G + 2;
                tk.out_on = false;
                tk.v_on = false;
                tk.init = 2;
                tk.fs_ptr = seg_slot(p, nh, 0, g);
            }
        } else if (p.phase == 3) {
            g = task + 1;
            tk.init = 1;
            tk.init_ptr = seg_slot(p, nh, 2, g);
            if (g != p.G - 1) tk.fs_ptr = nullptr;
        } else if (p.phase == 4) {
            tk.out_on = false;
            tk.v_on = false;
            tk.init = 2;
        }
        if (p.phase == 0 || p.phase == 4) {
            tk.t_begin = s_begin;
            tk.t_end = s_end;
        } else {
            const long long nc = (s_end - s_begin + kC - 1) / kC;
            const long long cps = (nc + p.G - 1) / p.G;
            const long long c_lo = min(nc, (long long)g * cps), c_hi = min(nc, c_lo + cps);
            tk.t_begin = s_begin + c_lo * kC;
            tk.t_end = min(s_end, s_begin + c_hi * kC);
            if (c_hi == c_lo) tk.t_end = tk.t_begin;
            if (p.dual && task == 0 && chain_b) tk.t_end = tk.t_begin;
        }
    }
    const long long t_begin = tk.t_begin, t_end = tk.t_end;
    const int n_chunks = (int)((t_end - t_begin + kC - 1) / kC);
    unsigned char* const ring = p.ring + (size_t)cl * 2 * P * kSlotStride;

    volatile uint32_t* const tmem_slot = reinterpret_cast<volatile uint32_t*>(sbase + OFF_MISC);
    volatile int* const abort_flag = reinterpret_cast<volatile int*>(sbase + OFF_MISC + 8);
    auto bar = [&](int i) -> uint32_t { return base + OFF_BAR + 8 * i; };
    const bool is_chain = rank == 0 || chain_b;
    const uint32_t tmem_cols = is_chain ? 512u : 256u;

    constexpr uint32_t ID_AP  = idesc_bf16(128, 64, false, false, false);
    constexpr uint32_t ID_W   = idesc_bf16(128, 64, true, false, false);   // MN-major A
    constexpr uint32_t ID_N64 = idesc_bf16(128, 64, false, false, false);
    constexpr uint32_t ID_C1  = idesc_bf16(128, 128, false, false, false);
    constexpr uint32_t ID_C2  = idesc_bf16(128, 128, false, true, false);  // MN-major B
    constexpr uint32_t ID_O2  = idesc_bf16(128, 64, false, false, false);  // K-major B (P)
    constexpr uint32_t ID_WP  = idesc_bf16(128, 128, false, true, false);  // MN-major B (Kt)

    if (tid == 0) {
        for (int i = 0; i < kNumBarsS; ++i)
            mbar_init(bar(i), (i == B_U_DONE || i == B_S_DONE0 || i == B_S_DONE1) ? kComputeWarps
                              : ((i == B_EMPTYG0 || i == B_EMPTYG1) && dual_task) ? 2 : 1);
        fence_mbar_init();
        *abort_flag = 0;
    }
    if (warp == 0) {
        tmem_alloc(base + OFF_MISC, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    // every barrier of the cluster is initialised before any CTA signals a peer
    cluster_sync_all();
    const uint32_t tmem = *tmem_slot;

    if (is_chain) {
        auto abuf = [&](int c) -> uint32_t { return base + C_A + (c & 1) * kPartA; };
        auto bbuf = [&](int c) -> uint32_t { return base + C_B + (c & 1) * kBStride; };
        auto vbuf = [&](int c) -> uint32_t { return base + C_V + (c % 3) * 16384; };
        if (warp < kComputeWarps) {
            // ============================================================ chain
            // Thread (warp, lane) holds half of row j of S^T: channels
            // 32 hf .. 32 hf + 31 in S[0..31] (the first half of the state
            // step, channels 0-63) and 64 + 32 hf .. in S[32..63] (the second).
            const int j = 32 * (warp & 3) + lane;        // row of S^T = value column = TMEM lane
            const int hf = warp >> 2;
            const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
            float S[64];
            if (tk.init == 1) {
                const float* s0 = tk.init_ptr + (size_t)(32 * hf) * kDv + j;
#pragma unroll
                for (int c = 0; c < 64; ++c) S[c] = s0[(size_t)((c & 31) + 64 * (c >> 5)) * kDv];
            } else {
                // zeros, or the identity (S[c] holds channel 32 hf + (c & 31) + 64 (c >> 5))
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    S[c] = (tk.init == 2 && 32 * hf + (c & 31) + 64 * (c >> 5) == j) ? 1.f : 0.f;
            }
            // bf16 S^T operand, channels 64 ph + 32 hf ..: columns 32 ph + 16 hf ..
            auto store_state_half = [&](int ph) {
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(S[32 * ph + 2 * i], S[32 * ph + 2 * i + 1]);
                tmem_st16(tmem + CT_S + lane_base + 32 * ph + 16 * hf, w);
                tmem_st_wait();
            };
            // one arrive per warp once all its lanes are done
            auto warp_arrive = [&](int bi) {
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(bi));
            };

            store_state_half(0);
            store_state_half(1);
            tc_fence_before_sync();
            warp_arrive(B_S_DONE0);
            warp_arrive(B_S_DONE1);
            bool failed = false;

            // Output rows of chunk c: O^T from columns 64-127 of its D1 buffer,
            // staged for a TMA store (full chunk) or written directly (partial
            // last chunk, so that nothing lands past the sequence).  Every
            // compute thread calls it.
            auto write_output = [&](int c) -> bool {
                const bool okw = wait_spin(bar(B_O_FULL0 + (c & 1)), (c >> 1) & 1, abort_flag, p.err);
                if (tid == 0) bulk_wait_group_read0();   // the last output store has read the staging
                if (named_barrier_or(BAR_ALL, kCompute, !okw)) return false;
                tc_fence_after_sync();
                const long long tc0 = t_begin + (long long)c * kC;
                const int Lc = (int)((t_end - tc0) < kC ? (t_end - tc0) : kC);
                float o[32];
                tmem_ld32(tmem + CT_D1 + 128 * (c & 1) + lane_base + 64 + 32 * hf, o);
                tmem_ld_wait();
                if (Lc == kC) {
                    unsigned short* ost = reinterpret_cast<unsigned short*>(sbase + C_OST) +
                                          (j >> 6) * 4096 + (j & 63);
#pragma unroll
                    for (int r = 0; r < 32; ++r)
                        ost[(32 * hf + r) * 64] = __bfloat16_as_ushort(__float2bfloat16_rn(o[r]));
                    fence_proxy_async_smem();
                } else {
                    const size_t rs = (size_t)H * kDv;
                    __nv_bfloat16* op = p.out + ((size_t)tc0 * H + h) * kDv + j + (size_t)(32 * hf) * rs;
#pragma unroll
                    for (int r = 0; r < 32; ++r)
                        if (32 * hf + r < Lc) op[r * rs] = __float2bfloat16_rn(o[r]);
                }
                tc_fence_before_sync();
                named_barrier(BAR_ALL, kCompute);
                if (tid == 0 && Lc == kC) {
                    tma_store_3d(&tm_o, base + C_OST, 0, h, (int)tc0);
                    tma_store_3d(&tm_o, base + C_OST + 8192, 64, h, (int)tc0);
                    bulk_commit_group();
                }
                return true;
            };

            for (int ci = 0; ci < n_chunks; ++ci) {
                const int b = ci & 1;
                const uint32_t d1 = CT_D1 + 128 * b;
                const bool has_next = ci + 1 < n_chunks;

                bool ok = wait_spin(bar(B_C1_FULL), ci & 1, abort_flag, p.err);
                if (warp == 0) ok = ok && wait_spin(bar(B_B_FULL0 + b), (ci >> 1) & 1, abort_flag, p.err);
                if (named_barrier_or(BAR_ALL, kCompute, !ok)) { failed = true; break; }
                tc_fence_after_sync();
                // ---- U^T to bf16 in place: half hf packs its 32 columns into
                // its own first 16, so that no warp writes columns another reads
                {
                    float x[32];
                    tmem_ld32(tmem + d1 + lane_base + 32 * hf, x);
                    tmem_ld_wait();
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
                    tmem_st16(tmem + d1 + lane_base + 32 * hf, w);
                    tmem_st_wait();
                }
                // Gamma out of part B, which is refilled once D^T and O^T are formed
                if (warp == 0)
                    reinterpret_cast<float4*>(sbase + C_GAM + b * 512)[lane] =
                        reinterpret_cast<const float4*>(sbase + (bbuf(ci) - base) + SL_GAM)[lane];
                tc_fence_before_sync();
                warp_arrive(B_U_DONE);

                // the previous chunk's output while this chunk's D^T is formed
                if (tk.out_on && ci > 0 && !write_output(ci - 1)) { failed = true; break; }

                ok = wait_spin(bar(B_C2_FULL), ci & 1, abort_flag, p.err);
                if (named_barrier_or(BAR_ALL, kCompute, !ok)) { failed = true; break; }
                tc_fence_after_sync();
                // ---- S^T_j = Gamma (S^T_j + D^T_j), one half of the channels
                // at a time: the issue warp starts the next chunk's [U^T | O^T]
                // on the first half while the second is updated
                {
                    float d0[32], d1[32];
                    tmem_ld32(tmem + CT_D2 + lane_base + 32 * hf, d0);
                    tmem_ld32(tmem + CT_D2 + lane_base + 64 + 32 * hf, d1);
                    tmem_ld_wait();
#pragma unroll
                    for (int ph = 0; ph < 2; ++ph) {
                        const float* gm = reinterpret_cast<const float*>(sbase + C_GAM + b * 512) + 64 * ph + 32 * hf;
#pragma unroll
                        for (int c = 0; c < 32; c += 4) {
                            const float4 g4 = *reinterpret_cast<const float4*>(gm + c);
                            const int o = 32 * ph + c;
                            add_mul_f32x2(S[o + 0], S[o + 1], ph ? d1[c + 0] : d0[c + 0], ph ? d1[c + 1] : d0[c + 1], g4.x, g4.y);
                            add_mul_f32x2(S[o + 2], S[o + 3], ph ? d1[c + 2] : d0[c + 2], ph ? d1[c + 3] : d0[c + 3], g4.z, g4.w);
                        }
                        // the products that read this chunk's S^T operand are done
                        if (has_next) store_state_half(ph);
                        tc_fence_before_sync();
                        warp_arrive(B_S_DONE0 + ph);
                    }
                }
            }
            if (!failed && tk.out_on && n_chunks > 0 && !write_output(n_chunks - 1)) failed = true;
            if (tid == 0) bulk_wait_group0();   // output stores complete before the CTA ends
            if (!failed && !*abort_flag && tk.fs_ptr) {
                float* fs = tk.fs_ptr + (size_t)(32 * hf) * kDv + j;
#pragma unroll
                for (int c = 0; c < 64; ++c) fs[(size_t)((c & 31) + 64 * (c >> 5)) * kDv] = S[c];
            }
        } else if (warp == kMmaWarp) {
            // ============================================================ chain issue
            if (lane == 0 && n_chunks > 0) {
                // operand descriptors of buffer 0 (buffers 1, 2 lie a fixed
                // number of bytes further on)
                const uint64_t dWQ = sw128_desc(abuf(0) + SL_WQ, 16);       // [-W; Qt], K-major
                const uint64_t dTB = sw128_desc(abuf(0) + SL_TB, 16);       // T, K-major
                const uint64_t dKP = sw128_desc(bbuf(0) + SL_KP, 8192);     // Kh, MN-major
                const uint64_t dPK = sw128_desc(bbuf(0) + SL_KP + 16384, 16);  // P, K-major
                const uint64_t dV  = sw128_desc(vbuf(0), 8192);             // v, MN-major
                // U'^T(c) = V^T T^T into columns 0-63 of D1 buffer c & 1; frees v buffer c % 3
                auto issue_uprime = [&](int c) {
                    const uint64_t vb = desc_add(dV, (c % 3) * 16384), tb = desc_add(dTB, (c & 1) * kPartA);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ss(tmem + CT_D1 + 128 * (c & 1), desc_add(vb, kk * 2048),
                                    desc_add(tb, kk * 32), ID_W, kk > 0);
                    mma_commit(bar(B_V_EMPTY0 + c % 3));
                };
                // [U^T | S^T Qt^T](c) = [U'^T | 0] + S^T(c) [-W; Qt]^T  (A = S^T bf16 in
                // tensor memory), K = channels 64 ph .. 64 ph + 63 once that half of
                // S^T(c) is written; the first K step adds to U'^T and starts
                // S^T Qt^T separately.  The second half frees part A.
                // with v = 0 (a transition run) there is no U'^T to add to
                const uint32_t acc_u = tk.v_on ? 1u : 0u;
                auto issue_c1 = [&](int c, int ph) {
                    const uint64_t wq = desc_add(dWQ, (c & 1) * kPartA);
                    const uint32_t dc = tmem + CT_D1 + 128 * (c & 1);
                    if (ph == 0) {
                        mma_bf16_ts(dc, tmem + CT_S, wq, ID_N64, acc_u);
                        mma_bf16_ts(dc + 64, tmem + CT_S, desc_add(wq, 8192), ID_N64, 0);
#pragma unroll
                        for (int kk = 1; kk < 4; ++kk)
                            mma_bf16_ts(dc, tmem + CT_S + kk * 8, desc_add(wq, kk * 32), ID_C1, 1);
                    } else {
#pragma unroll
                        for (int kk = 4; kk < 8; ++kk)
                            mma_bf16_ts(dc, tmem + CT_S + kk * 8, desc_add(wq, 16384 + (kk & 3) * 32), ID_C1, 1);
                        mma_commit(bar(B_C1_FULL));
                        mma_commit(bar(B_A_EMPTY0 + (c & 1)));
                    }
                };
                auto issue_c1_both = [&](int c, int parity) {
                    if (!wait_spin(bar(B_S_DONE0), parity, abort_flag, p.err)) return false;
                    tc_fence_after_sync();
                    issue_c1(c, 0);
                    if (!wait_spin(bar(B_S_DONE1), parity, abort_flag, p.err)) return false;
                    tc_fence_after_sync();
                    issue_c1(c, 1);
                    return true;
                };
                bool ok = wait_spin(bar(B_A_FULL0), 0, abort_flag, p.err) &&
                          (!tk.v_on || wait_spin(bar(B_V_FULL0), 0, abort_flag, p.err));
                if (ok) {
                    tc_fence_after_sync();
                    if (tk.v_on) issue_uprime(0);
                    ok = issue_c1_both(0, 0);
                }
                for (int ci = 0; ci < n_chunks && ok; ++ci) {
                    const int b = ci & 1;
                    const uint32_t d1 = CT_D1 + 128 * b;
                    const uint64_t kp = desc_add(dKP, b * kBStride), pk = desc_add(dPK, b * kBStride);
                    ok = wait_spin(bar(B_U_DONE), ci & 1, abort_flag, p.err) &&
                         wait_spin(bar(B_B_FULL0 + b), (ci >> 1) & 1, abort_flag, p.err);
                    if (!ok) break;
                    tc_fence_after_sync();
                    // D^T = U^T Kh, then O^T += U^T P^T  (K = 64 tokens: bf16 U^T
                    // columns 0-15, 32-47)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ts(tmem + CT_D2, tmem + d1 + 32 * (kk >> 1) + 8 * (kk & 1),
                                    desc_add(kp, kk * 2048), ID_C2, kk > 0);
                    mma_commit(bar(B_C2_FULL));
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ts(tmem + d1 + 64, tmem + d1 + 32 * (kk >> 1) + 8 * (kk & 1),
                                    desc_add(pk, kk * 32), ID_O2, 1);
                    mma_commit(bar(B_O_FULL0 + b));
                    mma_commit(bar(B_B_EMPTY0 + b));
                    if (ci + 1 < n_chunks) {
                        ok = wait_spin(bar(B_A_FULL0 + (b ^ 1)), ((ci + 1) >> 1) & 1, abort_flag, p.err) &&
                             (!tk.v_on ||
                              wait_spin(bar(B_V_FULL0 + (ci + 1) % 3), ((ci + 1) / 3) & 1, abort_flag, p.err));
                        if (!ok) break;
                        tc_fence_after_sync();
                        if (tk.v_on) issue_uprime(ci + 1);
                        ok = issue_c1_both(ci + 1, (ci + 1) & 1);
                    }
                }
                if (*abort_flag) {
                    mma_commit(bar(B_DRAIN));
                    mbar_wait_bounded(bar(B_DRAIN), 0, kWaitLimitNs);
                }
            }
        } else if (lane == 0) {
            // ============================================================ chain copy
            // Slot s of the ring holds chunks c = s (mod 2P), written by prep
            // rank 1 + c % P as its local chunk c / P.
            const int R = 2 * P;
            int n_v = 0;
            auto issue_v = [&](int c) {
                if (c >= 3 && !wait_bar(bar(B_V_EMPTY0 + c % 3), ((c - 3) / 3) & 1, abort_flag, p.err))
                    return false;
                const uint32_t fb = bar(B_V_FULL0 + c % 3);
                const int tok = (int)(t_begin + (long long)c * kC);
                mbar_arrive_expect_tx(fb, 16384);
                tma_load_3d(vbuf(c), &tm_v, fb, 0, h, tok);
                tma_load_3d(vbuf(c) + 8192, &tm_v, fb, 64, h, tok);
                ++n_v;
                return true;
            };
            // the chain holds both parts of chunk c: its slot goes back to the producer
            auto release = [&](int c) {
                if (!wait_bar(bar(B_A_FULL0 + (c & 1)), (c >> 1) & 1, abort_flag, p.err) ||
                    !wait_bar(bar(B_B_FULL0 + (c & 1)), (c >> 1) & 1, abort_flag, p.err))
                    return false;
                mbar_arrive_remote(mapa_shared(bar(B_EMPTYG0 + ((c / P) & 1)), 1 + c % P));
                return true;
            };
            bool ok = true;
            int n_a = 0, n_b = 0;                        // part loads issued
            if (n_chunks > 0 && tk.v_on) {
                prefetch_tensormap(&tm_v);
                ok = issue_v(0) && (n_chunks < 2 || issue_v(1));
            }
            for (int ci = 0; ci < n_chunks && ok; ++ci) {
                const int b = ci & 1, s = ci % R;
                const unsigned char* slot = ring + (size_t)s * kSlotStride;
                ok = wait_bar_cluster(bar(B_FULLG0 + s), (ci / R) & 1, abort_flag, p.err);
                if (!ok) break;
                fence_proxy_async_global();
                ok = ci < 2 || wait_bar(bar(B_A_EMPTY0 + b), ((ci - 2) >> 1) & 1, abort_flag, p.err);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(B_A_FULL0 + b), kPartA);
                bulk_load_g2s(abuf(ci), slot, kPartA, bar(B_A_FULL0 + b));
                ++n_a;
                ok = ci < 2 || wait_bar(bar(B_B_EMPTY0 + b), ((ci - 2) >> 1) & 1, abort_flag, p.err);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(B_B_FULL0 + b), kPartB);
                bulk_load_g2s(bbuf(ci), slot + kPartA, kPartB, bar(B_B_FULL0 + b));
                ++n_b;
                if (tk.v_on && ci + 2 < n_chunks) ok = issue_v(ci + 2);
                if (ok && ci >= 1) ok = release(ci - 1);
            }
            if (*abort_flag) {
                // copies still in flight land before the CTA ends
                for (int c = (n_v > 3 ? n_v - 3 : 0); c < n_v; ++c)
                    mbar_wait_bounded(bar(B_V_FULL0 + c % 3), (c / 3) & 1, kWaitLimitNs);
                for (int c = (n_a > 2 ? n_a - 2 : 0); c < n_a; ++c)
                    mbar_wait_bounded(bar(B_A_FULL0 + (c & 1)), (c >> 1) & 1, kWaitLimitNs);
                for (int c = (n_b > 2 ? n_b - 2 : 0); c < n_b; ++c)
                    mbar_wait_bounded(bar(B_B_FULL0 + (c & 1)), (c >> 1) & 1, kWaitLimitNs);
            }
        }
    } else {
        const int r = (int)rank - 1;
        const int M = (n_chunks > r) ? (n_chunks - r + P - 1) / P : 0;   // local chunks
        auto qk_buf = [&](int m) -> uint32_t { return base + P_QK + (m & 1) * 32768; };
        // k, q and g of local chunk m into buffers m & 1
        auto issue_qk = [&](int m) {
            const int row = (int)(t_begin + (long long)(r + P * m) * kC);
            const uint32_t dst = qk_buf(m), fb = bar(B_QK_FULL0 + (m & 1));
            mbar_arrive_expect_tx(fb, 65536);
            tma_load_3d(dst + 0, &tm_k, fb, 0, h, row);
            tma_load_3d(dst + 16384, &tm_k, fb, 64, h, row);
            tma_load_3d(dst + 8192, &tm_q, fb, 0, h, row);
            tma_load_3d(dst + 16384 + 8192, &tm_q, fb, 64, h, row);
            tma_load_3d(base + P_GS + (m & 1) * 32768, &tm_g, fb, 0, h, row);
        };
        if (warp < kComputeWarps) {
            // ============================================================ prep
            // Two groups of 4 warps on consecutive local chunks: group A (warps
            // 0-3) forms chunk m's decayed tiles, [A; P], the A rows and the P
            // tile and hands them to group B (warps 4-7), which forms T, W and
            // -W of chunk m while group A goes on with chunk m + 1.  Every
            // buffer of parity b is free again for chunk m + 2 once slot m went
            // out (k, q, g of m + 2 are loaded only then).
            const bool grp_a = warp < 4;
            const int gw = warp & 3;                      // warp within the group
            const int gt = tid & 127;                     // thread within the group
            const int c0 = lane * 4;                      // channels c0 .. c0 + 3
            const uint32_t lane_base = (uint32_t)(32 * gw) << 16;
            if (grp_a) {
                float* const tot_s = reinterpret_cast<float*>(sbase + P_TOT);
                auto beta_at = [&](int m) -> float {
                    const long long t = t_begin + (long long)(r + P * m) * kC + gt;
                    return (m < M && gt < kC && t < t_end) ? __ldg(p.beta + (size_t)t * H + h) : 0.f;
                };
                float beta_reg = beta_at(0);
                // byte offset of this thread's 4 channels in row i of a 128B-swizzled bf16 tile
                const uint32_t cq = (uint32_t)((c0 & 63) >> 3), cb = (uint32_t)((c0 & 7) << 1);
                auto swz = [&](int i) -> uint32_t { return ((cq ^ (uint32_t)(i & 7)) << 4) | cb; };
                const uint32_t in_off = (c0 >> 6) * 8192 + gw * 2048;    // Kh: rows 16 gw ..
                const uint32_t kq_off = (c0 >> 6) * 16384 + gw * 2048;   // [Kt; Qt]
                for (int m = 0; m < M; ++m) {
                    const int b = m & 1;
                    const long long t0 = t_begin + (long long)(r + P * m) * kC;
                    const int L = (int)((t_end - t0) < kC ? (t_end - t0) : kC);
                    const uint32_t kq = qk_buf(m);
                    const uint32_t kh = base + P_KP + b * 24576;    // Kh, then P at +16 KB
                    float* const gam_s = reinterpret_cast<float*>(sbase + P_GAM) + b * 128;
                    float* const beta_s = reinterpret_cast<float*>(sbase + P_BET) + b * 64;
                    float* const g_s = reinterpret_cast<float*>(sbase + P_GS + b * 32768);   // g, then A

                    bool ok = wait_bar(bar(B_QK_FULL0 + b), (m >> 1) & 1, abort_flag, p.err);
                    if (named_barrier_or(BAR_A, 128, !ok)) break;
                    if (gt < kC) beta_s[gt] = beta_reg;
                    beta_reg = beta_at(m + 1);
                    if (L < kC) {
                        // rows >= L belong to the next sequence or lie past the tensor
                        float4* gz = reinterpret_cast<float4*>(g_s);
                        uint4* kqz = reinterpret_cast<uint4*>(sbase + (kq - base));
                        for (int e = gt; e < (kC - L) * 32; e += 128) {
                            const int rr = L + e / 32, u = e % 32;
                            gz[rr * 32 + u] = make_float4(0.f, 0.f, 0.f, 0.f);
                        }
                        for (int e = gt; e < (kC - L) * 16; e += 128) {
                            const int rr = L + e / 16, u = e % 16;
                            const int off = (u >> 3) * 1024 + rr * 8 + (u & 7);
                            kqz[off] = make_uint4(0u, 0u, 0u, 0u);
                            kqz[off + 512] = make_uint4(0u, 0u, 0u, 0u);
                        }
                        named_barrier(BAR_A, 128);
                    }

                    // fused L2Norm: the inverse norms of this warp's 16 k rows and
                    // 16 q rows (lanes 2i, 2i + 1 hold row i's); the decayed tiles
                    // below take them as row factors of the decay factors, so k
                    // and q are never rewritten
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
                    // ---- decay factors e^{G}, e^{-G} per channel, decayed tiles -----
                    // The tiles: Kt = K e^G, Kh = K e^-G, Qt = scale Q e^G (with
                    // the L2Norm, the rows of K and Q scaled by their inverse norms).
                    auto decayed_row = [&](int i, const float (&e)[4], const float (&ei)[4]) {
                        const uint32_t o_in = in_off + i * 128 + swz(i);
                        const uint32_t o_kq = kq_off + i * 128 + swz(i);
                        const uint2 kw = ld_shared_v2(kq + o_kq);
                        const uint2 qw = ld_shared_v2(kq + o_kq + 8192);
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
                        float4* const gwt = reinterpret_cast<float4*>(g_s);
                        float pa[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll 4
                        for (int i = 0; i < 16; ++i) {
                            float4* const at = gwt + (gw * 16 + i) * 32 + (c0 >> 2);
                            const float4 z = *at;
                            const bool valid = gw * 16 + i < L;
                            const float4 a = valid ? make_float4(1.f + ex2_approx(-kLog2e * z.x),
                                                                 1.f + ex2_approx(-kLog2e * z.y),
                                                                 1.f + ex2_approx(-kLog2e * z.z),
                                                                 1.f + ex2_approx(-kLog2e * z.w))
                                                   : make_float4(1.f, 1.f, 1.f, 1.f);
                            *at = a;
                            pa[0] *= a.x; pa[1] *= a.y; pa[2] *= a.z; pa[3] *= a.w;
                        }
                        *reinterpret_cast<float4*>(tot_s + gw * 128 + c0) = make_float4(pa[0], pa[1], pa[2], pa[3]);
                        named_barrier(BAR_A, 128);
                        // the product of 1/alpha over the rows of the warps before
                        float ei[4] = {1.f, 1.f, 1.f, 1.f};
                        for (int w = 0; w < gw; ++w) {
                            const float4 t4 = *reinterpret_cast<const float4*>(tot_s + w * 128 + c0);
                            ei[0] *= t4.x; ei[1] *= t4.y; ei[2] *= t4.z; ei[3] *= t4.w;
                        }
                        if (gw == 3)
                            *reinterpret_cast<float4*>(gam_s + c0) =
                                make_float4(__frcp_rn(ei[0] * pa[0]), __frcp_rn(ei[1] * pa[1]),
                                            __frcp_rn(ei[2] * pa[2]), __frcp_rn(ei[3] * pa[3]));
#pragma unroll 4
                        for (int i = 0; i < 16; ++i) {
                            const float4 a = gwt[(gw * 16 + i) * 32 + (c0 >> 2)];
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
                            const float4 gi = *reinterpret_cast<const float4*>(g_s + (gw * 16 + i) * 128 + c0);
                            run[0] += gi.x; run[1] += gi.y; run[2] += gi.z; run[3] += gi.w;
                        }
                        *reinterpret_cast<float4*>(tot_s + gw * 128 + c0) =
                            make_float4(run[0] * kLog2e, run[1] * kLog2e, run[2] * kLog2e, run[3] * kLog2e);
                        named_barrier(BAR_A, 128);
                        float G[4] = {0.f, 0.f, 0.f, 0.f};
                        for (int w = 0; w < gw; ++w) {
                            const float4 t4 = *reinterpret_cast<const float4*>(tot_s + w * 128 + c0);
                            G[0] += t4.x; G[1] += t4.y; G[2] += t4.z; G[3] += t4.w;
                        }
                        if (gw == 3)
                            *reinterpret_cast<float4*>(gam_s + c0) =
                                make_float4(exp2f(fmaf(run[0], kLog2e, G[0])), exp2f(fmaf(run[1], kLog2e, G[1])),
                                            exp2f(fmaf(run[2], kLog2e, G[2])), exp2f(fmaf(run[3], kLog2e, G[3])));
#pragma unroll 2
                        for (int i = 0; i < 16; ++i) {
                            // rows reloaded (not kept from the totals above): a rolled
                            // loop keeps the prep's code small
                            const float4 gi = *reinterpret_cast<const float4*>(g_s + (gw * 16 + i) * 128 + c0);
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
                    named_barrier(BAR_A, 128);
                    if (gt == 0) {
                        tc_fence_after_sync();
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_bf16_ss(tmem + PT_AP, sw128_desc(kq + (kk >> 2) * 16384 + (kk & 3) * 32, 16),
                                        sw128_desc(kh + (kk >> 2) * 8192 + (kk & 3) * 32, 16), ID_AP, kk > 0);
                        mma_commit(bar(B_AP_FULL));
                    }

                    // ---- warp gw holds lanes 32 gw ..: the A rows (warps 0, 1) to
                    // fp32 scratch for the inverse, the P rows (warps 2, 3) to the
                    // K-major P tile
                    ok = wait_bar(bar(B_AP_FULL), m & 1, abort_flag, p.err);
                    if (named_barrier_or(BAR_A, 128, !ok)) break;
                    tc_fence_after_sync();
                    {
                        const int row = 32 * gw + lane;
#pragma unroll 1
                        for (int hh = 0; hh < 2; ++hh) {
                            float x[32];
                            tmem_ld32(tmem + PT_AP + lane_base + 32 * hh, x);
                            tmem_ld_wait();
                            if (gw < 2) {
                                const float bb = beta_s[row];
#pragma unroll
                                for (int i = 0; i < 32; i += 4)
                                    *reinterpret_cast<float4*>(g_s + sidx(row, 32 * hh + i)) =
                                        make_float4(bb * x[i], bb * x[i + 1], bb * x[i + 2], bb * x[i + 3]);
                            } else {
                                // P [i][j] (K-major B of U^T P^T): row i, j = 32 hh .., causal
                                const int rr = row - 64;
                                const uint32_t prow = kh + 16384 + rr * 128;
#pragma unroll
                                for (int u = 0; u < 4; ++u) {
                                    const int jj = 32 * hh + 8 * u;
                                    uint32_t w[4];
#pragma unroll
                                    for (int e = 0; e < 4; ++e)
                                        w[e] = pack_bf16x2(jj + 2 * e <= rr ? x[8 * u + 2 * e] : 0.f,
                                                           jj + 2 * e + 1 <= rr ? x[8 * u + 2 * e + 1] : 0.f);
                                    st_shared_v4(prow + (((4 * hh + u) ^ (rr & 7)) << 4), w[0], w[1], w[2], w[3]);
                                }
                            }
                        }
                    }
                    fence_proxy_async_smem();   // the P tile goes out by a bulk copy
                    tc_fence_before_sync();
                    named_barrier(BAR_A, 128);
                    if (gt == 0) mbar_arrive(bar(B_AB_FULL0 + b));
                }
                if (gt == 0 && *abort_flag) {
                    mma_commit(bar(B_DRAIN));
                    mbar_wait_bounded(bar(B_DRAIN), 0, kWaitLimitNs);
                }
            } else {
                for (int m = 0; m < M; ++m) {
                    const int b = m & 1;
                    const uint32_t kq = qk_buf(m);
                    const uint32_t tb = base + P_TB + b * 8192;
                    const float* const beta_s = reinterpret_cast<const float*>(sbase + P_BET) + b * 64;
                    float* const a_s = reinterpret_cast<float*>(sbase + P_GS + b * 32768);
                    float* const x_s = a_s + 4096;

                    bool ok = wait_bar(bar(B_AB_FULL0 + b), (m >> 1) & 1, abort_flag, p.err);
                    if (named_barrier_or(BAR_B, 128, !ok)) break;
                    // ---- T = (I + A)^-1 Diag(beta) -------------------------------
                    invert_unit_lower<BAR_SOLVE>(a_s, x_s, gt, gw, lane);
                    {
                        // row rr, columns 32 half ..; the upper-right 32 x 32 quadrant
                        // of X is never written (it is zero)
                        const int rr = gt >> 1, half = gt & 1;
                        float v[32];
                        if (rr < 32 && half == 1) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] = 0.f;
                        } else {
#pragma unroll
                            for (int q4 = 0; q4 < 8; ++q4) {
                                const int c = 32 * half + 4 * q4;
                                const float4 x4 = *reinterpret_cast<const float4*>(x_s + sidx(rr, c));
                                const float4 b4 = *reinterpret_cast<const float4*>(beta_s + c);
                                v[4 * q4 + 0] = x4.x * b4.x;
                                v[4 * q4 + 1] = x4.y * b4.y;
                                v[4 * q4 + 2] = x4.z * b4.z;
                                v[4 * q4 + 3] = x4.w * b4.w;
                            }
                        }
#pragma unroll
                        for (int ch = 0; ch < 4; ++ch) {
                            const int chunk = half * 4 + ch;
                            st_shared_v4(tb + rr * 128 + (((chunk ^ (rr & 7)) & 7) << 4),
                                         pack_bf16x2(v[8 * ch + 0], v[8 * ch + 1]),
                                         pack_bf16x2(v[8 * ch + 2], v[8 * ch + 3]),
                                         pack_bf16x2(v[8 * ch + 4], v[8 * ch + 5]),
                                         pack_bf16x2(v[8 * ch + 6], v[8 * ch + 7]));
                        }
                    }
                    fence_proxy_async_smem();
                    tc_fence_before_sync();
                    named_barrier(BAR_B, 128);
                    if (gt == 0) {
                        tc_fence_after_sync();
                        // W = T Kt in lanes 0-63 (B = Kt, MN-major: K rows = tokens).
                        // The A operand is 128 rows: rows 64-127 are whatever lies
                        // after T in shared memory, and their lanes are never read.
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_bf16_ss(tmem + PT_W, sw128_desc(tb + kk * 32, 16),
                                        sw128_desc(kq + kk * 2048, 16384), ID_WP, kk > 0);
                        mma_commit(bar(B_W_FULL));
                    }
                    ok = wait_bar(bar(B_W_FULL), m & 1, abort_flag, p.err);
                    if (named_barrier_or(BAR_B, 128, !ok)) break;
                    tc_fence_after_sync();
                    if (gw < 2) {
                        // -W [t][c] over Kt (rows 0-63 of the [Kt; Qt] tile, K-major):
                        // token t = this thread's lane row, 32 channels at a time
                        const int t = 32 * gw + lane;
#pragma unroll 1
                        for (int qq = 0; qq < 4; ++qq) {
                            float x[32];
                            tmem_ld32(tmem + PT_W + lane_base + 32 * qq, x);
                            tmem_ld_wait();
                            const uint32_t wrow = kq + (qq >> 1) * 16384 + t * 128;
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                uint32_t w[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    w[e] = pack_bf16x2(-x[8 * u + 2 * e], -x[8 * u + 2 * e + 1]);
                                st_shared_v4(wrow + (((4 * (qq & 1) + u) ^ (t & 7)) << 4), w[0], w[1], w[2], w[3]);
                            }
                        }
                    }
                    fence_proxy_async_smem();
                    tc_fence_before_sync();
                    named_barrier(BAR_B, 128);
                    if (gt == 0) {
                        // one READY ahead of the copy warp at most (a run-out wait
                        // aborts; the others leave at the next collective check)
                        if (m == 0 ||
                            wait_bar(bar(B_SENT0 + ((m - 1) & 1)), ((m - 1) >> 1) & 1, abort_flag, p.err))
                            mbar_arrive(bar(B_READY));
                    }
                }
                if (gt == 0 && *abort_flag) {
                    mma_commit(bar(B_DRAIN_B));
                    mbar_wait_bounded(bar(B_DRAIN_B), 0, kWaitLimitNs);
                }
            }
        } else if (warp == kCopyWarp && lane == 0) {
            // ============================================================ prep copy
            int n_qk = 0;
            if (M > 0) {
                prefetch_tensormap(&tm_q);
                prefetch_tensormap(&tm_k);
                prefetch_tensormap(&tm_g);
                issue_qk(0);
                ++n_qk;
                if (M > 1) { issue_qk(1); ++n_qk; }
            }
            for (int m = 0; m < M; ++m) {
                const int b = m & 1;
                const int s = r + P * b;                 // ring slot of local chunk m
                bool ok = wait_bar(bar(B_READY), m & 1, abort_flag, p.err);
                ok = ok && (m < 2 || wait_bar_cluster(bar(B_EMPTYG0 + b), ((m - 2) >> 1) & 1,
                                                      abort_flag, p.err));
                if (!ok) break;
                fence_proxy_async_global();
                unsigned char* dst = ring + (size_t)s * kSlotStride;
                const uint32_t kq = qk_buf(m);
                bulk_store_s2g(dst + SL_WQ, kq, 32768);
                bulk_store_s2g(dst + SL_TB, base + P_TB + b * 8192, 8192);
                unsigned char* dstb = dst + kPartA;
                bulk_store_s2g(dstb + SL_KP, base + P_KP + b * 24576, 24576);
                bulk_store_s2g(dstb + SL_GAM, base + P_GAM + b * 512, 512);
                bulk_commit_group();
                bulk_wait_group0();
                fence_proxy_async_global();
                mbar_arrive_remote(mapa_shared(bar(B_FULLG0 + s), 0));
                if (dual_task) mbar_arrive_remote(mapa_shared(bar(B_FULLG0 + s), P + 1));
                mbar_arrive(bar(B_SENT0 + b));
                if (m + 2 < M) { issue_qk(m + 2); ++n_qk; }
            }
            if (*abort_flag) {
                // the k, q loads still in flight land before the CTA ends
                for (int m = (n_qk > 2 ? n_qk - 2 : 0); m < n_qk; ++m)
                    mbar_wait_bounded(bar(B_QK_FULL0 + (m & 1)), (m >> 1) & 1, kWaitLimitNs);
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, tmem_cols);
    }
    // no CTA leaves while a peer may still signal one of its barriers
    cluster_sync_all();
}

// ------------------------------------------------------------------ host side
typedef void (*SplitKernel)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                            const CUtensorMap, const CUtensorMap, const SplitParams);

// The kernel's instantiation for the options of a call.
SplitKernel split_kernel(int l2norm, int raw_gate)
{
    return raw_gate ? (l2norm ? kda_chunk_split_kernel<true, true> : kda_chunk_split_kernel<false, true>)
                    : (l2norm ? kda_chunk_split_kernel<true, false> : kda_chunk_split_kernel<false, false>);
}

cudaError_t set_smem_attrs()
{
    for (int l2 = 0; l2 < 2; ++l2)
        for (int raw = 0; raw < 2; ++raw) {
            const cudaError_t e = cudaFuncSetAttribute(split_kernel(l2, raw),
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)kSmemBytesS);
            if (e != cudaSuccess) return e;
        }
    return cudaSuccess;
}

struct DeviceInfo {
    int sms = 0;
    int max_clusters[kMaxPrep + 1] = {0, 0, 0, 0};        // by P (one chain CTA)
    int max_clusters_dual[kMaxPrep + 1] = {0, 0, 0, 0};   // by P (two chain CTAs)
    bool ready = false;
};

std::mutex g_mutex;
DeviceInfo g_dev[64];

cudaError_t device_info(int dev, DeviceInfo** out)
{
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        cudaError_t e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        e = set_smem_attrs();
        if (e != cudaSuccess) return e;
        for (int P = 1; P <= kMaxPrep; ++P)
            for (int dual = 0; dual < 2; ++dual) {
                cudaLaunchConfig_t cfg = {};
                cudaLaunchAttribute at[1];
                at[0].id = cudaLaunchAttributeClusterDimension;
                at[0].val.clusterDim.x = P + 1 + dual;
                at[0].val.clusterDim.y = 1;
                at[0].val.clusterDim.z = 1;
                cfg.gridDim = dim3(P + 1 + dual);
                cfg.blockDim = dim3(kThreadsS);
                cfg.dynamicSmemBytes = kSmemBytesS;
                cfg.attrs = at;
                cfg.numAttrs = 1;
                int nc = 0;
                e = cudaOccupancyMaxActiveClusters(&nc, kda_chunk_split_kernel<false, false>, &cfg);
                if (e != cudaSuccess) return e;
                (dual ? d.max_clusters_dual : d.max_clusters)[P] = nc;
            }
        d.ready = true;
    }
    *out = &d;
    return cudaSuccess;
}

int g_forced_kernel = 0;     // 0 automatic, 1 one CTA per chain, 2 one cluster per chain,
                             // 3 segmented clusters
int g_forced_segments = 0;   // segments of a segmented run (0: by the cost model)
int g_dual_mode = 0;         // first pass: 0 cheaper layout, 1 separate clusters, 2 shared prep

// Relative cost of one chunk-step of a cluster with P prep CTAs, in
// thousands of cycles: the chain CTA needs about 2.9k per chunk and one prep
// CTA about 8.3k, so with three prep CTAs the chain sets the pace and with
// fewer the prep does (measured on the long-prefill workload).
double chunk_step_cost(int P)
{
    return P >= 3 ? 3.1 : (P == 2 ? 4.3 : 8.3);
}

// The most prep CTAs (<= kMaxPrep) with which `clusters` clusters of P CTAs
// and one chain CTA (two with `dual`) are all resident at once; 0 if not
// even P = 1 fits.
int resident_prep(const DeviceInfo& d, long long clusters, bool dual = false)
{
    for (int c = kMaxPrep; c >= 1; --c)
        if (clusters * (c + 1 + (dual ? 1 : 0)) <= d.sms &&
            clusters <= (dual ? d.max_clusters_dual : d.max_clusters)[c])
            return c;
    return 0;
}

// Segmented-run plan with G segments: prep CTAs of the two passes and the
// estimated time in chunk-step units (0 P: not every cluster fits at once).
struct SegPlan {
    int G = 0, P1 = 0, P3 = 0;
    bool dual = false;     // first pass with two chain CTAs per cluster
    double cost = 0.0;
};

// The first pass either runs the zero-start and transition runs of a
// segment in separate clusters (2G - 3 per chain) or in one cluster with
// two chain CTAs that share its prep CTAs (G - 1 per chain); the cheaper
// resident choice is taken.
SegPlan seg_plan(const DeviceInfo& d, long long chains, long long chunks, int G)
{
    SegPlan s;
    s.G = G;
    const int p_single = resident_prep(d, chains * (2 * G - 3 > 0 ? 2 * G - 3 : 1));
    const int p_dual = G >= 3 ? resident_prep(d, chains * (G - 1), true) : 0;
    // two chain CTAs on one prep set run at the chain's pace with three prep
    // CTAs but a third slower than one chain with fewer (measured)
    auto dual_cost = [](int P) { return chunk_step_cost(P) * (P < 3 ? 1.33 : 1.0); };
    if (g_dual_mode == 1 || G < 3) {
        s.dual = false;
    } else if (g_dual_mode == 2) {
        s.dual = true;
    } else {
        s.dual = p_dual > 0 && (p_single == 0 || dual_cost(p_dual) < chunk_step_cost(p_single));
    }
    s.P1 = s.dual ? p_dual : p_single;
    s.P3 = resident_prep(d, chains * (G - 1));
    const long long cps = (chunks + G - 1) / G;
    const double step1 = s.dual ? dual_cost(s.P1) : chunk_step_cost(s.P1);
    // the prefix pass between the two: about 3 chunk-steps per segment
    s.cost = (double)cps * (step1 + chunk_step_cost(s.P3)) + 3.0 * (G - 2);
    return s;
}

}  // namespace

void set_prefill_kernel(int kind) { g_forced_kernel = kind; }
int prefill_kernel_setting() { return g_forced_kernel; }
void set_prefill_segments(int segments) { g_forced_segments = segments; }
void set_prefill_dual(int mode) { g_dual_mode = mode; }

PrefillPlan plan_prefill(const ChunkArgs& a)
{
    PrefillPlan pl;
    const long long chains = (long long)a.N * a.H;
    const long long tokens = (long long)a.B * a.T;
    if (chains <= 0 || tokens == 0 || g_forced_kernel == 1) return pl;   // one CTA per chain
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return pl;
    DeviceInfo* d = nullptr;
    if (device_info(dev, &d) != cudaSuccess) return pl;
    // chunks per sequence (the mean for packed sequences)
    const long long chunks = (tokens / (a.N > 0 ? a.N : 1) + kC - 1) / kC;
    // Enough SMs for at least two per chain: as many prep CTAs per chain as
    // fit (at most kMaxPrep) with every cluster resident at once.
    int P = resident_prep(*d, chains);
    if (P == 0 && g_forced_kernel == 0) return pl;
    if (P == 0) P = 1;
    if (g_forced_kernel == 3 || (g_forced_kernel == 0 && chunks >= 64)) {
        // Segmented: worth it when the chains are so few that the SMs a
        // plain run leaves idle can carry the extra transition runs.
        SegPlan best;
        if (g_forced_kernel == 3 && g_forced_segments >= 2) {
            best = seg_plan(*d, chains, chunks, g_forced_segments);
        } else {
            for (int G = 3; G <= 64 && G <= chunks; ++G) {
                const SegPlan s = seg_plan(*d, chains, chunks, G);
                if (s.P1 == 0 || s.P3 == 0) continue;
                if (best.G == 0 || s.cost < best.cost) best = s;
            }
            if (g_forced_kernel == 3 && best.G == 0) best = seg_plan(*d, chains, chunks, 3);
        }
        const double plain = (double)chunks * chunk_step_cost(P);
        if (best.G >= 2 && (g_forced_kernel == 3 || best.cost < 0.85 * plain)) {
            pl.kind = 3;
            pl.G = best.G;
            pl.P1 = best.P1 > 0 ? best.P1 : 1;
            pl.P3 = best.P3 > 0 ? best.P3 : 1;
            pl.dual = best.dual;
            const long long c1 = chains * (pl.dual ? pl.G - 1 : (pl.G >= 3 ? 2 * pl.G - 3 : 1));
            const long long c3 = chains * (pl.G - 1);
            const size_t r1 = split_ring_bytes(c1, pl.P1), r3 = split_ring_bytes(c3, pl.P3);
            pl.ring_bytes = r1 > r3 ? r1 : r3;
            pl.seg_bytes = (size_t)chains * 3 * pl.G * kDk * kDv * sizeof(float);
            return pl;
        }
    }
    pl.kind = 2;
    pl.P = P;
    pl.ring_bytes = split_ring_bytes(chains, P);
    return pl;
}

int split_prep_ctas(const ChunkArgs& a)
{
    const PrefillPlan pl = plan_prefill(a);
    return pl.kind == 2 ? pl.P : 0;
}

size_t split_ring_bytes(long long chains, int P)
{
    return chains > 0 && P > 0 ? (size_t)chains * 2 * P * kSlotStride : 0;
}

namespace {

// One launch of the cluster kernel: `clusters` clusters of 1 + P CTAs.
cudaError_t launch_split(const ChunkArgs& a, int P, int phase, int G, unsigned char* ring,
                         float* seg, long long clusters, cudaStream_t stream, bool dual = false)
{
    if (P < 1 || P > kMaxPrep) return cudaErrorInvalidValue;
    if (clusters <= 0) return cudaSuccess;
    const long long tokens = (long long)a.B * a.T;
    if (tokens <= 0 || tokens > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (dual && phase != 1) return cudaErrorInvalidValue;
    const int csize = P + 1 + (dual ? 1 : 0);
    if (clusters * csize > 0x7fffffffLL) return cudaErrorInvalidValue;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    DeviceInfo* d = nullptr;
    e = device_info(dev, &d);
    if (e != cudaSuccess) return e;
    CUtensorMap tq, tk, tv, tg, to;
    if (!make_map(&tq, a.q, kDk, tokens, a.H, false) || !make_map(&tk, a.k, kDk, tokens, a.H, false) ||
        !make_map(&tv, a.v, kDv, tokens, a.H, false) ||
        !make_map(&tg, a.log_alpha, kDk, tokens, a.H, true) ||
        !make_map(&to, a.out, kDv, tokens, a.H, false, false))
        return cudaErrorInvalidValue;
    SplitParams p;
    p.beta = a.beta;
    p.initial_state = a.initial_state;
    p.cu_seqlens = a.cu_seqlens;
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.final_state = a.final_state;
    p.err = a.err;
    p.ring = ring;
    p.scale = a.scale;
    p.T = a.T;
    p.H = a.H;
    p.N = a.N;
    p.P = P;
    p.l2norm = a.l2norm;
    p.G = G;
    p.phase = phase;
    p.seg = seg;
    p.dual = dual ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = csize;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(clusters * csize));
    cfg.blockDim = dim3(kThreadsS);
    cfg.dynamicSmemBytes = kSmemBytesS;
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, split_kernel(p.l2norm, a.raw_gate), tq, tk, tv, tg, to, p);
}

// S_in(g + 1) = M_g S_in(g) + B_g for g = 1 .. G-2, in fp32, per chain: block
// (chain, cb) carries value columns 16 cb .. 16 cb + 15 of the state.
constexpr int kPrefixThreads = 256;
constexpr int kPrefixCols = 16;
constexpr int kPrefixLdM = kDk + 1;            // padded rows of M_g in shared memory

__global__ void __launch_bounds__(kPrefixThreads)
kda_segment_prefix_kernel(float* __restrict__ seg, int G)
{
    extern __shared__ float pm[];
    float* const Ms = pm;                                  // [dk][kPrefixLdM]
    float* const Ss = pm + kDk * kPrefixLdM;               // [dk][kPrefixCols]
    const int chain = blockIdx.x, cb = blockIdx.y, tid = threadIdx.x;
    const int col0 = cb * kPrefixCols;
    const size_t slot = (size_t)kDk * kDv;
    float* const base = seg + (size_t)chain * 3 * G * slot;
    const float* s1 = base + (size_t)(2 * G + 1) * slot;
    for (int e = tid; e < kDk * kPrefixCols; e += kPrefixThreads)
        Ss[e] = s1[(size_t)(e / kPrefixCols) * kDv + col0 + e % kPrefixCols];
    const int r = tid >> 1, c0 = 8 * (tid & 1);
    for (int g = 1; g <= G - 2; ++g) {
        const float* M = base + (size_t)g * slot;
        const float* Bg = base + (size_t)(G + g) * slot;
        for (int e = tid; e < kDk * kDk; e += kPrefixThreads)
            Ms[(e / kDk) * kPrefixLdM + e % kDk] = M[e];
        __syncthreads();
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = Bg[(size_t)r * kDv + col0 + c0 + c];
        for (int k = 0; k < kDk; ++k) {
            const float m = Ms[r * kPrefixLdM + k];
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[c] = fmaf(m, Ss[k * kPrefixCols + c0 + c], acc[c]);
        }
        __syncthreads();
        float* out = base + (size_t)(2 * G + g + 1) * slot;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            Ss[r * kPrefixCols + c0 + c] = acc[c];
            out[(size_t)r * kDv + col0 + c0 + c] = acc[c];
        }
        __syncthreads();
    }
}

// S_out = M S_in + B per chain (block (chain, cb): value columns 16 cb ..
// 16 cb + 15), in fp32; S_out may be B, not M or S_in.
__global__ void __launch_bounds__(kPrefixThreads)
kda_state_affine_kernel(const float* __restrict__ M, const float* B, const float* __restrict__ S_in,
                        float* S_out)
{
    extern __shared__ float pm[];
    float* const Ms = pm;
    float* const Ss = pm + kDk * kPrefixLdM;
    const int chain = blockIdx.x, cb = blockIdx.y, tid = threadIdx.x;
    const int col0 = cb * kPrefixCols;
    const size_t off = (size_t)chain * kDk * kDv;
    for (int e = tid; e < kDk * kPrefixCols; e += kPrefixThreads)
        Ss[e] = S_in[off + (size_t)(e / kPrefixCols) * kDv + col0 + e % kPrefixCols];
    for (int e = tid; e < kDk * kDk; e += kPrefixThreads)
        Ms[(e / kDk) * kPrefixLdM + e % kDk] = M[(size_t)chain * kDk * kDk + e];
    __syncthreads();
    const int r = tid >> 1, c0 = 8 * (tid & 1);
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = B[off + (size_t)r * kDv + col0 + c0 + c];
    for (int k = 0; k < kDk; ++k) {
        const float m = Ms[r * kPrefixLdM + k];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = fmaf(m, Ss[k * kPrefixCols + c0 + c], acc[c]);
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) S_out[off + (size_t)r * kDv + col0 + c0 + c] = acc[c];
}

// `units` identity matrices [dk][dk] (the transition of an empty sequence).
__global__ void kda_identity_kernel(float* __restrict__ M, long long n)
{
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n;
         e += (long long)gridDim.x * blockDim.x) {
        const int rc = (int)(e % (kDk * kDk));
        M[e] = (rc / kDk == rc % kDk) ? 1.f : 0.f;
    }
}

size_t prefix_smem_bytes()
{
    return (size_t)(kDk * kPrefixLdM + kDk * kPrefixCols) * sizeof(float);
}

}  // namespace

size_t transition_workspace_bytes(const ChunkArgs& a)
{
    const long long chains = (long long)a.N * a.H;
    if (chains <= 0 || (long long)a.B * a.T == 0) return 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    DeviceInfo* d = nullptr;
    if (device_info(dev, &d) != cudaSuccess) return 0;
    const int P = resident_prep(*d, chains);
    return split_ring_bytes(chains, P > 0 ? P : 1);
}

cudaError_t launch_chunk_transition(const ChunkArgs& a, float* transition, cudaStream_t stream)
{
    const long long chains = (long long)a.N * a.H;
    if (chains == 0) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    DeviceInfo* d = nullptr;
    e = device_info(dev, &d);
    if (e != cudaSuccess) return e;
    int P = resident_prep(*d, chains);
    if (P == 0) P = 1;
    if (!a.workspace || a.workspace_bytes < split_ring_bytes(chains, P) ||
        reinterpret_cast<uintptr_t>(a.workspace) % 256 != 0)
        return cudaErrorInvalidValue;
    // v and out are never touched (v = 0, no outputs); q stands in for them
    // so that their tensor maps are valid
    ChunkArgs t = a;
    t.v = a.q;
    t.out = const_cast<void*>(a.q);
    t.initial_state = nullptr;
    t.final_state = transition;
    return launch_split(t, P, 4, 1, static_cast<unsigned char*>(a.workspace), nullptr, chains, stream);
}

cudaError_t launch_identity_states(float* M, long long units, cudaStream_t stream)
{
    if (units <= 0) return cudaSuccess;
    const long long n = units * kDk * kDk;
    const long long blocks = (n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096;
    kda_identity_kernel<<<(unsigned)blocks, 256, 0, stream>>>(M, n);
    return cudaGetLastError();
}

cudaError_t launch_state_affine(const float* M, const float* B, const float* S_in, float* S_out,
                                long long chains, cudaStream_t stream)
{
    if (chains <= 0) return cudaSuccess;
    const size_t smem = prefix_smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(kda_state_affine_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kda_state_affine_kernel<<<dim3((unsigned)chains, kDv / kPrefixCols), kPrefixThreads, smem, stream>>>(
        M, B, S_in, S_out);
    return cudaGetLastError();
}

cudaError_t launch_chunk_split(const ChunkArgs& a, const PrefillPlan& pl, cudaStream_t stream)
{
    const long long chains = (long long)a.N * a.H;
    if (chains == 0) return cudaSuccess;
    const size_t need = pl.ring_bytes + pl.seg_bytes;
    // the hand-off ring (cluster k uses bytes [k, k + 1) * 2 P kSlotStride),
    // then the segment states, in the caller's workspace
    if (!a.workspace || a.workspace_bytes < need || reinterpret_cast<uintptr_t>(a.workspace) % 256 != 0)
        return cudaErrorInvalidValue;
    unsigned char* ring = static_cast<unsigned char*>(a.workspace);
    if (pl.kind == 2) return launch_split(a, pl.P, 0, 1, ring, nullptr, chains, stream);
    if (pl.kind != 3 || pl.G < 2) return cudaErrorInvalidValue;
    float* seg = reinterpret_cast<float*>(ring + pl.ring_bytes);
    const int G = pl.G;
    const long long c1 = chains * (pl.dual ? G - 1 : (G >= 3 ? 2 * G - 3 : 1));
    cudaError_t e = launch_split(a, pl.P1, 1, G, ring, seg, c1, stream, pl.dual);
    if (e != cudaSuccess) return e;
    if (G >= 3) {
        const size_t smem = prefix_smem_bytes();
        e = cudaFuncSetAttribute(kda_segment_prefix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        kda_segment_prefix_kernel<<<dim3((unsigned)chains, kDv / kPrefixCols), kPrefixThreads, smem,
                                    stream>>>(seg, G);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return launch_split(a, pl.P3, 3, G, ring, seg, chains * (G - 1), stream);
}

// ------------------------------------------------------------------ no-alloc variant
// kda_chunk_fwd_noalloc runs the same cluster kernel with its hand-off ring in
// this fixed device array instead of memory from the library's pool.  It
// serves callers that must not allocate device memory while they run: an
// engine that reserves nearly all of HBM for its per-request state caches up
// front and runs every step at a fixed footprint, where a pool that grows on
// first use could fail or push out other memory in the middle of a step.
// The array is the whole budget; rings that need more are rejected.  Nothing
// in it must start at zero: every ring slot is written by its prep CTA before
// the chain CTA reads it.  Every call uses the same array, so calls whose
// executions overlap in time race on it.
namespace {
constexpr size_t kNoAllocRingBytes = size_t(16) << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_ring[kNoAllocRingBytes];

struct NoAllocDevice {
    unsigned char* ring = nullptr;
    int sms = 0;
    int max_clusters[kMaxPrep + 1] = {0, 0, 0, 0};
};
NoAllocDevice g_noalloc[64];
std::mutex g_noalloc_mutex;

// Ring address, SM count and cluster residency of the current device, looked
// up once per device (none of these calls allocates).
cudaError_t noalloc_device(int dev, NoAllocDevice** out)
{
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    NoAllocDevice& d = g_noalloc[dev];
    if (!d.ring) {
        void* ptr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_ring);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        e = set_smem_attrs();
        if (e != cudaSuccess) return e;
        for (int P = 1; P <= kMaxPrep; ++P) {
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = P + 1;
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            cfg.gridDim = dim3(P + 1);
            cfg.blockDim = dim3(kThreadsS);
            cfg.dynamicSmemBytes = kSmemBytesS;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            e = cudaOccupancyMaxActiveClusters(&d.max_clusters[P], kda_chunk_split_kernel<false, false>, &cfg);
            if (e != cudaSuccess) return e;
        }
        d.ring = static_cast<unsigned char*>(ptr);
    }
    *out = &d;
    return cudaSuccess;
}
}  // namespace

bool noalloc_ring_fits(long long chains)
{
    return chains >= 0 && (size_t)chains * 2 * kSlotStride <= kNoAllocRingBytes;
}

cudaError_t launch_chunk_split_noalloc(const ChunkArgs& a, cudaStream_t stream)
{
    const long long chains = (long long)a.N * a.H;
    if (chains == 0) return cudaSuccess;
    if (!noalloc_ring_fits(chains)) return cudaErrorInvalidValue;
    const long long tokens = (long long)a.B * a.T;
    if (tokens <= 0 || tokens > 0x7fffffffLL) return cudaErrorInvalidValue;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    NoAllocDevice* d = nullptr;
    e = noalloc_device(dev, &d);
    if (e != cudaSuccess) return e;
    // as many prep CTAs as fit the SMs, the resident clusters and the array
    int P = 1;
    for (int c = kMaxPrep; c >= 1; --c) {
        if ((size_t)chains * 2 * c * kSlotStride <= kNoAllocRingBytes &&
            chains * (c + 1) <= d->sms && chains <= d->max_clusters[c]) {
            P = c;
            break;
        }
    }
    // Cluster k uses ring bytes [k, k + 1) * 2 P kSlotStride: every slot the
    // launch can touch must lie inside the array, whichever P was chosen.
    if ((size_t)chains * 2 * P * kSlotStride > kNoAllocRingBytes) return cudaErrorInvalidValue;
    CUtensorMap tq, tk, tv, tg, to;
    if (!make_map(&tq, a.q, kDk, tokens, a.H, false) || !make_map(&tk, a.k, kDk, tokens, a.H, false) ||
        !make_map(&tv, a.v, kDv, tokens, a.H, false) ||
        !make_map(&tg, a.log_alpha, kDk, tokens, a.H, true) ||
        !make_map(&to, a.out, kDv, tokens, a.H, false, false))
        return cudaErrorInvalidValue;
    SplitParams p;
    p.beta = a.beta;
    p.initial_state = a.initial_state;
    p.cu_seqlens = a.cu_seqlens;
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.final_state = a.final_state;
    p.err = a.err;
    p.ring = d->ring;
    p.scale = a.scale;
    p.T = a.T;
    p.H = a.H;
    p.N = a.N;
    p.P = P;
    p.l2norm = a.l2norm;
    p.G = 1;
    p.phase = 0;
    p.seg = nullptr;
    p.dual = 0;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = P + 1;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(chains * (P + 1)));
    cfg.blockDim = dim3(kThreadsS);
    cfg.dynamicSmemBytes = kSmemBytesS;
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, split_kernel(p.l2norm, a.raw_gate), tq, tk, tv, tg, to, p);
}

}  // namespace kda
