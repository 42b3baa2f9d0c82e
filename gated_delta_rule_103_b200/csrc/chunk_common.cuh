// Pieces shared by the tensor-core chunked prefill kernels: bf16 packing and
// shared-memory stores of 128B-swizzled operand rows, bounded mbarrier waits,
// the blocked triangular inverse (I + A)^-1, and the host-side TMA maps of the
// [tokens][H][d] tensors.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_internal.h"
#include "sm100_ptx.cuh"

namespace kda {
namespace tc {

using namespace ptx;

constexpr int kC = kChunk;                            // 64
constexpr uint64_t kWaitLimitNs = 2000000000ull;      // 2 s without progress
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// s = (s + d) * g on two fp32 values at once (packed f32x2 arithmetic of
// sm_100; each operation rounds to nearest like its scalar form).
__device__ __forceinline__ void add_mul_f32x2(float& s0, float& s1, float d0, float d1, float g0,
                                              float g1)
{
    asm("{\n\t.reg .b64 s, d, g;\n\t"
        "mov.b64 s, {%0, %1};\n\t"
        "mov.b64 d, {%2, %3};\n\t"
        "mov.b64 g, {%4, %5};\n\t"
        "add.rn.f32x2 s, s, d;\n\t"
        "mul.rn.f32x2 s, s, g;\n\t"
        "mov.b64 {%0, %1}, s;\n\t}"
        : "+f"(s0), "+f"(s1) : "f"(d0), "f"(d1), "f"(g0), "f"(g1));
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

// Sum of the squares of 4 bf16 values (two packed pairs): a lane's share of
// the squared norm of a q or k row in the fused L2Norm ("深度解读报告" 3.2,
// every row divided by max(||row||_2, 1e-6)).
__device__ __forceinline__ float sq_sum4(uint2 w)
{
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
    return fmaf(a.x, a.x, fmaf(a.y, a.y, fmaf(b.x, b.x, b.y * b.y)));
}

// One round of a transposing warp sum over an array of A values: N values
// remain, exchanged across lane bit S.
template <int A, int N, int S>
__device__ __forceinline__ void warp_sum_round(float (&v)[A], int lane)
{
    if constexpr (N > 1) {
        constexpr int half = N / 2;
        const bool up = (lane & S) != 0;
#pragma unroll
        for (int j = 0; j < half; ++j) {
            const float send = up ? v[j] : v[j + half];
            const float keep = up ? v[j + half] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, S);
        }
        if constexpr (S > 1) warp_sum_round<A, half, S / 2>(v, lane);
    } else {
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], S);
        if constexpr (S > 1) warp_sum_round<A, 1, S / 2>(v, lane);
    }
}

// Sums 16 values, each split over the 32 lanes of a warp, with one
// transposing butterfly: every round exchanges half of the values that
// remain, so the warp spends 16 shuffles instead of 5 per value.  Lanes 2i
// and 2i + 1 end with the total of value i.
__device__ __forceinline__ float warp_sum16(float (&v)[16], int lane)
{
    warp_sum_round<16, 16, 16>(v, lane);
    return v[0];
}

// The same for 8 values (11 shuffles): lanes 4i .. 4i + 3 end with the total
// of value i.
__device__ __forceinline__ float warp_sum8(float (&v)[8], int lane)
{
    warp_sum_round<8, 8, 16>(v, lane);
    return v[0];
}

// Elementwise product of two bf16 pairs, rounded to nearest.
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b)
{
    const __nv_bfloat162 r = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                                     *reinterpret_cast<const __nv_bfloat162*>(&b));
    return *reinterpret_cast<const uint32_t*>(&r);
}

// Writes 64 fp32 values as one 128-byte swizzled bf16 row.
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

// Index of element (r, c) of a 64 x 64 fp32 tile whose 16-byte groups are
// XOR-swizzled by (r & 7).
__device__ __forceinline__ int sidx(int r, int c)
{
    return r * 64 + ((((c >> 2) ^ (r & 7))) << 2) + (c & 3);
}

// Barrier-wide OR of `pred` over the `n` threads of named barrier `id`.
__device__ __forceinline__ bool named_barrier_or(int id, int n, bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r) : "r"((uint32_t)pred), "r"(id), "r"(n) : "memory");
    return r != 0;
}

// The polling loop of wait_bar, out of line, so that every wait costs the
// kernels' loops one poll of code: those loops are about as large as the SM's
// instruction cache (≈ 32 KB on B200).
static __device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           unsigned* err, uint64_t limit_ns)
{
    const uint64_t t0 = globaltimer();
    while (true) {
        // back off so that a waiting warp leaves its scheduler's issue slots
        // to the warps that work
        __nanosleep(64);
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit_ns) {
            *abort_flag = 1;
            atomicOr(err, kErrTimeout);
            return false;
        }
    }
}

// Waits (bounded) for completion of the mbarrier phase with parity `parity`.
// Gives up when the CTA has aborted or after limit_ns (2 s unless a caller
// passes less), aborting it.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned* err, uint64_t limit_ns = kWaitLimitNs)
{
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bar_slow(bar, parity, abort_flag, err, limit_ns);
}

// tf32 fragments of m16n8k8 tiles of a swizzled 64 x 64 fp32 tile (fp32
// bits are passed as they are; the tensor core uses their tf32 part).
__device__ __forceinline__ void frag_a(uint32_t (&a)[4], const float* M, int r0, int k0, int lane)
{
    const int g = lane >> 2, t = lane & 3;
    a[0] = __float_as_uint(M[sidx(r0 + g, k0 + t)]);
    a[1] = __float_as_uint(M[sidx(r0 + g + 8, k0 + t)]);
    a[2] = __float_as_uint(M[sidx(r0 + g, k0 + t + 4)]);
    a[3] = __float_as_uint(M[sidx(r0 + g + 8, k0 + t + 4)]);
}

__device__ __forceinline__ void frag_b(uint32_t (&b)[2], const float* M, int k0, int n0, int lane)
{
    const int g = lane >> 2, t = lane & 3;
    b[0] = __float_as_uint(M[sidx(k0 + t, n0 + g)]);
    b[1] = __float_as_uint(M[sidx(k0 + t + 4, n0 + g)]);
}

__device__ __forceinline__ void store_frag_d(float* M, const float (&d)[4], int r0, int n0, int lane,
                                             float sign)
{
    const int g = lane >> 2, t = lane & 3;
    M[sidx(r0 + g, n0 + 2 * t)] = sign * d[0];
    M[sidx(r0 + g, n0 + 2 * t + 1)] = sign * d[1];
    M[sidx(r0 + g + 8, n0 + 2 * t)] = sign * d[2];
    M[sidx(r0 + g + 8, n0 + 2 * t + 1)] = sign * d[3];
}

// X = (I + A)^-1 for strictly lower-triangular A (64 x 64, fp32, swizzled),
// by blocked forward substitution on the 4 prep warps (128 threads):
//   level 0: the 16 x 16 diagonal blocks X_ww = (I + A_ww)^-1 by forward
//            substitution, one column per thread (exact fp32);
//   level 1: X_{a,a-1} = -X_aa (A_{a,a-1} X_{a-1,a-1}) for a = 1, 3;
//   level 2: X_BA = -X_BB (A_BA X_AA) for the 32 x 32 halves;
// levels 1 and 2 with m16n8k8 tf32 mma.sync.  Upper blocks that level 2
// reads are zeroed.  Run by 4 warps (tid 0-127, warp 0-3) that synchronise on
// named barrier kBar; ends with that barrier.
template <int kBar>
__device__ __forceinline__ void invert_unit_lower(const float* __restrict__ A,
                                                  float* __restrict__ X, int tid, int warp, int lane)
{
    if (tid < 64) {
        const int b0 = 16 * (tid >> 4), m = tid & 15;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            // row i of the diagonal block, 4 elements per shared-memory access
            float a[16];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                if (4 * q4 < i) {
                    const float4 v = *reinterpret_cast<const float4*>(A + sidx(b0 + i, b0 + 4 * q4));
                    a[4 * q4] = v.x; a[4 * q4 + 1] = v.y; a[4 * q4 + 2] = v.z; a[4 * q4 + 3] = v.w;
                }
            }
            float acc0 = (i == m) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
            for (int q = 0; q + 1 < i; q += 2) {
                acc0 = fmaf(-a[q], x[q], acc0);
                acc1 = fmaf(-a[q + 1], x[q + 1], acc1);
            }
            if (i & 1) acc0 = fmaf(-a[i - 1], x[i - 1], acc0);
            x[i] = acc0 + acc1;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) X[sidx(b0 + i, b0 + m)] = x[i];
    } else {
        // zero blocks (0,1) and (2,3)
        const int z = tid - 64;             // 0..63
        const int r0 = (z < 32) ? 0 : 32;   // block row base
        const int rr = (z & 31) >> 1;       // 0..15
        const int cc = (z & 1) * 8;         // 0 or 8
#pragma unroll
        for (int e = 0; e < 8; ++e) X[sidx(r0 + rr, r0 + 16 + cc + e)] = 0.f;
    }
    named_barrier(kBar, 128);
    // level 1: warp w handles block a = 1 (w < 2) or 3, columns 8*(w&1)..+7 of it
    {
        const int a = (warp < 2) ? 1 : 3;
        const int ra = 16 * a, rb = ra - 16, n0 = rb + 8 * (warp & 1);
        float y[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t fa[4], fb[2];
#pragma unroll
        for (int k = 0; k < 16; k += 8) {
            frag_a(fa, A, ra, rb + k, lane);
            frag_b(fb, X, rb + k, n0, lane);
            mma_tf32_16x8x8(y, fa, fb);
        }
        store_frag_d(X, y, ra, n0, lane, 1.f);   // Y in the X_{a,a-1} block
        __syncwarp();
        float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < 16; k += 8) {
            frag_a(fa, X, ra, ra + k, lane);
            frag_b(fb, X, ra + k, n0, lane);     // Y rows (stored at rows ra..)
            mma_tf32_16x8x8(z, fa, fb);
        }
        __syncwarp();
        store_frag_d(X, z, ra, n0, lane, -1.f);
    }
    named_barrier(kBar, 128);
    // level 2: warp w handles rows 32 + 16*(w>>1).., columns 16*(w&1)..+15
    {
        const int r0 = 32 + 16 * (warp >> 1), c0 = 16 * (warp & 1);
        float y0[4] = {0.f, 0.f, 0.f, 0.f}, y1[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t fa[4], fb[2];
#pragma unroll
        for (int k = 0; k < 32; k += 8) {
            frag_a(fa, A, r0, k, lane);
            frag_b(fb, X, k, c0, lane);
            mma_tf32_16x8x8(y0, fa, fb);
            frag_b(fb, X, k, c0 + 8, lane);
            mma_tf32_16x8x8(y1, fa, fb);
        }
        store_frag_d(X, y0, r0, c0, lane, 1.f);
        store_frag_d(X, y1, r0, c0 + 8, lane, 1.f);
        named_barrier(kBar, 128);
        float z0[4] = {0.f, 0.f, 0.f, 0.f}, z1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < 32; k += 8) {
            frag_a(fa, X, r0, 32 + k, lane);
            frag_b(fb, X, 32 + k, c0, lane);
            mma_tf32_16x8x8(z0, fa, fb);
            frag_b(fb, X, 32 + k, c0 + 8, lane);
            mma_tf32_16x8x8(z1, fa, fb);
        }
        named_barrier(kBar, 128);
        store_frag_d(X, z0, r0, c0, lane, -1.f);
        store_frag_d(X, z1, r0, c0 + 8, lane, -1.f);
    }
    named_barrier(kBar, 128);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 3-D view [tokens][H][d] of a [B*T, H, d] tensor, moved in boxes of
// {box_d, 1, 64}: bf16 operand tiles with a 128-byte swizzle (box_d = 64),
// the bf16 output tiles as plain 128-byte rows (box_d = 64, no swizzle), the
// fp32 gate as plain 512-byte rows (box_d = 128).
inline bool make_map(CUtensorMap* m, const void* ptr, int d, long long tokens, int H, bool fp32,
              bool swizzle = true)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const int es = fp32 ? 4 : 2;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)tokens};
    const cuuint64_t strides[2] = {(cuuint64_t)d * es, (cuuint64_t)d * es * H};
    const cuuint32_t box[3] = {fp32 ? 128u : 64u, 1u, (cuuint32_t)kC};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
              const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              (fp32 || !swizzle) ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace kda
