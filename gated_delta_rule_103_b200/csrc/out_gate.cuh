// The output side of a KDA layer ("深度解读报告" 3.2: head-wise RMSNorm and a
// data-dependent sigmoid output gate), for one (token, head) row of kDv
// values held 4 per lane by a full warp:
//
//     o' = o / sqrt(mean(o^2) + eps) * w * sigmoid(g)
//
#pragma once

#include <cuda_runtime.h>

#include "kda_internal.h"

namespace kda {

// 1 / (1 + e^-x), the reciprocal correctly rounded (the same bits as an IEEE
// division of 1 by it, without the division's slow path)
__device__ __forceinline__ float out_sigmoid(float x) { return __frcp_rn(1.f + __expf(-x)); }

// x: the row's 4 values of this lane (in place); g: the gate pre-activations;
// w: the weight; eps > 0.  The mean square is a 5-step warp reduction.
__device__ __forceinline__ void out_norm_gate_row(float (&x)[4], const float (&g)[4],
                                                  const float (&w)[4], float eps)
{
    float ss = fmaf(x[0], x[0], fmaf(x[1], x[1], fmaf(x[2], x[2], x[3] * x[3])));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = rsqrtf(ss * (1.f / kDv) + eps);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = x[i] * inv * w[i] * out_sigmoid(g[i]);
}

}  // namespace kda
