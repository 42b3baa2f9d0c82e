// The forget gate from its pre-activation (KDA_FLAG_RAW_GATE).
//
// "深度解读报告" 3.2 obtains the per-channel gate alpha from a low-rank
// projection of the token and prints no activation; alpha must lie in
// (0, 1], and the logistic sigmoid is the map taken here:
// alpha = sigmoid(z), so log alpha = log sigmoid(z) = -softplus(-z).
#pragma once

#include <cuda_runtime.h>

namespace kda {

// log sigmoid(z) = min(z, 0) - log(1 + e^-|z|), in fp32 with the fast
// exponential and logarithm (absolute error about 1e-7, which is what the
// gate's prefix sums see).
__device__ __forceinline__ float log_sigmoid(float z)
{
    return fminf(z, 0.f) - __logf(1.f + __expf(-fabsf(z)));
}

}  // namespace kda
