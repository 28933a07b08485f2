// kda_common.cuh -- small device helpers shared by the KDA kernels (not by the oracle).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

// ---- element load / store for the two per-token dtypes -------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// ---- gate activation (KDA notes, "Gate 激活", table "两种 Gate") ------------------------------
// input = g_raw + dt_bias, rate = exp(A_log):
//   SAFE      g = L * sigmoid(rate * input)
//   STANDARD  g = -rate * softplus(input), softplus(x) = max(x,0) + log1p(exp(-|x|))
// NONE returns the input unchanged (it is already the log-space decay).
__device__ __forceinline__ float gate_value(float graw, float bias, float rate, int mode, float lower_bound) {
    const float x = graw + bias;
    if (mode == KDA_GATE_SAFE) {
        return lower_bound / (1.0f + expf(-rate * x));
    } else if (mode == KDA_GATE_STANDARD) {
        const float sp = fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
        return -rate * sp;
    }
    return graw;
}

// The same gate with the fast hardware exponential / division / logarithm (relative error ~1e-6,
// far below the tf32 operand rounding of the tensor-core path that uses it).
__device__ __forceinline__ float gate_value_fast(float graw, float bias, float rate, int mode, float lower_bound) {
    const float x = graw + bias;
    if (mode == KDA_GATE_SAFE) {
        return __fdividef(lower_bound, 1.0f + __expf(-rate * x));
    } else if (mode == KDA_GATE_STANDARD) {
        const float sp = fmaxf(x, 0.0f) + __logf(1.0f + __expf(-fabsf(x)));
        return -rate * sp;
    }
    return graw;
}

// ---- optional input-side steps (kda_input_flags) ---------------------------------------------
// 1 / max(||x||, 1e-6) from the sum of squares of x (KDA_INPUT_L2NORM_QK).
__device__ __forceinline__ float inv_l2norm(float sumsq) { return rsqrtf(fmaxf(sumsq, 1e-12f)); }
// Write strength from a logit (KDA_INPUT_BETA_LOGITS).
__device__ __forceinline__ float beta_from_logit(float x) { return 1.0f / (1.0f + expf(-x)); }

}  // namespace kda
