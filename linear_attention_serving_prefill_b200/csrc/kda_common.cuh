// Shared device helpers of libkda_b200 (storage conversions, the gate).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Lower bound of the per-step log-decay ("Kimi K3: Architecture, Training, and
// Million-Token Agentic RL", section 3.3 gate equation: g_min = -5).
constexpr float kGMin = -5.0f;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// g = g_min * sigmoid(exp(A) * z), given exp(A).  For exp(A)*z -> +inf the
// exponential underflows to 0 and g = g_min exactly; for -> -inf it overflows to
// +inf and g = -0 (alpha = 1 exactly), so g stays in [g_min, 0] -- the closed
// range that bounds a 16-token cumulative log-decay to [-80, 0].
__device__ __forceinline__ float gate_log_decay(float expA, float z) {
    return kGMin / (1.0f + expf(-expA * z));
}

// The unbounded gate of the earlier Kimi Linear design, which the same section
// contrasts with the bound: g = -softplus(exp(A) * z) = -log(1 + e^{exp(A) z}),
// evaluated as -(max(x, 0) + log1p(e^{-|x|})).  The result is clamped at
// kGClampSoftplus: below it e^{g} is already 0 in fp32, and the clamp keeps the
// cumulative log-decay of a chunk small enough that differences of it do not
// cancel catastrophically.
constexpr float kGClampSoftplus = -110.0f;

__device__ __forceinline__ float gate_log_decay_softplus(float expA, float z) {
    const float x = expA * z;
    return fmaxf(-(fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)))), kGClampSoftplus);
}

// Gate kinds of the C ABI (kda_gate).
enum GateKind : int { kGateBounded = 0, kGateSoftplus = 1 };

template <int GATE> __device__ __forceinline__ float gate_fn(float expA, float z) {
    return GATE == kGateSoftplus ? gate_log_decay_softplus(expA, z) : gate_log_decay(expA, z);
}

}  // namespace kda
