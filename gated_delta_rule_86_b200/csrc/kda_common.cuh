// Shared device helpers for the KDA kernels: element access for the two I/O
// dtypes, the device-side error word and bounded waits.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Error codes recorded in the device error word (mirror kda_status values).
constexpr int kDevErrTimeout = 4;

// Device-side error word (one per device and per translation unit that
// includes this header; the library is a single translation unit).  Kernels
// set it with atomicMax when a bounded wait runs out;
// kda_get_last_device_error reads and clears it.
static __device__ int g_device_error = 0;

__device__ __forceinline__ void record_device_error(int code) { atomicMax(&g_device_error, code); }

// Iteration limit of every spin on an mbarrier phase.  A try_wait suspends the
// thread for up to a system-dependent time per call, so this bounds a wait to
// well under a few seconds while never triggering on a healthy kernel.
constexpr uint32_t kSpinLimit = 1u << 24;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// How the inputs are given.  kGateChannel: one log-decay per key channel, log_alpha [..., d_k]
// (KDA).  kGateHead: one log-decay per head and token, log_g [...] (Gated DeltaNet, the
// scalar-gate case of the same recurrence); a null log_g means no decay at all, alpha == 1
// (DeltaNet).  kRawInputs: KDA from the raw projections (the fused prologue): q and k are
// L2-normalised over d_k here, log_alpha = logsigmoid(g) of a per-channel pre-activation g, and
// beta = sigmoid(b) of a pre-activation b.
enum GateKind : int { kGateChannel = 0, kGateHead = 1, kRawInputs = 2 };

// logsigmoid(x) = -log(1 + exp(-x)), in the form that neither overflows nor loses small values.
__device__ __forceinline__ float log_sigmoid(float x) { return fminf(x, 0.f) - log1pf(expf(-fabsf(x))); }
__device__ __forceinline__ float sigmoidf(float x) { return 1.f / (1.f + expf(-x)); }
// The same with the SFU intrinsics (__expf, __logf): an absolute error below 1e-6 in the log-decay
// (1 + y rounds y < 2^-24 away, a loss below 6e-8), for the per-element work of the decay scan.
__device__ __forceinline__ float log_sigmoid_fast(float x) {
    return fminf(x, 0.f) - __logf(1.f + __expf(-fabsf(x)));
}
// L2 normalisation of q and k (kRawInputs): x * rsqrt(sum x^2 + kNormEps)
constexpr float kNormEps = 1e-6f;

// Log-decay of key channel c at gate row `row` (token * H + head, or batch * H + head).
template <int GK, typename T>
__device__ __forceinline__ float gate_log(const T *gate, size_t row, int dk, int c) {
    if constexpr (GK == kGateChannel) return to_f32(gate[row * dk + c]);
    else if constexpr (GK == kRawInputs) return log_sigmoid(to_f32(gate[row * dk + c]));
    else return gate ? to_f32(gate[row]) : 0.f;
}
// beta of a row as the kernel uses it
template <int GK, typename T> __device__ __forceinline__ float beta_of(const T *beta, size_t row) {
    if constexpr (GK == kRawInputs) return sigmoidf(to_f32(beta[row]));
    else return to_f32(beta[row]);
}

// log2(e), used to turn exp(x) into exp2(x * log2e) for the ex2 unit.
constexpr float kLog2e = 1.4426950408889634f;

// 2^x on the SFU (ex2.approx: relative error ~2^-22, flushes subnormal results).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float fast_exp(float x) { return ex2_approx(x * kLog2e); }

}  // namespace kda
