// Small device helpers shared by the gated delta-rule kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr.h"

#include <algorithm>
#include <mutex>
#include <vector>

namespace gdr {

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) only when a kernel needs
// more than it was last given on this device: the call costs host time on
// every launch otherwise, and launches of short kernels are host-bound.
inline cudaError_t ensure_dynamic_smem(const void *fn, int bytes) {
    struct Entry {
        const void *fn;
        int dev;
        int bytes;
    };
    static std::mutex mu;
    static std::vector<Entry> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    Entry *hit = nullptr;
    for (auto &d : done)
        if (d.fn == fn && d.dev == dev) hit = &d;
    if (hit != nullptr && hit->bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    if (hit != nullptr) hit->bytes = bytes;
    else done.push_back(Entry{fn, dev, bytes});
    return cudaSuccess;
}

// Log-gates are clamped at this value per token: alpha >= e^-20 ~ 2e-9, so
// every exponent difference the chunked form takes stays finite.
constexpr float kLogGateMin = -20.0f;

__device__ __forceinline__ float clamp_log_gate(float g) { return fmaxf(g, kLogGateMin); }

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ void store_io(float *p, float x) { *p = x; }
__device__ __forceinline__ void store_io(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

// Token range [t0, t0 + len) of sequence n.  With cu_seqlens the range is
// clamped into [0, total_T] and a negative length counts as empty, so a
// malformed array cannot move any access out of bounds.
__device__ __forceinline__ void sequence_range(const int32_t *cu, int n, int num_seqs,
                                               int total_T, int &t0, int &len) {
    if (cu != nullptr) {
        int a = min(max(cu[n], 0), total_T);
        int b = min(max(cu[n + 1], 0), total_T);
        t0 = a;
        len = max(b - a, 0);
    } else {
        int L = total_T / num_seqs;
        t0 = n * L;
        len = L;
    }
}

// Maps and activations of the input-side prologue, shared by the standalone
// prologue kernel and the prefill's fused staging so that both give the same
// bits.  The approximations are single PTX instructions (denormals flushed:
// every operand here is either normal or its exact result is 0 or 1 to fp32
// precision).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rsqrt_approx(float x) {   // x >= 1e-6 where used
    float y;
    asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kNormEps = 1e-6f;   // q/k L2 norm: x / sqrt(sum x^2 + eps)

// SiLU y / (1 + e^-y) = y * 1 / (1 + 2^(-y log2 e)).  For y -> -inf the power
// overflows to inf and the reciprocal to 0.
__device__ __forceinline__ float silu_f(float y) {
    return y * rcp_approx(1.0f + ex2_approx(-kLog2e * y));
}

// SiLU on a pair of channels (the packed fp32x2 units), the same bits as silu_f.
__device__ __forceinline__ float2 silu2(float2 y) {
    float2 t = __fmul2_rn(y, make_float2(-kLog2e, -kLog2e));
    t = make_float2(ex2_approx(t.x), ex2_approx(t.y));
    t = __fadd2_rn(t, make_float2(1.f, 1.f));
    return __fmul2_rn(y, make_float2(rcp_approx(t.x), rcp_approx(t.y)));
}

// Sums over the 32 lanes of a warp of eight values per lane at once (eight
// tokens' sums of squares, 4 channels per lane, 128 channels per head): a
// transposed butterfly halves the tokens a lane carries at each of the
// xor-16/8/4 steps, finishes with xor 2/1, then fetches each token's total
// from a lane that holds it (token of lane l: 4 bit4(l) + 2 bit3(l) +
// bit2(l)).  17 shuffles instead of 40; the additions form the same tree as
// eight xor-16/8/4/2/1 reductions, so the totals have the same bits.
__device__ __forceinline__ void norm_sums8(const float (&ss)[8], int lane, float (&tot)[8]) {
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
    float v4[4], v2[2];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float send = b4 ? ss[k] : ss[k + 4], keep = b4 ? ss[k + 4] : ss[k];
        v4[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float send = b3 ? v4[k] : v4[k + 2], keep = b3 ? v4[k + 2] : v4[k];
        v2[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    float v = (b2 ? v2[1] : v2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? v2[0] : v2[1], 4);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 1);
#pragma unroll
    for (int k = 0; k < 8; ++k)
        tot[k] = __shfl_sync(0xffffffffu, v, ((k >> 2) & 1) * 16 + ((k >> 1) & 1) * 8 + (k & 1) * 4);
}

// log(1 + e^x), and the log-gate g = -c softplus(x_g); beta = sigmoid(x_beta).
__device__ __forceinline__ float softplus_f(float x) {
    return x > 20.f ? x : log1pf(expf(x));
}
__device__ __forceinline__ float log_gate_of(float c, float xg) { return -c * softplus_f(xg); }
__device__ __forceinline__ float beta_of(float xb) { return 1.0f / (1.0f + expf(-xb)); }

}  // namespace gdr
