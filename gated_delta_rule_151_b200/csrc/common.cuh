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

}  // namespace gdr
