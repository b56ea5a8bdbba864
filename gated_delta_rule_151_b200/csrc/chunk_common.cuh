// Pieces shared by the two tensor-core prefill plans (the single-kernel
// pipelined kernel and the two-kernel chunk-parallel plan): chunk and head
// sizes, instruction descriptors, shared-memory accessors, the 64 x 64
// unit-lower-triangular inverse, and the TMA descriptor of a bf16
// [T, heads, 128] tensor.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tc_ptx.cuh"

namespace gdr {
namespace {

using namespace tc;

constexpr int C = 64;     // chunk length (tokens)
constexpr int D = 128;    // d_k = d_v served by the tensor-core plans

constexpr uint32_t IDESC_BF16 = make_idesc(1, 128, 64);
constexpr uint32_t IDESC_F16 = make_idesc(0, 128, 64);
constexpr uint32_t IDESC_N64 = make_idesc(2, 128, 64);
constexpr uint32_t IDESC_N128 = make_idesc(2, 128, 128);

constexpr float kF16Limit = 60000.f;   // largest magnitude let into an fp16 operand

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}
__device__ __forceinline__ void st_shared_b32(uint32_t addr, uint32_t a) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
}
__device__ __forceinline__ void st_shared_b16(uint32_t addr, uint16_t a) {
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(a) : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}
__device__ __forceinline__ float ld_shared_bf16(uint32_t addr) {
    uint16_t v;
    asm volatile("ld.shared.b16 %0, [%1];" : "=h"(v) : "r"(addr));
    return __uint_as_float(static_cast<uint32_t>(v) << 16);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
    }
}

// Named barrier over one 256-thread warp group (ids 1 and 2; 0 is __syncthreads).
__device__ __forceinline__ void group_sync(int id) {
    asm volatile("bar.sync %0, 256;" ::"r"(id) : "memory");
}

// Element (i, j) of a 64 x 64 fp32 scratch matrix: rows of 64 floats whose
// 16-byte chunks are XOR-swizzled by the row, so float4 accesses by eight
// threads on eight different rows hit eight different bank groups.
__device__ __forceinline__ int ax(int i, int j) {
    return i * 64 + ((((j >> 2) ^ (i & 15))) << 2) + (j & 3);
}
__device__ __forceinline__ float4 ld4(const float *base, int i, int j) {
    return *reinterpret_cast<const float4 *>(base + ax(i, j));
}
__device__ __forceinline__ void st4(float *base, int i, int j, float4 v) {
    *reinterpret_cast<float4 *>(base + ax(i, j)) = v;
}

// acc[0..3] += sum_{s<16} X[xi][xj + s] * Y[yi + s][yj .. yj+3] for 16 x 16
// blocks of the swizzled scratch (Y may also be a plain 16 x 16 block).
template <bool Y_PLAIN>
__device__ __forceinline__ void block_row_times(float (&acc)[4], const float *X, int xi, int xj,
                                                const float *Y, int yi, int yj) {
#pragma unroll
    for (int s4 = 0; s4 < 16; s4 += 4) {
        const float4 a = ld4(X, xi, xj + s4);
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float4 t = Y_PLAIN ? *reinterpret_cast<const float4 *>(Y + (s4 + e) * 16 + yj)
                                     : ld4(Y, yi + s4 + e, yj);
            acc[0] = fmaf(av[e], t.x, acc[0]);
            acc[1] = fmaf(av[e], t.y, acc[1]);
            acc[2] = fmaf(av[e], t.z, acc[2]);
            acc[3] = fmaf(av[e], t.w, acc[3]);
        }
    }
}

// T = (I + A)^-1 for the strictly lower 64 x 64 A (fp32 scratch), recursively
// on halves: with A = [[A_a, 0], [A_ba, A_b]] (32 x 32 blocks),
//   T = [[T_a, 0], [-T_b A_ba T_a, T_b]],
// and the same on each 32 x 32 half down to 16 x 16 diagonal blocks, which
// are inverted by forward substitution (one thread per column).  Four
// dependent matrix steps after the diagonal blocks.  T lands in Tf (fp32,
// lower triangle and diagonal; the blocks above the diagonal are not
// written).  Xs: 4 KiB plain scratch (four 16 x 16 blocks).  Called by 256
// threads (p = thread index), which end synchronised.
__device__ __forceinline__ void unit_lower_inverse_f32(const float *Af, float *Tf, float *Xs, int p) {
    // diagonal 16 x 16 blocks, column c of block `blk`
    if (p < 64) {
        const int blk = p >> 4, c = p & 15, o = blk * 16;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float a[16];
#pragma unroll
            for (int s4 = 0; s4 < 16; s4 += 4) {
                if (s4 < r) {
                    const float4 v = ld4(Af, o + r, o + s4);
                    a[s4] = v.x; a[s4 + 1] = v.y; a[s4 + 2] = v.z; a[s4 + 3] = v.w;
                }
            }
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int s = 0; s < r; ++s) {
                if (s & 1) acc1 = fmaf(a[s], x[s], acc1);
                else acc0 = fmaf(a[s], x[s], acc0);
            }
            const float v = -(acc0 + acc1);
            x[r] = (r < c) ? 0.f : ((r == c) ? 1.f : v);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tf[ax(o + r, o + c)] = x[r];
    }
    group_sync(2);
    const int r = (p >> 2) & 15, cq = (p & 3) * 4;
    // T_10 = -T_11 A_10 T_00 and T_32 = -T_33 A_32 T_22
    if (p < 128) {
        const int I = (p >> 6) ? 3 : 1, J = I - 1;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        block_row_times<false>(acc, Af, 16 * I + r, 16 * J, Tf, 16 * J, 16 * J + cq);
        *reinterpret_cast<float4 *>(Xs + (p >> 6) * 256 + r * 16 + cq) =
            make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
    group_sync(2);
    if (p < 128) {
        const int I = (p >> 6) ? 3 : 1, J = I - 1;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        block_row_times<true>(acc, Tf, 16 * I + r, 16 * I, Xs + (p >> 6) * 256, 0, cq);
        st4(Tf, 16 * I + r, 16 * J + cq, make_float4(-acc[0], -acc[1], -acc[2], -acc[3]));
    }
    group_sync(2);
    // Y = A_ba T_a: blocks (I, J) in {2,3} x {0,1}
    {
        const int b = p >> 6, I = 2 + (b >> 1), J = b & 1;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int K = J; K < 2; ++K)
            block_row_times<false>(acc, Af, 16 * I + r, 16 * K, Tf, 16 * K, 16 * J + cq);
        *reinterpret_cast<float4 *>(Xs + b * 256 + r * 16 + cq) =
            make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
    group_sync(2);
    // T_ba = -T_b Y
    {
        const int b = p >> 6, I = 2 + (b >> 1), J = b & 1;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int K = 2; K <= I; ++K)
            block_row_times<true>(acc, Tf, 16 * I + r, 16 * K, Xs + ((K - 2) * 2 + J) * 256, 0, cq);
        st4(Tf, 16 * I + r, 16 * J + cq, make_float4(-acc[0], -acc[1], -acc[2], -acc[3]));
    }
    group_sync(2);
}

// unit_lower_inverse_f32, then T as the tf32 operand [i][j] (128-byte
// swizzled rows, zero above the diagonal) at shared address tm_addr.
__device__ __forceinline__ void unit_lower_inverse(const float *Af, float *Tf, float *Xs,
                                                   uint32_t tm_addr, int p) {
    unit_lower_inverse_f32(Af, Tf, Xs, p);
    for (int e = p; e < C * 16; e += 256) {
        const int i = e >> 4, q = e & 15, j0 = q * 4;
        const float4 t = ld4(Tf, i, j0);
        const float tv[4] = {t.x, t.y, t.z, t.w};
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) w[k] = to_tf32(j0 + k <= i ? tv[k] : 0.f);
        st_shared_v4(tm_addr + (j0 >> 5) * 8192 + sw128_offset(i, (j0 & 31) >> 2), w[0], w[1], w[2],
                     w[3]);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [total_T, H, 128] bf16 viewed as a 3-D tensor {128, H, total_T}; box
// {64, 1, 64} with 128-byte swizzle: one 64-token x 64-channel tile.
bool make_map(CUtensorMap *map, const void *base, int total_T, int H) {
    auto enc = get_encode();
    if (enc == nullptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)total_T};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// [total_T, H, 128] fp32 per-channel gates viewed as {128, H, total_T}; box
// {32, 1, 64} without swizzle: 64 tokens x 32 channels as rows of 128 bytes.
bool make_gate_map(CUtensorMap *map, const float *base, int total_T, int H) {
    auto enc = get_encode();
    if (enc == nullptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)total_T};
    cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)H * D * 4};
    cuuint32_t box[3] = {32, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace
}  // namespace gdr
