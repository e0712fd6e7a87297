// Device helpers shared by the tensor-core prefill kernels (internal to libkda):
// fp32 64 x 64 matrix indexing, bf16 packing, swizzled tile access, and the
// warp-level TF32 products used by the blocked triangular inverse.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "kda_sm100.cuh"

namespace kda {
namespace tc {

using sm100::sw128_off;

constexpr int C = 64;   // chunk rows
constexpr int D = 128;  // dk = dv

// fp32 64 x 64 matrices A and T: 4-float groups permuted per row, so that row
// vectors stay contiguous and 8 consecutive rows of one column group fall in
// different banks.
__device__ __forceinline__ int a_idx(int r, int c) { return r * C + (c ^ ((r & 7) << 2)); }
__device__ __forceinline__ int t_idx(int r, int c) { return r * C + (c ^ ((r & 7) << 2)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
    return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                      pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
}
__device__ __forceinline__ void unpack8(uint4 u, float (&x)[8]) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(p[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void load8(const float* p, float (&x)[8]) {
    *reinterpret_cast<float4*>(x) = *reinterpret_cast<const float4*>(p);
    *reinterpret_cast<float4*>(x + 4) = *reinterpret_cast<const float4*>(p + 4);
}
// bf16 element (row, col) of a [rows][128] swizzled tile whose two 64-column
// halves are `half_stride` bytes apart.
__device__ __forceinline__ float tile_elem(const uint8_t* base, uint32_t half_stride, int row,
                                           int col) {
    const uint8_t* p = base + (col >> 6) * half_stride + sw128_off(row, (col & 63) >> 3) +
                       (col & 7) * 2;
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// D = A B + D for one 16 x 8 x 8 TF32 tile (warp-level, legacy tensor path:
// used only for the small 16 x 16 block products of the triangular inverse).
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4],
                                         const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Off-diagonal blocks of T at distance DIST:
//   T_IJ = -T_II sum_{K=J}^{I-1} A_IK T_KJ,   I = J + DIST,  J = 0 .. 3 - DIST,
// one warp per block J.  Fragments (m16n8k8, tf32): lane = 4 g + t;
// A: (g, t), (g+8, t), (g, t+4), (g+8, t+4); B: (t, g), (t+4, g);
// C: (g, 2t), (g, 2t+1), (g+8, 2t), (g+8, 2t+1).
// Ends with a barrier over the thread group: `bar_id` 0 = the whole CTA,
// otherwise named barrier `bar_id` over `nthreads` threads.
template <int DIST>
__device__ __forceinline__ void offdiag_level(const float* Af, float* Tf, float* Ms, int warp,
                                              int lane, uint32_t bar_id = 0,
                                              uint32_t nthreads = 0) {
    constexpr int NB = 4 - DIST;
    if (warp < NB) {
        const int J = warp, I = J + DIST, g = lane >> 2, t = lane & 3;
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < DIST; ++kk) {
            const int K = J + kk;
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                const int c0 = 16 * K + 8 * ks + t;
                const uint32_t a[4] = {to_tf32(Af[a_idx(16 * I + g, c0)]),
                                       to_tf32(Af[a_idx(16 * I + g + 8, c0)]),
                                       to_tf32(Af[a_idx(16 * I + g, c0 + 4)]),
                                       to_tf32(Af[a_idx(16 * I + g + 8, c0 + 4)])};
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int col = 16 * J + 8 * nt + g;
                    const uint32_t b[2] = {to_tf32(Tf[t_idx(c0, col)]),
                                           to_tf32(Tf[t_idx(c0 + 4, col)])};
                    mma_tf32(acc[nt], a, b);
                }
            }
        }
        float* M = Ms + warp * 256;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            M[g * 16 + 8 * nt + 2 * t] = acc[nt][0];
            M[g * 16 + 8 * nt + 2 * t + 1] = acc[nt][1];
            M[(g + 8) * 16 + 8 * nt + 2 * t] = acc[nt][2];
            M[(g + 8) * 16 + 8 * nt + 2 * t + 1] = acc[nt][3];
        }
        __syncwarp();
        float out[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            const int c0 = 16 * I + 8 * ks + t;
            const uint32_t a[4] = {to_tf32(Tf[t_idx(16 * I + g, c0)]),
                                   to_tf32(Tf[t_idx(16 * I + g + 8, c0)]),
                                   to_tf32(Tf[t_idx(16 * I + g, c0 + 4)]),
                                   to_tf32(Tf[t_idx(16 * I + g + 8, c0 + 4)])};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const uint32_t b[2] = {to_tf32(M[(8 * ks + t) * 16 + 8 * nt + g]),
                                       to_tf32(M[(8 * ks + t + 4) * 16 + 8 * nt + g])};
                mma_tf32(out[nt], a, b);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int col = 16 * J + 8 * nt + 2 * t;
            Tf[t_idx(16 * I + g, col)] = -out[nt][0];
            Tf[t_idx(16 * I + g, col + 1)] = -out[nt][1];
            Tf[t_idx(16 * I + g + 8, col)] = -out[nt][2];
            Tf[t_idx(16 * I + g + 8, col + 1)] = -out[nt][3];
        }
    }
    if (bar_id == 0)
        __syncthreads();
    else
        sm100::group_sync(bar_id, nthreads);
}

}  // namespace tc
}  // namespace kda
