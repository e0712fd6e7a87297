// Device helpers shared by the tensor-core prefill kernels (internal to libkda):
// fp32 64 x 64 matrix indexing, bf16 packing, swizzled tile access, and the
// warp-level TF32 products and block steps of the triangular inverse.
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

// T = (I + A)^{-1} (A strictly lower, 4 x 4 blocks of 16 x 16) in three steps,
// each writing its blocks twice: in fp32 to Tf (the a_idx layout, read by the
// later steps) and as Tb = T diag(b) in bf16 to the [64][64] K-major operand
// tile `tb` (128-byte swizzle), so that no separate conversion pass is needed.
//   diag_inverse:       two diagonal blocks T_II, I = I0, I0 + 1, per warp
//                       (lane: one column of one block), forward substitution
//                       row by row, A's rows read as float4
//   inverse_pair:       T_10 = -T_11 A_10 T_00 or T_32 = -T_33 A_32 T_22 (one
//                       warp; M = A_IJ T_JJ through the warp's 16 x 16
//                       scratch, then -T_II M)
//   inverse_lower_left: the 32 x 32 block [T_20 T_21; T_30 T_31] =
//                       -T_hi (A_ll T_lo), T_lo = [T_00 0; T_10 T_11],
//                       T_hi = [T_22 0; T_32 T_33]: warp w (0-3) owns tile
//                       (i, j) = (2 + w / 2, w % 2), first M_ij = sum_k A_ik T_kj
//                       (k = j..1) into scratch tile w, then, after a named
//                       barrier of the four warps, T_ij = -sum_k T_ik M_kj
//                       (k = 2..i).
// The blocks above the diagonal of Tb are zeroed separately (tb_zero_upper).
// 16 x 16 tiles on the warp-level TF32 products above (fragments as there).
// acc[nt] += X[16 xi.., 16 xk..] * Y[16 xk.., 16 yj..], X and Y in the a_idx
// layout.
__device__ __forceinline__ void blk_mma(float (&acc)[2][4], const float* X, int xi, int xk,
                                        const float* Y, int yj, int g, int t) {
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const int c0 = 16 * xk + 8 * ks + t;
        const uint32_t a[4] = {to_tf32(X[a_idx(16 * xi + g, c0)]),
                               to_tf32(X[a_idx(16 * xi + g + 8, c0)]),
                               to_tf32(X[a_idx(16 * xi + g, c0 + 4)]),
                               to_tf32(X[a_idx(16 * xi + g + 8, c0 + 4)])};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int col = 16 * yj + 8 * nt + g;
            const uint32_t b[2] = {to_tf32(Y[a_idx(c0, col)]), to_tf32(Y[a_idx(c0 + 4, col)])};
            mma_tf32(acc[nt], a, b);
        }
    }
}
// acc[nt] += X[16 xi.., 16 xk..] * M, M a row-major 16 x 16 scratch tile.
__device__ __forceinline__ void blk_mma_scratch(float (&acc)[2][4], const float* X, int xi,
                                                int xk, const float* M, int g, int t) {
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const int c0 = 16 * xk + 8 * ks + t;
        const uint32_t a[4] = {to_tf32(X[a_idx(16 * xi + g, c0)]),
                               to_tf32(X[a_idx(16 * xi + g + 8, c0)]),
                               to_tf32(X[a_idx(16 * xi + g, c0 + 4)]),
                               to_tf32(X[a_idx(16 * xi + g + 8, c0 + 4)])};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t b[2] = {to_tf32(M[(8 * ks + t) * 16 + 8 * nt + g]),
                                   to_tf32(M[(8 * ks + t + 4) * 16 + 8 * nt + g])};
            mma_tf32(acc[nt], a, b);
        }
    }
}
__device__ __forceinline__ void acc_to_scratch(const float (&acc)[2][4], float* M, int g, int t) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        M[g * 16 + 8 * nt + 2 * t] = acc[nt][0];
        M[g * 16 + 8 * nt + 2 * t + 1] = acc[nt][1];
        M[(g + 8) * 16 + 8 * nt + 2 * t] = acc[nt][2];
        M[(g + 8) * 16 + 8 * nt + 2 * t + 1] = acc[nt][3];
    }
}
// Tb[row][col], Tb[row][col + 1] = x0 b[col], x1 b[col + 1] in bf16 (col even).
__device__ __forceinline__ void tb_store2(uint8_t* tb, int row, int col, float x0, float x1,
                                          const float* sb) {
    *reinterpret_cast<uint32_t*>(tb + sw128_off(row, col >> 3) + (col & 7) * 2) =
        pack_bf16x2(x0 * sb[col], x1 * sb[col + 1]);
}
__device__ __forceinline__ void acc_to_T_neg(const float (&acc)[2][4], float* Tf, uint8_t* tb,
                                             const float* sb, int I, int J, int g, int t) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int col = 16 * J + 8 * nt + 2 * t;
        Tf[a_idx(16 * I + g, col)] = -acc[nt][0];
        Tf[a_idx(16 * I + g, col + 1)] = -acc[nt][1];
        Tf[a_idx(16 * I + g + 8, col)] = -acc[nt][2];
        Tf[a_idx(16 * I + g + 8, col + 1)] = -acc[nt][3];
        tb_store2(tb, 16 * I + g, col, -acc[nt][0], -acc[nt][1], sb);
        tb_store2(tb, 16 * I + g + 8, col, -acc[nt][2], -acc[nt][3], sb);
    }
}

// Lane (I = I0 + lane / 16, jj = lane % 16) solves (I + A_II) t = e_jj:
// t_r = [r == jj] - sum_{c < r} A_II[r][c] t_c, r = 0..15 (t_r = 0 for r < jj).
// Row r of A_II is read as ceil(r / 4) float4 (the a_idx permutation moves
// whole 4-float groups); the 16 lanes of a block read the same addresses.
__device__ __forceinline__ void diag_inverse(const float* Af, float* Tf, uint8_t* tb,
                                             const float* sb, int I0, int lane) {
    const int I = I0 + (lane >> 4), jj = lane & 15, col = 16 * I + jj;
    float t[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const float* row = Af + (16 * I + r) * C;
        float s0 = (r == jj) ? 1.f : 0.f, s1 = 0.f;
#pragma unroll
        for (int q = 0; 4 * q < r; ++q) {
            const float4 a =
                *reinterpret_cast<const float4*>(row + ((16 * I + 4 * q) ^ ((r & 7) << 2)));
            s0 -= a.x * t[4 * q];
            if (4 * q + 1 < r) s1 -= a.y * t[4 * q + 1];
            if (4 * q + 2 < r) s0 -= a.z * t[4 * q + 2];
            if (4 * q + 3 < r) s1 -= a.w * t[4 * q + 3];
        }
        t[r] = s0 + s1;
    }
    const float b = sb[col];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        Tf[t_idx(16 * I + r, col)] = t[r];
        *reinterpret_cast<__nv_bfloat16*>(tb + sw128_off(16 * I + r, col >> 3) + (col & 7) * 2) =
            __float2bfloat16_rn(t[r] * b);
    }
}

// Zeros in the blocks of Tb above the diagonal: rows 16 I .., chunks of 8
// columns from 2 (I + 1) on (192 chunks of 16 bytes, one warp).
__device__ __forceinline__ void tb_zero_upper(uint8_t* tb, int lane) {
#pragma unroll
    for (int e = lane; e < 192; e += 32) {
        int row, ch;
        if (e < 96) {
            row = e / 6;
            ch = 2 + e % 6;
        } else if (e < 160) {
            row = 16 + (e - 96) / 4;
            ch = 4 + (e - 96) % 4;
        } else {
            row = 32 + (e - 160) / 2;
            ch = 6 + (e - 160) % 2;
        }
        *reinterpret_cast<uint4*>(tb + sw128_off(row, ch)) = make_uint4(0u, 0u, 0u, 0u);
    }
}

// One warp: T_{J+1,J} = -T_{J+1,J+1} A_{J+1,J} T_JJ (J even), M its 16 x 16
// scratch; the diagonal blocks written by this warp before (a __syncwarp
// between).
__device__ __forceinline__ void inverse_pair(const float* Af, float* Tf, float* M, uint8_t* tb,
                                             const float* sb, int J, int lane) {
    const int I = J + 1, g = lane >> 2, t = lane & 3;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    blk_mma(acc, Af, I, J, Tf, J, g, t);  // A_IJ T_JJ
    acc_to_scratch(acc, M, g, t);
    __syncwarp();
    float out[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    blk_mma_scratch(out, Tf, I, I, M, g, t);  // T_II M
    acc_to_T_neg(out, Tf, tb, sb, I, J, g, t);
}

__device__ __forceinline__ void inverse_lower_left(const float* Af, float* Tf, float* Ms,
                                                   uint8_t* tb, const float* sb, int warp,
                                                   int lane, uint32_t bar4) {
    if (warp >= 4) return;
    const int i = 2 + (warp >> 1), j = warp & 1, g = lane >> 2, t = lane & 3;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (int k = j; k < 2; ++k) blk_mma(acc, Af, i, k, Tf, j, g, t);  // M_ij
    acc_to_scratch(acc, Ms + warp * 256, g, t);
    sm100::group_sync(bar4, 128);
    float out[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    // T_ij = -(T_i2 M_2j [+ T_33 M_3j]); scratch tile of M_kj is 2 (k - 2) + j
    for (int k = 2; k <= i; ++k) blk_mma_scratch(out, Tf, i, k, Ms + (2 * (k - 2) + j) * 256, g, t);
    acc_to_T_neg(out, Tf, tb, sb, i, j, g, t);
}

}  // namespace tc
}  // namespace kda
