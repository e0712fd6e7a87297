// Composition of per-segment affine state maps: the step of a context-parallel
// prefill (one long sequence split into R token segments) that turns every
// segment's map into its entry state, and of its backward, which turns them
// into every segment's exit-state gradient.  Kimi Linear (aiwiki.ai), "The
// constrained DPLR form and the chunkwise algorithm": the state is carried
// recurrently between chunks, and the carry over a segment is affine in the
// state, S_out = M S_in + B, so segments compose.
//
//   forward:  S_0 given;  each[r] = S_r;  S_{r+1} = M_r S_r + B_r;  final = S_R
//   reverse:  g_R given;  each[r] = g_{r+1};  g_r = M_r^T g_{r+1} + B_r;  final = g_0
//
// One CTA per (sequence, head, 32 value columns), serial over the segments;
// the state slice [dk][32] in shared memory, fp32 on the CUDA cores (R dk x dk
// x 32 products per CTA: small next to the prefills around it).
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda_common.cuh"

namespace kda {
namespace {

template <int DK, bool kReverse>
__global__ void __launch_bounds__(256) fold_kernel(const float* __restrict__ M,
                                                   const float* __restrict__ Bm,
                                                   const float* __restrict__ S0, int R, int NH,
                                                   int dv, float* __restrict__ each,
                                                   float* __restrict__ final_state) {
    constexpr int CW = 32;                  // columns per CTA
    constexpr int RPT = DK * CW / 256 / 4;  // rows per thread (4 columns each)
    __shared__ __align__(16) float S[DK][CW];
    const int nh = blockIdx.x, j0 = blockIdx.y * CW, tid = threadIdx.x;
    const int c4 = tid & 7, rb = tid >> 3;  // columns 4 c4 .., rows RPT rb ..
    for (int i = tid; i < DK * CW; i += 256) {
        const int c = i / CW, j = i % CW;
        S[c][j] = S0 ? S0[((size_t)nh * DK + c) * dv + j0 + j] : 0.f;
    }
    __syncthreads();
    for (int step = 0; step < R; ++step) {
        const int r = kReverse ? R - 1 - step : step;
        const size_t mb = ((size_t)r * NH + nh) * DK * DK;
        const size_t sb = ((size_t)r * NH + nh) * DK * dv;
        float acc[RPT][4];
#pragma unroll
        for (int x = 0; x < RPT; ++x) {
            const int c = RPT * rb + x;
            const float4 b = *reinterpret_cast<const float4*>(Bm + sb + (size_t)c * dv + j0 + 4 * c4);
            const float4 sv = *reinterpret_cast<const float4*>(&S[c][4 * c4]);
            *reinterpret_cast<float4*>(each + sb + (size_t)c * dv + j0 + 4 * c4) = sv;
            acc[x][0] = b.x; acc[x][1] = b.y; acc[x][2] = b.z; acc[x][3] = b.w;
        }
        for (int k = 0; k < DK; ++k) {
            const float4 sv = *reinterpret_cast<const float4*>(&S[k][4 * c4]);
#pragma unroll
            for (int x = 0; x < RPT; ++x) {
                const int c = RPT * rb + x;
                const float m = kReverse ? M[mb + (size_t)k * DK + c] : M[mb + (size_t)c * DK + k];
                acc[x][0] += m * sv.x; acc[x][1] += m * sv.y;
                acc[x][2] += m * sv.z; acc[x][3] += m * sv.w;
            }
        }
        __syncthreads();  // every read of the old state is done
#pragma unroll
        for (int x = 0; x < RPT; ++x)
            *reinterpret_cast<float4*>(&S[RPT * rb + x][4 * c4]) =
                make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
        __syncthreads();
    }
    for (int i = tid; i < DK * CW; i += 256) {
        const int c = i / CW, j = i % CW;
        final_state[((size_t)nh * DK + c) * dv + j0 + j] = S[c][j];
    }
}

template <int DK>
cudaError_t fold_dispatch(const float* M, const float* Bm, const float* S0, int R, int NH, int dv,
                          bool reverse, float* each, float* fin, cudaStream_t st) {
    const dim3 grid(NH, dv / 32);
    if (reverse)
        fold_kernel<DK, true><<<grid, 256, 0, st>>>(M, Bm, S0, R, NH, dv, each, fin);
    else
        fold_kernel<DK, false><<<grid, 256, 0, st>>>(M, Bm, S0, R, NH, dv, each, fin);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fold_segments(const float* M, const float* Bm, const float* S0, int R, int NH,
                                 int dk, int dv, bool reverse, float* each, float* fin,
                                 cudaStream_t st) {
    if (NH == 0) return cudaSuccess;
    if (dk == 128) return fold_dispatch<128>(M, Bm, S0, R, NH, dv, reverse, each, fin, st);
    if (dk == 64) return fold_dispatch<64>(M, Bm, S0, R, NH, dv, reverse, each, fin, st);
    return fold_dispatch<32>(M, Bm, S0, R, NH, dv, reverse, each, fin, st);
}

}  // namespace kda
