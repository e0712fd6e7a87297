// KDA one-token recurrent decode step (fused, HBM-streaming).
//
// Kimi Linear (aiwiki.ai), "Why linear attention exists": decoding is a
// recurrent update whose per-token cost does not depend on the context read so
// far; "The constrained DPLR form and the chunkwise algorithm": the state per
// head is a fixed dk x dv (128 x 128) matrix.  Per (sequence, head):
//
//   Sbar = Diag(alpha) S                  alpha = exp(g)
//   u    = beta (v - Sbar^T k)            (delta-rule correction)
//   S   <- Sbar + k u^T                   == (I - b k k^T) Diag(alpha) S + b k v^T
//   o    = S^T q = Sbar^T q + u (k^T q)
//
// The state is the only large operand (64 KiB per head at 128 x 128, fp32);
// the kernel reads and writes it exactly once, so the step is bound by HBM
// bandwidth.  Both column reductions (Sbar^T k, Sbar^T q) run over dk only, so
// the dv columns of one (sequence, head) are independent: a CTA of 256 threads
// owns one (sequence, head) and a slice of DVS value columns (DVS = 64 for
// dv = 128: two CTAs per head, 32 state floats per thread, 4 CTAs per SM).
// Lane l of warp w holds columns [4 c4, 4 c4 + 4) of the slice in rows
// {w RPW + rw + 8 RPW p}, so every warp-wide load or store covers whole row
// slices with 16-byte vectors.  The column reductions are a shuffle inside the
// warp (when a warp spans several rows) and one shared-memory pass across the
// 8 warps.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_common.cuh"

namespace kda {

// kHeadGate: g is one value per (sequence, head) [units] (Gated DeltaNet)
// instead of one per key channel.
template <int DK, int DV, int DVS, typename TIn, bool kHeadGate>
__global__ void __launch_bounds__(256, (DK * DVS <= 8192) ? 4 : 2) decode_kernel(
    const TIn* __restrict__ q, const TIn* __restrict__ k, const TIn* __restrict__ v,
    const float* __restrict__ g, const float* __restrict__ beta, float* __restrict__ state,
    TIn* __restrict__ o) {
    constexpr int NW = 8;              // warps per CTA
    constexpr int LPR = DVS / 4;       // lanes per row slice (float4 each)
    constexpr int RPW = 32 / LPR;      // rows per warp per pass
    constexpr int RP = NW * RPW;       // rows per pass
    constexpr int NP = DK / RP;        // passes (float4 registers per thread)
    static_assert(DK % RP == 0, "DK must be a multiple of rows per pass");

    __shared__ float s_k[DK], s_q[DK], s_a[DK];
    __shared__ float4 s_redk[NW][LPR], s_redq[NW][LPR];
    __shared__ float s_kq;

    const int unit = blockIdx.x;  // (sequence, head)
    const int j0 = blockIdx.y * DVS;  // first value column of this slice
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int rw = lane / LPR, c4 = lane % LPR;
    // row r of the slice starts at float4 index r * (DV / 4) + j0 / 4
    float4* S = reinterpret_cast<float4*>(state + (size_t)unit * DK * DV + j0);

    // 1. stream the state in (independent of everything else: issue first)
    float4 x[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int row = p * RP + w * RPW + rw;
        x[p] = __ldcs(S + row * (DV / 4) + c4);
    }
    // 2. the token's vectors into shared memory
    for (int c = tid; c < DK; c += blockDim.x) {
        const size_t i = (size_t)unit * DK + c;
        s_k[c] = to_f32(k[i]);
        s_q[c] = to_f32(q[i]);
        s_a[c] = expf(kHeadGate ? g[unit] : g[i]);
    }
    __syncthreads();
    if (w == 0) {
        float kq = 0.f;
        for (int c = lane; c < DK; c += 32) kq += s_k[c] * s_q[c];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        if (lane == 0) s_kq = kq;
    }
    // 3. decay and partial column sums over this thread's rows
    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int row = p * RP + w * RPW + rw;
        const float a = s_a[row], kc = s_k[row], qc = s_q[row];
        x[p].x *= a; x[p].y *= a; x[p].z *= a; x[p].w *= a;
        pk.x += kc * x[p].x; pk.y += kc * x[p].y; pk.z += kc * x[p].z; pk.w += kc * x[p].w;
        pq.x += qc * x[p].x; pq.y += qc * x[p].y; pq.z += qc * x[p].z; pq.w += qc * x[p].w;
    }
    // lanes of one warp that hold the same columns (different rows) combine
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
        pk.x += __shfl_xor_sync(0xffffffffu, pk.x, off);
        pk.y += __shfl_xor_sync(0xffffffffu, pk.y, off);
        pk.z += __shfl_xor_sync(0xffffffffu, pk.z, off);
        pk.w += __shfl_xor_sync(0xffffffffu, pk.w, off);
        pq.x += __shfl_xor_sync(0xffffffffu, pq.x, off);
        pq.y += __shfl_xor_sync(0xffffffffu, pq.y, off);
        pq.z += __shfl_xor_sync(0xffffffffu, pq.z, off);
        pq.w += __shfl_xor_sync(0xffffffffu, pq.w, off);
    }
    if (rw == 0) {
        s_redk[w][c4] = pk;
        s_redq[w][c4] = pq;
    }
    __syncthreads();
    float4 sk = make_float4(0.f, 0.f, 0.f, 0.f), sq = sk;
#pragma unroll
    for (int i = 0; i < NW; ++i) {
        const float4 a = s_redk[i][c4], b = s_redq[i][c4];
        sk.x += a.x; sk.y += a.y; sk.z += a.z; sk.w += a.w;
        sq.x += b.x; sq.y += b.y; sq.z += b.z; sq.w += b.w;
    }
    // 4. u = beta (v - Sbar^T k) for this thread's four columns
    const float b = beta[unit];
    const size_t vo = (size_t)unit * DV + j0 + 4 * c4;
    float4 u;
    u.x = b * (to_f32(v[vo + 0]) - sk.x);
    u.y = b * (to_f32(v[vo + 1]) - sk.y);
    u.z = b * (to_f32(v[vo + 2]) - sk.z);
    u.w = b * (to_f32(v[vo + 3]) - sk.w);
    // 5. S = Sbar + k u^T, streamed back out
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int row = p * RP + w * RPW + rw;
        const float kc = s_k[row];
        float4 y = x[p];
        y.x += kc * u.x; y.y += kc * u.y; y.z += kc * u.z; y.w += kc * u.w;
        __stcs(S + row * (DV / 4) + c4, y);
    }
    // 6. o = Sbar^T q + u (k^T q)
    if (w == 0 && rw == 0) {
        const float kq = s_kq;
        o[vo + 0] = from_f32<TIn>(sq.x + u.x * kq);
        o[vo + 1] = from_f32<TIn>(sq.y + u.y * kq);
        o[vo + 2] = from_f32<TIn>(sq.z + u.z * kq);
        o[vo + 3] = from_f32<TIn>(sq.w + u.w * kq);
    }
}

template <typename TIn>
static cudaError_t decode_dispatch(const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, float* state, void* o, int units, int dk,
                                   int dv, bool head_gate, cudaStream_t st) {
    const TIn* Q = (const TIn*)q;
    const TIn* K = (const TIn*)k;
    const TIn* V = (const TIn*)v;
    TIn* O = (TIn*)o;
#define KDA_DECODE_CASE(A, B)                                                           \
    if (dk == A && dv == B) {                                                           \
        constexpr int DVS = (B == 128) ? 64 : B;                                        \
        const dim3 grid(units, B / DVS);                                                \
        if (head_gate)                                                                  \
            decode_kernel<A, B, DVS, TIn, true><<<grid, 256, 0, st>>>(Q, K, V, g, beta, state, O); \
        else                                                                            \
            decode_kernel<A, B, DVS, TIn, false><<<grid, 256, 0, st>>>(Q, K, V, g, beta, state, O); \
        return cudaGetLastError();                                                      \
    }
    KDA_DECODE_CASE(128, 128)
    KDA_DECODE_CASE(128, 64)
    KDA_DECODE_CASE(128, 32)
    KDA_DECODE_CASE(64, 128)
    KDA_DECODE_CASE(64, 64)
    KDA_DECODE_CASE(64, 32)
    KDA_DECODE_CASE(32, 128)
    KDA_DECODE_CASE(32, 64)
    KDA_DECODE_CASE(32, 32)
#undef KDA_DECODE_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, float* state, void* o, int N, int H, int dk,
                          int dv, kda_dtype_t dt, cudaStream_t st, bool head_gate) {
    const int units = N * H;
    if (units == 0) return cudaSuccess;
    if (dt == KDA_DTYPE_BF16)
        return decode_dispatch<__nv_bfloat16>(q, k, v, g, beta, state, o, units, dk, dv,
                                              head_gate, st);
    return decode_dispatch<float>(q, k, v, g, beta, state, o, units, dk, dv, head_gate, st);
}

}  // namespace kda
