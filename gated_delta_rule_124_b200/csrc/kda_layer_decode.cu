// One decode token of a KDA layer in one launch: the steps around the operator
// fused into the decode kernel's prologue and epilogue.
//
// Kimi Linear (aiwiki.ai), "The constrained DPLR form and the chunkwise
// algorithm" (the paragraph on what each KDA head applies): a depthwise causal
// convolution of kernel 4 with a Swish on q, k and v and the L2 normalisation
// of q and k before the operator; a head-wise RMSNorm and a sigmoid output gate
// after it.  Per (sequence n, head h), with c0..c2 the convolution state (the
// last three raw inputs, oldest first) and x the new raw input:
//
//   q = l2norm(Swish(w0 c0 + w1 c1 + w2 c2 + w3 x_q)),  k likewise,
//   v = Swish(w0 c0 + w1 c1 + w2 c2 + w3 x_v);  each state <- (c1, c2, x)
//   the decode step of kda_decode.cu on (q, k, v, g, beta, S)
//   y = o / sqrt(mean_j o_j^2 + rms_eps) * w_norm * sigmoid(gate)
//
// q, k, v and o never leave the chip.  One 256-thread CTA takes all DV value
// columns of one (sequence, head), so the q / k convolution, the convolution
// states (overwritten after a CTA barrier, once every thread has read them)
// and the RMSNorm's sum of o^2 over the DV columns stay inside the CTA.  The
// kernel is written for NS = DV / DVS 256-thread units per CTA (each unit a
// slice of DVS value columns, the slices' sums of squares combined in shared
// memory); the launch uses NS = 1.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_common.cuh"

namespace kda {
namespace {

struct LayerDecodeArgs {
    const void* xq;
    const void* xk;
    const void* xv;
    const float* wq;
    const float* wk;
    const float* wv;
    void* conv_q;
    void* conv_k;
    void* conv_v;
    const float* g;
    const float* beta;
    float* state;
    const void* gate;
    const float* w_norm;
    void* y;
    int H;
    float l2_eps;
    float rms_eps;
};

// Block-wide sum over NW warps (every thread gets the total).
template <int NW>
__device__ __forceinline__ float block_sum(float x, float* red) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
    __syncthreads();
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < NW; ++i) t += red[i];
    __syncthreads();
    return t;
}

template <int DK, int DV, int DVS, typename TIn>
__global__ void __launch_bounds__(256 * (DV / DVS), ((DK * DVS <= 8192) ? 4 : 2) / (DV / DVS))
    layer_decode_kernel(const LayerDecodeArgs a) {
    constexpr int NS = DV / DVS;       // value slices = 256-thread units per CTA
    constexpr int NW = 8;              // warps per unit
    constexpr int LPR = DVS / 4;
    constexpr int RPW = 32 / LPR;
    constexpr int RP = NW * RPW;
    constexpr int NP = DK / RP;
    static_assert(DK % RP == 0 && DK <= 256 && DVS <= 256, "shape");

    __shared__ float s_k[DK], s_q[DK], s_a[DK], s_v[NS][DVS];
    __shared__ float4 s_redk[NS][NW][LPR], s_redq[NS][NW][LPR];
    __shared__ float s_red[NS * NW];
    __shared__ float s_kq, s_ss[NS];

    const int unit = static_cast<int>(blockIdx.x);  // (sequence, head)
    const int n = unit / a.H, h = unit % a.H;
    const int sl = static_cast<int>(threadIdx.x) >> 8;  // value slice of this thread's unit
    const int j0 = sl * DVS;
    const int t = threadIdx.x;
    const int tid = t & 255, lane = tid & 31, w = tid >> 5;
    const int rw = lane / LPR, c4 = lane % LPR;
    float4* S = reinterpret_cast<float4*>(a.state + (size_t)unit * DK * DV + j0);

    // 1. stream the state in first (independent of everything else)
    float4 x[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int row = p * RP + w * RPW + rw;
        x[p] = __ldcs(S + row * (DV / 4) + c4);
    }
    // 2. prologue: convolution + Swish of q, k (threads t < DK, once per CTA)
    // and of each unit's DVS value columns
    const TIn* xq = static_cast<const TIn*>(a.xq);
    const TIn* xk = static_cast<const TIn*>(a.xk);
    const TIn* xv = static_cast<const TIn*>(a.xv);
    TIn* cq = static_cast<TIn*>(a.conv_q);
    TIn* ck = static_cast<TIn*>(a.conv_k);
    TIn* cv = static_cast<TIn*>(a.conv_v);
    // state row i of (n, h), channel c: ((n * 3 + i) * H + h) * d + c
    auto srow = [&](int i, int d) { return ((size_t)(n * 3 + i) * a.H + h) * d; };
    float nq[3] = {0.f, 0.f, 0.f}, nk[3] = {0.f, 0.f, 0.f}, nv[3] = {0.f, 0.f, 0.f};
    float yq = 0.f, yk = 0.f;
    if (t < DK) {
        const int c = t;
        const float4 wqv = *reinterpret_cast<const float4*>(a.wq + ((size_t)h * DK + c) * 4);
        const float4 wkv = *reinterpret_cast<const float4*>(a.wk + ((size_t)h * DK + c) * 4);
        const float q0 = to_f32(cq[srow(0, DK) + c]), q1 = to_f32(cq[srow(1, DK) + c]),
                    q2 = to_f32(cq[srow(2, DK) + c]);
        const float k0 = to_f32(ck[srow(0, DK) + c]), k1 = to_f32(ck[srow(1, DK) + c]),
                    k2 = to_f32(ck[srow(2, DK) + c]);
        const float qx = to_f32(xq[(size_t)unit * DK + c]), kx = to_f32(xk[(size_t)unit * DK + c]);
        yq = swish_for<TIn>(wqv.x * q0 + wqv.y * q1 + wqv.z * q2 + wqv.w * qx);
        yk = swish_for<TIn>(wkv.x * k0 + wkv.y * k1 + wkv.z * k2 + wkv.w * kx);
        nq[0] = q1; nq[1] = q2; nq[2] = qx;
        nk[0] = k1; nk[1] = k2; nk[2] = kx;
        s_a[c] = expf(a.g[(size_t)unit * DK + c]);
    }
    if (tid < DVS) {
        const int c = j0 + tid;
        const float4 wvv = *reinterpret_cast<const float4*>(a.wv + ((size_t)h * DV + c) * 4);
        const float v0 = to_f32(cv[srow(0, DV) + c]), v1 = to_f32(cv[srow(1, DV) + c]),
                    v2 = to_f32(cv[srow(2, DV) + c]);
        const float vx = to_f32(xv[(size_t)unit * DV + c]);
        s_v[sl][tid] = swish_for<TIn>(wvv.x * v0 + wvv.y * v1 + wvv.z * v2 + wvv.w * vx);
        nv[0] = v1; nv[1] = v2; nv[2] = vx;
    }
    const float sq = block_sum<NS * NW>(yq * yq, s_red);
    const float sk = block_sum<NS * NW>(yk * yk, s_red);
    // (block_sum ends with a barrier: every thread has read the old states)
    if (t < DK) {
        s_q[t] = yq * rsqrtf(sq + a.l2_eps);
        s_k[t] = yk * rsqrtf(sk + a.l2_eps);
        for (int i = 0; i < 3; ++i) {
            cq[srow(i, DK) + t] = from_f32<TIn>(nq[i]);
            ck[srow(i, DK) + t] = from_f32<TIn>(nk[i]);
        }
    }
    if (tid < DVS) {
        for (int i = 0; i < 3; ++i) cv[srow(i, DV) + j0 + tid] = from_f32<TIn>(nv[i]);
    }
    __syncthreads();
    if (t < 32) {
        float kq = 0.f;
        for (int c = lane; c < DK; c += 32) kq += s_k[c] * s_q[c];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        if (lane == 0) s_kq = kq;
    }
    // 3. the decode step: decay, the two column reductions over dk
    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int row = p * RP + w * RPW + rw;
        const float al = s_a[row], kc = s_k[row], qc = s_q[row];
        x[p].x *= al; x[p].y *= al; x[p].z *= al; x[p].w *= al;
        pk.x += kc * x[p].x; pk.y += kc * x[p].y; pk.z += kc * x[p].z; pk.w += kc * x[p].w;
        pq.x += qc * x[p].x; pq.y += qc * x[p].y; pq.z += qc * x[p].z; pq.w += qc * x[p].w;
    }
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
        s_redk[sl][w][c4] = pk;
        s_redq[sl][w][c4] = pq;
    }
    __syncthreads();
    float4 rk = make_float4(0.f, 0.f, 0.f, 0.f), rq = rk;
#pragma unroll
    for (int i = 0; i < NW; ++i) {
        const float4 u = s_redk[sl][i][c4], v = s_redq[sl][i][c4];
        rk.x += u.x; rk.y += u.y; rk.z += u.z; rk.w += u.w;
        rq.x += v.x; rq.y += v.y; rq.z += v.z; rq.w += v.w;
    }
    const float b = a.beta[unit];
    float4 u;
    u.x = b * (s_v[sl][4 * c4 + 0] - rk.x);
    u.y = b * (s_v[sl][4 * c4 + 1] - rk.y);
    u.z = b * (s_v[sl][4 * c4 + 2] - rk.z);
    u.w = b * (s_v[sl][4 * c4 + 3] - rk.w);
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        const int row = p * RP + w * RPW + rw;
        const float kc = s_k[row];
        float4 yv = x[p];
        yv.x += kc * u.x; yv.y += kc * u.y; yv.z += kc * u.z; yv.w += kc * u.w;
        __stcs(S + row * (DV / 4) + c4, yv);
    }
    // 4. epilogue: o of each slice (the unit's warp 0, lanes of row 0), the
    // slices' sums of squares, RMSNorm over all DV columns, weight and gate
    float o4[4] = {0.f, 0.f, 0.f, 0.f};
    if (w == 0 && rw == 0) {
        const float kq = s_kq;
        o4[0] = rq.x + u.x * kq;
        o4[1] = rq.y + u.y * kq;
        o4[2] = rq.z + u.z * kq;
        o4[3] = rq.w + u.w * kq;
        float ss = o4[0] * o4[0] + o4[1] * o4[1] + o4[2] * o4[2] + o4[3] * o4[3];
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1)
            ss += __shfl_xor_sync((LPR == 32) ? 0xffffffffu : ((1u << LPR) - 1u), ss, off);
        if (lane == 0) s_ss[sl] = ss;
    }
    __syncthreads();
    if (w == 0 && rw == 0) {
        float total = 0.f;
#pragma unroll
        for (int r = 0; r < NS; ++r) total += s_ss[r];
        const float inv = rsqrtf(total / DV + a.rms_eps);
        const TIn* gate = static_cast<const TIn*>(a.gate);
        TIn* y = static_cast<TIn*>(a.y);
        const size_t vo = (size_t)unit * DV + j0 + 4 * c4;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float gt = to_f32(gate[vo + i]);
            y[vo + i] = from_f32<TIn>(
                o4[i] * inv * a.w_norm[j0 + 4 * c4 + i] * sigmoid_for<TIn>(gt));
        }
    }
}

template <int DK, int DV, typename TIn>
cudaError_t launch_layer_decode_t(const LayerDecodeArgs& a, int units, cudaStream_t st) {
    // one 256-thread CTA per (sequence, head) over all DV columns: measured
    // 209 us against 237 us for two 256-thread units of DV / 2 columns in one
    // CTA (N = 256, H = 32, d = 128, bf16)
    constexpr int DVS = DV;
    layer_decode_kernel<DK, DV, DVS, TIn><<<units, 256 * (DV / DVS), 0, st>>>(a);
    return cudaGetLastError();
}

template <typename TIn>
cudaError_t layer_decode_dispatch(const LayerDecodeArgs& a, int units, int dk, int dv,
                                  cudaStream_t st) {
#define KDA_LD_CASE(A, B) \
    if (dk == A && dv == B) return launch_layer_decode_t<A, B, TIn>(a, units, st);
    KDA_LD_CASE(128, 128)
    KDA_LD_CASE(128, 64)
    KDA_LD_CASE(128, 32)
    KDA_LD_CASE(64, 128)
    KDA_LD_CASE(64, 64)
    KDA_LD_CASE(64, 32)
    KDA_LD_CASE(32, 128)
    KDA_LD_CASE(32, 64)
    KDA_LD_CASE(32, 32)
#undef KDA_LD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_layer_decode(const void* xq, const void* xk, const void* xv, const float* wq,
                                const float* wk, const float* wv, void* conv_q, void* conv_k,
                                void* conv_v, const float* g, const float* beta, float* state,
                                const void* gate, const float* w_norm, int N, int H, int dk,
                                int dv, kda_dtype_t dt, float l2_eps, float rms_eps, void* y,
                                cudaStream_t st) {
    const int units = N * H;
    if (units == 0) return cudaSuccess;
    const LayerDecodeArgs a{xq, xk, xv, wq, wk, wv, conv_q, conv_k, conv_v, g, beta,
                            state, gate, w_norm, y, H, l2_eps, rms_eps};
    if (dt == KDA_DTYPE_BF16) return layer_decode_dispatch<__nv_bfloat16>(a, units, dk, dv, st);
    return layer_decode_dispatch<float>(a, units, dk, dv, st);
}

}  // namespace kda
