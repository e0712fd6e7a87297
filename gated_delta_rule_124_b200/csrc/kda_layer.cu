// The per-head steps around the KDA operator (Kimi Linear (aiwiki.ai), "The
// constrained DPLR form and the chunkwise algorithm", the paragraph on what
// each KDA head applies): before it, a causal depthwise convolution of kernel
// size 4 with a Swish activation on q, k and v and the L2 normalisation of q
// and k; after it, a head-wise RMSNorm and a sigmoid output gate.
//
// Both kernels stream their tensors once (HBM-bound, a few flops per byte).
// Each lane holds d/32 consecutive channels of a head, so a warp reads and
// writes whole contiguous head rows; the per-(token, head) reductions (sum of
// squares over the channels) are warp shuffles.  The convolution gives a warp
// a run of consecutive tokens of one head, keeping the filter and the last
// three inputs in registers (never across the start of a sequence); the
// output step gives a warp one (token, head).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda_common.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace {

constexpr int kWarps = 8;  // warps (token, head pairs) per 256-thread CTA

template <int CPL, typename T>
struct Vec;
template <int CPL>
struct Vec<CPL, float> {
    __device__ static void load(const float* p, float (&x)[CPL]) {
#pragma unroll
        for (int i = 0; i < CPL; ++i) x[i] = p[i];
    }
    __device__ static void store(float* p, const float (&x)[CPL]) {
#pragma unroll
        for (int i = 0; i < CPL; ++i) p[i] = x[i];
    }
};
template <int CPL>
struct Vec<CPL, __nv_bfloat16> {
    __device__ static void load(const __nv_bfloat16* p, float (&x)[CPL]) {
#pragma unroll
        for (int i = 0; i < CPL; ++i) x[i] = __bfloat162float(p[i]);
    }
    __device__ static void store(__nv_bfloat16* p, const float (&x)[CPL]) {
#pragma unroll
        for (int i = 0; i < CPL; ++i) p[i] = __float2bfloat16_rn(x[i]);
    }
};
template <>
struct Vec<4, __nv_bfloat16> {  // 8-byte vectors
    __device__ static void load(const __nv_bfloat16* p, float (&x)[4]) {
        const uint2 u = *reinterpret_cast<const uint2*>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    }
    __device__ static void store(__nv_bfloat16* p, const float (&x)[4]) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(x[0], x[1]);
        const __nv_bfloat162 b = __floats2bfloat162_rn(x[2], x[3]);
        uint2 u;
        u.x = *reinterpret_cast<const uint32_t*>(&a);
        u.y = *reinterpret_cast<const uint32_t*>(&b);
        *reinterpret_cast<uint2*>(p) = u;
    }
};
template <>
struct Vec<4, float> {  // 16-byte vectors
    __device__ static void load(const float* p, float (&x)[4]) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    }
    __device__ static void store(float* p, const float (&x)[4]) {
        *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

constexpr int kRun = 32;  // consecutive tokens per warp in the convolution

// The sequence holding token t: its index s (the last s with cu[s] <= t) --
// clamped to [0, N - 1] so that a malformed cu_seqlens cannot send a read out
// of the tensors -- or, without cu_seqlens, t / T.
__device__ __forceinline__ int seq_of(const int32_t* cu, int N, int T, int t) {
    if (!cu) return T > 0 ? t / T : 0;
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}
// The same for a whole warp (every lane gets the answer): a 32-ary search, one
// load per lane and level, so one round trip per level instead of one per
// halving (at most 32 sequences: one level).  cu is non-decreasing with cu[0]
// = 0 <= t, so lane 0's entry always qualifies and the answer is the last
// entry <= t, as in seq_of.
__device__ __forceinline__ int warp_seq_of(const int32_t* cu, int N, int T, int t, int lane) {
    if (!cu) return T > 0 ? t / T : 0;
    int lo = 0, span = N;  // s lies in [lo, lo + span)
    while (true) {
        const int step = span <= 32 ? 1 : (span + 31) / 32;
        const int idx = lo + lane * step;
        const bool le = idx < lo + span && cu[idx] <= t;
        const unsigned m = __ballot_sync(0xffffffffu, le);
        const int k = m ? 31 - __clz(static_cast<int>(m)) : 0;
        if (step == 1) return lo + k;
        lo += k * step;
        span = min(step, N - lo);
    }
}
__device__ __forceinline__ int seq_begin(const int32_t* cu, int T, int s) {
    return cu ? max(0, cu[s]) : s * T;
}
__device__ __forceinline__ int seq_end(const int32_t* cu, int T, int s) {
    return cu ? cu[s + 1] : (s + 1) * T;
}

struct ConvArgs {
    const void* x[3];
    const float* w[3];
    void* y[3];
    int d[3];
};

// One warp per (tensor, head, run of kRun tokens): the filter stays in
// registers and the last three inputs slide along, so every input row is read
// once (plus a three-token halo per run).  y = Swish(causal depthwise
// conv4(x)), L2-normalised per (token, head) for q and k (tensors 0 and 1).
template <int CPL, typename TIn>
__device__ __forceinline__ void conv_run(const TIn* __restrict__ x, const float* __restrict__ w,
                                         TIn* __restrict__ y, const int32_t* __restrict__ cu,
                                         int N, int T, int total, int H, int h, int t0, bool l2,
                                         float eps) {
    constexpr int D = 32 * CPL;
    const int lane = threadIdx.x & 31, c0 = lane * CPL;
    float wt[CPL][4];
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        const float4 v = *reinterpret_cast<const float4*>(w + ((size_t)h * D + c0 + j) * 4);
        wt[j][0] = v.x; wt[j][1] = v.y; wt[j][2] = v.z; wt[j][3] = v.w;
    }
    // the halo rows and the first row are requested before the sequence
    // lookup (which only decides whether the halo belongs to t0's sequence)
    float win[3][CPL];  // inputs of tokens t - 3, t - 2, t - 1
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const int src = t0 - 3 + i;
        if (src >= 0) {
            Vec<CPL, TIn>::load(x + ((size_t)src * H + h) * D + c0, win[i]);
        } else {
#pragma unroll
            for (int j = 0; j < CPL; ++j) win[i][j] = 0.f;
        }
    }
    const int t1 = min(total, t0 + kRun);
    float nxt[CPL];  // the next token's row, requested one token ahead
    Vec<CPL, TIn>::load(x + ((size_t)t0 * H + h) * D + c0, nxt);
    int s = warp_seq_of(cu, N, T, t0, lane);
    int begin = seq_begin(cu, T, s), end = seq_end(cu, T, s);
#pragma unroll
    for (int i = 0; i < 3; ++i)
        if (t0 - 3 + i < begin)
#pragma unroll
            for (int j = 0; j < CPL; ++j) win[i][j] = 0.f;
    for (int t = t0; t < t1; ++t) {
        float cur[CPL];
#pragma unroll
        for (int j = 0; j < CPL; ++j) cur[j] = nxt[j];
        if (t + 1 < t1) Vec<CPL, TIn>::load(x + ((size_t)(t + 1) * H + h) * D + c0, nxt);
        while (t >= end && s < N - 1) {  // t starts a new sequence: no history
            ++s;
            begin = seq_begin(cu, T, s);
            end = seq_end(cu, T, s);
#pragma unroll
            for (int i = 0; i < 3; ++i)
#pragma unroll
                for (int j = 0; j < CPL; ++j) win[i][j] = 0.f;
        }
        float out[CPL], ss = 0.f;
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            float acc = wt[j][3] * cur[j];
            acc = fmaf(wt[j][2], win[2][j], acc);
            acc = fmaf(wt[j][1], win[1][j], acc);
            acc = fmaf(wt[j][0], win[0][j], acc);
            out[j] = swish_for<TIn>(acc);
            ss = fmaf(out[j], out[j], ss);
            win[0][j] = win[1][j];
            win[1][j] = win[2][j];
            win[2][j] = cur[j];
        }
        if (l2) {
            const float inv = rsqrtf(warp_sum(ss) + eps);
#pragma unroll
            for (int j = 0; j < CPL; ++j) out[j] *= inv;
        }
        Vec<CPL, TIn>::store(y + ((size_t)t * H + h) * D + c0, out);
    }
}

// One decode token per (tensor, sequence, head), one warp: the filter's first
// three taps read the sequence's last three inputs from its convolution state
// [N, 3, H, D] (oldest first), the fourth the new input; the state then drops
// its oldest row and appends the input.
template <int CPL, typename TIn>
__device__ __forceinline__ void conv_step(const TIn* __restrict__ x, const float* __restrict__ w,
                                          TIn* __restrict__ state, TIn* __restrict__ y, int H,
                                          int n, int h, bool l2, float eps) {
    constexpr int D = 32 * CPL;
    const int lane = threadIdx.x & 31, c0 = lane * CPL;
    float wt[CPL][4];
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        const float4 v = *reinterpret_cast<const float4*>(w + ((size_t)h * D + c0 + j) * 4);
        wt[j][0] = v.x; wt[j][1] = v.y; wt[j][2] = v.z; wt[j][3] = v.w;
    }
    float win[3][CPL], cur[CPL];
#pragma unroll
    for (int i = 0; i < 3; ++i)
        Vec<CPL, TIn>::load(state + (((size_t)n * 3 + i) * H + h) * D + c0, win[i]);
    Vec<CPL, TIn>::load(x + ((size_t)n * H + h) * D + c0, cur);
    float out[CPL], ss = 0.f;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        float acc = wt[j][3] * cur[j];
        acc = fmaf(wt[j][2], win[2][j], acc);
        acc = fmaf(wt[j][1], win[1][j], acc);
        acc = fmaf(wt[j][0], win[0][j], acc);
        out[j] = swish_for<TIn>(acc);
        ss = fmaf(out[j], out[j], ss);
    }
    Vec<CPL, TIn>::store(state + (((size_t)n * 3 + 0) * H + h) * D + c0, win[1]);
    Vec<CPL, TIn>::store(state + (((size_t)n * 3 + 1) * H + h) * D + c0, win[2]);
    Vec<CPL, TIn>::store(state + (((size_t)n * 3 + 2) * H + h) * D + c0, cur);
    if (l2) {
        const float inv = rsqrtf(warp_sum(ss) + eps);
#pragma unroll
        for (int j = 0; j < CPL; ++j) out[j] *= inv;
    }
    Vec<CPL, TIn>::store(y + ((size_t)n * H + h) * D + c0, out);
}

struct StepArgs {
    const void* x[3];
    const float* w[3];
    void* state[3];
    void* y[3];
    int d[3];
};

template <typename TIn>
__global__ void __launch_bounds__(32 * kWarps) conv_step_kernel(const StepArgs a, int N, int H,
                                                                float eps) {
    const int tensor = blockIdx.y;  // 0 q, 1 k, 2 v
    const long long task = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (task >= (long long)N * H) return;
    const int h = static_cast<int>(task % H), n = static_cast<int>(task / H);
    const TIn* x = static_cast<const TIn*>(tensor == 0 ? a.x[0] : tensor == 1 ? a.x[1] : a.x[2]);
    TIn* y = static_cast<TIn*>(tensor == 0 ? a.y[0] : tensor == 1 ? a.y[1] : a.y[2]);
    TIn* st = static_cast<TIn*>(tensor == 0 ? a.state[0] : tensor == 1 ? a.state[1] : a.state[2]);
    const float* w = tensor == 0 ? a.w[0] : tensor == 1 ? a.w[1] : a.w[2];
    const int d = tensor == 0 ? a.d[0] : tensor == 1 ? a.d[1] : a.d[2];
    const bool l2 = tensor < 2;
    switch (d) {
        case 128: conv_step<4, TIn>(x, w, st, y, H, n, h, l2, eps); break;
        case 64: conv_step<2, TIn>(x, w, st, y, H, n, h, l2, eps); break;
        default: conv_step<1, TIn>(x, w, st, y, H, n, h, l2, eps); break;
    }
}

template <typename TIn>
__global__ void __launch_bounds__(32 * kWarps) conv_swish_kernel(
    const ConvArgs a, const int32_t* __restrict__ cu, int N, int T, int total, int H, float eps) {
    const int tensor = blockIdx.y;  // 0 q, 1 k, 2 v
    const long long task = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const long long runs = (total + kRun - 1) / kRun;
    if (task >= runs * H) return;
    const int h = static_cast<int>(task % H), t0 = static_cast<int>(task / H) * kRun;
    // (selects rather than an indexed parameter array, which would go through
    // the stack)
    const TIn* x = static_cast<const TIn*>(tensor == 0 ? a.x[0] : tensor == 1 ? a.x[1] : a.x[2]);
    TIn* y = static_cast<TIn*>(tensor == 0 ? a.y[0] : tensor == 1 ? a.y[1] : a.y[2]);
    const float* w = tensor == 0 ? a.w[0] : tensor == 1 ? a.w[1] : a.w[2];
    const int d = tensor == 0 ? a.d[0] : tensor == 1 ? a.d[1] : a.d[2];
    const bool l2 = tensor < 2;
    switch (d) {
        case 128: conv_run<4, TIn>(x, w, y, cu, N, T, total, H, h, t0, l2, eps); break;
        case 64: conv_run<2, TIn>(x, w, y, cu, N, T, total, H, h, t0, l2, eps); break;
        default: conv_run<1, TIn>(x, w, y, cu, N, T, total, H, h, t0, l2, eps); break;
    }
}

// bf16, d = 128 (q, k and v): the same warp per (tensor, head, run of kRun
// tokens), but the run's rows and the three before it are first copied into
// the warp's part of shared memory at once (16-byte cp.async, 35 rows of 256 B;
// zeros outside [0, total)), so that every warp has its whole run in flight
// instead of one row ahead; the sliding window then reads the rows there.
constexpr int kStageRows = kRun + 3;
constexpr int kStageBytes = kWarps * kStageRows * 128 * 2;

__global__ void __launch_bounds__(32 * kWarps) conv_staged_kernel(
    const ConvArgs a, const int32_t* __restrict__ cu, int N, int T, int total, int H, float eps) {
    constexpr int D = 128, CPL = 4;
    extern __shared__ __align__(16) uint8_t conv_smem[];
    const int tensor = blockIdx.y;  // 0 q, 1 k, 2 v
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, c0 = lane * CPL;
    const long long task = (long long)blockIdx.x * kWarps + warp;
    const long long runs = (total + kRun - 1) / kRun;
    if (task >= runs * H) return;  // (per warp; no block-wide barrier below)
    const int h = static_cast<int>(task % H), t0 = static_cast<int>(task / H) * kRun;
    const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(
        tensor == 0 ? a.x[0] : tensor == 1 ? a.x[1] : a.x[2]);
    __nv_bfloat16* y = static_cast<__nv_bfloat16*>(tensor == 0 ? a.y[0] : tensor == 1 ? a.y[1] : a.y[2]);
    const float* w = tensor == 0 ? a.w[0] : tensor == 1 ? a.w[1] : a.w[2];
    const bool l2 = tensor < 2;
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(conv_smem) + warp * kStageRows * D;
    for (int e = lane; e < kStageRows * (D / 8); e += 32) {  // rows t0 - 3 .. t0 + kRun - 1
        const int row = e >> 4, ch = e & 15, t = t0 - 3 + row;
        __nv_bfloat16* dst = xs + row * D + ch * 8;
        if (t >= 0 && t < total)
            sm100::cp_async16(dst, x + ((size_t)t * H + h) * D + ch * 8);
        else
            *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
    sm100::cp_async_commit();
    float wt[CPL][4];
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        const float4 v = *reinterpret_cast<const float4*>(w + ((size_t)h * D + c0 + j) * 4);
        wt[j][0] = v.x; wt[j][1] = v.y; wt[j][2] = v.z; wt[j][3] = v.w;
    }
    int s = warp_seq_of(cu, N, T, t0, lane);
    int begin = seq_begin(cu, T, s), end = seq_end(cu, T, s);
    sm100::cp_async_wait_all();
    __syncwarp();
    float win[3][CPL];  // inputs of tokens t - 3, t - 2, t - 1
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        Vec<CPL, __nv_bfloat16>::load(xs + i * D + c0, win[i]);
        if (t0 - 3 + i < begin)
#pragma unroll
            for (int j = 0; j < CPL; ++j) win[i][j] = 0.f;
    }
    const int t1 = min(total, t0 + kRun);
    for (int t = t0; t < t1; ++t) {
        float cur[CPL];
        Vec<CPL, __nv_bfloat16>::load(xs + (t - t0 + 3) * D + c0, cur);
        while (t >= end && s < N - 1) {  // t starts a new sequence: no history
            ++s;
            begin = seq_begin(cu, T, s);
            end = seq_end(cu, T, s);
#pragma unroll
            for (int i = 0; i < 3; ++i)
#pragma unroll
                for (int j = 0; j < CPL; ++j) win[i][j] = 0.f;
        }
        float out[CPL], ss = 0.f;
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            float acc = wt[j][3] * cur[j];
            acc = fmaf(wt[j][2], win[2][j], acc);
            acc = fmaf(wt[j][1], win[1][j], acc);
            acc = fmaf(wt[j][0], win[0][j], acc);
            out[j] = swish_for<__nv_bfloat16>(acc);
            ss = fmaf(out[j], out[j], ss);
            win[0][j] = win[1][j];
            win[1][j] = win[2][j];
            win[2][j] = cur[j];
        }
        if (l2) {
            const float inv = rsqrtf(warp_sum(ss) + eps);
#pragma unroll
            for (int j = 0; j < CPL; ++j) out[j] *= inv;
        }
        Vec<CPL, __nv_bfloat16>::store(y + ((size_t)t * H + h) * D + c0, out);
    }
}

// y = o / sqrt(mean o^2 + eps) * w * sigmoid(gate), per (token, head); a warp
// takes kPairs consecutive (token, head) rows, all loads issued first.
constexpr int kPairs = 4;
template <int CPL, typename TIn>
__global__ void __launch_bounds__(32 * kWarps) norm_gate_kernel(
    const TIn* o, const TIn* gate, const float* __restrict__ w, int total, int H, float eps,
    TIn* y) {  // y may be o
    constexpr int D = 32 * CPL;
    const int lane = threadIdx.x & 31;
    const long long rows = (long long)total * H;
    const long long first = ((long long)blockIdx.x * kWarps + (threadIdx.x >> 5)) * kPairs;
    if (first >= rows) return;
    float ov[kPairs][CPL], gv[kPairs][CPL], wv[CPL];
#pragma unroll
    for (int j = 0; j < CPL; ++j) wv[j] = w[lane * CPL + j];
#pragma unroll
    for (int p = 0; p < kPairs; ++p) {
        if (first + p < rows) {
            const size_t base = (size_t)(first + p) * D + lane * CPL;
            Vec<CPL, TIn>::load(o + base, ov[p]);
            Vec<CPL, TIn>::load(gate + base, gv[p]);
        }
    }
#pragma unroll
    for (int p = 0; p < kPairs; ++p) {
        if (first + p >= rows) break;
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < CPL; ++j) ss = fmaf(ov[p][j], ov[p][j], ss);
        const float r = rsqrtf(warp_sum(ss) * (1.f / D) + eps);
        float out[CPL];
#pragma unroll
        for (int j = 0; j < CPL; ++j)
            out[j] = ov[p][j] * r * wv[j] * sigmoid_for<TIn>(gv[p][j]);
        Vec<CPL, TIn>::store(y + (size_t)(first + p) * D + lane * CPL, out);
    }
}

unsigned grid_for(int total, int H) {
    const long long per_block = (long long)kWarps * kPairs;
    return static_cast<unsigned>(((long long)total * H + per_block - 1) / per_block);
}

template <typename TIn>
cudaError_t gate_dispatch(const void* o, const void* gate, const float* w, int total, int H,
                          int d, float eps, void* y, cudaStream_t st) {
    const unsigned g = grid_for(total, H);
    const TIn* O = static_cast<const TIn*>(o);
    const TIn* G = static_cast<const TIn*>(gate);
    TIn* Y = static_cast<TIn*>(y);
    if (d == 128)
        norm_gate_kernel<4, TIn><<<g, 32 * kWarps, 0, st>>>(O, G, w, total, H, eps, Y);
    else if (d == 64)
        norm_gate_kernel<2, TIn><<<g, 32 * kWarps, 0, st>>>(O, G, w, total, H, eps, Y);
    else
        norm_gate_kernel<1, TIn><<<g, 32 * kWarps, 0, st>>>(O, G, w, total, H, eps, Y);
    return cudaGetLastError();
}

__global__ void spread_gate_kernel(const float* __restrict__ g, long long n, int dk,
                                   float* __restrict__ out) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = g[i / dk];
}

}  // namespace

cudaError_t launch_spread_gate(const float* g, int total, int H, int dk, float* out,
                               cudaStream_t st) {
    const long long n = (long long)total * H * dk;
    if (n == 0) return cudaSuccess;
    spread_gate_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(g, n, dk, out);
    return cudaGetLastError();
}

cudaError_t launch_qkv_conv(const void* const x[3], const float* const w[3], void* const y[3],
                            int dk, int dv, const int32_t* cu, int N, int T, int total, int H,
                            float eps, kda_dtype_t dt, cudaStream_t st) {
    if ((long long)total * H == 0) return cudaSuccess;
    ConvArgs a;
    for (int i = 0; i < 3; ++i) {
        a.x[i] = x[i];
        a.w[i] = w[i];
        a.y[i] = y[i];
        a.d[i] = i < 2 ? dk : dv;
    }
    const long long runs = (total + kRun - 1) / kRun;
    const dim3 grid(static_cast<unsigned>((runs * H + kWarps - 1) / kWarps), 3);
    if (dt == KDA_DTYPE_BF16 && dk == 128 && dv == 128) {
        const cudaError_t attr = cudaFuncSetAttribute(
            conv_staged_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kStageBytes);
        if (attr != cudaSuccess) return attr;
        conv_staged_kernel<<<grid, 32 * kWarps, kStageBytes, st>>>(a, cu, N, T, total, H, eps);
    } else if (dt == KDA_DTYPE_BF16)
        conv_swish_kernel<__nv_bfloat16><<<grid, 32 * kWarps, 0, st>>>(a, cu, N, T, total, H, eps);
    else
        conv_swish_kernel<float><<<grid, 32 * kWarps, 0, st>>>(a, cu, N, T, total, H, eps);
    return cudaGetLastError();
}

cudaError_t launch_qkv_conv_step(const void* const x[3], const float* const w[3],
                                 void* const state[3], void* const y[3], int dk, int dv, int N,
                                 int H, float eps, kda_dtype_t dt, cudaStream_t st) {
    if ((long long)N * H == 0) return cudaSuccess;
    StepArgs a;
    for (int i = 0; i < 3; ++i) {
        a.x[i] = x[i];
        a.w[i] = w[i];
        a.state[i] = state[i];
        a.y[i] = y[i];
        a.d[i] = i < 2 ? dk : dv;
    }
    const dim3 grid(static_cast<unsigned>(((long long)N * H + kWarps - 1) / kWarps), 3);
    if (dt == KDA_DTYPE_BF16)
        conv_step_kernel<__nv_bfloat16><<<grid, 32 * kWarps, 0, st>>>(a, N, H, eps);
    else
        conv_step_kernel<float><<<grid, 32 * kWarps, 0, st>>>(a, N, H, eps);
    return cudaGetLastError();
}

cudaError_t launch_norm_gate(const void* o, const void* gate, const float* w, int total, int H,
                             int d, float eps, kda_dtype_t dt, void* y, cudaStream_t st) {
    if ((long long)total * H == 0) return cudaSuccess;
    if (dt == KDA_DTYPE_BF16)
        return gate_dispatch<__nv_bfloat16>(o, gate, w, total, H, d, eps, y, st);
    return gate_dispatch<float>(o, gate, w, total, H, d, eps, y, st);
}

}  // namespace kda
