// Shared device helpers of libkda (not part of the public ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

// ---------------------------------------------------------------- workspace
// Layout of the caller's workspace (all offsets 256-byte aligned):
//   [0, 256)              status word (uint32 at offset 0); at offset 4 the
//                         largest number of chunks of one sequence (written
//                         by the chunk-table kernel); padding
//   chunk_start[N + 1]    int32: global index of each sequence's first chunk
//   seq_order[N]          int32: the sequences by descending chunk count (ties
//                         by index; the identity beyond kMaxOrderedSeqs)
//   chunk_info[maxc]      int4 {seq, first token, rows, chunk-in-sequence};
//                         unused slots hold seq = -1, rows = 0
//   then, for the CUDA-core path only: G, W, U (token-major fp32) and the
//   per-chunk states [maxc, H, dk, dv] fp32; for the split tensor-core path
//   only: one operand blob per (chunk slot, head), then one uint32 ready flag
//   per (chunk slot, head).
constexpr size_t kAlign = 256;
// Sequences the chunk-table kernel sorts by length (it ranks them in shared
// memory); larger batches keep their order.
constexpr int kMaxOrderedSeqs = 4096;

__host__ __device__ inline size_t align_up(size_t x, size_t a = kAlign) {
    return (x + a - 1) / a * a;
}

// Device status bits (OR-ed by kernels; the first error wins on the host).
enum : uint32_t { STATUS_BAD_SEQLENS = 1u, STATUS_TIMEOUT = 2u };

struct Workspace {
    uint32_t* status;
    int* chunk_start;
    int* seq_order;
    int4* chunk_info;
    float* G;
    float* W;
    float* U;
    float* states;
    uint8_t* blobs;
    uint32_t* flags;
    size_t header_bytes;  // status + tables
    size_t total_bytes;   // header + CUDA-core path intermediates
};

inline int max_chunks(int total_tokens, int num_seqs, int chunk) {
    // sum_s ceil(len_s / C) <= (total + N (C - 1)) / C
    return (int)(((long long)total_tokens + (long long)num_seqs * (chunk - 1)) / chunk);
}

inline Workspace carve(void* base, int total, int N, int H, int dk, int dv, int chunk,
                       bool with_intermediates, size_t blob_bytes = 0) {
    Workspace w{};
    const int maxc = max_chunks(total, N, chunk);
    char* p = static_cast<char*>(base);
    size_t off = 0;
    w.status = reinterpret_cast<uint32_t*>(p + off);
    off += kAlign;
    w.chunk_start = reinterpret_cast<int*>(p + off);
    off = align_up(off + sizeof(int) * (size_t)(N + 1));
    w.seq_order = reinterpret_cast<int*>(p + off);
    off = align_up(off + sizeof(int) * (size_t)N);
    w.chunk_info = reinterpret_cast<int4*>(p + off);
    off = align_up(off + sizeof(int4) * (size_t)maxc);
    w.header_bytes = off;
    if (with_intermediates) {
        w.G = reinterpret_cast<float*>(p + off);
        off = align_up(off + sizeof(float) * (size_t)total * H * dk);
        w.W = reinterpret_cast<float*>(p + off);
        off = align_up(off + sizeof(float) * (size_t)total * H * dk);
        w.U = reinterpret_cast<float*>(p + off);
        off = align_up(off + sizeof(float) * (size_t)total * H * dv);
        w.states = reinterpret_cast<float*>(p + off);
        off = align_up(off + sizeof(float) * (size_t)maxc * H * dk * dv);
    }
    if (blob_bytes) {
        off = align_up(off, 1024);
        w.blobs = reinterpret_cast<uint8_t*>(p + off);
        off = align_up(off + blob_bytes * (size_t)maxc * H);
        w.flags = reinterpret_cast<uint32_t*>(p + off);
        off = align_up(off + sizeof(uint32_t) * (size_t)maxc * H);
    }
    w.total_bytes = off;
    return w;
}

// ------------------------------------------------------------- conversions
// x rounded to the nearest tf32 value (10-bit mantissa, ties away from zero;
// the low 13 bits zero): operands of kind::tf32 products are written rounded,
// since the tensor cores drop those bits, a bias that adds up over a sum.
__device__ __forceinline__ float round_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
    return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Logistic function with one MUFU operation: sigmoid(x) = (1 + tanh(x / 2)) / 2
// (tanh.approx.f32, max relative error about 2^-11, so an absolute error of at
// most about 2.5e-4 here); Swish is x * sigmoid(x).
__device__ __forceinline__ float fast_sigmoid(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * x));
    return fmaf(0.5f, t, 0.5f);
}
__device__ __forceinline__ float fast_swish(float x) { return x * fast_sigmoid(x); }
// The forms the layer kernels use per output type: bf16 outputs (rounded to 8
// mantissa bits anyway) take the one-MUFU logistic, fp32 outputs the
// exponential and a fast division.
template <typename TOut>
__device__ __forceinline__ float sigmoid_for(float x) {
    return fast_sigmoid(x);
}
template <>
__device__ __forceinline__ float sigmoid_for<float>(float x) {
    return __fdividef(1.f, 1.f + __expf(-x));
}
template <typename TOut>
__device__ __forceinline__ float swish_for(float x) {
    return x * sigmoid_for<TOut>(x);
}

__device__ __forceinline__ bool status_bad(const uint32_t* status) {
    return *reinterpret_cast<const volatile uint32_t*>(status) != 0u;
}

}  // namespace kda

// Host-side prefill helpers shared by the entry points (kda_api.cu defines them).
namespace kda {
// Tokens and sequences of one prefill call.
struct Prefill {
    int total, N;
};
// The argument rules every prefill entry point shares (sizes, dtype, the
// cu_seqlens / B / T / num_seqs combination, supported dk, dv and chunk).
kda_status_t check_prefill_shape(const int32_t* cu, int B, int T, int num_seqs, int H, int dk,
                                 int dv, int chunk, kda_dtype_t dt, Prefill* out);
// Clear the status word and build the chunk table (two stream operations).
kda_status_t begin_prefill(const Workspace& w, const int32_t* cu, int B, int T, int N, int chunk,
                           int maxc, cudaStream_t st);
// The CUDA-core plan after the chunk table: a1 .. a4 as four kernels on the
// intermediates of `w` (carved with_intermediates).
kda_status_t run_simt(const void* q, const void* k, const void* v, const float* g,
                      const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                      int B, int T, const Prefill& p, int H, int dk, int dv, int chunk,
                      kda_dtype_t dtype, void* o, float* final_state, const Workspace& w,
                      int maxc, cudaStream_t st);
}  // namespace kda

// Launchers implemented in the .cu files (host side, return cudaError_t).
namespace kda {
cudaError_t launch_build_chunk_table(const int32_t* cu_seqlens, int B, int T, int N, int chunk,
                                     int maxc, uint32_t* status, int* chunk_start,
                                     int4* chunk_info, cudaStream_t st,
                                     int* seq_order = nullptr);
cudaError_t launch_gate_cumsum(const float* g, const int4* info, int maxc, int H, int dk,
                               const uint32_t* status, float* G, cudaStream_t st);
cudaError_t launch_intra(const void* k, const void* v, const float* G, const float* beta,
                         const int4* info, int maxc, int H, int dk, int dv, int chunk,
                         kda_dtype_t dt, const uint32_t* status, float* W, float* U,
                         cudaStream_t st);
cudaError_t launch_inter(const void* k, const float* G, const float* W, float* U,
                         const float* h0, const int32_t* cu_seqlens, int B, int T, int N,
                         const int* chunk_start, int H, int dk, int dv, int chunk,
                         kda_dtype_t dt, const uint32_t* status, float* states, float* hN,
                         cudaStream_t st, int dv_slice = 0);
cudaError_t launch_output(const void* q, const void* k, const float* G, const float* U,
                          const float* states, const int4* info, int maxc, int H, int dk,
                          int dv, int chunk, kda_dtype_t dt, const uint32_t* status, void* o,
                          cudaStream_t st);
cudaError_t launch_qkv_conv(const void* const x[3], const float* const w[3], void* const y[3],
                            int dk, int dv, const int32_t* cu, int N, int T, int total, int H,
                            float eps, kda_dtype_t dt, cudaStream_t st);
cudaError_t launch_qkv_conv_step(const void* const x[3], const float* const w[3],
                                 void* const state[3], void* const y[3], int dk, int dv, int N,
                                 int H, float eps, kda_dtype_t dt, cudaStream_t st);
cudaError_t launch_norm_gate(const void* o, const void* gate, const float* w, int total, int H,
                             int d, float eps, kda_dtype_t dt, void* y, cudaStream_t st);
cudaError_t launch_layer_decode(const void* xq, const void* xk, const void* xv, const float* wq,
                                const float* wk, const float* wv, void* conv_q, void* conv_k,
                                void* conv_v, const float* g, const float* beta, float* state,
                                const void* gate, const float* w_norm, int N, int H, int dk,
                                int dv, kda_dtype_t dt, float l2_eps, float rms_eps, void* y,
                                cudaStream_t st);
cudaError_t launch_decode(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, float* state, void* o, int N, int H, int dk,
                          int dv, kda_dtype_t dt, cudaStream_t st, bool head_gate = false);
size_t bwd_workspace_bytes(int total, int N, int H, int dk, int dv);
// Composition of per-segment state maps (kda_segments.cu): forward entry
// states, or (reverse) exit-state gradients; see kda_fold_segment_states.
cudaError_t launch_fold_segments(const float* M, const float* Bm, const float* S0, int R, int NH,
                                 int dk, int dv, bool reverse, float* each, float* fin,
                                 cudaStream_t st);
// The backward's two chains on the tensor cores (dk = dv = 128): the forward
// pass (U in place of Ut, the entry state of every chunk) and the backward
// pass (dU, the exit-state gradient of every chunk, dS_0); kda_bwd_tc.cu.
bool bwd_tc_available();
cudaError_t launch_bwd_chains_tc(const float* W, const float* Kb, const float* G, const float* S0,
                                 const float* dS_end, float* U_in_out, const float* E,
                                 const float* F, const int32_t* cu, int T, int N, int H,
                                 const int* chunk_start, uint32_t* status, float* states,
                                 float* dU, float* dSx, float* dS0, cudaStream_t st);
// E = P^T dO and F = Qt^T dO - W^T E, and the dense products after the back
// substitution (dQt, dKt, dKb, dGam, dbeta) on the tensor cores (dk = dv =
// 128); kda_bwd_tc.cu.
template <typename TIn>
cudaError_t launch_bwd_ef_tc(const TIn* q, const TIn* dout, const float* G, const float* P,
                             const float* W, const int4* info, int total, int maxc, int H,
                             uint32_t* status, float* E, float* F, cudaStream_t st);
template <typename TIn>
cudaError_t launch_bwd_dense_tc(const TIn* k, const TIn* dout, const float* G, const float* beta,
                                const float* U, const float* Y, const float* states,
                                const float* dSx, const float* dbB, const int4* info, int total,
                                int maxc, int H, uint32_t* status, float* dQt, float* dKt,
                                float* dKb, float* dGam, float* dbeta, cudaStream_t st);
// G, Kb, the right-hand sides b K exp(G), and A, P as a three-pass tf32
// product under a per-channel exponent reference (slow[] = 1: the chunk is
// left to the exact kernel); kda_bwd_tc.cu.
template <typename TIn>
cudaError_t launch_bwd_apkb_tc(const TIn* q, const TIn* k, const float* g, const float* beta,
                               const int4* info, int total, int maxc, int H, uint32_t* status,
                               int* slow, float* G, float* Ar, float* P, float* Kb, float* Rk,
                               cudaStream_t st);
// The two triangular solves through T = (I + A)^-1 (fp32, per chunk):
// [W | Ut] = T [b Kt | b V] (W holds b Kt on entry), then Y = T^T dU, dv,
// dA, dP and the partial dbeta, with the products in three tf32 passes;
// kda_bwd_tc.cu.
template <typename TIn>
cudaError_t launch_bwd_subst_tc(const TIn* v, const float* beta, const float* Ar,
                                const int4* info, int total, int maxc, int H, uint32_t* status,
                                float* W, float* Ut, float* Tm, cudaStream_t st);
template <typename TIn>
cudaError_t launch_bwd_solve_tc(const TIn* v, const TIn* dout, const float* Ar,
                                const float* beta, const float* U, const float* dU,
                                const float* Tm, const int4* info, int total, int maxc, int H,
                                uint32_t* status, float* Y, float* dv, float* dAr, float* dP,
                                float* dbB, cudaStream_t st);
// The pair sums (dq, dk, dg) as tensor-core products under a per-channel
// exponent reference; a chunk whose gate range exceeds it gets slow[] = 1 and
// is left to the exact CUDA-core kernel; kda_bwd_tc.cu.
template <typename TIn>
cudaError_t launch_bwd_pair_tc(const TIn* q, const TIn* k, const float* G, const float* dAr,
                               const float* dP, const float* dQt, const float* dKt,
                               const float* dKb, const float* dGam, const int4* info, int total,
                               int maxc, int H, uint32_t* status, int* slow, float* dq,
                               float* dk, float* dg, cudaStream_t st);
cudaError_t launch_bwd(const void* q, const void* k, const void* v, const float* g,
                       const float* beta, const float* h0, const void* dout, const float* dhT,
                       const int32_t* cu, int T, int N, int H, int dk, int dv, kda_dtype_t dt,
                       float* dq, float* dkk, float* dvv, float* dg, float* db, float* dh0,
                       void* workspace, cudaStream_t st);
// the backward with a head-uniform gate g [total, H]: spread over the channels,
// the per-channel backward, the channel gradients summed into dg_head [total, H]
size_t bwd_head_gate_workspace_bytes(int total, int N, int H, int dk, int dv);
cudaError_t launch_bwd_head_gate(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, const float* h0, const void* dout,
                                 const float* dhT, const int32_t* cu, int T, int N, int H, int dk,
                                 int dv, kda_dtype_t dt, float* dq, float* dkk, float* dvv,
                                 float* dg_head, float* db, float* dh0, void* workspace,
                                 cudaStream_t st);
// G_full[t, h, c] = g[t, h] (a head-uniform gate spread over dk channels)
cudaError_t launch_spread_gate(const float* g, int total, int H, int dk, float* out,
                               cudaStream_t st);
}  // namespace kda
