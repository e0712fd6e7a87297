// Tensor-core (tcgen05 / TMEM / TMA) chunkwise prefill for bf16, dk = dv = 128,
// chunk = 64.  Internal to libkda.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// True when the tensor-core prefill kernels can run (the driver entry point
// that encodes TMA tensor maps is available).
bool tc_path_available();

// The steps around the operator fused into the split plan's kernels
// (kda_layer_chunk_fwd): the raw inputs (read by the tensor maps instead of
// q, k, v), their depthwise filters [H * 128, 4], the L2-norm epsilon; the
// output gate, the RMSNorm weights [128] and epsilon, and y (written instead
// of o).
struct LayerArgs {
    const void* xq;
    const void* xk;
    const void* xv;
    const float* wq;
    const float* wk;
    const float* wv;
    float l2_eps;
    const void* gate;
    const float* w_norm;
    float rms_eps;
    void* y;
};

// The chunkwise prefill as two tensor-core kernels: chunk-parallel
// intra-chunk kernel + per-chain kernel, handing over through `blobs`
// (split_blob_bytes() per (chunk slot, head)).
size_t split_blob_bytes();
// gh != NULL: the gate is head-uniform, gh [total, H] (g is then unused).
cudaError_t launch_chunk_fwd_split(const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, const float* h0,
                                   const int32_t* cu_seqlens, int T, int N, int H,
                                   const int4* chunk_info, int maxc, const int* chunk_start,
                                   uint32_t* status, void* blobs, void* o, float* hN,
                                   cudaStream_t st, const float* gh = nullptr,
                                   const int* seq_order = nullptr,
                                   const LayerArgs* layer = nullptr);
// Its two kernels one at a time (the chain kernel reads what the intra kernel
// wrote, on the same stream).
cudaError_t launch_split_intra(const void* q, const void* k, const float* g, const float* beta,
                               int total, int H, const int4* chunk_info, int maxc,
                               uint32_t* status, void* blobs, cudaStream_t st,
                               const float* gh = nullptr, const LayerArgs* layer = nullptr);
// seq_order (the chunk table's longest-first order of the sequences, or NULL):
// the order in which the chains are launched.
cudaError_t launch_split_chain(const void* v, const float* h0, const int32_t* cu_seqlens, int T,
                               int N, int H, const int* chunk_start, uint32_t* status,
                               const void* blobs, void* o, float* hN, cudaStream_t st,
                               const int* seq_order = nullptr,
                               const LayerArgs* layer = nullptr);
// The affine map of the prefill on the state, per (sequence, head): final
// state = M S_0 + Bm (M = the product of the chunk transitions, dk x dk; Bm =
// the final state from S_0 = 0): the intra-chunk kernel once, then the chain
// kernel twice without outputs -- from a zero state with V (Bm) and from the
// identity with V = 0 (M).
cudaError_t launch_split_state_maps(const void* q, const void* k, const void* v, const float* g,
                                    const float* beta, const int32_t* cu_seqlens, int T, int N,
                                    int H, const int4* chunk_info, int maxc,
                                    const int* chunk_start, uint32_t* status, void* blobs,
                                    float* M, float* Bm, cudaStream_t st,
                                    const int* seq_order = nullptr);
// The two kernels co-scheduled in one cooperative launch (chains wait for the
// blobs of their chunks through `flags`, one uint32 per (chunk slot, head)).
// withheld_flag >= 0 (testing the bounded-wait error path only): the flag of
// that (slot * H + head) is never released; flag_wait_ns != 0 bounds the
// chains' wait on one flag (default 2 s).
// gh != nullptr: the head-uniform gate [total, H] of Gated DeltaNet (g unused).
// overlap_grid() is its grid size, or 0 when the launch does not apply.
int overlap_grid(int N, int H);
cudaError_t launch_chunk_fwd_overlap(const void* q, const void* k, const void* v, const float* g,
                                     const float* beta, const float* h0,
                                     const int32_t* cu_seqlens, int T, int N, int H,
                                     const int4* chunk_info, int maxc, const int* chunk_start,
                                     uint32_t* status, void* blobs, uint32_t* flags, void* o,
                                     float* hN, cudaStream_t st, long long withheld_flag = -1,
                                     unsigned long long flag_wait_ns = 0,
                                     const float* gh = nullptr);

}  // namespace kda
