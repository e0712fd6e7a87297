// kda_chunk_fwd_noalloc: chunkwise prefill that allocates nothing and takes no
// workspace.
//
// Who needs it: callers that are handed only their input and output buffers
// and may not obtain device memory themselves -- for example an operator
// plugged into an inference engine or graph runtime whose interface has no
// workspace slot and whose memory planner owns all of the device's memory, or
// a serving loop that reserved nearly all HBM for its state pool up front, so
// that a cudaMalloc would fail, fragment that pool, or stall the other streams
// while the driver synchronises.  For them this file keeps the scratch that
// kda_chunk_fwd takes from its workspace (status word, chunk table and the
// CUDA-core path's intermediates) in one statically sized device array.
//
// Costs and rules:
//  * Every GPU on which this file's device module is loaded holds the array
//    (KDA_NOALLOC_SCRATCH_BYTES) until the process exits.  When the driver
//    loads that module is CUDA's choice: with lazy module loading (the
//    default of CUDA 12, CUDA_MODULE_LOADING=LAZY) it is the first
//    cudaGetSymbolAddress below, i.e. the first call of this entry point on
//    the device, so the 64 MiB are committed by that call; with eager loading
//    they are committed when the context is created.  A caller that reserves
//    nearly all HBM up front should therefore make its first call (on a tiny
//    problem, if need be) before taking that reservation.
//  * The first call on a device looks up the array's device address (one
//    cudaGetSymbolAddress with that device current) and caches it; make that
//    first call before any stream capture begins.
//  * All calls share the one array, which keeps the previous call's contents.
//    Everything a call reads is written earlier in the same call (the status
//    word is cleared on entry), so results never depend on an earlier call;
//    but two calls whose work overlaps on the GPU (different streams, no
//    ordering between them) race on the array.
//  * Problems whose scratch would exceed the array are rejected on the host
//    with KDA_ERR_WORKSPACE before anything is enqueued.
//  * No cudaMalloc, cudaFree or allocating library routine is called.
// It runs the same CUDA-core kernels as kda_chunk_fwd's CUDA-core path, for
// every dtype; device-side cu_seqlens errors make those kernels skip their work
// (o and final_state are then left unwritten) and, since the status word is
// inside the private array, are not reported -- callers who need that report
// use kda_chunk_fwd with kda_get_device_status.
#include <cuda_runtime.h>
#include <stdint.h>

#include <initializer_list>
#include <mutex>

#include "kda.h"
#include "kda_common.cuh"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name is only a host-side stand-in; the real address comes from
// cudaGetSymbolAddress, looked up once per device and cached.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" kda_status_t kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                              const float* g, const float* beta,
                                              const float* initial_state,
                                              const int32_t* cu_seqlens, int B, int T,
                                              int num_seqs, int H, int dk, int dv, int chunk,
                                              kda_dtype_t dtype, void* o, float* final_state,
                                              void* stream) {
    // --- the same argument rules as kda_chunk_fwd
    kda::Prefill pf;
    const kda_status_t chk =
        kda::check_prefill_shape(cu_seqlens, B, T, num_seqs, H, dk, dv, chunk, dtype, &pf);
    if (chk != KDA_OK) return chk;
    const int total = pf.total, N = pf.N;
    for (const void* p : {q, k, v, (const void*)g, (const void*)beta, (const void*)o})
        if (!p || !al16(p)) return KDA_ERR_INVALID_ARG;
    if ((initial_state && !al16(initial_state)) || (final_state && !al16(final_state)))
        return KDA_ERR_INVALID_ARG;
    // --- does the problem fit the static scratch?
    const kda::Workspace need = kda::carve(nullptr, total, N, H, dk, dv, chunk, true);
    if (need.total_bytes > (size_t)KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_WORKSPACE;
    // --- set-up (first call per device), then the CUDA-core launch sequence
    void* base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return KDA_ERR_CUDA;
    const kda::Workspace w = kda::carve(base, total, N, H, dk, dv, chunk, true);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int maxc = kda::max_chunks(total, N, chunk);
    kda_status_t r = kda::begin_prefill(w, cu_seqlens, B, T, N, chunk, maxc, st);
    if (r != KDA_OK) return r;
    if (total == 0 && !final_state) return KDA_OK;
    return kda::run_simt(q, k, v, g, beta, initial_state, cu_seqlens, B, T, pf, H, dk, dv, chunk,
                         dtype, o, final_state, w, maxc, st);
}
