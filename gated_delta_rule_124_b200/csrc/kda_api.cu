// C ABI of libkda: argument validation, workspace layout and launch order.
// Everything here runs on the host and only enqueues work; see include/kda.h.
#include <cuda_runtime.h>
#include <stdint.h>

#include <stdlib.h>
#include <string.h>

#include <initializer_list>

#include "kda.h"
#include "kda_common.cuh"
#include "kda_chunk_tc.cuh"

namespace {

using kda::Workspace;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
bool dim_ok(int d) { return d == 32 || d == 64 || d == 128; }
bool chunk_ok(int c) { return c == 16 || c == 32 || c == 64; }
bool dtype_ok(kda_dtype_t t) { return t == KDA_DTYPE_F32 || t == KDA_DTYPE_BF16; }

}  // namespace

namespace kda {

kda_status_t check_prefill_shape(const int32_t* cu, int B, int T, int num_seqs, int H, int dk,
                                 int dv, int chunk, kda_dtype_t dt, Prefill* out) {
    if (B < 1 || T < 0 || num_seqs < 1 || H < 1) return KDA_ERR_INVALID_ARG;
    if (!dtype_ok(dt)) return KDA_ERR_INVALID_ARG;
    if (cu) {
        if (B != 1) return KDA_ERR_INVALID_ARG;
        if (!aligned16(cu)) return KDA_ERR_INVALID_ARG;
        out->total = T;
        out->N = num_seqs;
    } else {
        if (num_seqs != B) return KDA_ERR_INVALID_ARG;
        if ((long long)B * T > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
        out->total = B * T;
        out->N = B;
    }
    if (!dim_ok(dk) || !dim_ok(dv) || !chunk_ok(chunk)) return KDA_ERR_UNSUPPORTED;
    return KDA_OK;
}

kda_status_t begin_prefill(const Workspace& w, const int32_t* cu, int B, int T, int N, int chunk,
                           int maxc, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(w.status, 0, sizeof(uint32_t), st);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    e = launch_build_chunk_table(cu, B, T, N, chunk, maxc, w.status, w.chunk_start,
                                 w.chunk_info, st, w.seq_order);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status_t run_simt(const void* q, const void* k, const void* v, const float* g,
                      const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                      int B, int T, const Prefill& p, int H, int dk, int dv, int chunk,
                      kda_dtype_t dtype, void* o, float* final_state, const Workspace& w,
                      int maxc, cudaStream_t st) {
    cudaError_t e = launch_gate_cumsum(g, w.chunk_info, maxc, H, dk, w.status, w.G, st);
    if (e == cudaSuccess)
        e = launch_intra(k, v, w.G, beta, w.chunk_info, maxc, H, dk, dv, chunk, dtype, w.status,
                         w.W, w.U, st);
    if (e == cudaSuccess)
        e = launch_inter(k, w.G, w.W, w.U, initial_state, cu_seqlens, B, T, p.N, w.chunk_start,
                         H, dk, dv, chunk, dtype, w.status, w.states, final_state, st);
    if (e == cudaSuccess)
        e = launch_output(q, k, w.G, w.U, w.states, w.chunk_info, maxc, H, dk, dv, chunk, dtype,
                          w.status, o, st);
    return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace kda

namespace {

using kda::Prefill;
using kda::begin_prefill;
using kda::check_prefill_shape;
using kda::run_simt;

// Which kernels kda_chunk_fwd runs (the values of the KDA_PLAN_* constants).
enum class Path { Simt = KDA_PLAN_SIMT, Split = KDA_PLAN_SPLIT, Overlap = KDA_PLAN_OVERLAP };

bool tc_shape(int dk, int dv, int chunk, kda_dtype_t dt) {
    return dt == KDA_DTYPE_BF16 && dk == 128 && dv == 128 && chunk == 64 &&
           kda::tc_path_available();
}

// Whether co-scheduling the two split kernels pays: the chains get one SM per
// unit (2 N H SMs) and the intra-chunk items the rest, against the two kernels
// back to back on every SM.  Cost model in units of one chain step, from
// B200 measurements: an intra-chunk item costs about 4.8 chain steps of one
// unit, and two intra units share an SM.  Needs the chain length, so only
// when every sequence has the same length (B x T, or one packed sequence).
bool overlap_pays(long long items, long long rounds, long long NH, int sms) {
    const double rho = 4.8;
    const double intra_split = items * rho / (2.0 * sms);
    const double intra_ov = items * rho / (2.0 * (sms - 2 * NH));
    const double chain = static_cast<double>(rounds);
    return (intra_ov > chain ? intra_ov : chain) <= 0.85 * (intra_split + chain);
}

// Whether `path` can run a problem of these shapes on the current device.
bool path_applies(Path path, int N, int H, int dk, int dv, int chunk, kda_dtype_t dt) {
    switch (path) {
        case Path::Simt: return true;
        case Path::Split: return tc_shape(dk, dv, chunk, dt);
        case Path::Overlap: return tc_shape(dk, dv, chunk, dt) && kda::overlap_grid(N, H) > 0;
    }
    return false;
}

// The default plan, a function of the arguments and the device only: bf16,
// dk = dv = 128, chunk 64 runs on the tensor cores as the split plan -- the
// chunk-parallel intra-chunk kernel and the per-chain kernel -- co-scheduled
// in one launch on disjoint SMs where overlap_pays(), else as two launches;
// every other supported shape runs the CUDA-core plan.
Path select_path(int total, int N, bool packed, int H, int dk, int dv, int chunk,
                 kda_dtype_t dt) {
    if (!tc_shape(dk, dv, chunk, dt)) return Path::Simt;
    const int sms = kda::overlap_grid(N, H);
    if (sms == 0) return Path::Split;
    if (packed && N > 1) return Path::Split;
    const long long rounds = ((long long)total / N + chunk - 1) / chunk;
    const long long items = rounds * N * H;
    return overlap_pays(items, rounds, (long long)N * H, sms) ? Path::Overlap : Path::Split;
}

bool plan_from_int(int plan, Path* out) {
    switch (plan) {
        case KDA_PLAN_SIMT: *out = Path::Simt; return true;
        case KDA_PLAN_SPLIT: *out = Path::Split; return true;
        case KDA_PLAN_OVERLAP: *out = Path::Overlap; return true;
    }
    return false;
}

Workspace carve_for(void* base, const Prefill& p, int H, int dk, int dv, int chunk, Path path) {
    return kda::carve(base, p.total, p.N, H, dk, dv, chunk, path == Path::Simt,
                      (path == Path::Split || path == Path::Overlap) ? kda::split_blob_bytes()
                                                                     : 0);
}

size_t workspace_bytes_for(int total, int N, int H, int dk, int dv, int chunk, Path path) {
    const Prefill p{total, N};
    return carve_for(nullptr, p, H, dk, dv, chunk, path).total_bytes;
}

kda_status_t check_ws(void* ws, size_t bytes, const Prefill& p, int H, int dk, int dv,
                      int chunk, Path path, Workspace* out) {
    if (!ws) return KDA_ERR_WORKSPACE;
    if (!aligned256(ws)) return KDA_ERR_INVALID_ARG;
    Workspace w = carve_for(ws, p, H, dk, dv, chunk, path);
    if (bytes < w.total_bytes) return KDA_ERR_WORKSPACE;
    *out = w;
    return KDA_OK;
}

// The step calls keep only the status word and the chunk table in the
// workspace (their intermediates are the caller's buffers).
kda_status_t check_ws_header(void* ws, size_t bytes, const Prefill& p, int H, int dk, int dv,
                             int chunk, Workspace* out) {
    if (!ws) return KDA_ERR_WORKSPACE;
    if (!aligned256(ws)) return KDA_ERR_INVALID_ARG;
    Workspace w = kda::carve(ws, p.total, p.N, H, dk, dv, chunk, false);
    if (bytes < w.total_bytes) return KDA_ERR_WORKSPACE;
    *out = w;
    return KDA_OK;
}

kda_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

// Gated DeltaNet (head-uniform gate): the split plan reads the gate per
// (token, head) directly; every other shape spreads it over the dk channels
// into the workspace, after the CUDA-core plan's own part, and runs that plan.
// Gated DeltaNet takes the plans of KDA by the same rule (its intra-chunk
// kernel is the head-gate variant of the same kernel).
Path gdn_path(int total, int N, bool packed, int H, int dk, int dv, int chunk, kda_dtype_t dt) {
    return select_path(total, N, packed, H, dk, dv, chunk, dt);
}

size_t gdn_workspace_bytes(const Prefill& p, int H, int dk, int dv, int chunk, Path path,
                           size_t* spread_offset) {
    const size_t base = carve_for(nullptr, p, H, dk, dv, chunk, path).total_bytes;
    *spread_offset = base;
    if (path != Path::Simt) return base;
    return kda::align_up(base + sizeof(float) * (size_t)p.total * H * dk);
}

}  // namespace

extern "C" {

const char* kda_status_string(kda_status_t s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: invalid argument";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: shape or dtype not supported";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA: CUDA runtime error";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a bounded device-side wait gave up";
        case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing or too small";
        case KDA_ERR_BAD_SEQLENS:
            return "KDA_ERR_BAD_SEQLENS: cu_seqlens is not 0..T non-decreasing";
    }
    return "KDA_ERR_UNKNOWN";
}

int kda_num_chunks_upper_bound(int total_tokens, int num_seqs, int chunk) {
    if (total_tokens < 0 || num_seqs < 1 || chunk < 1) return 0;
    return kda::max_chunks(total_tokens, num_seqs, chunk);
}

int kda_chunk_fwd_plan(int total_tokens, int num_seqs, int packed, int H, int dk, int dv,
                       int chunk, kda_dtype_t dtype) {
    if (total_tokens < 0 || num_seqs < 1 || H < 1 || !dim_ok(dk) || !dim_ok(dv) ||
        !chunk_ok(chunk) || !dtype_ok(dtype))
        return -1;
    return static_cast<int>(
        select_path(total_tokens, num_seqs, packed != 0, H, dk, dv, chunk, dtype));
}

size_t kda_chunk_fwd_workspace_size(int total_tokens, int num_seqs, int H, int dk, int dv,
                                    int chunk, kda_dtype_t dtype) {
    if (total_tokens < 0 || num_seqs < 1 || H < 1 || !dim_ok(dk) || !dim_ok(dv) ||
        !chunk_ok(chunk) || !dtype_ok(dtype))
        return 0;
    // the split and co-scheduled plans share one layout, so packing does not matter
    return workspace_bytes_for(total_tokens, num_seqs, H, dk, dv, chunk,
                               select_path(total_tokens, num_seqs, false, H, dk, dv, chunk,
                                           dtype));
}

size_t kda_chunk_fwd_plan_workspace_size(int plan, int total_tokens, int num_seqs, int H, int dk,
                                         int dv, int chunk, kda_dtype_t dtype) {
    Path path;
    if (!plan_from_int(plan, &path) || total_tokens < 0 || num_seqs < 1 || H < 1 ||
        !dim_ok(dk) || !dim_ok(dv) || !chunk_ok(chunk) || !dtype_ok(dtype) ||
        !path_applies(path, num_seqs, H, dk, dv, chunk, dtype))
        return 0;
    return workspace_bytes_for(total_tokens, num_seqs, H, dk, dv, chunk, path);
}

}  // extern "C"

namespace {

// kda_chunk_fwd's body on a given plan (checked to apply).
kda_status_t chunk_fwd_on(Path path, const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* initial_state,
                          const int32_t* cu_seqlens, int B, int T, const Prefill& p, int H,
                          int dk, int dv, int chunk, kda_dtype_t dtype, void* o,
                          float* final_state, void* workspace, size_t workspace_bytes,
                          void* stream) {
    if (!q || !k || !v || !g || !beta || !o) return KDA_ERR_INVALID_ARG;
    for (const void* ptr : {q, k, v, (const void*)g, (const void*)beta, (const void*)o})
        if (!aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
        return KDA_ERR_INVALID_ARG;
    Workspace w;
    kda_status_t s = check_ws(workspace, workspace_bytes, p, H, dk, dv, chunk, path, &w);
    if (s != KDA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int maxc = kda::max_chunks(p.total, p.N, chunk);
    s = begin_prefill(w, cu_seqlens, B, T, p.N, chunk, maxc, st);
    if (s != KDA_OK) return s;
    if (p.total == 0 && !final_state) return KDA_OK;
    if (path == Path::Overlap) {
        return from_cuda(kda::launch_chunk_fwd_overlap(q, k, v, g, beta, initial_state,
                                                       cu_seqlens, T, p.N, H, w.chunk_info,
                                                       maxc, w.chunk_start, w.status, w.blobs,
                                                       w.flags, o, final_state, st));
    }
    if (path == Path::Split) {
        return from_cuda(kda::launch_chunk_fwd_split(q, k, v, g, beta, initial_state,
                                                     cu_seqlens, T, p.N, H, w.chunk_info, maxc,
                                                     w.chunk_start, w.status, w.blobs, o,
                                                     final_state, st, nullptr, w.seq_order));
    }
    return run_simt(q, k, v, g, beta, initial_state, cu_seqlens, B, T, p, H, dk, dv, chunk,
                    dtype, o, final_state, w, maxc, st);
}

}  // namespace

extern "C" {

kda_status_t kda_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, const float* initial_state,
                           const int32_t* cu_seqlens, int B, int T, int num_seqs, int H,
                           int dk, int dv, int chunk, kda_dtype_t dtype, void* o,
                           float* final_state, void* workspace, size_t workspace_bytes,
                           void* stream) {
    Prefill p;
    kda_status_t s =
        check_prefill_shape(cu_seqlens, B, T, num_seqs, H, dk, dv, chunk, dtype, &p);
    if (s != KDA_OK) return s;
    const Path path = select_path(p.total, p.N, cu_seqlens != nullptr, H, dk, dv, chunk, dtype);
    return chunk_fwd_on(path, q, k, v, g, beta, initial_state, cu_seqlens, B, T, p, H, dk, dv,
                        chunk, dtype, o, final_state, workspace, workspace_bytes, stream);
}

kda_status_t kda_chunk_fwd_with_plan(int plan, const void* q, const void* k, const void* v,
                                     const float* g, const float* beta,
                                     const float* initial_state, const int32_t* cu_seqlens, int B,
                                     int T, int num_seqs, int H, int dk, int dv, int chunk,
                                     kda_dtype_t dtype, void* o, float* final_state,
                                     void* workspace, size_t workspace_bytes, void* stream) {
    Path path;
    if (!plan_from_int(plan, &path)) return KDA_ERR_INVALID_ARG;
    Prefill p;
    kda_status_t s =
        check_prefill_shape(cu_seqlens, B, T, num_seqs, H, dk, dv, chunk, dtype, &p);
    if (s != KDA_OK) return s;
    if (!path_applies(path, p.N, H, dk, dv, chunk, dtype)) return KDA_ERR_UNSUPPORTED;
    return chunk_fwd_on(path, q, k, v, g, beta, initial_state, cu_seqlens, B, T, p, H, dk, dv,
                        chunk, dtype, o, final_state, workspace, workspace_bytes, stream);
}

}  // extern "C"

namespace {
// kda_layer_chunk_fwd's workspace: the plan's own, then (composed path only)
// q, k, v and o in the input dtype.
size_t layer_workspace_bytes(const Prefill& p, int H, int dk, int dv, int chunk,
                             kda_dtype_t dt, Path path, size_t* extra_off) {
    const size_t base = carve_for(nullptr, p, H, dk, dv, chunk, path).total_bytes;
    *extra_off = kda::align_up(base);
    if (path != Path::Simt) return base;
    const size_t es = dt == KDA_DTYPE_BF16 ? 2 : 4;
    return kda::align_up(*extra_off + es * (size_t)p.total * H * (2 * dk + 2 * dv));
}
}  // namespace

extern "C" {

size_t kda_layer_chunk_fwd_workspace_size(int total_tokens, int num_seqs, int H, int dk, int dv,
                                          int chunk, kda_dtype_t dtype) {
    if (total_tokens < 0 || num_seqs < 1 || H < 1 || !dim_ok(dk) || !dim_ok(dv) ||
        !chunk_ok(chunk) || !dtype_ok(dtype))
        return 0;
    const Prefill p{total_tokens, num_seqs};
    size_t off;
    return layer_workspace_bytes(p, H, dk, dv, chunk, dtype,
                                 tc_shape(dk, dv, chunk, dtype) ? Path::Split : Path::Simt, &off);
}

kda_status_t kda_layer_chunk_fwd(const void* xq, const void* xk, const void* xv, const float* wq,
                                 const float* wk, const float* wv, const float* g,
                                 const float* beta, const float* initial_state,
                                 const int32_t* cu_seqlens, int B, int T, int num_seqs, int H,
                                 int dk, int dv, int chunk, kda_dtype_t dtype, const void* gate,
                                 const float* w_norm, float l2_eps, float rms_eps, void* y,
                                 float* final_state, void* workspace, size_t workspace_bytes,
                                 void* stream) {
    Prefill p;
    kda_status_t s =
        check_prefill_shape(cu_seqlens, B, T, num_seqs, H, dk, dv, chunk, dtype, &p);
    if (s != KDA_OK) return s;
    if (!(l2_eps > 0.f) || !(l2_eps < 1e30f) || !(rms_eps > 0.f) || !(rms_eps < 1e30f))
        return KDA_ERR_INVALID_ARG;
    for (const void* ptr : std::initializer_list<const void*>{
             xq, xk, xv, (const void*)wq, (const void*)wk, (const void*)wv, (const void*)g,
             (const void*)beta, gate, (const void*)w_norm, y})
        if (!ptr || !aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
        return KDA_ERR_INVALID_ARG;
    const Path path = tc_shape(dk, dv, chunk, dtype) ? Path::Split : Path::Simt;
    size_t extra = 0;
    const size_t need = layer_workspace_bytes(p, H, dk, dv, chunk, dtype, path, &extra);
    if (!workspace) return KDA_ERR_WORKSPACE;
    if (!aligned256(workspace)) return KDA_ERR_INVALID_ARG;
    if (workspace_bytes < need) return KDA_ERR_WORKSPACE;
    const Workspace w = carve_for(workspace, p, H, dk, dv, chunk, path);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int maxc = kda::max_chunks(p.total, p.N, chunk);
    s = begin_prefill(w, cu_seqlens, B, T, p.N, chunk, maxc, st);
    if (s != KDA_OK) return s;
    if (p.total == 0 && !final_state) return KDA_OK;
    if (path == Path::Split) {
        const kda::LayerArgs la{xq, xk, xv, wq, wk, wv, l2_eps, gate, w_norm, rms_eps, y};
        return from_cuda(kda::launch_chunk_fwd_split(nullptr, nullptr, nullptr, g, beta,
                                                     initial_state, cu_seqlens, T, p.N, H,
                                                     w.chunk_info, maxc, w.chunk_start, w.status,
                                                     w.blobs, nullptr, final_state, st, nullptr,
                                                     w.seq_order, &la));
    }
    // every other shape: the three steps one after another, q, k, v and o in
    // the workspace
    const size_t es = dtype == KDA_DTYPE_BF16 ? 2 : 4;
    char* base = static_cast<char*>(workspace) + extra;
    void* q = base;
    void* k = base + es * (size_t)p.total * H * dk;
    void* v = base + es * (size_t)p.total * H * 2 * dk;
    void* o = base + es * (size_t)p.total * H * (2 * dk + dv);
    const void* const x3[3] = {xq, xk, xv};
    const float* const w3[3] = {wq, wk, wv};
    void* const y3[3] = {q, k, v};
    cudaError_t e = kda::launch_qkv_conv(x3, w3, y3, dk, dv, cu_seqlens, p.N, cu_seqlens ? 0 : T,
                                         p.total, H, l2_eps, dtype, st);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    s = run_simt(q, k, v, g, beta, initial_state, cu_seqlens, B, T, p, H, dk, dv, chunk, dtype, o,
                 final_state, w, maxc, st);
    if (s != KDA_OK) return s;
    return from_cuda(kda::launch_norm_gate(o, gate, w_norm, p.total, H, dv, rms_eps, dtype, y, st));
}

kda_status_t kda_test_overlap_flag_timeout(const void* q, const void* k, const void* v,
                                           const float* g, const float* beta,
                                           const float* initial_state,
                                           const int32_t* cu_seqlens, int B, int T,
                                           int num_seqs, int H, void* o, float* final_state,
                                           void* workspace, size_t workspace_bytes,
                                           int withheld_chunk, int withheld_head,
                                           unsigned long long flag_wait_ns, void* stream) {
    Prefill p;
    kda_status_t s = check_prefill_shape(cu_seqlens, B, T, num_seqs, H, 128, 128, 64,
                                         KDA_DTYPE_BF16, &p);
    if (s != KDA_OK) return s;
    if (!path_applies(Path::Overlap, p.N, H, 128, 128, 64, KDA_DTYPE_BF16))
        return KDA_ERR_UNSUPPORTED;
    const int maxc = kda::max_chunks(p.total, p.N, 64);
    if (withheld_chunk < 0 || withheld_chunk >= maxc || withheld_head < 0 ||
        withheld_head >= H || flag_wait_ns == 0 || flag_wait_ns > 2000000000ull)
        return KDA_ERR_INVALID_ARG;
    for (const void* ptr : {q, k, v, (const void*)g, (const void*)beta, (const void*)o})
        if (!ptr || !aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
        return KDA_ERR_INVALID_ARG;
    Workspace w;
    s = check_ws(workspace, workspace_bytes, p, H, 128, 128, 64, Path::Overlap, &w);
    if (s != KDA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    s = begin_prefill(w, cu_seqlens, B, T, p.N, 64, maxc, st);
    if (s != KDA_OK) return s;
    if (p.total == 0) return KDA_OK;
    return from_cuda(kda::launch_chunk_fwd_overlap(
        q, k, v, g, beta, initial_state, cu_seqlens, T, p.N, H, w.chunk_info, maxc,
        w.chunk_start, w.status, w.blobs, w.flags, o, final_state, st,
        (long long)withheld_chunk * H + withheld_head, flag_wait_ns));
}

// ------------------------------------------------- one step per call (a1-a4)

#define KDA_PREFILL_PROLOGUE(...)                                                   \
    Prefill p;                                                                            \
    kda_status_t s =                                                                      \
        check_prefill_shape(cu_seqlens, B, T, num_seqs, H, dk, dv, chunk, dtype, &p);     \
    if (s != KDA_OK) return s;                                                            \
    for (const void* ptr : std::initializer_list<const void*>{__VA_ARGS__})              \
        if (!ptr || !aligned16(ptr)) return KDA_ERR_INVALID_ARG;                          \
    Workspace w;                                                                          \
    s = check_ws_header(workspace, workspace_bytes, p, H, dk, dv, chunk, &w);          \
    if (s != KDA_OK) return s;                                                            \
    cudaStream_t st = static_cast<cudaStream_t>(stream);                                  \
    const int maxc = kda::max_chunks(p.total, p.N, chunk);

// First enqueue of a step call; every argument check must come before it.
#define KDA_PREFILL_BEGIN()                                                               \
    s = begin_prefill(w, cu_seqlens, B, T, p.N, chunk, maxc, st);                         \
    if (s != KDA_OK) return s;

kda_status_t kda_chunk_gate_cumsum(const float* g, const int32_t* cu_seqlens, int B, int T,
                                   int num_seqs, int H, int dk, int chunk, float* G,
                                   void* workspace, size_t workspace_bytes, void* stream) {
    const int dv = dk;
    const kda_dtype_t dtype = KDA_DTYPE_F32;
    KDA_PREFILL_PROLOGUE((const void*)g, (const void*)G)
    KDA_PREFILL_BEGIN()
    return from_cuda(kda::launch_gate_cumsum(g, w.chunk_info, maxc, H, dk, w.status, G, st));
}

kda_status_t kda_chunk_intra(const void* k, const void* v, const float* G, const float* beta,
                             const int32_t* cu_seqlens, int B, int T, int num_seqs, int H,
                             int dk, int dv, int chunk, kda_dtype_t dtype, float* W, float* Ut,
                             void* workspace, size_t workspace_bytes, void* stream) {
    KDA_PREFILL_PROLOGUE(k, v, (const void*)G, (const void*)beta, (const void*)W,
                         (const void*)Ut)
    KDA_PREFILL_BEGIN()
    return from_cuda(kda::launch_intra(k, v, G, beta, w.chunk_info, maxc, H, dk, dv, chunk,
                                       dtype, w.status, W, Ut, st));
}

kda_status_t kda_chunk_inter(const void* k, const float* G, const float* W, float* U,
                             const float* initial_state, const int32_t* cu_seqlens, int B,
                             int T, int num_seqs, int H, int dk, int dv, int chunk,
                             kda_dtype_t dtype, float* chunk_states, float* final_state,
                             void* workspace, size_t workspace_bytes, void* stream) {
    KDA_PREFILL_PROLOGUE(k, (const void*)G, (const void*)W, (const void*)U,
                         (const void*)chunk_states)
    if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
        return KDA_ERR_INVALID_ARG;
    KDA_PREFILL_BEGIN()
    return from_cuda(kda::launch_inter(k, G, W, U, initial_state, cu_seqlens, B, T, p.N,
                                       w.chunk_start, H, dk, dv, chunk, dtype, w.status,
                                       chunk_states, final_state, st));
}

kda_status_t kda_chunk_output(const void* q, const void* k, const float* G, const float* U,
                              const float* chunk_states, const int32_t* cu_seqlens, int B,
                              int T, int num_seqs, int H, int dk, int dv, int chunk,
                              kda_dtype_t dtype, void* o, void* workspace,
                              size_t workspace_bytes, void* stream) {
    KDA_PREFILL_PROLOGUE(q, k, (const void*)G, (const void*)U, (const void*)chunk_states,
                         (const void*)o)
    KDA_PREFILL_BEGIN()
    return from_cuda(kda::launch_output(q, k, G, U, chunk_states, w.chunk_info, maxc, H, dk, dv,
                                        chunk, dtype, w.status, o, st));
}

#undef KDA_PREFILL_PROLOGUE
#undef KDA_PREFILL_BEGIN

// ------------------------------- tensor-core split path, one kernel per call

namespace {
constexpr int kTcD = 128, kTcC = 64;

kda_status_t split_prologue(const int32_t* cu_seqlens, int B, int T, int num_seqs, int H,
                            std::initializer_list<const void*> ptrs, void* workspace,
                            size_t workspace_bytes, Prefill* p, Workspace* w) {
    kda_status_t s = check_prefill_shape(cu_seqlens, B, T, num_seqs, H, kTcD, kTcD, kTcC,
                                         KDA_DTYPE_BF16, p);
    if (s != KDA_OK) return s;
    for (const void* ptr : ptrs)
        if (!ptr || !aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    if (!kda::tc_path_available()) return KDA_ERR_UNSUPPORTED;
    return check_ws(workspace, workspace_bytes, *p, H, kTcD, kTcD, kTcC, Path::Split, w);
}
}  // namespace

size_t kda_chunk_split_workspace_size(int total_tokens, int num_seqs, int H) {
    if (total_tokens < 0 || num_seqs < 1 || H < 1) return 0;
    const Prefill p{total_tokens, num_seqs};
    return carve_for(nullptr, p, H, kTcD, kTcD, kTcC, Path::Split).total_bytes;
}

kda_status_t kda_chunk_split_intra(const void* q, const void* k, const float* g,
                                   const float* beta, const int32_t* cu_seqlens, int B, int T,
                                   int num_seqs, int H, void* workspace, size_t workspace_bytes,
                                   void* stream) {
    Prefill p;
    Workspace w;
    kda_status_t s = split_prologue(cu_seqlens, B, T, num_seqs, H,
                                    {q, k, (const void*)g, (const void*)beta}, workspace,
                                    workspace_bytes, &p, &w);
    if (s != KDA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int maxc = kda::max_chunks(p.total, p.N, kTcC);
    s = begin_prefill(w, cu_seqlens, B, T, p.N, kTcC, maxc, st);
    if (s != KDA_OK) return s;
    return from_cuda(kda::launch_split_intra(q, k, g, beta, p.total, H, w.chunk_info, maxc,
                                             w.status, w.blobs, st));
}

kda_status_t kda_chunk_split_chain(const void* v, const float* initial_state,
                                   const int32_t* cu_seqlens, int B, int T, int num_seqs, int H,
                                   void* o, float* final_state, void* workspace,
                                   size_t workspace_bytes, void* stream) {
    Prefill p;
    Workspace w;
    kda_status_t s = split_prologue(cu_seqlens, B, T, num_seqs, H, {v, (const void*)o},
                                    workspace, workspace_bytes, &p, &w);
    if (s != KDA_OK) return s;
    if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
        return KDA_ERR_INVALID_ARG;
    return from_cuda(kda::launch_split_chain(v, initial_state, cu_seqlens, T, p.N, H,
                                             w.chunk_start, w.status, w.blobs, o, final_state,
                                             static_cast<cudaStream_t>(stream), w.seq_order));
}

// ------------------------------------------- state maps of a prefill (CP)

kda_status_t kda_chunk_state_maps(const void* q, const void* k, const void* v, const float* g,
                                  const float* beta, const int32_t* cu_seqlens, int B, int T,
                                  int num_seqs, int H, float* M, float* Bm, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    Prefill p;
    Workspace w;
    kda_status_t s = split_prologue(cu_seqlens, B, T, num_seqs, H,
                                    {q, k, v, (const void*)g, (const void*)beta, (const void*)M,
                                     (const void*)Bm},
                                    workspace, workspace_bytes, &p, &w);
    if (s != KDA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int maxc = kda::max_chunks(p.total, p.N, kTcC);
    s = begin_prefill(w, cu_seqlens, B, T, p.N, kTcC, maxc, st);
    if (s != KDA_OK) return s;
    return from_cuda(kda::launch_split_state_maps(q, k, v, g, beta, cu_seqlens, T, p.N, H,
                                                  w.chunk_info, maxc, w.chunk_start, w.status,
                                                  w.blobs, M, Bm, st, w.seq_order));
}

kda_status_t kda_fold_segment_states(const float* M, const float* Bm, const float* S0, int R,
                                     int N, int H, int dk, int dv, int reverse, float* each,
                                     float* final_state, void* stream) {
    if (R < 0 || N < 0 || H < 1) return KDA_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    if (!final_state || !aligned16(final_state) || (S0 && !aligned16(S0))) return KDA_ERR_INVALID_ARG;
    if (R > 0)
        for (const void* ptr : {(const void*)M, (const void*)Bm, (const void*)each})
            if (!ptr || !aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    return from_cuda(kda::launch_fold_segments(M, Bm, S0, R, N * H, dk, dv, reverse != 0, each,
                                               final_state, static_cast<cudaStream_t>(stream)));
}

// ----------------------------------------------------------------- decode

kda_status_t kda_decode_step(const void* q, const void* k, const void* v, const float* g,
                             const float* beta, float* state, void* o, int N, int H, int dk,
                             int dv, kda_dtype_t dtype, void* stream) {
    if (N < 0 || H < 1 || !dtype_ok(dtype)) return KDA_ERR_INVALID_ARG;
    if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (N == 0) return KDA_OK;
    for (const void* ptr : {q, k, v, (const void*)g, (const void*)beta, (const void*)state,
                            (const void*)o})
        if (!ptr || !aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    return from_cuda(kda::launch_decode(q, k, v, g, beta, state, o, N, H, dk, dv, dtype,
                                        static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------- Gated DeltaNet (head-uniform gate)

size_t kda_gdn_chunk_fwd_workspace_size(int total_tokens, int num_seqs, int H, int dk, int dv,
                                        int chunk, kda_dtype_t dtype) {
    if (total_tokens < 0 || num_seqs < 1 || H < 1 || !dim_ok(dk) || !dim_ok(dv) ||
        !chunk_ok(chunk) || !dtype_ok(dtype))
        return 0;
    const Prefill p{total_tokens, num_seqs};
    size_t off;
    return gdn_workspace_bytes(p, H, dk, dv, chunk,
                               gdn_path(p.total, p.N, false, H, dk, dv, chunk, dtype), &off);
}

kda_status_t kda_gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, const float* initial_state,
                               const int32_t* cu_seqlens, int B, int T, int num_seqs, int H,
                               int dk, int dv, int chunk, kda_dtype_t dtype, void* o,
                               float* final_state, void* workspace, size_t workspace_bytes,
                               void* stream) {
    Prefill p;
    kda_status_t s =
        check_prefill_shape(cu_seqlens, B, T, num_seqs, H, dk, dv, chunk, dtype, &p);
    if (s != KDA_OK) return s;
    if (!q || !k || !v || !g || !beta || !o) return KDA_ERR_INVALID_ARG;
    for (const void* ptr : {q, k, v, (const void*)g, (const void*)beta, (const void*)o})
        if (!aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
        return KDA_ERR_INVALID_ARG;
    const Path path = gdn_path(p.total, p.N, cu_seqlens != nullptr, H, dk, dv, chunk, dtype);
    size_t spread_off = 0;
    const size_t need = gdn_workspace_bytes(p, H, dk, dv, chunk, path, &spread_off);
    if (!workspace) return KDA_ERR_WORKSPACE;
    if (!aligned256(workspace)) return KDA_ERR_INVALID_ARG;
    if (workspace_bytes < need) return KDA_ERR_WORKSPACE;
    const Workspace w = carve_for(workspace, p, H, dk, dv, chunk, path);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int maxc = kda::max_chunks(p.total, p.N, chunk);
    s = begin_prefill(w, cu_seqlens, B, T, p.N, chunk, maxc, st);
    if (s != KDA_OK) return s;
    if (p.total == 0 && !final_state) return KDA_OK;
    if (path == Path::Overlap)
        return from_cuda(kda::launch_chunk_fwd_overlap(q, k, v, nullptr, beta, initial_state,
                                                       cu_seqlens, T, p.N, H, w.chunk_info,
                                                       maxc, w.chunk_start, w.status, w.blobs,
                                                       w.flags, o, final_state, st, -1, 0, g));
    if (path == Path::Split)
        return from_cuda(kda::launch_chunk_fwd_split(q, k, v, nullptr, beta, initial_state,
                                                     cu_seqlens, T, p.N, H, w.chunk_info, maxc,
                                                     w.chunk_start, w.status, w.blobs, o,
                                                     final_state, st, g, w.seq_order));
    float* gfull = reinterpret_cast<float*>(static_cast<char*>(workspace) + spread_off);
    const cudaError_t e = kda::launch_spread_gate(g, p.total, H, dk, gfull, st);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    return run_simt(q, k, v, gfull, beta, initial_state, cu_seqlens, B, T, p, H, dk, dv, chunk,
                    dtype, o, final_state, w, maxc, st);
}

kda_status_t kda_gdn_decode_step(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, float* state, void* o, int N, int H, int dk,
                                 int dv, kda_dtype_t dtype, void* stream) {
    if (N < 0 || H < 1 || !dtype_ok(dtype)) return KDA_ERR_INVALID_ARG;
    if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (N == 0) return KDA_OK;
    for (const void* ptr : {q, k, v, (const void*)g, (const void*)beta, (const void*)state,
                            (const void*)o})
        if (!ptr || !aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    return from_cuda(kda::launch_decode(q, k, v, g, beta, state, o, N, H, dk, dv, dtype,
                                        static_cast<cudaStream_t>(stream), true));
}

// ------------------------------------------------------------- backward

size_t kda_chunk_bwd_workspace_size(int total_tokens, int num_seqs, int H, int dk, int dv) {
    if (total_tokens < 0 || num_seqs < 1 || H < 1 || !dim_ok(dk) || !dim_ok(dv)) return 0;
    return kda::bwd_workspace_bytes(total_tokens, num_seqs, H, dk, dv);
}

kda_status_t kda_chunk_bwd(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, const float* initial_state, const void* dout,
                           const float* dfinal_state, const int32_t* cu_seqlens, int B, int T,
                           int num_seqs, int H, int dk, int dv, kda_dtype_t dtype, float* dq,
                           float* dk_out, float* dv_out, float* dg, float* dbeta,
                           float* dinitial_state, void* workspace, size_t workspace_bytes,
                           void* stream) {
    Prefill p;
    kda_status_t s = check_prefill_shape(cu_seqlens, B, T, num_seqs, H, dk, dv, 64, dtype, &p);
    if (s != KDA_OK) return s;
    for (const void* ptr : std::initializer_list<const void*>{
             q, k, v, (const void*)g, (const void*)beta, dout, (const void*)dq,
             (const void*)dk_out, (const void*)dv_out, (const void*)dg, (const void*)dbeta})
        if (!ptr || !aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    for (const void* ptr : std::initializer_list<const void*>{
             (const void*)initial_state, (const void*)dfinal_state, (const void*)dinitial_state})
        if (ptr && !aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    if (!workspace) return KDA_ERR_WORKSPACE;
    if (!aligned256(workspace)) return KDA_ERR_INVALID_ARG;
    if (workspace_bytes < kda::bwd_workspace_bytes(p.total, p.N, H, dk, dv))
        return KDA_ERR_WORKSPACE;
    return from_cuda(kda::launch_bwd(q, k, v, g, beta, initial_state, dout, dfinal_state,
                                     cu_seqlens, T, p.N, H, dk, dv, dtype, dq, dk_out, dv_out, dg,
                                     dbeta, dinitial_state, workspace,
                                     static_cast<cudaStream_t>(stream)));
}

size_t kda_gdn_chunk_bwd_workspace_size(int total_tokens, int num_seqs, int H, int dk, int dv) {
    if (total_tokens < 0 || num_seqs < 1 || H < 1 || !dim_ok(dk) || !dim_ok(dv)) return 0;
    return kda::bwd_head_gate_workspace_bytes(total_tokens, num_seqs, H, dk, dv);
}

kda_status_t kda_gdn_chunk_bwd(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, const float* initial_state, const void* dout,
                               const float* dfinal_state, const int32_t* cu_seqlens, int B, int T,
                               int num_seqs, int H, int dk, int dv, kda_dtype_t dtype, float* dq,
                               float* dk_out, float* dv_out, float* dg, float* dbeta,
                               float* dinitial_state, void* workspace, size_t workspace_bytes,
                               void* stream) {
    Prefill p;
    kda_status_t s = check_prefill_shape(cu_seqlens, B, T, num_seqs, H, dk, dv, 64, dtype, &p);
    if (s != KDA_OK) return s;
    for (const void* ptr : std::initializer_list<const void*>{
             q, k, v, (const void*)g, (const void*)beta, dout, (const void*)dq,
             (const void*)dk_out, (const void*)dv_out, (const void*)dg, (const void*)dbeta})
        if (!ptr || !aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    for (const void* ptr : std::initializer_list<const void*>{
             (const void*)initial_state, (const void*)dfinal_state, (const void*)dinitial_state})
        if (ptr && !aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    if (!workspace) return KDA_ERR_WORKSPACE;
    if (!aligned256(workspace)) return KDA_ERR_INVALID_ARG;
    if (workspace_bytes < kda::bwd_head_gate_workspace_bytes(p.total, p.N, H, dk, dv))
        return KDA_ERR_WORKSPACE;
    return from_cuda(kda::launch_bwd_head_gate(
        q, k, v, g, beta, initial_state, dout, dfinal_state, cu_seqlens, T, p.N, H, dk, dv, dtype,
        dq, dk_out, dv_out, dg, dbeta, dinitial_state, workspace,
        static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------ layer steps (NEXT-2)

kda_status_t kda_qkv_conv_norm(const void* xq, const void* xk, const void* xv, const float* wq,
                               const float* wk, const float* wv, const int32_t* cu_seqlens,
                               int B, int T, int num_seqs, int H, int dk, int dv,
                               kda_dtype_t dtype, float eps, void* q, void* k, void* v,
                               void* stream) {
    Prefill p;
    kda_status_t s = check_prefill_shape(cu_seqlens, B, T, num_seqs, H, dk, dv, 64, dtype, &p);
    if (s != KDA_OK) return s;
    if (!(eps > 0.f) || !(eps < 1e30f)) return KDA_ERR_INVALID_ARG;
    for (const void* ptr : std::initializer_list<const void*>{
             xq, xk, xv, (const void*)wq, (const void*)wk, (const void*)wv, q, k, v})
        if (!ptr || !aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    const void* const x[3] = {xq, xk, xv};
    const float* const w[3] = {wq, wk, wv};
    void* const y[3] = {q, k, v};
    return from_cuda(kda::launch_qkv_conv(x, w, y, dk, dv, cu_seqlens, p.N,
                                          cu_seqlens ? 0 : T, p.total, H, eps, dtype,
                                          static_cast<cudaStream_t>(stream)));
}

kda_status_t kda_qkv_conv_norm_step(const void* xq, const void* xk, const void* xv,
                                    const float* wq, const float* wk, const float* wv,
                                    void* conv_q, void* conv_k, void* conv_v, int N, int H,
                                    int dk, int dv, kda_dtype_t dtype, float eps, void* q,
                                    void* k, void* v, void* stream) {
    if (N < 0 || H < 1 || !dtype_ok(dtype)) return KDA_ERR_INVALID_ARG;
    if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (!(eps > 0.f) || !(eps < 1e30f)) return KDA_ERR_INVALID_ARG;
    if (N == 0) return KDA_OK;
    for (const void* ptr : std::initializer_list<const void*>{
             xq, xk, xv, (const void*)wq, (const void*)wk, (const void*)wv, conv_q, conv_k,
             conv_v, q, k, v})
        if (!ptr || !aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    const void* const x[3] = {xq, xk, xv};
    const float* const w[3] = {wq, wk, wv};
    void* const state[3] = {conv_q, conv_k, conv_v};
    void* const y[3] = {q, k, v};
    return from_cuda(kda::launch_qkv_conv_step(x, w, state, y, dk, dv, N, H, eps, dtype,
                                               static_cast<cudaStream_t>(stream)));
}

kda_status_t kda_output_norm_gate(const void* o, const void* gate, const float* w,
                                  int total_tokens, int H, int dv, kda_dtype_t dtype, float eps,
                                  void* y, void* stream) {
    if (total_tokens < 0 || H < 1 || !dtype_ok(dtype)) return KDA_ERR_INVALID_ARG;
    if ((long long)total_tokens * H > 0x7fffffffLL) return KDA_ERR_INVALID_ARG;
    if (!dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (!(eps > 0.f) || !(eps < 1e30f)) return KDA_ERR_INVALID_ARG;
    for (const void* ptr : std::initializer_list<const void*>{o, gate, (const void*)w, y})
        if (!ptr || !aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    return from_cuda(kda::launch_norm_gate(o, gate, w, total_tokens, H, dv, eps, dtype, y,
                                           static_cast<cudaStream_t>(stream)));
}

kda_status_t kda_layer_decode_step(const void* xq, const void* xk, const void* xv,
                                  const float* wq, const float* wk, const float* wv,
                                  void* conv_q, void* conv_k, void* conv_v, const float* g,
                                  const float* beta, float* state, const void* gate,
                                  const float* w_norm, int N, int H, int dk, int dv,
                                  kda_dtype_t dtype, float l2_eps, float rms_eps, void* y,
                                  void* stream) {
    if (N < 0 || H < 1 || !dtype_ok(dtype)) return KDA_ERR_INVALID_ARG;
    if ((long long)N * H > 0x3fffffffLL) return KDA_ERR_INVALID_ARG;
    if (!dim_ok(dk) || !dim_ok(dv)) return KDA_ERR_UNSUPPORTED;
    if (!(l2_eps > 0.f) || !(l2_eps < 1e30f) || !(rms_eps > 0.f) || !(rms_eps < 1e30f))
        return KDA_ERR_INVALID_ARG;
    if (N == 0) return KDA_OK;
    for (const void* ptr : std::initializer_list<const void*>{
             xq, xk, xv, (const void*)wq, (const void*)wk, (const void*)wv, conv_q, conv_k,
             conv_v, (const void*)g, (const void*)beta, (const void*)state, gate,
             (const void*)w_norm, y})
        if (!ptr || !aligned16(ptr)) return KDA_ERR_INVALID_ARG;
    return from_cuda(kda::launch_layer_decode(xq, xk, xv, wq, wk, wv, conv_q, conv_k, conv_v, g,
                                              beta, state, gate, w_norm, N, H, dk, dv, dtype,
                                              l2_eps, rms_eps, y,
                                              static_cast<cudaStream_t>(stream)));
}

// ----------------------------------------------------------------- status

kda_status_t kda_get_device_status(void* workspace, void* stream) {
    if (!workspace || !aligned256(workspace)) return KDA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    if (word & kda::STATUS_BAD_SEQLENS) return KDA_ERR_BAD_SEQLENS;
    if (word & kda::STATUS_TIMEOUT) return KDA_ERR_TIMEOUT;
    return KDA_OK;
}

}  // extern "C"
