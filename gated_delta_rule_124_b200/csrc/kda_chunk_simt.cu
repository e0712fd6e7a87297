// KDA chunkwise prefill on CUDA cores (fp32 arithmetic), one kernel per step.
//
// Steps (Kimi Linear, aiwiki.ai, "The constrained DPLR form and the chunkwise
// algorithm": chunks, WY representation, UT transform, recurrent between
// chunks and parallel inside one):
//   a1 gate_cumsum : G = per-chunk inclusive cumulative sum of g = log(alpha)
//   a2 intra       : A (strictly lower, beta-weighted, gate-rescaled K K^T),
//                    (I + A) X = [diag(b)(K * Gam) | diag(b) V] solved by
//                    forward substitution  ->  W, Ut
//   a3 inter       : per (sequence, head, dv slice), serial over chunks:
//                    U = Ut - W S;  S <- Diag(Gam_last) S + (K * exp(G_last - G))^T U
//   a4 output      : O = (Q * Gam) S_n + (P masked to i <= r) U
// These kernels serve the fp32 path and every shape the tensor-core kernel
// does not take; the exponent differences exp(G_r - G_i) (i <= r, so never
// positive for g <= 0) are evaluated directly, never as a ratio of
// cumulative decays.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kda_common.cuh"

namespace kda {

// ------------------------------------------------------------- chunk table
// One block.  Validates cu_seqlens (or synthesises B equal sequences of T),
// writes chunk_start[N + 1], fills chunk_info[maxc] and, when `order` is
// given, the sequences by descending chunk count (ties by index) -- per-chain
// work launched in that order starts with the longest chains, so that the
// last one to start is short.
__global__ void build_chunk_table_kernel(const int32_t* __restrict__ cu, int B, int T, int N,
                                         int chunk, int maxc, uint32_t* status,
                                         int* __restrict__ chunk_start,
                                         int4* __restrict__ info, int* __restrict__ order) {
    __shared__ int warp_sums[32];
    __shared__ int s_nch[kMaxOrderedSeqs];
    __shared__ int bad, most;
    const int tid = threadIdx.x, nt = blockDim.x;
    if (tid == 0) bad = most = 0;
    __syncthreads();
    auto seq_lo = [&](int s) -> int { return cu ? cu[s] : s * T; };
    const int total = cu ? T : B * T;
    // validation
    for (int s = tid; s < N; s += nt) {
        int a = seq_lo(s), b = seq_lo(s + 1);
        if (b < a) atomicOr(&bad, 1);
    }
    if (tid == 0 && (seq_lo(0) != 0 || seq_lo(N) != total)) atomicOr(&bad, 1);
    __syncthreads();
    if (bad) {
        if (tid == 0) atomicOr(status, STATUS_BAD_SEQLENS);
        for (int c = tid; c < maxc; c += nt) info[c] = make_int4(-1, 0, 0, 0);
        return;
    }
    // exclusive scan of per-sequence chunk counts: each thread owns a
    // contiguous run of sequences
    const int per = (N + nt - 1) / nt;
    const int s0 = min(N, tid * per), s1 = min(N, s0 + per);
    int local = 0, lmax = 0;
    for (int s = s0; s < s1; ++s) {
        const int c = (seq_lo(s + 1) - seq_lo(s) + chunk - 1) / chunk;
        local += c;
        lmax = max(lmax, c);
    }
    if (lmax > 0) atomicMax(&most, lmax);
    // block exclusive scan of `local`
    const int lane = tid & 31, wid = tid >> 5;
    int x = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int nw = (nt + 31) / 32;
        int w = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        warp_sums[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    int excl = x - local + (wid > 0 ? warp_sums[wid - 1] : 0);
    for (int s = s0; s < s1; ++s) {
        chunk_start[s] = excl;
        excl += (seq_lo(s + 1) - seq_lo(s) + chunk - 1) / chunk;
    }
    if (s1 == N && s0 < s1) chunk_start[N] = excl;
    if (order) {
        if (N <= kMaxOrderedSeqs) {
            for (int s = tid; s < N; s += nt)
                s_nch[s] = (seq_lo(s + 1) - seq_lo(s) + chunk - 1) / chunk;
            __syncthreads();
            for (int s = tid; s < N; s += nt) {
                const int c = s_nch[s];
                int rank = 0;
                for (int u = 0; u < N; ++u) {
                    const int cu2 = s_nch[u];
                    rank += (cu2 > c) || (cu2 == c && u < s);
                }
                order[rank] = s;
            }
        } else {
            for (int s = tid; s < N; s += nt) order[s] = s;
        }
    }
    if (N == 0 && tid == 0) chunk_start[0] = 0;
    __syncthreads();
    if (tid == 0 && per * nt >= N && s0 >= N) {
        // nothing: chunk_start[N] written by the owner of the last run
    }
    __syncthreads();
    // status word 1: the largest number of chunks of one sequence
    if (tid == 0) status[1] = static_cast<uint32_t>(most);
    const int used = chunk_start[N];
    for (int c = tid; c < maxc; c += nt) {
        if (c >= used) {
            info[c] = make_int4(-1, 0, 0, 0);
            continue;
        }
        // last sequence with chunk_start[s] <= c (binary search; zero-length
        // sequences share a start and are skipped by taking the last match)
        int lo = 0, hi = N - 1;
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (chunk_start[mid] <= c) lo = mid; else hi = mid - 1;
        }
        const int n = c - chunk_start[lo];
        const int t0 = seq_lo(lo) + n * chunk;
        const int rows = min(chunk, seq_lo(lo + 1) - t0);
        info[c] = make_int4(lo, t0, rows, n);
    }
}

cudaError_t launch_build_chunk_table(const int32_t* cu_seqlens, int B, int T, int N, int chunk,
                                     int maxc, uint32_t* status, int* chunk_start,
                                     int4* chunk_info, cudaStream_t st, int* seq_order) {
    build_chunk_table_kernel<<<1, 1024, 0, st>>>(cu_seqlens, B, T, N, chunk, maxc, status,
                                                 chunk_start, chunk_info, seq_order);
    return cudaGetLastError();
}

// ------------------------------------------------------------ a1: cumsum
__global__ void gate_cumsum_kernel(const float* __restrict__ g, const int4* __restrict__ info,
                                   int H, int dk, const uint32_t* status,
                                   float* __restrict__ G) {
    if (status_bad(status)) return;
    const int4 ci = info[blockIdx.x];
    const int h = blockIdx.y;
    if (ci.z <= 0) return;
    for (int c = threadIdx.x; c < dk; c += blockDim.x) {
        float acc = 0.f;
        for (int r = 0; r < ci.z; ++r) {
            const size_t idx = ((size_t)(ci.y + r) * H + h) * dk + c;
            acc += g[idx];
            G[idx] = acc;
        }
    }
}

cudaError_t launch_gate_cumsum(const float* g, const int4* info, int maxc, int H, int dk,
                               const uint32_t* status, float* G, cudaStream_t st) {
    if (maxc == 0) return cudaSuccess;
    dim3 grid(maxc, H);
    gate_cumsum_kernel<<<grid, 128, 0, st>>>(g, info, H, dk, status, G);
    return cudaGetLastError();
}

// ------------------------------------------------------------- a2: intra
// Shared memory: K, G as [C][dk+1] (padded: consecutive rows hit different
// banks), X = [C][dk + dv + 1] right-hand sides / solution, A [C][C+1], beta[C].
template <typename TIn>
__global__ void __launch_bounds__(256) intra_kernel(
    const TIn* __restrict__ k, const TIn* __restrict__ v, const float* __restrict__ G,
    const float* __restrict__ beta, const int4* __restrict__ info, int H, int dk, int dv,
    int C, const uint32_t* status, float* __restrict__ W, float* __restrict__ Ut) {
    if (status_bad(status)) return;
    const int4 ci = info[blockIdx.x];
    const int h = blockIdx.y;
    const int L = ci.z;
    if (L <= 0) return;
    extern __shared__ float sm[];
    const int ldk = dk + 1, ldx = dk + dv + 1, lda = C + 1;
    float* Ks = sm;
    float* Gs = Ks + C * ldk;
    float* X = Gs + C * ldk;
    float* As = X + C * ldx;
    float* bs = As + C * lda;
    const int tid = threadIdx.x, nt = blockDim.x;
    for (int idx = tid; idx < L * dk; idx += nt) {
        const int r = idx / dk, c = idx % dk;
        const size_t gi = ((size_t)(ci.y + r) * H + h) * dk + c;
        Ks[r * ldk + c] = to_f32(k[gi]);
        Gs[r * ldk + c] = G[gi];
    }
    for (int r = tid; r < L; r += nt) bs[r] = beta[(size_t)(ci.y + r) * H + h];
    __syncthreads();
    // right-hand sides: [b_r k_r * exp(G_r) | b_r v_r]
    for (int idx = tid; idx < L * dk; idx += nt) {
        const int r = idx / dk, c = idx % dk;
        X[r * ldx + c] = bs[r] * Ks[r * ldk + c] * expf(Gs[r * ldk + c]);
    }
    for (int idx = tid; idx < L * dv; idx += nt) {
        const int r = idx / dv, j = idx % dv;
        X[r * ldx + dk + j] = bs[r] * to_f32(v[((size_t)(ci.y + r) * H + h) * dv + j]);
    }
    // A[r][i] = b_r sum_c k_rc k_ic exp(G_rc - G_ic), i < r
    for (int idx = tid; idx < L * L; idx += nt) {
        const int r = idx / L, i = idx % L;
        float acc = 0.f;
        if (i < r) {
            const float* kr = Ks + r * ldk;
            const float* ki = Ks + i * ldk;
            const float* gr = Gs + r * ldk;
            const float* gi = Gs + i * ldk;
            for (int c = 0; c < dk; ++c) acc += kr[c] * ki[c] * expf(gr[c] - gi[c]);
            acc *= bs[r];
        }
        As[r * lda + i] = acc;
    }
    __syncthreads();
    // UT transform: forward substitution, one column per thread,
    // x_r = rhs_r - sum_{i<r} A[r][i] x_i
    for (int col = tid; col < dk + dv; col += nt) {
        for (int r = 1; r < L; ++r) {
            float acc = X[r * ldx + col];
            const float* ar = As + r * lda;
            for (int i = 0; i < r; ++i) acc -= ar[i] * X[i * ldx + col];
            X[r * ldx + col] = acc;
        }
    }
    __syncthreads();
    for (int idx = tid; idx < L * dk; idx += nt) {
        const int r = idx / dk, c = idx % dk;
        W[((size_t)(ci.y + r) * H + h) * dk + c] = X[r * ldx + c];
    }
    for (int idx = tid; idx < L * dv; idx += nt) {
        const int r = idx / dv, j = idx % dv;
        Ut[((size_t)(ci.y + r) * H + h) * dv + j] = X[r * ldx + dk + j];
    }
}

static size_t intra_smem(int dk, int dv, int C) {
    return sizeof(float) * ((size_t)2 * C * (dk + 1) + (size_t)C * (dk + dv + 1) +
                            (size_t)C * (C + 1) + C);
}

cudaError_t launch_intra(const void* k, const void* v, const float* G, const float* beta,
                         const int4* info, int maxc, int H, int dk, int dv, int chunk,
                         kda_dtype_t dt, const uint32_t* status, float* W, float* U,
                         cudaStream_t st) {
    if (maxc == 0) return cudaSuccess;
    const size_t smem = intra_smem(dk, dv, chunk);
    dim3 grid(maxc, H);
    if (dt == KDA_DTYPE_BF16) {
        auto kern = intra_kernel<__nv_bfloat16>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, 256, smem, st>>>((const __nv_bfloat16*)k, (const __nv_bfloat16*)v, G, beta,
                                      info, H, dk, dv, chunk, status, W, U);
    } else {
        auto kern = intra_kernel<float>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, 256, smem, st>>>((const float*)k, (const float*)v, G, beta, info, H, dk, dv,
                                      chunk, status, W, U);
    }
    return cudaGetLastError();
}

// ------------------------------------------------------------- a3: inter
// One block per (sequence, head, dv slice of width DVS).  Shared memory:
// S [dk][DVS], W [C][dk+1], Kd = K * exp(G_last - G) [C][dk+1], U [C][DVS+1],
// exp(G_last) [dk].
constexpr int kInterDVS = 32;

template <typename TIn>
__global__ void __launch_bounds__(256) inter_kernel(
    const TIn* __restrict__ k, const float* __restrict__ G, const float* __restrict__ W,
    float* __restrict__ U, const float* __restrict__ h0, const int32_t* __restrict__ cu, int T,
    const int* __restrict__ chunk_start, int H, int dk, int dv, int C, int dvs,
    const uint32_t* status, float* __restrict__ states, float* __restrict__ hN) {
    if (status_bad(status)) return;
    const int s = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * dvs;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int t_begin = cu ? cu[s] : s * T;
    const int t_end = cu ? cu[s + 1] : (s + 1) * T;
    extern __shared__ float sm[];
    const int ldk = dk + 1, ldu = dvs + 1;
    float* S = sm;                  // [dk][dvs]
    float* Ws = S + dk * dvs;       // [C][ldk]
    float* Kd = Ws + C * ldk;       // [C][ldk]
    float* Us = Kd + C * ldk;       // [C][ldu]
    float* eGl = Us + C * ldu;      // [dk]
    const size_t st_base = ((size_t)s * H + h) * dk * dv;
    for (int idx = tid; idx < dk * dvs; idx += nt) {
        const int c = idx / dvs, j = idx % dvs;
        S[idx] = h0 ? h0[st_base + (size_t)c * dv + j0 + j] : 0.f;
    }
    __syncthreads();
    int n = 0;
    for (int t0 = t_begin; t0 < t_end; t0 += C, ++n) {
        const int L = min(C, t_end - t0);
        const size_t cs = (size_t)chunk_start[s] + n;
        float* Sn = states + (cs * H + h) * dk * dv;
        for (int idx = tid; idx < dk * dvs; idx += nt) {
            const int c = idx / dvs, j = idx % dvs;
            Sn[(size_t)c * dv + j0 + j] = S[idx];
        }
        const float* Glast = G + ((size_t)(t0 + L - 1) * H + h) * dk;
        for (int c = tid; c < dk; c += nt) eGl[c] = expf(Glast[c]);
        for (int idx = tid; idx < L * dk; idx += nt) {
            const int r = idx / dk, c = idx % dk;
            const size_t gi = ((size_t)(t0 + r) * H + h) * dk + c;
            Ws[r * ldk + c] = W[gi];
            Kd[r * ldk + c] = to_f32(k[gi]) * expf(Glast[c] - G[gi]);
        }
        for (int idx = tid; idx < L * dvs; idx += nt) {
            const int r = idx / dvs, j = idx % dvs;
            Us[r * ldu + j] = U[((size_t)(t0 + r) * H + h) * dv + j0 + j];
        }
        __syncthreads();
        // U = Ut - W S
        for (int idx = tid; idx < L * dvs; idx += nt) {
            const int r = idx / dvs, j = idx % dvs;
            float acc = Us[r * ldu + j];
            const float* wr = Ws + r * ldk;
            for (int c = 0; c < dk; ++c) acc -= wr[c] * S[c * dvs + j];
            Us[r * ldu + j] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < L * dvs; idx += nt) {
            const int r = idx / dvs, j = idx % dvs;
            U[((size_t)(t0 + r) * H + h) * dv + j0 + j] = Us[r * ldu + j];
        }
        // S <- Diag(exp(G_last)) S + Kd^T U
        for (int idx = tid; idx < dk * dvs; idx += nt) {
            const int c = idx / dvs, j = idx % dvs;
            float acc = eGl[c] * S[idx];
            for (int r = 0; r < L; ++r) acc += Kd[r * ldk + c] * Us[r * ldu + j];
            S[idx] = acc;
        }
        __syncthreads();
    }
    if (hN) {
        for (int idx = tid; idx < dk * dvs; idx += nt) {
            const int c = idx / dvs, j = idx % dvs;
            hN[st_base + (size_t)c * dv + j0 + j] = S[idx];
        }
    }
}

cudaError_t launch_inter(const void* k, const float* G, const float* W, float* U,
                         const float* h0, const int32_t* cu_seqlens, int B, int T, int N,
                         const int* chunk_start, int H, int dk, int dv, int chunk,
                         kda_dtype_t dt, const uint32_t* status, float* states, float* hN,
                         cudaStream_t st, int dv_slice) {
    (void)B;
    if (N == 0) return cudaSuccess;
    const int want = dv_slice > 0 ? dv_slice : kInterDVS;
    const int dvs = dv < want ? dv : want;
    const size_t smem = sizeof(float) * ((size_t)dk * dvs + (size_t)2 * chunk * (dk + 1) +
                                         (size_t)chunk * (dvs + 1) + dk);
    dim3 grid(N, H, dv / dvs);
    if (dt == KDA_DTYPE_BF16) {
        auto kern = inter_kernel<__nv_bfloat16>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, 256, smem, st>>>((const __nv_bfloat16*)k, G, W, U, h0, cu_seqlens, T,
                                      chunk_start, H, dk, dv, chunk, dvs, status, states, hN);
    } else {
        auto kern = inter_kernel<float>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, 256, smem, st>>>((const float*)k, G, W, U, h0, cu_seqlens, T, chunk_start,
                                      H, dk, dv, chunk, dvs, status, states, hN);
    }
    return cudaGetLastError();
}

// ------------------------------------------------------------ a4: output
// One block per (chunk, head).  Shared memory: Q*Gam, K, G as [C][dk+1],
// P [C][C+1], then per dv slice S_n [dk][DVS] and U [C][DVS+1].
template <typename TIn>
__global__ void __launch_bounds__(256) output_kernel(
    const TIn* __restrict__ q, const TIn* __restrict__ k, const float* __restrict__ G,
    const float* __restrict__ U, const float* __restrict__ states,
    const int4* __restrict__ info, int H, int dk, int dv, int C, int dvs,
    const uint32_t* status, TIn* __restrict__ o) {
    if (status_bad(status)) return;
    const int cidx = blockIdx.x, h = blockIdx.y;
    const int4 ci = info[cidx];
    const int L = ci.z;
    if (L <= 0) return;
    const int tid = threadIdx.x, nt = blockDim.x;
    extern __shared__ float sm[];
    const int ldk = dk + 1, lda = C + 1, ldu = dvs + 1;
    float* Qs = sm;
    float* Ks = Qs + C * ldk;
    float* Gs = Ks + C * ldk;
    float* Ps = Gs + C * ldk;
    float* Ss = Ps + C * lda;       // [dk][dvs]
    float* Us = Ss + dk * dvs;      // [C][ldu]
    for (int idx = tid; idx < L * dk; idx += nt) {
        const int r = idx / dk, c = idx % dk;
        const size_t gi = ((size_t)(ci.y + r) * H + h) * dk + c;
        Qs[r * ldk + c] = to_f32(q[gi]);
        Ks[r * ldk + c] = to_f32(k[gi]);
        Gs[r * ldk + c] = G[gi];
    }
    __syncthreads();
    // P[r][i] = sum_c q_rc k_ic exp(G_rc - G_ic), i <= r (diagonal included:
    // the read-out uses the state after token r's own write)
    for (int idx = tid; idx < L * L; idx += nt) {
        const int r = idx / L, i = idx % L;
        float acc = 0.f;
        if (i <= r) {
            const float* qr = Qs + r * ldk;
            const float* ki = Ks + i * ldk;
            const float* gr = Gs + r * ldk;
            const float* gi = Gs + i * ldk;
            for (int c = 0; c < dk; ++c) acc += qr[c] * ki[c] * expf(gr[c] - gi[c]);
        }
        Ps[r * lda + i] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < L * dk; idx += nt) {
        const int r = idx / dk, c = idx % dk;
        Qs[r * ldk + c] *= expf(Gs[r * ldk + c]);
    }
    const float* Sn = states + ((size_t)cidx * H + h) * dk * dv;
    for (int j0 = 0; j0 < dv; j0 += dvs) {
        __syncthreads();
        for (int idx = tid; idx < dk * dvs; idx += nt) {
            const int c = idx / dvs, j = idx % dvs;
            Ss[idx] = Sn[(size_t)c * dv + j0 + j];
        }
        for (int idx = tid; idx < L * dvs; idx += nt) {
            const int r = idx / dvs, j = idx % dvs;
            Us[r * ldu + j] = U[((size_t)(ci.y + r) * H + h) * dv + j0 + j];
        }
        __syncthreads();
        for (int idx = tid; idx < L * dvs; idx += nt) {
            const int r = idx / dvs, j = idx % dvs;
            float acc = 0.f;
            const float* qr = Qs + r * ldk;
            for (int c = 0; c < dk; ++c) acc += qr[c] * Ss[c * dvs + j];
            const float* pr = Ps + r * lda;
            for (int i = 0; i <= r; ++i) acc += pr[i] * Us[i * ldu + j];
            o[((size_t)(ci.y + r) * H + h) * dv + j0 + j] = from_f32<TIn>(acc);
        }
    }
}

cudaError_t launch_output(const void* q, const void* k, const float* G, const float* U,
                          const float* states, const int4* info, int maxc, int H, int dk,
                          int dv, int chunk, kda_dtype_t dt, const uint32_t* status, void* o,
                          cudaStream_t st) {
    if (maxc == 0) return cudaSuccess;
    const int dvs = dv < kInterDVS ? dv : kInterDVS;
    const size_t smem = sizeof(float) * ((size_t)3 * chunk * (dk + 1) +
                                         (size_t)chunk * (chunk + 1) + (size_t)dk * dvs +
                                         (size_t)chunk * (dvs + 1));
    dim3 grid(maxc, H);
    if (dt == KDA_DTYPE_BF16) {
        auto kern = output_kernel<__nv_bfloat16>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, 256, smem, st>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, G, U,
                                      states, info, H, dk, dv, chunk, dvs, status,
                                      (__nv_bfloat16*)o);
    } else {
        auto kern = output_kernel<float>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, 256, smem, st>>>((const float*)q, (const float*)k, G, U, states, info, H,
                                      dk, dv, chunk, dvs, status, (float*)o);
    }
    return cudaGetLastError();
}

}  // namespace kda
