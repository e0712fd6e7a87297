// KDA backward (gradients of the chunkwise forward's outputs), recurrent form.
//
// The pages give no backward equations; these are derived from the forward
// step (Kimi Linear (aiwiki.ai), "Kimi Delta Attention"):
//   S_bar = Diag(alpha) S_prev,  w = S_bar^T k,  u = beta (v - w),
//   S = S_bar + k u^T,  o = S^T q,  alpha = exp(g).
// Going backwards over the tokens with dS the gradient of the state after the
// token:
//   dS += q do^T;  dq = S do;  du = dS^T k;  dk = dS u + S_bar dw;
//   dv = beta du;  dbeta = du . (v - w);  dw = -beta du;
//   dS_bar = dS + k dw^T;  dg = alpha * rowsum(dS_bar * S_prev);
//   dS <- Diag(alpha) dS_bar;  after the first token dS is d initial_state.
//
// One CTA of 256 threads per (sequence, head, 32 value columns): the columns
// of a state evolve independently, so a slice needs only its own columns,
// while dq, dk, dg and dbeta sum over all columns -- each slice writes its
// partial sums and a second kernel adds the slices.  The states the backward
// sweep needs (S before each token) are rebuilt: a forward sweep stores the
// state every 8 tokens in the workspace, and each 8-token block is rebuilt
// from its checkpoint into shared memory before it is walked backwards.  This
// is the plain recurrent form: correct, and far slower than the forward's
// chunked tensor-core form.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int NTB = 256;  // threads
constexpr int DVS = 32;   // value columns per CTA
constexpr int SB = 8;     // tokens per checkpoint block

// Thread (warp w, lane l) holds float4 column group c4 = l & 7 of rows
// p * 32 + w * 4 + (l >> 3), p < DK / 32.
template <int DK>
struct Layout {
    static constexpr int NP = DK / 32;
    __device__ static int row(int p, int warp, int lane) { return p * 32 + warp * 4 + (lane >> 3); }
};

__device__ __forceinline__ float4 f4(float a) { return make_float4(a, a, a, a); }
__device__ __forceinline__ float dot4(float4 a, float4 b) {
    return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}
// sum over the 8 lanes that hold one row (lanes of equal l >> 3)
__device__ __forceinline__ float row_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    return x;
}

struct BwdParams {
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    const float* h0;
    const void* dout;
    const float* dhT;
    const int32_t* cu;
    int T, N, H, DV, total;
    float* ckpt;   // [total / SB + N + 1][H][DK][DV]
    float* dq_p;   // [slices][total][H][DK]
    float* dk_p;
    float* dg_p;
    float* db_p;   // [slices][total][H]
    float* dv;     // [total][H][DV]
    float* dh0;    // [N][H][DK][DV] (may be NULL)
};

template <typename TIn>
__device__ __forceinline__ float ld(const TIn* p, size_t i) {
    return to_f32(p[i]);
}

template <int DK, typename TIn>
__global__ void __launch_bounds__(NTB, 1) bwd_kernel(const BwdParams p) {
    using Lo = Layout<DK>;
    constexpr int NP = Lo::NP;
    extern __shared__ float4 smem_f4[];
    float4* sbuf = smem_f4;  // [SB][DK][8] float4: the state before each token of a block
    __shared__ float s_q[DK], s_k[DK], s_a[DK];
    __shared__ float s_v[DVS], s_do[DVS], s_col[DVS], s_du[DVS];
    __shared__ float4 s_red[8][8];
    __shared__ float s_beta;

    const int unit = blockIdx.x, slice = blockIdx.y;
    const int seq = unit / p.H, h = unit % p.H;
    const int j0 = slice * DVS;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, c4 = lane & 7;
    const int t_begin = p.cu ? p.cu[seq] : seq * p.T;
    const int t_end = p.cu ? p.cu[seq + 1] : (seq + 1) * p.T;
    const int nslice = p.DV / DVS;
    const TIn* Q = static_cast<const TIn*>(p.q);
    const TIn* K = static_cast<const TIn*>(p.k);
    const TIn* V = static_cast<const TIn*>(p.v);
    const TIn* DO = static_cast<const TIn*>(p.dout);

    auto state_ptr = [&](float* base, size_t block) {  // float4 row starts of this slice
        return reinterpret_cast<float4*>(base + ((block * p.H + h) * DK) * p.DV + j0);
    };
    // token t's vectors into shared memory (q, k, alpha over DK; v, do over the slice)
    auto load_token = [&](int t, bool with_do) {
        const size_t bk = ((size_t)t * p.H + h) * DK;
        for (int c = tid; c < DK; c += NTB) {
            s_q[c] = ld(Q, bk + c);
            s_k[c] = ld(K, bk + c);
            s_a[c] = expf(p.g[bk + c]);
        }
        if (tid < DVS) {
            const size_t bv = ((size_t)t * p.H + h) * p.DV + j0 + tid;
            s_v[tid] = ld(V, bv);
            s_do[tid] = with_do ? ld(DO, bv) : 0.f;
        }
        if (tid == 0) s_beta = p.beta[(size_t)t * p.H + h];
        __syncthreads();
    };
    // column sums over the DK rows of x (one value per row of this thread's
    // float4 group, weighted by wrow[p]) -> s_out[32]
    auto col_sum = [&](const float4 (&x)[NP], const float (&wrow)[NP], float* s_out) {
        float4 acc = f4(0.f);
#pragma unroll
        for (int i = 0; i < NP; ++i) {
            acc.x += x[i].x * wrow[i]; acc.y += x[i].y * wrow[i];
            acc.z += x[i].z * wrow[i]; acc.w += x[i].w * wrow[i];
        }
#pragma unroll
        for (int o = 8; o < 32; o <<= 1) {
            acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
            acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
            acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
            acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
        }
        if (lane < 8) s_red[warp][c4] = acc;
        __syncthreads();
        if (tid < 8) {
            float4 s = f4(0.f);
#pragma unroll
            for (int w2 = 0; w2 < 8; ++w2) {
                const float4 y = s_red[w2][tid];
                s.x += y.x; s.y += y.y; s.z += y.z; s.w += y.w;
            }
            s_out[4 * tid] = s.x; s_out[4 * tid + 1] = s.y;
            s_out[4 * tid + 2] = s.z; s_out[4 * tid + 3] = s.w;
        }
        __syncthreads();
    };
    // one forward step on S (registers): S <- Diag(a) S + k (beta (v - S_bar^T k))^T
    auto forward_step = [&](float4 (&S)[NP]) {
        float kr[NP];
#pragma unroll
        for (int i = 0; i < NP; ++i) {
            const int r = Lo::row(i, warp, lane);
            const float a = s_a[r];
            S[i].x *= a; S[i].y *= a; S[i].z *= a; S[i].w *= a;
            kr[i] = s_k[r];
        }
        col_sum(S, kr, s_col);  // w
        const float b = s_beta;
        const float4 u = make_float4(b * (s_v[4 * c4] - s_col[4 * c4]),
                                     b * (s_v[4 * c4 + 1] - s_col[4 * c4 + 1]),
                                     b * (s_v[4 * c4 + 2] - s_col[4 * c4 + 2]),
                                     b * (s_v[4 * c4 + 3] - s_col[4 * c4 + 3]));
#pragma unroll
        for (int i = 0; i < NP; ++i) {
            S[i].x += kr[i] * u.x; S[i].y += kr[i] * u.y;
            S[i].z += kr[i] * u.z; S[i].w += kr[i] * u.w;
        }
    };

    // ---------------- forward sweep: a checkpoint every SB tokens
    float4 S[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        const int r = Lo::row(i, warp, lane);
        S[i] = p.h0 ? reinterpret_cast<const float4*>(
                          p.h0 + (((size_t)seq * p.H + h) * DK + r) * p.DV + j0)[c4]
                    : f4(0.f);
    }
    const size_t blk0 = (size_t)(t_begin / SB) + seq;
    for (int t = t_begin; t < t_end; ++t) {
        if ((t - t_begin) % SB == 0) {
            float4* dst = state_ptr(p.ckpt, blk0 + (t - t_begin) / SB);
#pragma unroll
            for (int i = 0; i < NP; ++i)
                dst[(size_t)Lo::row(i, warp, lane) * (p.DV / 4) + c4] = S[i];
        }
        load_token(t, false);
        forward_step(S);
        __syncthreads();
    }
    __syncthreads();

    // ---------------- backward sweep, block by block
    float4 dS[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        const int r = Lo::row(i, warp, lane);
        dS[i] = p.dhT ? reinterpret_cast<const float4*>(
                            p.dhT + (((size_t)seq * p.H + h) * DK + r) * p.DV + j0)[c4]
                      : f4(0.f);
    }
    const int nblk = (t_end - t_begin + SB - 1) / SB;
    for (int bi = nblk - 1; bi >= 0; --bi) {
        const int t0 = t_begin + bi * SB, cnt = min(SB, t_end - t0);
        // rebuild the block's states from its checkpoint
        const float4* src = state_ptr(p.ckpt, blk0 + bi);
#pragma unroll
        for (int i = 0; i < NP; ++i) S[i] = src[(size_t)Lo::row(i, warp, lane) * (p.DV / 4) + c4];
        for (int i = 0; i < cnt; ++i) {
#pragma unroll
            for (int pp = 0; pp < NP; ++pp)
                sbuf[((size_t)i * DK + Lo::row(pp, warp, lane)) * 8 + c4] = S[pp];
            if (i + 1 < cnt) {
                load_token(t0 + i, false);
                forward_step(S);
                __syncthreads();
            }
        }
        // walk it backwards
        for (int i = cnt - 1; i >= 0; --i) {
            const int t = t0 + i;
            load_token(t, true);
            float4 Sp[NP], Sb[NP], St[NP];
            float kr[NP], qr[NP], ar[NP];
#pragma unroll
            for (int pp = 0; pp < NP; ++pp) {
                const int r = Lo::row(pp, warp, lane);
                Sp[pp] = sbuf[((size_t)i * DK + r) * 8 + c4];
                ar[pp] = s_a[r];
                kr[pp] = s_k[r];
                qr[pp] = s_q[r];
                Sb[pp] = make_float4(Sp[pp].x * ar[pp], Sp[pp].y * ar[pp], Sp[pp].z * ar[pp],
                                     Sp[pp].w * ar[pp]);
            }
            col_sum(Sb, kr, s_col);  // w
            const float b = s_beta;
            const float4 w = make_float4(s_col[4 * c4], s_col[4 * c4 + 1], s_col[4 * c4 + 2],
                                         s_col[4 * c4 + 3]);
            const float4 vv = make_float4(s_v[4 * c4], s_v[4 * c4 + 1], s_v[4 * c4 + 2],
                                          s_v[4 * c4 + 3]);
            const float4 u = make_float4(b * (vv.x - w.x), b * (vv.y - w.y), b * (vv.z - w.z),
                                         b * (vv.w - w.w));
            const float4 dov = make_float4(s_do[4 * c4], s_do[4 * c4 + 1], s_do[4 * c4 + 2],
                                           s_do[4 * c4 + 3]);
            const size_t part = ((size_t)slice * p.total + t) * p.H + h;
#pragma unroll
            for (int pp = 0; pp < NP; ++pp) {
                St[pp] = make_float4(Sb[pp].x + kr[pp] * u.x, Sb[pp].y + kr[pp] * u.y,
                                     Sb[pp].z + kr[pp] * u.z, Sb[pp].w + kr[pp] * u.w);
                dS[pp].x += qr[pp] * dov.x; dS[pp].y += qr[pp] * dov.y;
                dS[pp].z += qr[pp] * dov.z; dS[pp].w += qr[pp] * dov.w;
                const float dq = row_sum(dot4(St[pp], dov));
                if (c4 == 0) p.dq_p[part * DK + Lo::row(pp, warp, lane)] = dq;
            }
            col_sum(dS, kr, s_du);  // du
            const float4 du = make_float4(s_du[4 * c4], s_du[4 * c4 + 1], s_du[4 * c4 + 2],
                                          s_du[4 * c4 + 3]);
            if (tid < DVS)
                p.dv[((size_t)t * p.H + h) * p.DV + j0 + tid] = b * s_du[tid];
            if (warp == 0) {  // this slice's part of dbeta
                float x = lane < DVS ? s_du[lane] * (s_v[lane] - s_col[lane]) : 0.f;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                if (lane == 0) p.db_p[part] = x;
            }
            const float4 dw = make_float4(-b * du.x, -b * du.y, -b * du.z, -b * du.w);
#pragma unroll
            for (int pp = 0; pp < NP; ++pp) {
                const int r = Lo::row(pp, warp, lane);
                const float dk = row_sum(dot4(dS[pp], u) + dot4(Sb[pp], dw));
                const float4 dSb = make_float4(dS[pp].x + kr[pp] * dw.x, dS[pp].y + kr[pp] * dw.y,
                                               dS[pp].z + kr[pp] * dw.z, dS[pp].w + kr[pp] * dw.w);
                const float da = row_sum(dot4(dSb, Sp[pp]));
                if (c4 == 0) {
                    p.dk_p[part * DK + r] = dk;
                    p.dg_p[part * DK + r] = ar[pp] * da;
                }
                dS[pp] = make_float4(ar[pp] * dSb.x, ar[pp] * dSb.y, ar[pp] * dSb.z,
                                     ar[pp] * dSb.w);
            }
            __syncthreads();
        }
    }
    if (p.dh0) {
#pragma unroll
        for (int i = 0; i < NP; ++i) {
            const int r = Lo::row(i, warp, lane);
            reinterpret_cast<float4*>(p.dh0 + (((size_t)seq * p.H + h) * DK + r) * p.DV + j0)[c4] =
                dS[i];
        }
    }
    (void)nslice;
}

// dq, dk, dg [total, H, DK] and dbeta [total, H]: the slices' partial sums added.
__global__ void bwd_reduce_kernel(const float* __restrict__ dq_p, const float* __restrict__ dk_p,
                                  const float* __restrict__ dg_p, const float* __restrict__ db_p,
                                  int nslice, long long rows, int DK, float* dq, float* dk,
                                  float* dg, float* db) {
    const long long n = rows * DK;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        float a = 0.f, b = 0.f, c = 0.f;
        for (int s = 0; s < nslice; ++s) {
            a += dq_p[s * n + i];
            b += dk_p[s * n + i];
            c += dg_p[s * n + i];
        }
        dq[i] = a;
        dk[i] = b;
        dg[i] = c;
        if (i < rows) {
            float d = 0.f;
            for (int s = 0; s < nslice; ++s) d += db_p[s * rows + i];
            db[i] = d;
        }
    }
}

template <int DK, typename TIn>
cudaError_t bwd_launch(const BwdParams& p, cudaStream_t st) {
    const size_t smem = (size_t)SB * DK * DVS * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(bwd_kernel<DK, TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_kernel<DK, TIn><<<dim3(p.N * p.H, p.DV / DVS), NTB, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace_bytes(int total, int N, int H, int dk, int dv) {
    const size_t ck = ((size_t)total / SB + N + 1) * H * dk * dv * sizeof(float);
    const size_t slices = dv / DVS;
    const size_t part = slices * (size_t)total * H * (3 * dk + 1) * sizeof(float);
    return align_up(ck) + align_up(part);
}

cudaError_t launch_bwd(const void* q, const void* k, const void* v, const float* g,
                       const float* beta, const float* h0, const void* dout, const float* dhT,
                       const int32_t* cu, int T, int N, int H, int dk, int dv, kda_dtype_t dt,
                       float* dq, float* dkk, float* dvv, float* dg, float* db, float* dh0,
                       void* workspace, cudaStream_t st) {
    const int total = cu ? T : N * T;
    if (N * H == 0) return cudaSuccess;
    char* ws = static_cast<char*>(workspace);
    const size_t ck = align_up(((size_t)total / SB + N + 1) * H * dk * dv * sizeof(float));
    const int slices = dv / DVS;
    const size_t n = (size_t)total * H * dk;
    float* part = reinterpret_cast<float*>(ws + ck);
    BwdParams p{q, k, v, g, beta, h0, dout, dhT, cu, T, N, H, dv, total,
                reinterpret_cast<float*>(ws), part, part + slices * n, part + 2 * slices * n,
                part + 3 * slices * n, dvv, dh0};
    cudaError_t e;
    if (dt == KDA_DTYPE_BF16) {
        e = dk == 128 ? bwd_launch<128, __nv_bfloat16>(p, st)
            : dk == 64 ? bwd_launch<64, __nv_bfloat16>(p, st)
                       : bwd_launch<32, __nv_bfloat16>(p, st);
    } else {
        e = dk == 128 ? bwd_launch<128, float>(p, st)
            : dk == 64 ? bwd_launch<64, float>(p, st)
                       : bwd_launch<32, float>(p, st);
    }
    if (e != cudaSuccess || total == 0) return e;
    const long long rows = (long long)total * H;
    const long long work = rows * dk;
    const unsigned grid = static_cast<unsigned>(work / 256 + 1 < 148 * 16 ? work / 256 + 1
                                                                          : 148 * 16);
    bwd_reduce_kernel<<<grid, 256, 0, st>>>(p.dq_p, p.dk_p, p.dg_p, p.db_p, slices, rows, dk, dq,
                                            dkk, dg, db);
    return cudaGetLastError();
}

}  // namespace kda
