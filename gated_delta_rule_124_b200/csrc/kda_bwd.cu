// KDA backward (gradients of the chunkwise prefill), chunked form on CUDA cores.
//
// The pages give no backward equations; these follow from the chunk form of
// Kimi Linear (aiwiki.ai), "The constrained DPLR form and the chunkwise
// algorithm".  Per (sequence, head) and chunk of C tokens with entry state S,
// G the inclusive cumulative sum of g inside the chunk and Gam = exp(G_last):
//   A[r][i] = b_r sum_c k_rc k_ic exp(G_rc - G_ic)   (i < r),  T = (I + A)^-1
//   P[r][i] = sum_c q_rc k_ic exp(G_rc - G_ic)       (i <= r)
//   W = T diag(b) (K * exp(G)),  Ut = T diag(b) V,  U = Ut - W S
//   O = (Q * exp(G)) S + P U,    S' = Diag(Gam) S + (K * exp(G_last - G))^T U
// Going backwards with dS' the gradient of the exit state and dO of the
// chunk's outputs (Qt = Q * exp(G), Kt = K * exp(G), Kb = K * exp(G_last - G)):
//   E  = P^T dO,  F = Qt^T dO - W^T E                              (b1 intra)
//   X  = Kb dS',  dU = E + X,  dS = Diag(Gam) dS' - W^T X + F      (b2 chain)
//   Y  = T^T dU (back substitution),  dv = b Y,
//   dA = -strict_lower(Y U^T),  dP = lower(dO U^T)                 (b3 solve)
//   dQt = dO S^T,  dKt = -b (Y S^T),  dKb = U dS'^T,
//   dbeta = Y.V + sum_i dA[r][i] A[r][i] / b_r - Kt.(Y S^T)         (b4 dense)
//   then the pair sums over (r, i, c) of A and P give dq, dk and dG, and
//   dg is the reverse cumulative sum of dG inside the chunk          (b5 pairs)
// The gradient of T = (I + A)^-1 never appears on its own: T^T dT T^T reduces
// to Y U^T because the gradient reaching W is -dU S^T.  The forward half is
// recomputed: b1 forms G, A, P, Kb, W and Ut of each chunk (the forward's a1
// and a2, with A and P from one pass over the token pairs) and the forward
// pass of the b2 chain kernel gives U and the entry state of every chunk.
// Launches per call: chunk table, b1a/b1b/b1c, b2 forward and backward, b3,
// b4, b5.  Every exponent is a difference exp(G_r - G_i) with i <= r, so
// never positive for g <= 0; all arithmetic is fp32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int CB = 64;   // chunk length of the backward
constexpr int DVS = 32;  // value columns per slice

struct BwdBufs {
    Workspace w;
    float* E;     // [total, H, dv]
    float* dU;    // [total, H, dv]
    float* Y;     // [total, H, dv]
    float* F;     // [maxc, H, dk, dv]
    float* Ar;    // [maxc, H, C, C]     A without the b_r factor
    float* Kb;    // [total, H, dk]      K * exp(G_last - G)
    float* Pm;    // [maxc, H, C, C]     P
    float* dSx;   // [maxc, H, dk, dv]   gradient of each chunk's exit state
    float* dAr;   // [maxc, H, C, C]     b_r dA[r][i]
    float* dP;    // [maxc, H, C, C]
    float* dQt;   // [total, H, dk]
    float* dKt;   // [total, H, dk]
    float* dKb;   // [total, H, dk]
    float* dGam;  // [maxc, H, dk]
    float* dbB;   // [total, H]
    int* slow;    // [maxc, H]  (tensor-core pair sums) 1: the chunk is left to the exact kernel
    float* Tm;    // [maxc, H, C, C]     (tensor-core solves) T = (I + A)^-1
    size_t bytes;
};

BwdBufs carve_bwd(void* base, int total, int N, int H, int dk, int dv) {
    BwdBufs b{};
    b.w = carve(base, total, N, H, dk, dv, CB, true);
    const size_t maxc = (size_t)max_chunks(total, N, CB);
    char* p = static_cast<char*>(base);
    size_t off = b.w.total_bytes;
    auto take = [&](size_t floats) {
        float* r = reinterpret_cast<float*>(p + off);
        off = align_up(off + floats * sizeof(float));
        return r;
    };
    const size_t tv = (size_t)total * H * dv, tk = (size_t)total * H * dk;
    const size_t cs = maxc * H * dk * dv, cc = maxc * H * CB * CB;
    b.E = take(tv);
    b.dU = take(tv);
    b.Y = take(tv);
    b.F = take(cs);
    b.Ar = take(cc);
    b.Kb = take(tk);
    b.Pm = take(cc);
    b.dSx = take(cs);
    b.dAr = take(cc);
    b.dP = take(cc);
    b.dQt = take(tk);
    b.dKt = take(tk);
    b.dKb = take(tk);
    b.dGam = take(maxc * H * dk);
    b.dbB = take((size_t)total * H);
    b.slow = reinterpret_cast<int*>(take(maxc * H));
    b.Tm = take(cc);
    b.bytes = off;
    return b;
}

// ------------------------------------------------------------ b1: intra
// Three kernels, one block per (chunk, head) each, small enough in shared
// memory for two blocks per SM.  Rows past the chunk's end are zero.
//   b1a: G (a1), A without b and P from one exponent per (r, i, c), Kb, and
//        the right-hand sides b Kt (into the W buffer).  Shared: Q, K, G
//        [C][dk+1].
//   b1b: (I + A) [W | Ut] = [b Kt | b V] by forward substitution (a2).
//        Shared: A [C][C+1], X [C][dk+dv+1], b [C].
//   b1c: E = P^T dO and F = Qt^T dO - W^T E.  Shared: P [C][C+1], Qt and W
//        [C][dk+4], dO and E slices [C][DVS+4] (16-byte rows for the F tiles).
constexpr int kPairTiles = (CB / 4) * (CB / 4 + 1) / 2;  // 4 x 4 tiles with i <= r

template <int DK, typename TIn>
__global__ void __launch_bounds__(256) bwd_apkb_kernel(
    const TIn* __restrict__ q, const TIn* __restrict__ k, const float* __restrict__ g,
    const float* __restrict__ beta, const int4* __restrict__ info, int H,
    const uint32_t* status, float* __restrict__ G, float* __restrict__ Ar_out,
    float* __restrict__ P_out, float* __restrict__ Kb, float* __restrict__ Rk, bool rt,
    const int* __restrict__ slow) {
    // rt: P and Kb are tf32 operands of the tensor-core kernels after this one;
    // slow != NULL: only the chunks the tensor-core kernel left (flag 1)
    constexpr int LDK = DK + 1;
    if (status_bad(status)) return;
    const int cidx = blockIdx.x, h = blockIdx.y;
    const int4 ci = info[cidx];
    const int L = ci.z;
    if (L <= 0) return;
    if (slow && !slow[(size_t)cidx * H + h]) return;
    const int tid = threadIdx.x;
    extern __shared__ __align__(16) float sm[];
    float* Qs = sm;
    float* Ks = Qs + CB * LDK;
    float* Gs = Ks + CB * LDK;
    const size_t row0 = ((size_t)ci.y * H + h) * DK;  // element (r, c) at row0 + r H DK + c
    const size_t rstride = (size_t)H * DK;
    for (int idx = tid; idx < CB * DK; idx += 256) {
        const int r = idx / DK, c = idx % DK;
        const bool in = r < L;
        const size_t gi = row0 + r * rstride + c;
        Qs[r * LDK + c] = in ? to_f32(q[gi]) : 0.f;
        Ks[r * LDK + c] = in ? to_f32(k[gi]) : 0.f;
        Gs[r * LDK + c] = in ? g[gi] : 0.f;
    }
    __syncthreads();
    // a1: G = inclusive cumulative sum of g over the chunk's rows
    for (int c = tid; c < DK; c += 256) {
        float acc = 0.f;
        for (int r = 0; r < L; ++r) {
            acc += Gs[r * LDK + c];
            Gs[r * LDK + c] = acc;
            G[row0 + r * rstride + c] = acc;
        }
    }
    __syncthreads();
    float* Ac = Ar_out + ((size_t)cidx * H + h) * CB * CB;
    float* Pc = P_out + ((size_t)cidx * H + h) * CB * CB;
    // A[r][i] (i < r) and P[r][i] (i <= r): work item = (4 x 4 tile of
    // pairs, channels c = q4 mod 4), the four items of a tile on adjacent lanes
    for (int item = tid; item < kPairTiles * 4; item += 256) {
        const int tile = item >> 2, q4 = item & 3;
        int bi = 0;
        while ((bi + 1) * (bi + 2) / 2 <= tile) ++bi;
        const int bj = tile - bi * (bi + 1) / 2;
        const int r0 = 4 * bi, i0 = 4 * bj;
        float aA[4][4], aP[4][4];
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) aA[x][y] = aP[x][y] = 0.f;
#pragma unroll 2
        for (int c = q4; c < DK; c += 4) {
            float kr[4], qr[4], gr[4], ki[4], gi[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                kr[x] = Ks[(r0 + x) * LDK + c];
                qr[x] = Qs[(r0 + x) * LDK + c];
                gr[x] = Gs[(r0 + x) * LDK + c];
                ki[x] = Ks[(i0 + x) * LDK + c];
                gi[x] = Gs[(i0 + x) * LDK + c];
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    // pairs with i > r may overflow here; they are not kept
                    const float ke = ki[y] * __expf(gr[x] - gi[y]);
                    aA[x][y] += kr[x] * ke;
                    aP[x][y] += qr[x] * ke;
                }
        }
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) {
                aA[x][y] += __shfl_xor_sync(0xffffffffu, aA[x][y], 1);
                aA[x][y] += __shfl_xor_sync(0xffffffffu, aA[x][y], 2);
                aP[x][y] += __shfl_xor_sync(0xffffffffu, aP[x][y], 1);
                aP[x][y] += __shfl_xor_sync(0xffffffffu, aP[x][y], 2);
            }
        // lane q4 writes row r0 + q4 of the tile
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            if (x != q4) continue;
            const int r = r0 + x;
            float4 va, vp;
            float* pa = &va.x;
            float* pp = &vp.x;
#pragma unroll
            for (int y = 0; y < 4; ++y) {
                const int i = i0 + y;
                pa[y] = (r < L && i < r) ? aA[x][y] : 0.f;
                pp[y] = (r < L && i <= r) ? (rt ? round_tf32(aP[x][y]) : aP[x][y]) : 0.f;
            }
            *reinterpret_cast<float4*>(Ac + r * CB + i0) = va;
            *reinterpret_cast<float4*>(Pc + r * CB + i0) = vp;
        }
    }
    // the tiles above the diagonal are zero
    for (int idx = tid; idx < CB * CB / 4; idx += 256) {
        const int r = idx / (CB / 4), i4 = idx % (CB / 4);
        if (i4 > r / 4) {
            *reinterpret_cast<float4*>(Ac + r * CB + 4 * i4) = make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4*>(Pc + r * CB + 4 * i4) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    // Kb = K exp(G_last - G) and the right-hand sides b K exp(G)
    for (int idx = tid; idx < L * DK; idx += 256) {
        const int r = idx / DK, c = idx % DK;
        const size_t gi = row0 + r * rstride + c;
        const float gr = Gs[r * LDK + c], kr = Ks[r * LDK + c];
        const float kb = kr * __expf(Gs[(L - 1) * LDK + c] - gr);
        Kb[gi] = rt ? round_tf32(kb) : kb;
        Rk[gi] = beta[(size_t)(ci.y + r) * H + h] * kr * __expf(gr);
    }
}

template <int DK, typename TIn>
__global__ void __launch_bounds__(256) bwd_subst_kernel(
    const TIn* __restrict__ v, const float* __restrict__ beta, const float* __restrict__ Ain,
    const int4* __restrict__ info, int H, int dv, const uint32_t* status,
    float* __restrict__ W, float* __restrict__ Ut, bool rt) {  // rt: W rounded to tf32
    if (status_bad(status)) return;
    const int cidx = blockIdx.x, h = blockIdx.y;
    const int4 ci = info[cidx];
    const int L = ci.z;
    if (L <= 0) return;
    const int tid = threadIdx.x;
    extern __shared__ __align__(16) float sm[];
    const int lda = CB + 1, ldx = DK + dv + 4, nc = DK + dv;
    float* As = sm;
    float* X = As + CB * lda;
    float* bs = X + CB * ldx;
    const float* Ac = Ain + ((size_t)cidx * H + h) * CB * CB;
    for (int idx = tid; idx < CB * CB; idx += 256) As[(idx / CB) * lda + idx % CB] = Ac[idx];
    for (int r = tid; r < L; r += 256) bs[r] = beta[(size_t)(ci.y + r) * H + h];
    for (int idx = tid; idx < L * DK; idx += 256) {
        const int r = idx / DK, c = idx % DK;
        X[r * ldx + c] = W[((size_t)(ci.y + r) * H + h) * DK + c];
    }
    __syncthreads();
    for (int idx = tid; idx < L * dv; idx += 256) {
        const int r = idx / dv, j = idx % dv;
        X[r * ldx + DK + j] = bs[r] * to_f32(v[((size_t)(ci.y + r) * H + h) * dv + j]);
    }
    __syncthreads();
    // blocks of 16 rows: first the rows above the block (4 x 4 register
    // tiles, one task per 4 rows and 4 columns), then the block itself, one
    // column per thread
    for (int r0 = 0; r0 < L; r0 += 16) {
        if (r0 > 0) {
            for (int t = tid; t < 4 * (nc / 4); t += 256) {
                const int rq = t / (nc / 4), cq = t % (nc / 4);
                const int ra = r0 + 4 * rq;
                if (ra >= L) continue;
                float acc[4][4];
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
#pragma unroll 4
                for (int i = 0; i < r0; ++i) {
                    const float4 xv = *reinterpret_cast<const float4*>(X + i * ldx + 4 * cq);
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const float a = As[(ra + x) * lda + i];
                        acc[x][0] += a * xv.x; acc[x][1] += a * xv.y;
                        acc[x][2] += a * xv.z; acc[x][3] += a * xv.w;
                    }
                }
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    if (ra + x >= L) break;
                    float4* dst = reinterpret_cast<float4*>(X + (ra + x) * ldx + 4 * cq);
                    float4 cur = *dst;
                    const float b = bs[ra + x];
                    cur.x -= b * acc[x][0]; cur.y -= b * acc[x][1];
                    cur.z -= b * acc[x][2]; cur.w -= b * acc[x][3];
                    *dst = cur;
                }
            }
            __syncthreads();
        }
        const int r1 = min(r0 + 16, L);
        for (int col = tid; col < nc; col += 256) {
            for (int r = r0 + 1; r < r1; ++r) {
                float acc = 0.f;
                for (int i = r0; i < r; ++i) acc += As[r * lda + i] * X[i * ldx + col];
                X[r * ldx + col] -= bs[r] * acc;
            }
        }
        __syncthreads();
    }
    __syncthreads();
    for (int idx = tid; idx < L * DK; idx += 256) {
        const int r = idx / DK, c = idx % DK;
        W[((size_t)(ci.y + r) * H + h) * DK + c] = rt ? round_tf32(X[r * ldx + c]) : X[r * ldx + c];
    }
    for (int idx = tid; idx < L * dv; idx += 256) {
        const int r = idx / dv, j = idx % dv;
        Ut[((size_t)(ci.y + r) * H + h) * dv + j] = X[r * ldx + DK + j];
    }
}

template <int DK, typename TIn>
__global__ void __launch_bounds__(256) bwd_ef_kernel(
    const TIn* __restrict__ q, const TIn* __restrict__ dout, const float* __restrict__ G,
    const float* __restrict__ Pin, const float* __restrict__ W, const int4* __restrict__ info,
    int H, int dv, const uint32_t* status, float* __restrict__ E, float* __restrict__ F) {
    constexpr int LDQ = DK + 4, LDS = DVS + 4, LDA = CB + 1;
    if (status_bad(status)) return;
    const int cidx = blockIdx.x, h = blockIdx.y;
    const int4 ci = info[cidx];
    const int L = ci.z;
    if (L <= 0) return;
    const int tid = threadIdx.x;
    extern __shared__ __align__(16) float sm[];
    float* Qs = sm;                // Qt [C][LDQ]
    float* Ws = Qs + CB * LDQ;     // [C][LDQ]
    float* Ps = Ws + CB * LDQ;     // [C][LDA]
    float* Ds = Ps + CB * LDA;     // [C][LDS]
    float* Es = Ds + CB * LDS;     // [C][LDS]
    const float* Pc = Pin + ((size_t)cidx * H + h) * CB * CB;
    for (int idx = tid; idx < CB * CB; idx += 256) Ps[(idx / CB) * LDA + idx % CB] = Pc[idx];
    for (int idx = tid; idx < L * DK; idx += 256) {
        const int r = idx / DK, c = idx % DK;
        const size_t gi = ((size_t)(ci.y + r) * H + h) * DK + c;
        Qs[r * LDQ + c] = to_f32(q[gi]) * __expf(G[gi]);
        Ws[r * LDQ + c] = W[gi];
    }
    float* Fc = F + ((size_t)cidx * H + h) * DK * dv;
    for (int j0 = 0; j0 < dv; j0 += DVS) {
        __syncthreads();
        for (int idx = tid; idx < CB * DVS; idx += 256) {
            const int r = idx / DVS, j = idx % DVS;
            Ds[r * LDS + j] =
                r < L ? to_f32(dout[((size_t)(ci.y + r) * H + h) * dv + j0 + j]) : 0.f;
        }
        __syncthreads();
        // E rows 2 ip, 2 ip + 1, columns jq + 8 y (P[r][i] = 0 for i > r
        // inside a diagonal 4 x 4 tile, so both rows start at r = 2 ip)
        for (int t = tid; t < (CB / 2) * (DVS / 4); t += 256) {
            const int jq = t % (DVS / 4), ip = t / (DVS / 4);
            const int i = 2 * ip;
            float e0[4] = {0.f, 0.f, 0.f, 0.f}, e1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
            for (int r = i; r < L; ++r) {
                const float p0 = Ps[r * LDA + i], p1 = Ps[r * LDA + i + 1];
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    const float d = Ds[r * LDS + jq + 8 * y];
                    e0[y] += p0 * d;
                    e1[y] += p1 * d;
                }
            }
#pragma unroll
            for (int y = 0; y < 4; ++y) {
                const int j = jq + 8 * y;
                Es[i * LDS + j] = e0[y];
                Es[(i + 1) * LDS + j] = e1[y];
                if (i < L) E[((size_t)(ci.y + i) * H + h) * dv + j0 + j] = e0[y];
                if (i + 1 < L) E[((size_t)(ci.y + i + 1) * H + h) * dv + j0 + j] = e1[y];
            }
        }
        __syncthreads();
        // F by 4 x 4 register tiles (channels 4 c4 + x, columns 4 j4 + y)
        for (int t = tid; t < (DK / 4) * (DVS / 4); t += 256) {
            const int j4 = t % (DVS / 4), c4 = t / (DVS / 4);
            float acc[4][4];
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
            for (int r = 0; r < L; ++r) {
                const float4 q4 = *reinterpret_cast<const float4*>(Qs + r * LDQ + 4 * c4);
                const float4 w4 = *reinterpret_cast<const float4*>(Ws + r * LDQ + 4 * c4);
                const float4 d4 = *reinterpret_cast<const float4*>(Ds + r * LDS + 4 * j4);
                const float4 e4 = *reinterpret_cast<const float4*>(Es + r * LDS + 4 * j4);
                const float qv[4] = {q4.x, q4.y, q4.z, q4.w}, wv[4] = {w4.x, w4.y, w4.z, w4.w};
                const float dd[4] = {d4.x, d4.y, d4.z, d4.w}, ev[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) acc[x][y] += qv[x] * dd[y] - wv[x] * ev[y];
            }
#pragma unroll
            for (int x = 0; x < 4; ++x)
                *reinterpret_cast<float4*>(Fc + (size_t)(4 * c4 + x) * dv + j0 + 4 * j4) =
                    make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
        }
    }
}

size_t apkb_smem(int dk) { return sizeof(float) * (size_t)3 * CB * (dk + 1); }
size_t subst_smem(int dk, int dv) {
    return sizeof(float) * ((size_t)CB * (CB + 1) + (size_t)CB * (dk + dv + 4) + CB);
}
size_t ef_smem(int dk) {
    return sizeof(float) * ((size_t)2 * CB * (dk + 4) + (size_t)CB * (CB + 1) +
                            (size_t)2 * CB * (DVS + 4));
}

// ------------------------------------------------------------ b2: chains
// Both serial passes over a sequence's chunks, one block per (sequence, head,
// slice of 32 value columns), the state slice in shared memory:
//   forward  (first to last):  S_n -> states;  U = Ut - W S;
//                              S <- Diag(Gam) S + Kb^T U
//   backward (last to first):  dS' -> dSx;  X = Kb dS';  dU = E + X;
//                              dS <- Diag(Gam) dS' - W^T X + F
// Each chunk: W and Kb rows staged in shared memory with 16-byte loads, then
// two small products on 4-column register tiles (M1: rows 2 rg, 2 rg + 1;
// M2: channels 4 cg .. 4 cg + 3).  Shared: W, Kb [C][dk+4], state [dk][36],
// M1 result [C][36], Gam [dk].
constexpr int kChainDVS = 32;
constexpr int kLdA = 128 + 4;  // row stride of the staged W and Kb (floats)
constexpr int kLdS = kChainDVS + 4;

template <bool kBack, typename TIn>
__global__ void __launch_bounds__(256) chain_kernel(
    const float* __restrict__ Wg, const float* __restrict__ Kbg, const float* __restrict__ G,
    const float* __restrict__ S0, const float* EF_rows, const float* __restrict__ F,
    const int32_t* __restrict__ cu, int T, const int* __restrict__ chunk_start, int H, int dk,
    int dv, const uint32_t* status, float* rows_out, float* __restrict__ per_chunk,
    float* __restrict__ S_end) {
    // EF_rows and rows_out are the same buffer in the forward pass (Ut is
    // replaced by U): each element is read and then written by one thread
    if (status_bad(status)) return;
    const int s = blockIdx.x, h = blockIdx.y, j0 = blockIdx.z * kChainDVS;
    const int tid = threadIdx.x;
    const int t_begin = cu ? cu[s] : s * T;
    const int t_end = cu ? cu[s + 1] : (s + 1) * T;
    extern __shared__ __align__(16) float sm[];
    float* Ws = sm;                 // [C][kLdA]
    float* Kb = Ws + CB * kLdA;     // [C][kLdA]
    float* Ss = Kb + CB * kLdA;     // [dk][kLdS]
    float* Rs = Ss + 128 * kLdS;    // [C][kLdS]
    float* Gam = Rs + CB * kLdS;    // [dk]
    const size_t st_base = ((size_t)s * H + h) * dk * dv;
    for (int idx = tid; idx < dk * kChainDVS; idx += 256) {
        const int c = idx / kChainDVS, j = idx % kChainDVS;
        Ss[c * kLdS + j] = S0 ? S0[st_base + (size_t)c * dv + j0 + j] : 0.f;
    }
    const int jg = tid & 7, rg = tid >> 3;
    const int nch = (t_end - t_begin + CB - 1) / CB;
    const int dk4 = dk / 4;
    for (int step = 0; step < nch; ++step) {
        const int n = kBack ? nch - 1 - step : step;
        const int t0 = t_begin + n * CB;
        const int L = min(CB, t_end - t0);
        const size_t cbase = (((size_t)chunk_start[s] + n) * H + h) * dk * dv;
        __syncthreads();
        // the state entering this step: the forward's S_n, the backward's dS'
        for (int idx = tid; idx < dk * kChainDVS; idx += 256) {
            const int c = idx / kChainDVS, j = idx % kChainDVS;
            per_chunk[cbase + (size_t)c * dv + j0 + j] = Ss[c * kLdS + j];
        }
        for (int idx = tid; idx < L * dk4; idx += 256) {
            const int r = idx / dk4, c4 = idx % dk4;
            const size_t gi = ((size_t)(t0 + r) * H + h) * dk + 4 * c4;
            *reinterpret_cast<float4*>(Ws + r * kLdA + 4 * c4) =
                *reinterpret_cast<const float4*>(Wg + gi);
            *reinterpret_cast<float4*>(Kb + r * kLdA + 4 * c4) =
                *reinterpret_cast<const float4*>(Kbg + gi);
        }
        for (int c = tid; c < dk; c += 256) Gam[c] = expf(G[((size_t)(t0 + L - 1) * H + h) * dk + c]);
        __syncthreads();
        // M1: rows 2 rg, 2 rg + 1, columns 4 jg .. 4 jg + 3
        {
            const float* A1 = kBack ? Kb : Ws;
            float acc[2][4];
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
#pragma unroll 4
            for (int c = 0; c < dk; ++c) {
                const float a0 = A1[(2 * rg) * kLdA + c], a1 = A1[(2 * rg + 1) * kLdA + c];
                const float4 sv = *reinterpret_cast<const float4*>(Ss + c * kLdS + 4 * jg);
                acc[0][0] += a0 * sv.x; acc[0][1] += a0 * sv.y;
                acc[0][2] += a0 * sv.z; acc[0][3] += a0 * sv.w;
                acc[1][0] += a1 * sv.x; acc[1][1] += a1 * sv.y;
                acc[1][2] += a1 * sv.z; acc[1][3] += a1 * sv.w;
            }
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int r = 2 * rg + x;
                if (r < L) {
                    const size_t vi = ((size_t)(t0 + r) * H + h) * dv + j0 + 4 * jg;
                    const float4 base = *reinterpret_cast<const float4*>(EF_rows + vi);
                    float4 m;  // forward: U = Ut - W S; backward: X = Kb dS'
                    if (kBack) {
                        m = make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
                        *reinterpret_cast<float4*>(rows_out + vi) =
                            make_float4(base.x + m.x, base.y + m.y, base.z + m.z, base.w + m.w);
                    } else {
                        m = make_float4(base.x - acc[x][0], base.y - acc[x][1],
                                        base.z - acc[x][2], base.w - acc[x][3]);
                        *reinterpret_cast<float4*>(rows_out + vi) = m;
                    }
                    *reinterpret_cast<float4*>(Rs + r * kLdS + 4 * jg) = m;
                }
            }
        }
        __syncthreads();
        // M2: channels 4 cg .. 4 cg + 3, columns 4 jg .. 4 jg + 3
        for (int cg = rg; cg < dk4; cg += 32) {
            const float* A2 = kBack ? Ws : Kb;
            float acc[4][4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int c = 4 * cg + x;
                const float4 sv = *reinterpret_cast<const float4*>(Ss + c * kLdS + 4 * jg);
                float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
                if (kBack) f = *reinterpret_cast<const float4*>(F + cbase + (size_t)c * dv + j0 + 4 * jg);
                acc[x][0] = Gam[c] * sv.x + f.x; acc[x][1] = Gam[c] * sv.y + f.y;
                acc[x][2] = Gam[c] * sv.z + f.z; acc[x][3] = Gam[c] * sv.w + f.w;
            }
            const float sg = kBack ? -1.f : 1.f;
#pragma unroll 4
            for (int r = 0; r < L; ++r) {
                const float4 a4 = *reinterpret_cast<const float4*>(A2 + r * kLdA + 4 * cg);
                const float4 m4 = *reinterpret_cast<const float4*>(Rs + r * kLdS + 4 * jg);
                const float av[4] = {sg * a4.x, sg * a4.y, sg * a4.z, sg * a4.w};
                const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) acc[x][y] += av[x] * mv[y];
            }
            // every thread reads only its own tile of the state in M2
#pragma unroll
            for (int x = 0; x < 4; ++x)
                *reinterpret_cast<float4*>(Ss + (4 * cg + x) * kLdS + 4 * jg) =
                    make_float4(acc[x][0], acc[x][1], acc[x][2], acc[x][3]);
        }
    }
    __syncthreads();
    if (S_end) {
        for (int idx = tid; idx < dk * kChainDVS; idx += 256) {
            const int c = idx / kChainDVS, j = idx % kChainDVS;
            S_end[st_base + (size_t)c * dv + j0 + j] = Ss[c * kLdS + j];
        }
    }
}

size_t chain_smem() {
    return sizeof(float) * ((size_t)2 * CB * kLdA + (size_t)128 * kLdS + (size_t)CB * kLdS + 128);
}

// ------------------------------------------------------------ b3: solve
// One block per (chunk, head).  Shared: A without b [C][C+1], b [C], Y
// [C][dv+1], then U, dO, V slices [C][DVS+1].
template <typename TIn>
__global__ void __launch_bounds__(256) bwd_solve_kernel(
    const TIn* __restrict__ v, const TIn* __restrict__ dout, const float* __restrict__ Ain,
    const float* __restrict__ beta, const float* __restrict__ U,
    const float* __restrict__ dU, const int4* __restrict__ info, int H, int dv,
    const uint32_t* status, float* __restrict__ Y, float* __restrict__ dv_out,
    float* __restrict__ dAr, float* __restrict__ dP, float* __restrict__ dbB, bool rt) {
    // rt: Y is written rounded to tf32 (an operand of the tensor-core dense kernel)
    if (status_bad(status)) return;
    const int cidx = blockIdx.x, h = blockIdx.y;
    const int4 ci = info[cidx];
    const int L = ci.z;
    if (L <= 0) return;
    const int tid = threadIdx.x, nt = blockDim.x;
    extern __shared__ float sm[];
    const int lda = CB + 1, ldy = dv + 4, lds = DVS + 1;
    float* Ar = sm;
    float* bs = Ar + CB * lda;
    float* Ys = bs + CB;
    float* Us = Ys + CB * ldy;
    float* Ds = Us + CB * lds;
    float* Vs = Ds + CB * lds;
    {
        const float* Ac = Ain + ((size_t)cidx * H + h) * CB * CB;
        for (int idx = tid; idx < CB * CB; idx += nt) Ar[(idx / CB) * lda + idx % CB] = Ac[idx];
    }
    for (int r = tid; r < L; r += nt) bs[r] = beta[(size_t)(ci.y + r) * H + h];
    for (int idx = tid; idx < L * dv; idx += nt) {
        const int r = idx / dv, j = idx % dv;
        Ys[r * ldy + j] = dU[((size_t)(ci.y + r) * H + h) * dv + j];
    }
    __syncthreads();
    // (I + A)^T Y = dU by back substitution, Y_r = dU_r - sum_{i > r} b_i
    // A[i][r] Y_i, in blocks of 16 rows from the last: first the rows below
    // the block (4 x 4 register tiles), then the block, one column per thread
    for (int r1 = L; r1 > 0; r1 -= 16) {
        const int r0 = max(r1 - 16, 0);
        if (r1 < L) {
            for (int t = tid; t < 4 * (dv / 4); t += nt) {
                const int rq = t / (dv / 4), cq = t % (dv / 4);
                const int ra = r0 + 4 * rq;
                if (ra >= r1) continue;
                float acc[4][4];
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
#pragma unroll 4
                for (int i = r1; i < L; ++i) {
                    const float4 yv = *reinterpret_cast<const float4*>(Ys + i * ldy + 4 * cq);
                    const float bi = bs[i];
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const float a = bi * Ar[i * lda + ra + x];
                        acc[x][0] += a * yv.x; acc[x][1] += a * yv.y;
                        acc[x][2] += a * yv.z; acc[x][3] += a * yv.w;
                    }
                }
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    if (ra + x >= r1) break;
                    float4* dst = reinterpret_cast<float4*>(Ys + (ra + x) * ldy + 4 * cq);
                    float4 cur = *dst;
                    cur.x -= acc[x][0]; cur.y -= acc[x][1];
                    cur.z -= acc[x][2]; cur.w -= acc[x][3];
                    *dst = cur;
                }
            }
            __syncthreads();
        }
        for (int col = tid; col < dv; col += nt) {
            for (int r = r1 - 2; r >= r0; --r) {
                float acc = 0.f;
                for (int i = r + 1; i < r1; ++i) acc += bs[i] * Ar[i * lda + r] * Ys[i * ldy + col];
                Ys[r * ldy + col] -= acc;
            }
        }
        __syncthreads();
    }
    for (int idx = tid; idx < L * dv; idx += nt) {
        const int r = idx / dv, j = idx % dv;
        const size_t vi = ((size_t)(ci.y + r) * H + h) * dv + j;
        Y[vi] = rt ? round_tf32(Ys[r * ldy + j]) : Ys[r * ldy + j];
        dv_out[vi] = bs[r] * Ys[r * ldy + j];
    }
    // dA[i][j] = -(Y U^T)[i][j] (j < i), dP[i][j] = (dO U^T)[i][j] (j <= i):
    // thread (i = tid / 4, jl = tid % 4) takes j = jl + 4 m
    const int i = tid >> 2, jl = tid & 3;
    float accA[CB / 4], accP[CB / 4];
#pragma unroll
    for (int m = 0; m < CB / 4; ++m) accA[m] = accP[m] = 0.f;
    float yv = 0.f;
    for (int j0 = 0; j0 < dv; j0 += DVS) {
        __syncthreads();
        for (int idx = tid; idx < CB * DVS; idx += nt) {
            const int r = idx / DVS, j = idx % DVS;
            const bool in = r < L;
            const size_t vi = ((size_t)(ci.y + r) * H + h) * dv + j0 + j;
            Us[r * lds + j] = in ? U[vi] : 0.f;
            Ds[r * lds + j] = in ? to_f32(dout[vi]) : 0.f;
            Vs[r * lds + j] = in ? to_f32(v[vi]) : 0.f;
        }
        __syncthreads();
        if (i < L) {
            for (int j = 0; j < DVS; ++j) {
                const float y = Ys[i * ldy + j0 + j], d = Ds[i * lds + j];
#pragma unroll
                for (int m = 0; m < CB / 4; ++m) {
                    const float u = Us[(jl + 4 * m) * lds + j];
                    accA[m] += y * u;
                    accP[m] += d * u;
                }
            }
            for (int j = jl; j < DVS; j += 4) yv += Ys[i * ldy + j0 + j] * Vs[i * lds + j];
        }
    }
    const size_t cc = ((size_t)cidx * H + h) * CB * CB + (size_t)i * CB;
    float part = yv;
    if (i < L) {
#pragma unroll
        for (int m = 0; m < CB / 4; ++m) {
            const int j = jl + 4 * m;
            const float da = j < i ? -accA[m] : 0.f;
            part += da * Ar[i * lda + j];
            dAr[cc + j] = bs[i] * da;
            dP[cc + j] = j <= i ? accP[m] : 0.f;
        }
    }
    // the four threads of one row are adjacent lanes of one warp
    part += __shfl_xor_sync(0xffffffffu, part, 1);
    part += __shfl_xor_sync(0xffffffffu, part, 2);
    if (i < L && jl == 0) dbB[(size_t)(ci.y + i) * H + h] = part;
}

size_t solve_smem(int dv) {
    return sizeof(float) * ((size_t)CB * (CB + 1) + CB +
                            (size_t)CB * (dv + 4) + (size_t)3 * CB * (DVS + 1));
}

// ------------------------------------------------------------ b4: dense
// One block per (chunk, head).  dQt = dO S^T, YS = Y S^T, dKb = U dS'^T over
// the dv columns, and dGam = rowsum(S * dS').  Thread (rg = tid / 16, cl =
// tid % 16) owns rows 4 rg .. 4 rg + 3 and channels cl + 16 m.  Shared:
// S and dS' slices [DK][DVS+1], dO, Y, U slices [C][DVS+1].
template <int DK, typename TIn>
__global__ void __launch_bounds__(256) bwd_dense_kernel(
    const TIn* __restrict__ k, const TIn* __restrict__ dout, const float* __restrict__ G,
    const float* __restrict__ beta, const float* __restrict__ U, const float* __restrict__ Y,
    const float* __restrict__ states, const float* __restrict__ dSx,
    const float* __restrict__ dbB, const int4* __restrict__ info, int H, int dv,
    const uint32_t* status, float* __restrict__ dQt, float* __restrict__ dKt,
    float* __restrict__ dKb, float* __restrict__ dGam, float* __restrict__ dbeta) {
    constexpr int NM = DK / 16;
    constexpr int LD = DVS + 1;
    if (status_bad(status)) return;
    const int cidx = blockIdx.x, h = blockIdx.y;
    const int4 ci = info[cidx];
    const int L = ci.z;
    if (L <= 0) return;
    const int tid = threadIdx.x, nt = blockDim.x;
    const int rg = tid >> 4, cl = tid & 15;
    extern __shared__ float sm[];
    float* Ss = sm;             // [DK][LD]
    float* Xs = Ss + DK * LD;   // [DK][LD]
    float* Ds = Xs + DK * LD;   // [C][LD]
    float* Ysl = Ds + CB * LD;  // [C][LD]
    float* Us = Ysl + CB * LD;  // [C][LD]
    float aQ[4][NM], aY[4][NM], aK[4][NM];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int m = 0; m < NM; ++m) aQ[a][m] = aY[a][m] = aK[a][m] = 0.f;
    float gam = 0.f;
    const size_t cbase = ((size_t)cidx * H + h) * DK * dv;
    for (int j0 = 0; j0 < dv; j0 += DVS) {
        __syncthreads();
        for (int idx = tid; idx < DK * DVS; idx += nt) {
            const int c = idx / DVS, j = idx % DVS;
            Ss[c * LD + j] = states[cbase + (size_t)c * dv + j0 + j];
            Xs[c * LD + j] = dSx[cbase + (size_t)c * dv + j0 + j];
        }
        for (int idx = tid; idx < CB * DVS; idx += nt) {
            const int r = idx / DVS, j = idx % DVS;
            const bool in = r < L;
            const size_t vi = ((size_t)(ci.y + r) * H + h) * dv + j0 + j;
            Ds[r * LD + j] = in ? to_f32(dout[vi]) : 0.f;
            Ysl[r * LD + j] = in ? Y[vi] : 0.f;
            Us[r * LD + j] = in ? U[vi] : 0.f;
        }
        __syncthreads();
        if (tid < DK)
            for (int j = 0; j < DVS; ++j) gam += Ss[tid * LD + j] * Xs[tid * LD + j];
        for (int j = 0; j < DVS; ++j) {
            float d[4], y[4], u[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                d[a] = Ds[(4 * rg + a) * LD + j];
                y[a] = Ysl[(4 * rg + a) * LD + j];
                u[a] = Us[(4 * rg + a) * LD + j];
            }
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                const float sv = Ss[(cl + 16 * m) * LD + j], xv = Xs[(cl + 16 * m) * LD + j];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    aQ[a][m] += d[a] * sv;
                    aY[a][m] += y[a] * sv;
                    aK[a][m] += u[a] * xv;
                }
            }
        }
    }
    if (tid < DK) dGam[((size_t)cidx * H + h) * DK + tid] = gam;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int r = 4 * rg + a;
        float part = 0.f;
        if (r < L) {
            const size_t row = ((size_t)(ci.y + r) * H + h) * DK;
            const float b = beta[(size_t)(ci.y + r) * H + h];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                const int c = cl + 16 * m;
                dQt[row + c] = aQ[a][m];
                dKt[row + c] = -b * aY[a][m];
                dKb[row + c] = aK[a][m];
                part += to_f32(k[row + c]) * expf(G[row + c]) * aY[a][m];
            }
        }
        // the sixteen threads of one row group are one half of a warp
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (cl == 0 && r < L) {
            const size_t bi = (size_t)(ci.y + r) * H + h;
            dbeta[bi] = dbB[bi] - part;
        }
    }
}

size_t dense_smem(int dk) { return sizeof(float) * (size_t)(2 * dk + 3 * CB) * (DVS + 1); }

// ------------------------------------------------------------ b5: pairs
// One block per (chunk, head, 32 channels).  Thread (grp = tid / 32, lane)
// takes channel c0 + lane and the rows r = grp + 8 n: first as the later
// token of each pair (sums over i <= r), then as the earlier one (sums over
// r' >= r); then it adds the elementwise terms, and a reverse scan over the
// chunk's rows turns dG into dg.  Shared: Q, K, G, dG [C][32], b dA and dP
// [C][C+1], and the per-group sums for the last row [8][32].
template <typename TIn>
__global__ void __launch_bounds__(256) bwd_pair_kernel(
    const TIn* __restrict__ q, const TIn* __restrict__ k, const float* __restrict__ G,
    const float* __restrict__ dAr, const float* __restrict__ dP, const float* __restrict__ dQt,
    const float* __restrict__ dKt, const float* __restrict__ dKb,
    const float* __restrict__ dGam, const int4* __restrict__ info, int H, int dk,
    const uint32_t* status, float* __restrict__ dq, float* __restrict__ dk_out,
    float* __restrict__ dg, const int* __restrict__ slow) {
    // slow != NULL: only the chunks the tensor-core pair kernel left (flag 1)
    constexpr int NR = CB / 8;
    constexpr int LA = CB + 1;
    if (status_bad(status)) return;
    const int cidx = blockIdx.x, h = blockIdx.y, c0 = blockIdx.z * 32;
    const int4 ci = info[cidx];
    const int L = ci.z;
    if (L <= 0) return;
    if (slow && !slow[(size_t)cidx * H + h]) return;
    const int tid = threadIdx.x, lane = tid & 31, grp = tid >> 5;
    extern __shared__ float sm[];
    float* Qs = sm;              // [C][32]
    float* Ks = Qs + CB * 32;    // [C][32]
    float* Gs = Ks + CB * 32;    // [C][32]
    float* dGs = Gs + CB * 32;   // [C][32]
    float* sA = dGs + CB * 32;   // [C][LA]
    float* sP = sA + CB * LA;    // [C][LA]
    float* lastred = sP + CB * LA;  // [8][32]
    for (int idx = tid; idx < CB * 32; idx += 256) {
        const int r = idx / 32, c = idx % 32;
        const bool in = r < L;
        const size_t gi = ((size_t)(ci.y + r) * H + h) * dk + c0 + c;
        Qs[idx] = in ? to_f32(q[gi]) : 0.f;
        Ks[idx] = in ? to_f32(k[gi]) : 0.f;
        Gs[idx] = in ? G[gi] : 0.f;
    }
    const size_t cc = ((size_t)cidx * H + h) * CB * CB;
    for (int idx = tid; idx < CB * CB; idx += 256) {
        const int r = idx / CB, i = idx % CB;
        const bool in = r < L && i < L;
        sA[r * LA + i] = in ? dAr[cc + idx] : 0.f;
        sP[r * LA + i] = in ? dP[cc + idx] : 0.f;
    }
    __syncthreads();
    float rowA[NR], dQp[NR], col[NR];
#pragma unroll
    for (int n = 0; n < NR; ++n) {
        const int r = grp + 8 * n;
        float a = 0.f, p = 0.f, cs = 0.f;
        if (r < L) {
            const float gr = Gs[r * 32 + lane];
            // r as the later token: i < r (A) and i <= r (P)
#pragma unroll 4
            for (int i = 0; i < r; ++i) {
                const float e = Ks[i * 32 + lane] * __expf(gr - Gs[i * 32 + lane]);
                a += sA[r * LA + i] * e;
                p += sP[r * LA + i] * e;
            }
            p += sP[r * LA + r] * Ks[r * 32 + lane];
            // r as the earlier token: r' > r (A and P) and r' = r (P)
#pragma unroll 4
            for (int i = r + 1; i < L; ++i) {
                const float e = __expf(Gs[i * 32 + lane] - gr);
                cs += (sA[i * LA + r] * Ks[i * 32 + lane] + sP[i * LA + r] * Qs[i * 32 + lane]) * e;
            }
            cs += sP[r * LA + r] * Qs[r * 32 + lane];
        }
        rowA[n] = a;
        dQp[n] = p;
        col[n] = cs;
    }
    const float glast = Gs[(L - 1) * 32 + lane];
    float lastsum = 0.f;
#pragma unroll
    for (int n = 0; n < NR; ++n) {
        const int r = grp + 8 * n;
        if (r < L) {
            const size_t gi = ((size_t)(ci.y + r) * H + h) * dk + c0 + lane;
            const float gr = Gs[r * 32 + lane], qr = Qs[r * 32 + lane], kr = Ks[r * 32 + lane];
            const float eg = expf(gr), eb = expf(glast - gr);
            const float a = dQt[gi], b = dKt[gi], d = dKb[gi];
            dq[gi] = dQp[n] + a * eg;
            dk_out[gi] = rowA[n] + col[n] + b * eg + d * eb;
            dGs[r * 32 + lane] = kr * (rowA[n] - col[n]) + qr * dQp[n] + a * qr * eg +
                                 b * kr * eg - d * kr * eb;
            lastsum += d * kr * eb;
        }
    }
    lastred[grp * 32 + lane] = lastsum;
    __syncthreads();
    if (grp == 0) {
        float acc = expf(glast) * dGam[((size_t)cidx * H + h) * dk + c0 + lane];
#pragma unroll
        for (int g2 = 0; g2 < 8; ++g2) acc += lastred[g2 * 32 + lane];
        for (int r = L - 1; r >= 0; --r) {
            acc += dGs[r * 32 + lane];
            dg[((size_t)(ci.y + r) * H + h) * dk + c0 + lane] = acc;
        }
    }
}

size_t pair_smem() {
    return sizeof(float) * ((size_t)4 * CB * 32 + (size_t)2 * CB * (CB + 1) + 8 * 32);
}

template <typename Kern>
cudaError_t set_smem(Kern* kern, size_t bytes) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int DK, typename TIn>
cudaError_t launch_dense(const BwdBufs& b, const TIn* K, const TIn* DO, const float* beta,
                         int maxc, int H, int dv, float* db, cudaStream_t st) {
    const size_t sm = dense_smem(DK);
    cudaError_t e = set_smem(bwd_dense_kernel<DK, TIn>, sm);
    if (e != cudaSuccess) return e;
    bwd_dense_kernel<DK, TIn><<<dim3(maxc, H), 256, sm, st>>>(
        K, DO, b.w.G, beta, b.w.U, b.Y, b.w.states, b.dSx, b.dbB, b.w.chunk_info, H, dv,
        b.w.status, b.dQt, b.dKt, b.dKb, b.dGam, db);
    return cudaGetLastError();
}

template <int DK, typename TIn>
cudaError_t launch_intra3(const BwdBufs& b, const TIn* Q, const TIn* K, const TIn* V,
                          const TIn* DO, const float* g, const float* beta, int maxc, int H,
                          int dv, int total, bool tc, cudaStream_t st) {
    const Workspace& w = b.w;
    const dim3 grid(maxc, H);
    cudaError_t e;
    if (tc) {  // A and P as products; chunks outside the exponent range stay exact
        e = launch_bwd_apkb_tc<TIn>(Q, K, g, beta, w.chunk_info, total, maxc, H, w.status, b.slow,
                                    w.G, b.Ar, b.Pm, b.Kb, w.W, st);
        if (e != cudaSuccess) return e;
    }
    size_t sm = apkb_smem(DK);
    if ((e = set_smem(bwd_apkb_kernel<DK, TIn>, sm)) != cudaSuccess) return e;
    bwd_apkb_kernel<DK, TIn><<<grid, 256, sm, st>>>(Q, K, g, beta, w.chunk_info, H, w.status,
                                                    w.G, b.Ar, b.Pm, b.Kb, w.W, tc,
                                                    tc ? b.slow : nullptr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (tc) {
        e = launch_bwd_subst_tc<TIn>(V, beta, b.Ar, w.chunk_info, total, maxc, H, w.status, w.W,
                                     w.U, b.Tm, st);
    } else {
        sm = subst_smem(DK, dv);
        if ((e = set_smem(bwd_subst_kernel<DK, TIn>, sm)) != cudaSuccess) return e;
        bwd_subst_kernel<DK, TIn><<<grid, 256, sm, st>>>(V, beta, b.Ar, w.chunk_info, H, dv,
                                                         w.status, w.W, w.U, tc);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    if (tc)
        return launch_bwd_ef_tc<TIn>(Q, DO, w.G, b.Pm, w.W, w.chunk_info, total, maxc, H,
                                     w.status, b.E, b.F, st);
    sm = ef_smem(DK);
    if ((e = set_smem(bwd_ef_kernel<DK, TIn>, sm)) != cudaSuccess) return e;
    bwd_ef_kernel<DK, TIn><<<grid, 256, sm, st>>>(Q, DO, w.G, b.Pm, w.W, w.chunk_info, H, dv,
                                                  w.status, b.E, b.F);
    return cudaGetLastError();
}

template <typename TIn>
cudaError_t run_bwd(const BwdBufs& b, const void* q, const void* k, const void* v,
                    const float* g, const float* beta, const float* h0, const void* dout,
                    const float* dhT, const int32_t* cu, int T, int N, int H, int dk, int dv,
                    kda_dtype_t dt, int maxc, float* dq, float* dkk, float* dvv, float* dg,
                    float* db, float* dh0, cudaStream_t st) {
    const TIn* Q = static_cast<const TIn*>(q);
    const TIn* K = static_cast<const TIn*>(k);
    const TIn* V = static_cast<const TIn*>(v);
    const TIn* DO = static_cast<const TIn*>(dout);
    const Workspace& w = b.w;
    const int total = cu ? T : N * T;
    // dk = dv = 128: the chains, E/F and the dense products on the tensor cores
    const bool tc = dk == 128 && dv == 128 && bwd_tc_available();
    cudaError_t e;
    if (maxc > 0) {
        e = dk == 128 ? launch_intra3<128, TIn>(b, Q, K, V, DO, g, beta, maxc, H, dv, total, tc, st)
            : dk == 64 ? launch_intra3<64, TIn>(b, Q, K, V, DO, g, beta, maxc, H, dv, total, tc, st)
                       : launch_intra3<32, TIn>(b, Q, K, V, DO, g, beta, maxc, H, dv, total, tc, st);
        if (e != cudaSuccess) return e;
    }
    if (tc) {
        e = launch_bwd_chains_tc(w.W, b.Kb, w.G, h0, dhT, w.U, b.E, b.F, cu, T, N, H,
                                 w.chunk_start, w.status, w.states, b.dU, b.dSx, dh0, st);
        if (e != cudaSuccess) return e;
    } else {
        const size_t sm = chain_smem();
        const dim3 grid(N, H, dv / kChainDVS);
        if ((e = set_smem(chain_kernel<false, TIn>, sm)) != cudaSuccess) return e;
        if ((e = set_smem(chain_kernel<true, TIn>, sm)) != cudaSuccess) return e;
        // forward: U = Ut - W S (in place) and every chunk's entry state
        chain_kernel<false, TIn><<<grid, 256, sm, st>>>(w.W, b.Kb, w.G, h0, w.U, nullptr, cu, T,
                                                       w.chunk_start, H, dk, dv, w.status, w.U,
                                                       w.states, nullptr);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        // backward: dU, the exit-state gradient of every chunk, dS_0
        chain_kernel<true, TIn><<<grid, 256, sm, st>>>(w.W, b.Kb, w.G, dhT, b.E, b.F, cu, T,
                                                      w.chunk_start, H, dk, dv, w.status, b.dU,
                                                      b.dSx, dh0);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (maxc == 0) return cudaSuccess;
    if (tc) {
        e = launch_bwd_solve_tc<TIn>(V, DO, b.Ar, beta, w.U, b.dU, b.Tm, w.chunk_info, total, maxc,
                                     H, w.status, b.Y, dvv, b.dAr, b.dP, b.dbB, st);
        if (e != cudaSuccess) return e;
    } else {
        const size_t sm = solve_smem(dv);
        if ((e = set_smem(bwd_solve_kernel<TIn>, sm)) != cudaSuccess) return e;
        bwd_solve_kernel<TIn><<<dim3(maxc, H), 256, sm, st>>>(V, DO, b.Ar, beta, w.U, b.dU,
                                                             w.chunk_info, H, dv, w.status, b.Y,
                                                             dvv, b.dAr, b.dP, b.dbB, tc);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    e = tc ? launch_bwd_dense_tc<TIn>(K, DO, w.G, beta, w.U, b.Y, w.states, b.dSx, b.dbB,
                                      w.chunk_info, total, maxc, H, w.status, b.dQt, b.dKt,
                                      b.dKb, b.dGam, db, st)
        : dk == 128 ? launch_dense<128, TIn>(b, K, DO, beta, maxc, H, dv, db, st)
        : dk == 64 ? launch_dense<64, TIn>(b, K, DO, beta, maxc, H, dv, db, st)
                   : launch_dense<32, TIn>(b, K, DO, beta, maxc, H, dv, db, st);
    if (e != cudaSuccess) return e;
    if (tc) {  // the pair sums as products; chunks outside the exponent range stay exact
        e = launch_bwd_pair_tc<TIn>(Q, K, w.G, b.dAr, b.dP, b.dQt, b.dKt, b.dKb, b.dGam,
                                    w.chunk_info, total, maxc, H, w.status, b.slow, dq, dkk, dg,
                                    st);
        if (e != cudaSuccess) return e;
    }
    const size_t sm = pair_smem();
    if ((e = set_smem(bwd_pair_kernel<TIn>, sm)) != cudaSuccess) return e;
    bwd_pair_kernel<TIn><<<dim3(maxc, H, dk / 32), 256, sm, st>>>(
        Q, K, w.G, b.dAr, b.dP, b.dQt, b.dKt, b.dKb, b.dGam, w.chunk_info, H, dk, w.status, dq,
        dkk, dg, tc ? b.slow : nullptr);
    return cudaGetLastError();
}

// dg_head[row] = sum over the dk channels of dg[row, :] (one warp per row):
// the gradient of a head-uniform gate spread over the channels
__global__ void sum_channels_kernel(const float* __restrict__ x, long long rows, int dk,
                                    float* __restrict__ out) {
    const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float acc = 0.f;
    for (int c = lane; c < dk; c += 32) acc += x[row * dk + c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) out[row] = acc;
}

}  // namespace

size_t bwd_head_gate_workspace_bytes(int total, int N, int H, int dk, int dv) {
    return align_up(bwd_workspace_bytes(total, N, H, dk, dv)) +
           2 * align_up(sizeof(float) * (size_t)total * H * dk);
}

cudaError_t launch_bwd_head_gate(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, const float* h0, const void* dout,
                                 const float* dhT, const int32_t* cu, int T, int N, int H, int dk,
                                 int dv, kda_dtype_t dt, float* dq, float* dkk, float* dvv,
                                 float* dg_head, float* db, float* dh0, void* workspace,
                                 cudaStream_t st) {
    const int total = cu ? T : N * T;
    char* base = static_cast<char*>(workspace);
    const size_t off = align_up(bwd_workspace_bytes(total, N, H, dk, dv));
    float* g_full = reinterpret_cast<float*>(base + off);
    float* dg_full =
        reinterpret_cast<float*>(base + off + align_up(sizeof(float) * (size_t)total * H * dk));
    cudaError_t e = launch_spread_gate(g, total, H, dk, g_full, st);
    if (e == cudaSuccess)
        e = launch_bwd(q, k, v, g_full, beta, h0, dout, dhT, cu, T, N, H, dk, dv, dt, dq, dkk,
                       dvv, dg_full, db, dh0, workspace, st);
    if (e != cudaSuccess || total == 0) return e;
    const long long rows = (long long)total * H;
    sum_channels_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(dg_full, rows, dk,
                                                                              dg_head);
    return cudaGetLastError();
}

size_t bwd_workspace_bytes(int total, int N, int H, int dk, int dv) {
    return carve_bwd(nullptr, total, N, H, dk, dv).bytes;
}

cudaError_t launch_bwd(const void* q, const void* k, const void* v, const float* g,
                       const float* beta, const float* h0, const void* dout, const float* dhT,
                       const int32_t* cu, int T, int N, int H, int dk, int dv, kda_dtype_t dt,
                       float* dq, float* dkk, float* dvv, float* dg, float* db, float* dh0,
                       void* workspace, cudaStream_t st) {
    const int total = cu ? T : N * T;
    const BwdBufs b = carve_bwd(workspace, total, N, H, dk, dv);
    const Workspace& w = b.w;
    const int maxc = max_chunks(total, N, CB);
    cudaError_t e = cudaMemsetAsync(w.status, 0, sizeof(uint32_t), st);
    if (e == cudaSuccess)
        e = launch_build_chunk_table(cu, cu ? 1 : N, T, N, CB, maxc, w.status, w.chunk_start,
                                     w.chunk_info, st);
    if (e != cudaSuccess) return e;
    return dt == KDA_DTYPE_BF16
               ? run_bwd<__nv_bfloat16>(b, q, k, v, g, beta, h0, dout, dhT, cu, T, N, H, dk, dv,
                                        dt, maxc, dq, dkk, dvv, dg, db, dh0, st)
               : run_bwd<float>(b, q, k, v, g, beta, h0, dout, dhT, cu, T, N, H, dk, dv, dt,
                                maxc, dq, dkk, dvv, dg, db, dh0, st);
}

}  // namespace kda
