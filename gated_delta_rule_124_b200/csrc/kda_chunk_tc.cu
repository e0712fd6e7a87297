// KDA chunkwise prefill on the 5th-generation tensor cores (tcgen05 + TMEM,
// operands staged by TMA), bf16 q/k/v/o, fp32 g/beta/state, dk = dv = 128,
// chunk C = 64.  One CTA of 128 threads owns one (sequence, head) and walks its
// chunks in order, carrying the fp32 state S (128 x 128) in tensor memory.
//
// Kimi Linear (aiwiki.ai), "The constrained DPLR form and the chunkwise
// algorithm": inside a chunk the per-token corrections are gathered into a WY
// form and the unit-triangular system is solved once (UT transform); between
// chunks the state is carried recurrently.  Per chunk (rows r, i; G = in-chunk
// inclusive cumsum of g; Gam = exp(G)):
//
//   A[r,i] = b_r sum_c k_rc k_ic exp(G_rc - G_ic)  (i < r)
//   P[r,i] = sum_c q_rc k_ic exp(G_rc - G_ic)      (i <= r)
//   Tb     = (I + A)^{-1} diag(b)                  (UT transform, CUDA cores)
//   [W | Ut] = Tb [K * Gam | V]                    (one MMA, N = 256)
//   X      = [W ; Q * Gam] S                       (one MMA, M = 128)
//   U      = Ut - X[0:64]                          (epilogue)
//   O      = X[64:128] + [0 ; P] U                 (MMA accumulate)
//   S     <- Diag(Gam_last) S + (K * exp(G_last - G))^T U
//
// A and P come from one M = 128 MMA [b K * E ; Q * E] (K * E^-1)^T with
// E = exp(G - Gm) and a per-channel reference Gm = max_r G - 80: every factor
// is then within exp(+-80) whenever the chunk's per-channel log-decay range is
// at most 160 (for the gates of all benchmark configurations it is below 100).
// A chunk outside that range takes an exact CUDA-core evaluation of A and P
// instead (exp of each difference), so any finite g is handled.
//
// Shared-memory operand tiles use the 128-byte swizzle; a [rows][128] tile of
// bf16 is two 64-column halves, each rows x 128 B, and serves as a K-major
// operand (contraction over its 128 columns) or as an MN-major one
// (contraction over its rows).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "kda_chunk_tc.cuh"
#include "kda_common.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = 64;          // chunk rows
constexpr int D = 128;         // dk = dv
constexpr int NT = 128;        // threads per CTA
constexpr float kRef = 80.f;   // exponent headroom of the A / P factors
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s bound on every wait

// shared-memory map (byte offsets from a 1024-aligned base)
constexpr uint32_t OFF_K = 0;          // K tile -> K*E^-1 (RAP) -> [garbage ; P] (PM)
constexpr uint32_t OFF_WQ = 16384;     // [W kb0 | Q kb0 | W kb1 | Q kb1]  (Q -> Q*Gam)
constexpr uint32_t OFF_KG = 49152;     // K*Gam (then V directly after it)
constexpr uint32_t OFF_V = 65536;      // V tile
constexpr uint32_t OFF_G = 81920;      // g -> G (fp32 [64][128]) -> Tb (bf16) + T (fp32)
constexpr uint32_t OFF_LAP = 114688;   // [b K*E ; Q*E] per 64-col half (128 rows) -> A, P fp32
constexpr uint32_t OFF_KT = 147456;    // K * exp(G_last - G)
constexpr uint32_t OFF_SB = 163840;    // S (bf16, [dk][dv], MN-major B operand)
constexpr uint32_t OFF_UB = 196608;    // U (bf16, [token][dv], MN-major B operand)
constexpr uint32_t OFF_BETA = 212992;  // 64 floats
constexpr uint32_t OFF_GM = OFF_BETA + 256;    // 128 floats: Gm
constexpr uint32_t OFF_EGM = OFF_GM + 512;     // exp(Gm)
constexpr uint32_t OFF_EGLM = OFF_EGM + 512;   // exp(G_last - Gm)
constexpr uint32_t OFF_GC = OFF_EGLM + 512;    // exp(G_last)
constexpr uint32_t OFF_GL = OFF_GC + 512;      // G_last
constexpr uint32_t OFF_BAR = OFF_GL + 512;     // 2 mbarriers + tmem base
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack

// TMEM columns (512 allocated)
constexpr uint32_t TM_W = 0;      // W (cols 0-127) | Ut (128-255); later K~^T U (0-127)
constexpr uint32_t TM_UT = 128;
constexpr uint32_t TM_X = 256;    // A|P (256-319) early; then [W;QGam] S and O
constexpr uint32_t TM_S = 384;    // fp32 state

constexpr uint32_t TX_BYTES = 3 * 16384 + 32768;

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
    return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                      pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
}
__device__ __forceinline__ void unpack8(uint4 u, float (&x)[8]) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(p[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}
// bf16 element (row, col) of a [rows][128] swizzled tile whose two 64-column
// halves are `half_stride` bytes apart.
__device__ __forceinline__ float tile_elem(const uint8_t* base, uint32_t half_stride, int row,
                                           int col) {
    const uint8_t* p = base + (col >> 6) * half_stride + sw128_off(row, (col & 63) >> 3) +
                       (col & 7) * 2;
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
}

struct TcParams {
    const float* beta;
    const float* h0;
    const int32_t* cu;
    int T;
    int H;
    const uint32_t* status;
    uint32_t* status_out;
    __nv_bfloat16* o;
    float* hN;
};

__global__ void __launch_bounds__(NT, 1)
    chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                        const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv,
                        const __grid_constant__ CUtensorMap tmg, const TcParams p) {
    if (status_bad(p.status)) return;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    float* sbeta = reinterpret_cast<float*>(sm + OFF_BETA);
    float* sGm = reinterpret_cast<float*>(sm + OFF_GM);
    float* seGm = reinterpret_cast<float*>(sm + OFF_EGM);
    float* seGLm = reinterpret_cast<float*>(sm + OFF_EGLM);
    float* sGC = reinterpret_cast<float*>(sm + OFF_GC);
    float* sGL = reinterpret_cast<float*>(sm + OFF_GL);
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint64_t* bar_mma = bar_tma + 1;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + OFF_BAR + 16);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int seq = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int t_begin = p.cu ? p.cu[seq] : seq * p.T;
    const int t_end = p.cu ? p.cu[seq + 1] : (seq + 1) * p.T;

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem;
    const uint32_t tlane = static_cast<uint32_t>(32 * warp) << 16;  // this warp's lane quarter
    bool failed = false;
    uint32_t mma_phase = 0;

    // ---- initial state: fp32 into TMEM (row c = lane c), bf16 copy into Sb
    {
        const int c = tid;
        const float* src = p.h0 ? p.h0 + (((size_t)seq * p.H + h) * D + c) * D : nullptr;
#pragma unroll 1
        for (int piece = 0; piece < 4; ++piece) {
            uint32_t r[32];
            float x[32];
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                float4 v = src ? *reinterpret_cast<const float4*>(src + piece * 32 + i)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
                x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(x[i]);
            tmem_st32(tbase + tlane + TM_S + piece * 32, r);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                float y[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) y[i] = x[q4 * 8 + i];
                const int col = piece * 32 + q4 * 8;
                *reinterpret_cast<uint4*>(sm + OFF_SB + (col >> 6) * 16384 +
                                          sw128_off(c, (col & 63) >> 3)) = pack8(y);
            }
        }
        tmem_wait_st();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    int n = 0;
    for (int t0 = t_begin; t0 < t_end && !failed; t0 += C, ++n) {
        const int L = min(C, t_end - t0);
        // ---------------------------------------------------------- loads
        if (tid == 0) {
            mbar_arrive_expect_tx(bar_tma, TX_BYTES);
            tma_load_3d(sm + OFF_K, &tmk, bar_tma, 0, h, t0);
            tma_load_3d(sm + OFF_K + 8192, &tmk, bar_tma, 64, h, t0);
            tma_load_3d(sm + OFF_WQ + 8192, &tmq, bar_tma, 0, h, t0);
            tma_load_3d(sm + OFF_WQ + 16384 + 8192, &tmq, bar_tma, 64, h, t0);
            tma_load_3d(sm + OFF_V, &tmv, bar_tma, 0, h, t0);
            tma_load_3d(sm + OFF_V + 8192, &tmv, bar_tma, 64, h, t0);
            tma_load_3d(sm + OFF_G, &tmg, bar_tma, 0, h, t0);
        }
        if (tid < C) sbeta[tid] = tid < L ? p.beta[(size_t)(t0 + tid) * p.H + h] : 0.f;
        bool ok = mbar_wait(bar_tma, n & 1, kWaitNs);
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        // ---------------------------- E1: cumulative log-gate, per channel
        bool slow;
        {
            const int c = tid;
            float* g = reinterpret_cast<float*>(sm + OFF_G);
            float G = 0.f, gmax = -INFINITY, gmin = INFINITY;
            for (int r = 0; r < L; ++r) {
                G += g[r * D + c];
                g[r * D + c] = G;
                gmax = fmaxf(gmax, G);
                gmin = fminf(gmin, G);
            }
            const float Gm = gmax - kRef;
            sGm[c] = Gm;
            seGm[c] = expf(Gm);
            seGLm[c] = expf(G - Gm);
            sGC[c] = expf(G);
            sGL[c] = G;
            const bool s = !(gmax - gmin <= 2.f * kRef) || !(gmax <= 60.f);
            slow = __syncthreads_or(s);
        }
        // ---------------- exact A and P on CUDA cores (rare: extreme decay)
        if (slow) {
            const float* G = reinterpret_cast<const float*>(sm + OFF_G);
            float* Af = reinterpret_cast<float*>(sm + OFF_LAP);
            float* Pf = Af + C * C;
            for (int idx = tid; idx < C * C; idx += NT) {
                const int r = idx >> 6, i = idx & 63;
                float a = 0.f, pp = 0.f;
                if (r < L && i <= r) {
                    for (int c = 0; c < D; ++c) {
                        const float e = expf(G[r * D + c] - G[i * D + c]);
                        const float ki = tile_elem(sm + OFF_K, 8192, i, c);
                        a += tile_elem(sm + OFF_K, 8192, r, c) * ki * e;
                        pp += tile_elem(sm + OFF_WQ + 8192, 16384, r, c) * ki * e;
                    }
                }
                Af[idx] = (i < r) ? sbeta[r] * a : 0.f;
                Pf[idx] = pp;
            }
            __syncthreads();
        }
        // ------------------------------ E2: operand tiles, row-parallel
        {
            const float* G = reinterpret_cast<const float*>(sm + OFF_G);
#pragma unroll 1
            for (int s = 0; s < 8; ++s) {
                const int it = tid + NT * s;
                const int r = it >> 4, j = it & 15, kb = j >> 3, ch = j & 7, c0 = 8 * j;
                const uint32_t o64 = sw128_off(r, ch);
                uint8_t* pk = sm + OFF_K + kb * 8192 + o64;
                uint8_t* pq = sm + OFF_WQ + kb * 16384 + 8192 + o64;
                float lb[8], lq[8], rk[8], kg[8], qg[8], kt[8];
                if (r < L) {
                    float k8[8], q8[8];
                    unpack8(*reinterpret_cast<const uint4*>(pk), k8);
                    unpack8(*reinterpret_cast<const uint4*>(pq), q8);
                    const float b = sbeta[r];
                    if (!slow) {
                        // all factors within exp(+-80): products stay accurate
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int c = c0 + i;
                            const float x = G[r * D + c] - sGm[c];
                            const float E = expf(x), Ei = expf(-x);
                            lb[i] = b * k8[i] * E;
                            lq[i] = q8[i] * E;
                            rk[i] = k8[i] * Ei;
                            kg[i] = k8[i] * E * seGm[c];
                            qg[i] = q8[i] * E * seGm[c];
                            kt[i] = k8[i] * Ei * seGLm[c];
                        }
                    } else {
                        // extreme decay: Gam and exp(G_last - G) evaluated directly
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int c = c0 + i;
                            const float Gr = G[r * D + c];
                            const float gam = expf(Gr);
                            lb[i] = lq[i] = rk[i] = 0.f;
                            kg[i] = k8[i] * gam;
                            qg[i] = q8[i] * gam;
                            kt[i] = k8[i] * expf(sGL[c] - Gr);
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) lb[i] = lq[i] = rk[i] = kg[i] = qg[i] = kt[i] = 0.f;
                }
                if (!slow) {
                    *reinterpret_cast<uint4*>(sm + OFF_LAP + kb * 16384 + o64) = pack8(lb);
                    *reinterpret_cast<uint4*>(sm + OFF_LAP + kb * 16384 + 8192 + o64) =
                        pack8(lq);
                }
                *reinterpret_cast<uint4*>(pk) = pack8(rk);
                *reinterpret_cast<uint4*>(pq) = pack8(qg);
                *reinterpret_cast<uint4*>(sm + OFF_KG + kb * 8192 + o64) = pack8(kg);
                *reinterpret_cast<uint4*>(sm + OFF_KT + kb * 8192 + o64) = pack8(kt);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ------------------------------------------------ A, P (M=128, N=64)
        if (!slow) {
            if (tid == 0) {
                constexpr uint32_t id = idesc_bf16_f32(128, 64, false, false);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const int kb = ks >> 2, kk = ks & 3;
                    mma_bf16(tbase + TM_X,
                             sdesc_sw128(sbase + OFF_LAP + kb * 16384 + kk * 32, 16, 1024),
                             sdesc_sw128(sbase + OFF_K + kb * 8192 + kk * 32, 16, 1024), id,
                             ks > 0);
                }
                mma_commit(bar_mma);
            }
            ok = mbar_wait(bar_mma, mma_phase & 1, kWaitNs);
            ++mma_phase;
            if (__syncthreads_or(!ok)) {
                failed = true;
                break;
            }
            tc_fence_after();
        }
        // ---------------- A -> fp32 (rows 0-63), P -> bf16 PM rows 64-127
        {
            float* Af = reinterpret_cast<float*>(sm + OFF_LAP);
            const float* Pf = Af + C * C;
            const int m = tid;  // TMEM lane == row of the 128-row result
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t v[32];
                if (!slow) {
                    tmem_ld32(tbase + tlane + TM_X + half * 32, v);
                    tmem_wait_ld();
                }
                if (m < C) {
                    if (!slow) {
                        const int r = m;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int col = half * 32 + i;
                            Af[r * C + col] = (r < L && col < r) ? __uint_as_float(v[i]) : 0.f;
                        }
                    }
                } else {
                    const int r = m - C;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        float y[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int col = half * 32 + q4 * 8 + i;
                            const float val = slow ? Pf[r * C + col] : __uint_as_float(v[q4 * 8 + i]);
                            y[i] = (r < L && col <= r) ? val : 0.f;
                        }
                        const int col = half * 32 + q4 * 8;
                        *reinterpret_cast<uint4*>(sm + OFF_K + sw128_off(m, col >> 3)) = pack8(y);
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ----------------------- UT transform: T = (I + A)^{-1}, blocked 16x16
        {
            const float* Af = reinterpret_cast<const float*>(sm + OFF_LAP);
            float* Mf = reinterpret_cast<float*>(sm + OFF_LAP) + C * C;  // scratch
            float* Tf = reinterpret_cast<float*>(sm + OFF_G + 16384);
            if (tid < C) {
                const int I = tid >> 4, jj = tid & 15, col = 16 * I + jj;
                float x[16];
#pragma unroll
                for (int rr = 0; rr < 16; ++rr) {
                    const int row = 16 * I + rr;
                    float val = (rr == jj) ? 1.f : 0.f;
#pragma unroll
                    for (int ii = 0; ii < rr; ++ii)
                        val -= (ii >= jj) ? Af[row * C + 16 * I + ii] * x[ii] : 0.f;
                    x[rr] = (rr >= jj) ? val : 0.f;
                    Tf[row * C + col] = x[rr];
                }
            }
            __syncthreads();
#pragma unroll 1
            for (int d = 1; d < 4; ++d) {
                const int nel = (4 - d) * 256;
                // M_IJ = sum_{K=J}^{I-1} A_IK T_KJ, I = J + d
                for (int e = tid; e < nel; e += NT) {
                    const int J = e >> 8, a = (e >> 4) & 15, b = e & 15, I = J + d;
                    float acc = 0.f;
                    for (int x = 16 * J; x < 16 * I; ++x)
                        acc += Af[(16 * I + a) * C + x] * Tf[x * C + 16 * J + b];
                    Mf[e] = acc;
                }
                __syncthreads();
                // T_IJ = -T_II M_IJ
                for (int e = tid; e < nel; e += NT) {
                    const int J = e >> 8, a = (e >> 4) & 15, b = e & 15, I = J + d;
                    float acc = 0.f;
#pragma unroll
                    for (int y = 0; y < 16; ++y)
                        acc += Tf[(16 * I + a) * C + 16 * I + y] * Mf[(J << 8) + y * 16 + b];
                    Tf[(16 * I + a) * C + 16 * J + b] = -acc;
                }
                __syncthreads();
            }
            // Tb = T diag(beta) -> bf16, K-major rows of 64 (rows 0-63)
            for (int e = tid; e < C * 8; e += NT) {
                const int r = e >> 3, ch = e & 7;
                float y[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int col = ch * 8 + i;
                    y[i] = (col <= r) ? Tf[r * C + col] * sbeta[col] : 0.f;
                }
                *reinterpret_cast<uint4*>(sm + OFF_G + sw128_off(r, ch)) = pack8(y);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ------------------------- [W | Ut] = Tb [K*Gam | V]   (M=128, N=256)
        if (tid == 0) {
            constexpr uint32_t id = idesc_bf16_f32(128, 256, false, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tbase + TM_W, sdesc_sw128(sbase + OFF_G + ks * 32, 16, 1024),
                         sdesc_sw128(sbase + OFF_KG + ks * 2048, 8192, 1024), id, ks > 0);
            mma_commit(bar_mma);
        }
        ok = mbar_wait(bar_mma, mma_phase & 1, kWaitNs);
        ++mma_phase;
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        tc_fence_after();
        // W (rows 0-63) -> bf16 into the W rows of the [W ; Q*Gam] tile
        if (warp < 2) {
            const int r = tid;
#pragma unroll 1
            for (int piece = 0; piece < 4; ++piece) {
                uint32_t v[32];
                tmem_ld32(tbase + tlane + TM_W + piece * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float y[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) y[i] = __uint_as_float(v[q4 * 8 + i]);
                    const int col = piece * 32 + q4 * 8;
                    *reinterpret_cast<uint4*>(sm + OFF_WQ + (col >> 6) * 16384 +
                                              sw128_off(r, (col & 63) >> 3)) = pack8(y);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ------------------------------- X = [W ; Q*Gam] S   (M=128, N=128)
        if (tid == 0) {
            constexpr uint32_t id = idesc_bf16_f32(128, 128, false, true);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int kb = ks >> 2, kk = ks & 3;
                mma_bf16(tbase + TM_X, sdesc_sw128(sbase + OFF_WQ + kb * 16384 + kk * 32, 16, 1024),
                         sdesc_sw128(sbase + OFF_SB + ks * 2048, 16384, 1024), id, ks > 0);
            }
            mma_commit(bar_mma);
        }
        ok = mbar_wait(bar_mma, mma_phase & 1, kWaitNs);
        ++mma_phase;
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        tc_fence_after();
        // U = Ut - W S  (rows 0-63) -> bf16 Ub
        if (warp < 2) {
            const int r = tid;
#pragma unroll 1
            for (int piece = 0; piece < 4; ++piece) {
                uint32_t a[32], b[32];
                tmem_ld32(tbase + tlane + TM_UT + piece * 32, a);
                tmem_ld32(tbase + tlane + TM_X + piece * 32, b);
                tmem_wait_ld();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float y[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        y[i] = __uint_as_float(a[q4 * 8 + i]) - __uint_as_float(b[q4 * 8 + i]);
                    const int col = piece * 32 + q4 * 8;
                    *reinterpret_cast<uint4*>(sm + OFF_UB + (col >> 6) * 8192 +
                                              sw128_off(r, (col & 63) >> 3)) = pack8(y);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ---- O = X[64:] + [. ; P] U  (accumulate);  K~^T U -> TM_W  (M=128)
        if (tid == 0) {
            constexpr uint32_t idP = idesc_bf16_f32(128, 128, false, true);
            constexpr uint32_t idK = idesc_bf16_f32(128, 128, true, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tbase + TM_X, sdesc_sw128(sbase + OFF_K + ks * 32, 16, 1024),
                         sdesc_sw128(sbase + OFF_UB + ks * 2048, 8192, 1024), idP, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tbase + TM_W, sdesc_sw128(sbase + OFF_KT + ks * 2048, 8192, 1024),
                         sdesc_sw128(sbase + OFF_UB + ks * 2048, 8192, 1024), idK, ks > 0);
            mma_commit(bar_mma);
        }
        ok = mbar_wait(bar_mma, mma_phase & 1, kWaitNs);
        ++mma_phase;
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        tc_fence_after();
        // S <- Gam_last * S + K~^T U  (every lane = state row c); O rows out
        {
            const int c = tid;
            const float gc = sGC[c];
#pragma unroll 1
            for (int piece = 0; piece < 4; ++piece) {
                uint32_t a[32], s[32];
                tmem_ld32(tbase + tlane + TM_W + piece * 32, a);
                tmem_ld32(tbase + tlane + TM_S + piece * 32, s);
                tmem_wait_ld();
                float x[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    x[i] = fmaf(gc, __uint_as_float(s[i]), __uint_as_float(a[i]));
                    s[i] = __float_as_uint(x[i]);
                }
                tmem_st32(tbase + tlane + TM_S + piece * 32, s);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float y[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) y[i] = x[q4 * 8 + i];
                    const int col = piece * 32 + q4 * 8;
                    *reinterpret_cast<uint4*>(sm + OFF_SB + (col >> 6) * 16384 +
                                              sw128_off(c, (col & 63) >> 3)) = pack8(y);
                }
            }
            tmem_wait_st();
            if (warp >= 2) {
                const int r = tid - C;
#pragma unroll 1
                for (int piece = 0; piece < 4; ++piece) {
                    uint32_t v[32];
                    tmem_ld32(tbase + tlane + TM_X + piece * 32, v);
                    tmem_wait_ld();
                    if (r < L) {
                        __nv_bfloat16* dst =
                            p.o + ((size_t)(t0 + r) * p.H + h) * D + piece * 32;
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            float y[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) y[i] = __uint_as_float(v[q4 * 8 + i]);
                            *reinterpret_cast<uint4*>(dst + q4 * 8) = pack8(y);
                        }
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (!failed && p.hN) {
        const int c = tid;
        float* dst = p.hN + (((size_t)seq * p.H + h) * D + c) * D;
#pragma unroll 1
        for (int piece = 0; piece < 4; ++piece) {
            uint32_t s[32];
            tmem_ld32(tbase + tlane + TM_S + piece * 32, s);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4*>(dst + piece * 32 + i) =
                    make_float4(__uint_as_float(s[i]), __uint_as_float(s[i + 1]),
                                __uint_as_float(s[i + 2]), __uint_as_float(s[i + 3]));
        }
    }
    if (failed) {
        // Let any copy or MMA still in flight land before the memory is given
        // back (bounded again), then report.
        if (tid == 0) {
            mbar_wait(bar_tma, n & 1, kWaitNs);
            atomicOr(p.status_out, STATUS_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

// ------------------------------------------------------------------- host
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }();
    return fn;
}

// [total][H][128] tensor, box = box0 channels x 1 head x 64 tokens.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int total,
              int H, int box0, CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)total};
    cuuint64_t strides[2] = {(cuuint64_t)D * esize, (cuuint64_t)D * esize * H};
    cuuint32_t box[3] = {(cuuint32_t)box0, 1, (cuuint32_t)C};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

bool tc_path_available() { return encode_fn() != nullptr; }

cudaError_t launch_chunk_fwd_tc(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, const float* h0, const int32_t* cu_seqlens,
                                int T, int N, int H, const int* chunk_start, uint32_t* status,
                                void* o, float* hN, cudaStream_t st) {
    (void)chunk_start;
    const int total = cu_seqlens ? T : N * T;
    if (total == 0) {
        // nothing to read; the state passes through
        if (hN) {
            if (h0) return cudaMemcpyAsync(hN, h0, sizeof(float) * (size_t)N * H * D * D,
                                           cudaMemcpyDeviceToDevice, st);
            return cudaMemsetAsync(hN, 0, sizeof(float) * (size_t)N * H * D * D, st);
        }
        return cudaSuccess;
    }
    CUtensorMap mq, mk, mv, mg;
    if (!make_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, total, H, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, total, H, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, total, H, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, total, H, 128,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_fwd_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    TcParams prm{beta, h0, cu_seqlens, T, H, status, status, (__nv_bfloat16*)o, hN};
    chunk_fwd_tc_kernel<<<N * H, NT, SMEM_BYTES, st>>>(mq, mk, mv, mg, prm);
    return cudaGetLastError();
}

}  // namespace kda
