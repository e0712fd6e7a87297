// The contractions of the chunked KDA backward on the 5th-generation tensor
// cores (tcgen05, kind::tf32, accumulators in tensor memory), for dk = dv =
// 128 and chunks of 64 tokens: the two serial chains, E and F, and the dense
// products after the back substitution.  See kda_bwd.cu for the derivation
// (Kimi Linear (aiwiki.ai), "The constrained DPLR form and the chunkwise
// algorithm", differentiated).  Per (sequence, head) and half of the value
// columns, over the chunks of the sequence:
//
//   forward  (first to last):  S_n -> per_chunk;  U = Ut - W S;
//                              S <- Diag(Gam) S + Kb^T U
//   backward (last to first):  dS' -> per_chunk;  X = Kb dS';  dU = E + X;
//                              dS <- Diag(Gam) dS' - W^T X + F
//
// Each step is two products: M1 = A1 St (A1 = W forward, Kb backward; M = 64
// tokens padded to 128 rows, K = 128 channels, N = 64 columns) and M2 =
// A2^T R (A2 = Kb forward, W backward; R = U forward, X backward; M = 128
// channels, K = 64 tokens, N = 64), with the combination of M1 with the per-token rows between them
// and the state update after M2 on the CUDA cores in fp32.  The operands are
// fp32 in shared memory, read by the tensor cores as tf32 (10-bit mantissa);
// the state is carried in fp32 registers.
//
// Shared memory (one fp32 tile row of 32 values is one 128-byte swizzle row):
// per stage (double-buffered across steps) the chunk's W and Kb [64 tokens]
// [128 channels], loaded by TMA as four 32-channel blocks of 8 KB -- A1 as a
// K-major operand of M1 (the 128-byte swizzle with 16-byte granules) and A2
// as an MN-major operand (M = channel) of M2; the state St [128 channels][64
// columns] as two 32-column blocks of 16 KB (MN-major B of M1); the combined
// rows R [64 tokens][64 columns] as two blocks of 8 KB (MN-major B of M2).
// An MN-major tf32 operand must use the 128-byte swizzle with 32-byte
// granules (4-row atoms), so A2, St and R are written in that layout: each
// pass loads its A2 tile through a tensor map of that swizzle and its A1 tile
// through one of the 16-byte-granule swizzle.  M1's padding rows 64-127 read
// the next 8 KB of shared memory (the following block or tile); their results
// are never read.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>
#include <string.h>

#include "kda_common.cuh"
#include "kda_sm100.cuh"
#include "kda_tc_util.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int CB = 64;   // chunk tokens
constexpr int DD = 128;  // dk = dv
constexpr int NS = 64;   // value columns per CTA
constexpr int NTB = 256;
constexpr uint64_t kWaitNs = 2000000000ull;

constexpr uint32_t TILE = 32768;             // [64][128] fp32
constexpr uint32_t STAGE = 2 * TILE;         // W, Kb
constexpr uint32_t OFF_ST = 2 * STAGE;       // St: 2 blocks [128][32] fp32
constexpr uint32_t OFF_RW = OFF_ST + 32768;  // R: 2 blocks [64][32] fp32
constexpr uint32_t OFF_BAR = OFF_RW + 16384;
constexpr uint32_t SMEM = OFF_BAR + 64 + 1024;
static_assert(SMEM <= 232448, "one CTA per SM");
constexpr uint32_t TM_R1 = 0, TM_R2 = 64;    // tensor-memory columns of M1, M2

// kind::tf32 instruction descriptor: fp32 accumulate, tf32 A and B.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((b_mn ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32_tc(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

struct ChainArgs {
    const float* G;        // [total, H, 128] in-chunk cumulative gate
    const float* S0;       // entry state (forward: S_0; backward: dS of the end) or NULL
    const float* EF_rows;  // forward: Ut; backward: E   [total, H, 128]
    const float* F;        // backward: F [chunks, H, 128, 128]
    const int32_t* cu;
    int T;
    const int* chunk_start;
    int H;
    const uint32_t* status;
    uint32_t* status_out;
    float* rows_out;       // forward: U (may be EF_rows); backward: dU
    float* per_chunk;      // forward: S_n; backward: dS' of chunk n
    float* S_end;          // forward: NULL; backward: dS_0 (or NULL)
};

// x as the sum of two tf32 values: hi = x rounded, lo = the remainder rounded
// (operands of three-pass products: hi hi + hi lo + lo hi is within a few
// fp32 ulps of the exact product).
__device__ __forceinline__ void split_tf32(float x, float& hi, float& lo) {
    hi = round_tf32(x);
    lo = round_tf32(x - hi);
}

// One 32-value row of an MN-major tf32 operand block, rounded to tf32.
__device__ __forceinline__ void store_row32(uint8_t* blk, int row, const float (&x)[32]) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
        *reinterpret_cast<float4*>(blk + sw128_32b_off(row, q)) =
            make_float4(round_tf32(x[4 * q]), round_tf32(x[4 * q + 1]), round_tf32(x[4 * q + 2]),
                        round_tf32(x[4 * q + 3]));
}

template <bool kBack>
__global__ void __launch_bounds__(NTB, 1)
    chain_tc_kernel(const __grid_constant__ CUtensorMap tmw,
                    const __grid_constant__ CUtensorMap tmkb, const ChainArgs a) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t s_tmem;
    __shared__ int s_skip;  // one reading of the status for the whole CTA
    if (threadIdx.x == 0) s_skip = status_bad(a.status);
    __syncthreads();
    if (s_skip) return;
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + OFF_BAR);  // [2]
    uint64_t* bar_mma = bar_ld + 2;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, cq = warp >> 2;
    const int trow = 32 * quarter + lane;  // tensor-memory lane == channel (M2) / token (M1)
    const uint32_t tlane = static_cast<uint32_t>(32 * quarter) << 16;
    const int seq = blockIdx.x, h = blockIdx.y, j0 = NS * blockIdx.z;
    const int t_begin = a.cu ? a.cu[seq] : seq * a.T;
    const int t_end = a.cu ? a.cu[seq + 1] : (seq + 1) * a.T;
    const int nch = (t_end - t_begin + CB - 1) / CB;
    const size_t st_base = (((size_t)seq * a.H + h) * DD) * DD + j0 + 32 * cq;

    if (warp == 0) {
        tmem_alloc(&s_tmem, 128);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_ld + 1, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    // the entry state, this thread's 32 values of channel row trow
    float st[32];
    {
        const float* src = a.S0 ? a.S0 + st_base + (size_t)trow * DD : nullptr;
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            const float4 v = src ? *reinterpret_cast<const float4*>(src + i)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            st[i] = v.x; st[i + 1] = v.y; st[i + 2] = v.z; st[i + 3] = v.w;
        }
        store_row32(sm + OFF_ST + cq * 16384, trow, st);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = s_tmem;
    auto chunk_of = [&](int step) { return kBack ? nch - 1 - step : step; };
    auto issue_loads = [&](int step) {  // thread 0: W and Kb of that step's chunk
        const int s = step & 1, tt0 = t_begin + chunk_of(step) * CB;
        uint8_t* stg = sm + s * STAGE;
        mbar_arrive_expect_tx(bar_ld + s, STAGE);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
            tma_load_3d(stg + kb * 8192, &tmw, bar_ld + s, 32 * kb, h, tt0);
            tma_load_3d(stg + TILE + kb * 8192, &tmkb, bar_ld + s, 32 * kb, h, tt0);
        }
    };
    bool failed = false;
    uint32_t mma_phase = 0;
    int loads_issued = 0;
    if (tid == 0 && nch > 0) {
        issue_loads(0);
        loads_issued = 1;
    }
    constexpr uint32_t id1 = idesc_tf32(128, NS, false, true);
    constexpr uint32_t id2 = idesc_tf32(128, NS, true, true);
    for (int step = 0; step < nch && !failed; ++step) {
        const int n = chunk_of(step), s = step & 1;
        const int t0 = t_begin + n * CB, L = min(CB, t_end - t0);
        const size_t cbase = (((size_t)a.chunk_start[seq] + n) * a.H + h) * DD * DD;
        if (tid == 0 && step + 1 < nch) {  // that stage was last read by step - 1's products
            issue_loads(step + 1);
            ++loads_issued;
        }
        // this chunk's per-token rows (M1 lanes 0-63), F row, exp(G_last) of channel trow
        float base[32], fr[32];
        const bool row_ok = quarter < 2 && trow < L;
        if (row_ok) {
            const float* src = a.EF_rows + ((size_t)(t0 + trow) * a.H + h) * DD + j0 + 32 * cq;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 v = *reinterpret_cast<const float4*>(src + i);
                base[i] = v.x; base[i + 1] = v.y; base[i + 2] = v.z; base[i + 3] = v.w;
            }
        }
        if (kBack) {
            const float* src = a.F + cbase + (size_t)trow * DD + j0 + 32 * cq;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 v = *reinterpret_cast<const float4*>(src + i);
                fr[i] = v.x; fr[i + 1] = v.y; fr[i + 2] = v.z; fr[i + 3] = v.w;
            }
        }
        const float gam = expf(a.G[((size_t)(t0 + L - 1) * a.H + h) * DD + trow]);
        {  // the state entering this step (a tf32 operand of the dense kernel)
            float* dst = a.per_chunk + cbase + (size_t)trow * DD + j0 + 32 * cq;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4*>(dst + i) =
                    make_float4(round_tf32(st[i]), round_tf32(st[i + 1]), round_tf32(st[i + 2]),
                                round_tf32(st[i + 3]));
        }
        bool ok = mbar_wait(bar_ld + s, (step >> 1) & 1, kWaitNs);
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        // ---- M1 = A1 St
        const uint32_t stg = sbase + s * STAGE;
        const uint32_t a1 = stg + (kBack ? TILE : 0), a2 = stg + (kBack ? 0 : TILE);
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 16; ++ks) {
                const int kb = ks >> 2, kk = ks & 3;
                mma_tf32_tc(tbase + TM_R1, sdesc_sw128(a1 + kb * 8192 + kk * 32, 16, 1024),
                            sdesc_sw128_32b(sbase + OFF_ST + ks * 1024, 16384, 512), id1,
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
        // ---- the rows: U = Ut - M1 (forward) or dU = E + M1 (backward); zero
        // past the chunk's last token so that they add nothing to M2
        if (quarter < 2) {
            uint32_t v[32];
            tmem_ld32(tbase + tlane + TM_R1 + 32 * cq, v);
            tmem_wait_ld();
            float m[32];  // the rows M2 takes: U (forward), X (backward)
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float x = __uint_as_float(v[i]);
                m[i] = row_ok ? (kBack ? x : round_tf32(base[i] - x)) : 0.f;
            }
            if (row_ok) {
                float* dst = a.rows_out + ((size_t)(t0 + trow) * a.H + h) * DD + j0 + 32 * cq;
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4*>(dst + i) =
                        kBack ? make_float4(base[i] + m[i], base[i + 1] + m[i + 1],
                                            base[i + 2] + m[i + 2], base[i + 3] + m[i + 3])
                              : make_float4(m[i], m[i + 1], m[i + 2], m[i + 3]);
            }
            store_row32(sm + OFF_RW + cq * 8192, trow, m);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ---- M2 = A2^T R
        if (tid == 0) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_tf32_tc(tbase + TM_R2, sdesc_sw128_32b(a2 + ks * 1024, 8192, 512),
                            sdesc_sw128_32b(sbase + OFF_RW + ks * 1024, 8192, 512), id2, ks > 0);
            mma_commit(bar_mma);
        }
        ok = mbar_wait(bar_mma, mma_phase & 1, kWaitNs);
        ++mma_phase;
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        tc_fence_after();
        // ---- the state: S <- Gam S + M2 (forward); dS <- Gam dS' - M2 + F
        {
            uint32_t v[32];
            tmem_ld32(tbase + tlane + TM_R2 + 32 * cq, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float z = __uint_as_float(v[i]);
                st[i] = kBack ? fmaf(gam, st[i], fr[i] - z) : fmaf(gam, st[i], z);
            }
            store_row32(sm + OFF_ST + cq * 16384, trow, st);
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (!failed && a.S_end) {
        float* dst = a.S_end + st_base + (size_t)trow * DD;
#pragma unroll
        for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + i) = make_float4(st[i], st[i + 1], st[i + 2], st[i + 3]);
    }
    if (failed && tid == 0) {
        // wait (bounded) for the products and copies still in flight
        if (mma_phase > 0) mbar_wait(bar_mma, (mma_phase - 1) & 1, kWaitNs);
        for (int k = loads_issued - 2; k < loads_issued; ++k)
            if (k >= 0) mbar_wait(bar_ld + (k & 1), (k >> 1) & 1, kWaitNs);
        atomicOr(a.status_out, STATUS_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 128);
}

// ------------------------------------------------------------ E and F
// Per (chunk, head): E = P^T dO [64 tokens][128] and F = Qt^T dO - W^T E
// [128 channels][128], the value columns in two halves of 64.  Every operand
// is MN-major (the token index is K): P [r][i] (M = i, padded to 128 rows,
// whose results are never read), Qt and W [r][c] (M = c), dO and -E [r][j]
// (N = j), all in the 32-byte-granule swizzle.  Per half: E and the Qt^T dO
// part of F in one commit; -E replaces dO in shared memory; then W^T (-E)
// accumulates into F.  P and W come by TMA, Qt = q exp(G) and dO (widened
// to fp32) are written by the threads.
namespace ef {
constexpr uint32_t OFF_P = 0;          // P: 2 blocks [64 r][32 i]
constexpr uint32_t OFF_D = 16384;      // dO, then -E, of the half: 2 blocks [64 r][32 j]
constexpr uint32_t OFF_Q = 32768;      // Qt: 4 blocks [64 r][32 c]
constexpr uint32_t OFF_W = 65536;      // W: 4 blocks [64 r][32 c]
constexpr uint32_t OFF_BAR = 98304;
constexpr uint32_t SMEM = OFF_BAR + 64 + 1024;
constexpr uint32_t TM_E = 0, TM_F = 128;  // half jh at +64 jh
}  // namespace ef

// Store 16 consecutive fp32 values of row `row` (16-byte chunks q0 .. q0 + 3)
// into a [rows][32] block in the 32-byte-granule swizzle.
// (rounded to tf32)
__device__ __forceinline__ void store16_32b(uint8_t* blk, int row, int q0, const float (&x)[16]) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
        *reinterpret_cast<float4*>(blk + sw128_32b_off(row, q0 + q)) =
            make_float4(round_tf32(x[4 * q]), round_tf32(x[4 * q + 1]), round_tf32(x[4 * q + 2]),
                        round_tf32(x[4 * q + 3]));
}

template <typename TIn>
__device__ __forceinline__ void load16_f32(const TIn* src, float (&x)[16]);
template <>
__device__ __forceinline__ void load16_f32<float>(const float* src, float (&x)[16]) {
#pragma unroll
    for (int i = 0; i < 16; i += 4) {
        const float4 v = *reinterpret_cast<const float4*>(src + i);
        x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
    }
}
template <>
__device__ __forceinline__ void load16_f32<__nv_bfloat16>(const __nv_bfloat16* src,
                                                          float (&x)[16]) {
#pragma unroll
    for (int i = 0; i < 16; i += 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(src + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            x[i + 2 * p] = __uint_as_float(w[p] << 16);
            x[i + 2 * p + 1] = __uint_as_float(w[p] & 0xFFFF0000u);
        }
    }
}

struct EfArgs {
    const void* q;
    const void* dout;
    const float* G;
    const int4* info;  // per chunk slot: (sequence, first token, rows, -)
    int H;
    const uint32_t* status;
    uint32_t* status_out;
    float* E;  // [total, H, 128]
    float* F;  // [chunks, H, 128, 128]
};

template <typename TIn>
__global__ void __launch_bounds__(NTB, 1)
    ef_tc_kernel(const __grid_constant__ CUtensorMap tmp, const __grid_constant__ CUtensorMap tmw,
                 const EfArgs a) {
    using namespace ef;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t s_tmem;
    __shared__ int s_skip;
    const int cidx = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int4 ci = a.info[cidx];
    const int t0 = ci.y, L = ci.z;
    if (tid == 0) s_skip = status_bad(a.status) || L <= 0;
    __syncthreads();
    if (s_skip) return;
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + ef::OFF_BAR);
    uint64_t* bar_mma = bar_ld + 1;
    const int warp = tid >> 5, lane = tid & 31, quarter = warp & 3, cw = warp >> 2;
    const uint32_t tlane = static_cast<uint32_t>(32 * quarter) << 16;
    const TIn* Qg = static_cast<const TIn*>(a.q);
    const TIn* Dg = static_cast<const TIn*>(a.dout);
    if (warp == 0) {
        tmem_alloc(&s_tmem, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_ld, 16384 + 32768);
        tma_load_3d(sm + OFF_P, &tmp, bar_ld, 0, 0, cidx * a.H + h);
        tma_load_3d(sm + OFF_P + 8192, &tmp, bar_ld, 32, 0, cidx * a.H + h);
#pragma unroll
        for (int kb = 0; kb < 4; ++kb)
            tma_load_3d(sm + OFF_W + kb * 8192, &tmw, bar_ld, 32 * kb, h, t0);
    }
    // Qt = q exp(G): row r = tid / 4, channels 32 (tid % 4) .. + 31 (block tid % 4)
    {
        const int r = tid >> 2, kb = tid & 3;
        const bool ok = r < L;
        const size_t gi = ((size_t)(t0 + r) * a.H + h) * DD + 32 * kb;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float x[16], gv[16];
            if (ok) {
                load16_f32<TIn>(Qg + gi + 16 * half, x);
                load16_f32<float>(a.G + gi + 16 * half, gv);
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] *= __expf(gv[i]);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = 0.f;
            }
            store16_32b(sm + OFF_Q + kb * 8192, r, 4 * half, x);
        }
    }
    const uint32_t tbase = s_tmem;
    bool failed = false;
    uint32_t mma_phase = 0;
    constexpr uint32_t idn = idesc_tf32(128, 64, true, true);
    for (int jh = 0; jh < 2 && !failed; ++jh) {
        // dO of this half: row r = tid / 4, columns 64 jh + 16 (tid % 4) .. + 15
        {
            const int r = tid >> 2, part = tid & 3;
            float x[16];
            if (r < L) {
                load16_f32<TIn>(Dg + ((size_t)(t0 + r) * a.H + h) * DD + 64 * jh + 16 * part, x);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = 0.f;
            }
            store16_32b(sm + OFF_D + (part >> 1) * 8192, r, 4 * (part & 1), x);
        }
        fence_async_smem();
        bool ok = jh > 0 || mbar_wait(bar_ld, 0, kWaitNs);
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_tf32_tc(tbase + TM_E + 64 * jh, sdesc_sw128_32b(sbase + OFF_P + ks * 1024, 8192, 512),
                            sdesc_sw128_32b(sbase + OFF_D + ks * 1024, 8192, 512), idn, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_tf32_tc(tbase + TM_F + 64 * jh, sdesc_sw128_32b(sbase + OFF_Q + ks * 1024, 8192, 512),
                            sdesc_sw128_32b(sbase + OFF_D + ks * 1024, 8192, 512), idn, ks > 0);
            mma_commit(bar_mma);
        }
        ok = mbar_wait(bar_mma, mma_phase & 1, kWaitNs);
        ++mma_phase;
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        tc_fence_after();
        // E rows (token i = lane of quarters 0, 1), 32 columns per warp: to
        // global, and -E over dO in shared memory
        if (quarter < 2) {
            const int i = 32 * quarter + lane;
            uint32_t v[32];
            tmem_ld32(tbase + tlane + TM_E + 64 * jh + 32 * cw, v);
            tmem_wait_ld();
            float e[32];
#pragma unroll
            for (int x = 0; x < 32; ++x) e[x] = i < L ? __uint_as_float(v[x]) : 0.f;
            if (i < L) {
                float* dst = a.E + ((size_t)(t0 + i) * a.H + h) * DD + 64 * jh + 32 * cw;
#pragma unroll
                for (int x = 0; x < 32; x += 4)
                    *reinterpret_cast<float4*>(dst + x) = make_float4(e[x], e[x + 1], e[x + 2], e[x + 3]);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4*>(sm + OFF_D + cw * 8192 + sw128_32b_off(i, q)) =
                    make_float4(-round_tf32(e[4 * q]), -round_tf32(e[4 * q + 1]),
                                -round_tf32(e[4 * q + 2]), -round_tf32(e[4 * q + 3]));
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_tf32_tc(tbase + TM_F + 64 * jh, sdesc_sw128_32b(sbase + OFF_W + ks * 1024, 8192, 512),
                            sdesc_sw128_32b(sbase + OFF_D + ks * 1024, 8192, 512), idn, 1);
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
    if (!failed) {  // F: channel c = lane of the warp's quarter, 64 columns per warp
        const int c = 32 * quarter + lane;
        float* dst = a.F + (((size_t)cidx * a.H + h) * DD + c) * DD + 64 * cw;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            uint32_t v[32];
            tmem_ld32(tbase + tlane + TM_F + 64 * cw + 32 * x, v);
            tmem_wait_ld();
#pragma unroll
            for (int y = 0; y < 32; y += 4)
                *reinterpret_cast<float4*>(dst + 32 * x + y) =
                    make_float4(__uint_as_float(v[y]), __uint_as_float(v[y + 1]),
                                __uint_as_float(v[y + 2]), __uint_as_float(v[y + 3]));
        }
    } else if (tid == 0) {
        if (mma_phase > 0) mbar_wait(bar_mma, (mma_phase - 1) & 1, kWaitNs);
        mbar_wait(bar_ld, 0, kWaitNs);
        atomicOr(a.status_out, STATUS_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 256);
}

// ------------------------------------------------------------ dense
// Per (chunk, head), after the back substitution: [dO ; Y] S^T (one M = 128
// product: rows 0-63 dQt = dO S^T, rows 64-127 Y S^T) and U dS'^T (M = 64
// padded to 128), over the value columns in four quarters of 32 (K).  All
// operands K-major in the 16-byte-granule swizzle: dO widened to fp32 by the
// threads; Y, U, S and dS' by TMA.  Epilogue: dQt, dKt = -b (Y S^T), dKb =
// U dS'^T, dbeta = dbB - sum_c Kt (Y S^T), and dGam = rowsum(S * dS') from
// the staged quarters.
namespace dn {
constexpr uint32_t OFF_A = 0;       // [dO ; Y] quarter [128][32]
constexpr uint32_t OFF_U = 16384;   // U quarter [64][32]; padding rows read OFF_S
constexpr uint32_t OFF_S = 24576;   // S quarter [128 c][32 j]
constexpr uint32_t OFF_X = 40960;   // dS' quarter [128 c][32 j]
constexpr uint32_t OFF_RED = 57344; // dbeta partials [2][64]
constexpr uint32_t OFF_BAR = OFF_RED + 512;
constexpr uint32_t SMEM_USED = OFF_BAR + 64 + 1024;
// requested size: at most two CTAs per SM (each holds 256 tensor-memory columns)
constexpr uint32_t SMEM = 96 * 1024;
static_assert(SMEM_USED <= SMEM, "dense tile");
constexpr uint32_t TM_1 = 0, TM_2 = 128;
}  // namespace dn

struct DenseArgs {
    const void* k;
    const void* dout;
    const float* G;
    const float* beta;
    const float* dbB;
    const int4* info;
    int H;
    const uint32_t* status;
    uint32_t* status_out;
    float* dQt;
    float* dKt;
    float* dKb;
    float* dGam;
    float* dbeta;
};

template <typename TIn>
__global__ void __launch_bounds__(NTB, 1)
    dense_tc_kernel(const __grid_constant__ CUtensorMap tmy, const __grid_constant__ CUtensorMap tmu,
                    const __grid_constant__ CUtensorMap tms, const __grid_constant__ CUtensorMap tmx,
                    const DenseArgs a) {
    using namespace dn;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t s_tmem;
    __shared__ int s_skip;
    const int cidx = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int4 ci = a.info[cidx];
    const int t0 = ci.y, L = ci.z;
    if (tid == 0) s_skip = status_bad(a.status) || L <= 0;
    __syncthreads();
    if (s_skip) return;
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + dn::OFF_BAR);
    uint64_t* bar_mma = bar_ld + 1;
    float* s_red = reinterpret_cast<float*>(sm + OFF_RED);
    const int warp = tid >> 5, lane = tid & 31, quarter = warp & 3, cw = warp >> 2;
    const uint32_t tlane = static_cast<uint32_t>(32 * quarter) << 16;
    const TIn* Dg = static_cast<const TIn*>(a.dout);
    const TIn* Kg = static_cast<const TIn*>(a.k);
    if (warp == 0) {
        tmem_alloc(&s_tmem, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    __syncthreads();
    const uint32_t tbase = s_tmem;
    const int mat = cidx * a.H + h;
    bool failed = false;
    int fail_ld = -1, fail_mma = -1;  // the quarter whose copies / products were in flight
    float gam = 0.f;
    constexpr uint32_t idk = idesc_tf32(128, 128, false, false);
    for (int qk = 0; qk < 4; ++qk) {
        if (tid == 0) {
            mbar_arrive_expect_tx(bar_ld, 8192 + 8192 + 16384 + 16384);
            tma_load_3d(sm + OFF_A + 8192, &tmy, bar_ld, 32 * qk, h, t0);
            tma_load_3d(sm + OFF_U, &tmu, bar_ld, 32 * qk, h, t0);
            tma_load_3d(sm + OFF_S, &tms, bar_ld, 32 * qk, 0, mat);
            tma_load_3d(sm + OFF_X, &tmx, bar_ld, 32 * qk, 0, mat);
        }
        {  // dO quarter: row r = tid / 4, columns 32 qk + 8 (tid % 4) .. + 7
            const int r = tid >> 2, part = tid & 3;
            float x[16];
            if (r < L) {
                const TIn* src = Dg + ((size_t)(t0 + r) * a.H + h) * DD + 32 * qk + 8 * part;
                if constexpr (sizeof(TIn) == 2) {
                    const uint4 v = *reinterpret_cast<const uint4*>(src);
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        x[2 * p] = __uint_as_float(w[p] << 16);
                        x[2 * p + 1] = __uint_as_float(w[p] & 0xFFFF0000u);
                    }
                } else {
                    const float4 v0 = *reinterpret_cast<const float4*>(src);
                    const float4 v1 = *reinterpret_cast<const float4*>(src + 4);
                    x[0] = v0.x; x[1] = v0.y; x[2] = v0.z; x[3] = v0.w;
                    x[4] = v1.x; x[5] = v1.y; x[6] = v1.z; x[7] = v1.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = 0.f;
            }
            *reinterpret_cast<float4*>(sm + OFF_A + sw128_off(r, 2 * part)) =
                make_float4(round_tf32(x[0]), round_tf32(x[1]), round_tf32(x[2]), round_tf32(x[3]));
            *reinterpret_cast<float4*>(sm + OFF_A + sw128_off(r, 2 * part + 1)) =
                make_float4(round_tf32(x[4]), round_tf32(x[5]), round_tf32(x[6]), round_tf32(x[7]));
        }
        fence_async_smem();
        bool ok = mbar_wait(bar_ld, qk & 1, kWaitNs);
        if (__syncthreads_or(!ok)) {
            failed = true;
            fail_ld = qk;
            break;
        }
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t acc = (qk | kk) > 0;
                mma_tf32_tc(tbase + TM_1, sdesc_sw128(sbase + OFF_A + kk * 32, 16, 1024),
                            sdesc_sw128(sbase + OFF_S + kk * 32, 16, 1024), idk, acc);
                mma_tf32_tc(tbase + TM_2, sdesc_sw128(sbase + OFF_U + kk * 32, 16, 1024),
                            sdesc_sw128(sbase + OFF_X + kk * 32, 16, 1024), idk, acc);
            }
            mma_commit(bar_mma);
        }
        if (tid < DD) {  // dGam: channel tid, this quarter's 32 columns
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 sv = *reinterpret_cast<const float4*>(sm + OFF_S + sw128_off(tid, q));
                const float4 xv = *reinterpret_cast<const float4*>(sm + OFF_X + sw128_off(tid, q));
                gam += sv.x * xv.x + sv.y * xv.y + sv.z * xv.z + sv.w * xv.w;
            }
        }
        ok = mbar_wait(bar_mma, qk & 1, kWaitNs);
        if (__syncthreads_or(!ok)) {
            failed = true;
            fail_mma = qk;
            break;
        }
        tc_fence_after();
    }
    if (!failed) {
        if (tid < DD) a.dGam[(size_t)mat * DD + tid] = gam;
        const int r = 32 * (quarter & 1) + lane;  // token row of this thread
        const bool row_ok = r < L;
        const size_t row = ((size_t)(t0 + r) * a.H + h) * DD + 64 * cw;
        float part = 0.f;
        float b = 0.f;
        if (quarter >= 2 && row_ok) b = a.beta[(size_t)(t0 + r) * a.H + h];
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            uint32_t v[32];
            tmem_ld32(tbase + tlane + TM_1 + 64 * cw + 32 * x, v);
            tmem_wait_ld();
            if (quarter < 2) {  // dQt = dO S^T
                if (row_ok) {
#pragma unroll
                    for (int y = 0; y < 32; y += 4)
                        *reinterpret_cast<float4*>(a.dQt + row + 32 * x + y) =
                            make_float4(__uint_as_float(v[y]), __uint_as_float(v[y + 1]),
                                        __uint_as_float(v[y + 2]), __uint_as_float(v[y + 3]));
                }
            } else if (row_ok) {  // Y S^T: dKt and the Kt . (Y S^T) part of dbeta
                float kv[16], gv[16];
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    load16_f32<TIn>(Kg + row + 32 * x + 16 * hf, kv);
                    load16_f32<float>(a.G + row + 32 * x + 16 * hf, gv);
#pragma unroll
                    for (int y = 0; y < 16; ++y)
                        part += kv[y] * expf(gv[y]) * __uint_as_float(v[16 * hf + y]);
                }
#pragma unroll
                for (int y = 0; y < 32; y += 4)
                    *reinterpret_cast<float4*>(a.dKt + row + 32 * x + y) =
                        make_float4(-b * __uint_as_float(v[y]), -b * __uint_as_float(v[y + 1]),
                                    -b * __uint_as_float(v[y + 2]), -b * __uint_as_float(v[y + 3]));
            }
            if (quarter < 2) {  // dKb = U dS'^T
                tmem_ld32(tbase + tlane + TM_2 + 64 * cw + 32 * x, v);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int y = 0; y < 32; y += 4)
                        *reinterpret_cast<float4*>(a.dKb + row + 32 * x + y) =
                            make_float4(__uint_as_float(v[y]), __uint_as_float(v[y + 1]),
                                        __uint_as_float(v[y + 2]), __uint_as_float(v[y + 3]));
                }
            }
        }
        if (quarter >= 2) s_red[cw * 64 + r] = part;
        __syncthreads();
        if (quarter >= 2 && cw == 0 && row_ok) {
            const size_t bi = (size_t)(t0 + r) * a.H + h;
            a.dbeta[bi] = a.dbB[bi] - (s_red[r] + s_red[64 + r]);
        }
    } else if (tid == 0) {  // wait (bounded) for what is still in flight
        if (fail_ld >= 0) mbar_wait(bar_ld, fail_ld & 1, kWaitNs);
        if (fail_mma >= 0) mbar_wait(bar_mma, fail_mma & 1, kWaitNs);
        atomicOr(a.status_out, STATUS_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 256);
}

// ------------------------------------------------------------ pair sums
// Per (chunk, head), with E = exp(G - Gm) under a per-channel reference Gm =
// max_r G_r - 80 (every factor within exp(+-80) when the chunk's per-channel
// log-decay range is at most 160 and max G <= 60, as in the forward's A/P):
//   [rowA ; dQp] = ([bdA ; dP] (K * E^-1)) * [E ; E]     (one M = 128 product)
//   col          = ([bdA ; dP]^T [K * E ; Q * E]) * E^-1  (M = 64 padded to 128)
// i.e. rowA[r] = sum_{i<r} bdA[r][i] k_i e^{G_r - G_i}, dQp[r] = sum_{i<=r}
// dP[r][i] k_i e^{G_r - G_i}, col[r] = sum_{i'>=r} (bdA[i'][r] k_i' + dP[i'][r]
// q_i') e^{G_i' - G_r} (the masks are the zeros of bdA and dP), then the same
// epilogue as the exact kernel: dq, dk, dG and the reverse cumulative sum dg.
// X = [bdA ; dP] [128 rows][64 columns] is the K-major A operand of the first
// product and the MN-major A operand of the second (the 16-byte- and the
// 32-byte-granule swizzle).  Both products are taken in three tf32 passes
// (each operand split into a rounded high part and the rounded remainder:
// hi hi + hi lo + lo hi): in one pass the pair sums carried most of the
// gradients' error (dg is their reverse cumulative sum).  The two products
// are staged one after the other in the same shared memory (the values of
// the second kept in registers meanwhile).  A chunk outside the range sets
// slow = 1 and is left to the exact kernel.
namespace pr {
// first product
constexpr uint32_t OFF_X1H = 0;       // X high, 2 blocks [128][32] (16-byte granules)
constexpr uint32_t OFF_X1L = 32768;   // X low
constexpr uint32_t OFF_B1H = 65536;   // K * E^-1 high [64 i][128 c]: 4 blocks [64][32]
constexpr uint32_t OFF_B1L = 98304;   // low
// second product (over the first's operands)
constexpr uint32_t OFF_X2H = 0;       // X high, 2 blocks [128][32] (32-byte granules)
constexpr uint32_t OFF_X2L = 32768;   // X low
constexpr uint32_t OFF_B2H = 65536;   // [K * E ; Q * E] high: 4 blocks [128][32]
constexpr uint32_t OFF_B2L = 131072;  // low
constexpr uint32_t OFF_GM = 196608;   // Gm [128]
constexpr uint32_t OFF_RED = OFF_GM + 512;   // max, min [4][128] each; later the epilogue's exchange
constexpr uint32_t OFF_BAR = OFF_RED + 4096;
constexpr uint32_t SMEM = OFF_BAR + 64 + 1024;
// after the products, the accumulators as fp32 [rows][LDD] over the operands
constexpr int LDD = 132;
constexpr uint32_t OFF_D1 = 0;                       // rows 0-63 rowA, 64-127 dQp
constexpr uint32_t OFF_D2 = 128 * LDD * 4;           // rows 0-63 col
static_assert(OFF_D2 + 64 * LDD * 4 <= OFF_GM, "accumulator dump");
constexpr uint32_t TM_1 = 0, TM_2 = 128;
constexpr float kRefPair = 80.f;
constexpr int NTP = 512;  // threads: one CTA per SM (shared memory), so 16 warps
}  // namespace pr

struct PairArgs {
    const void* q;
    const void* k;
    const float* G;
    const float* dAr;
    const float* dP;
    const float* dQt;
    const float* dKt;
    const float* dKb;
    const float* dGam;
    const int4* info;
    int H;
    const uint32_t* status;
    uint32_t* status_out;
    int* slow;
    float* dq;
    float* dk;
    float* dg;
};

template <typename TIn>
__device__ __forceinline__ float4 load4_f32(const TIn* p);
template <>
__device__ __forceinline__ float4 load4_f32<float>(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}
template <>
__device__ __forceinline__ float4 load4_f32<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                       __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u));
}

__device__ __forceinline__ float4 round4_tf32(float4 v) {
    return make_float4(round_tf32(v.x), round_tf32(v.y), round_tf32(v.z), round_tf32(v.w));
}

template <typename TIn>
__global__ void __launch_bounds__(pr::NTP, 1) pair_tc_kernel(const PairArgs a) {
    using namespace pr;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t s_tmem;
    __shared__ int s_skip;
    const int cidx = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int4 ci = a.info[cidx];
    const int t0 = ci.y, L = ci.z;
    if (tid == 0) s_skip = status_bad(a.status) || L <= 0;
    __syncthreads();
    if (s_skip) return;
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    float* sGm = reinterpret_cast<float*>(sm + OFF_GM);
    float* sRed = reinterpret_cast<float*>(sm + OFF_RED);
    uint64_t* bar_mma = reinterpret_cast<uint64_t*>(sm + pr::OFF_BAR);
    const TIn* Qg = static_cast<const TIn*>(a.q);
    const TIn* Kg = static_cast<const TIn*>(a.k);
    // channel c, a quarter `part` of the chunk's rows (16 each)
    const int c = tid & 127, part = tid >> 7;
    const size_t rowH = (size_t)a.H * DD;  // stride between tokens
    const size_t base = ((size_t)t0 * a.H + h) * DD;
    // 1. per-channel max / min of G over the chunk's rows, the reference and
    // the range test (the exact kernel reads the flag this writes)
    {
        float gv[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {  // all 16 loads in flight at once
            const int r = 16 * part + j;
            gv[j] = r < L ? __ldg(a.G + base + r * rowH + c) : 0.f;
        }
        float mx = -INFINITY, mn = INFINITY;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (16 * part + j < L) {
                mx = fmaxf(mx, gv[j]);
                mn = fminf(mn, gv[j]);
            }
        }
        sRed[part * 128 + c] = mx;
        sRed[512 + part * 128 + c] = mn;
    }
    __syncthreads();
    bool bad = false;
    if (tid < 128) {
        const float mx = fmaxf(fmaxf(sRed[c], sRed[128 + c]), fmaxf(sRed[256 + c], sRed[384 + c]));
        const float mn = fminf(fminf(sRed[512 + c], sRed[640 + c]), fminf(sRed[768 + c], sRed[896 + c]));
        sGm[c] = mx - kRefPair;
        bad = !(mx - mn <= 2.f * kRefPair) || !(mx <= 60.f);
    }
    const bool slow = __syncthreads_or(bad);
    if (tid == 0) a.slow[(size_t)cidx * a.H + h] = slow ? 1 : 0;
    if (slow) return;
    const int warp = tid >> 5, lane = tid & 31, quarter = warp & 3, cg = warp >> 2;
    if (warp == 0) {
        tmem_alloc(&s_tmem, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    // 2. the first product's operands.  X rows m (< 64: bdA row m; >= 64: dP
    // row m - 64), four columns per float4; K * E^-1 rows r, channels 4 c4 ..;
    // X and K * E, Q * E stay in registers for the second product
    constexpr int NX = 2048 / NTP;
    float4 xv[NX], kev[NX], qev[NX];
    {
        const size_t cc = ((size_t)cidx * a.H + h) * 64 * 64;
#pragma unroll
        for (int it = 0; it < NX; ++it) {
            const int idx = tid + NTP * it;  // 0 .. 2047
            const int m = idx >> 4, c4 = idx & 15;
            const int r = m & 63;
            xv[it] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r < L)
                xv[it] = __ldg(reinterpret_cast<const float4*>((m < 64 ? a.dAr : a.dP) + cc + r * 64 + 4 * c4));
            float4 hi, lo;
            split_tf32(xv[it].x, hi.x, lo.x);
            split_tf32(xv[it].y, hi.y, lo.y);
            split_tf32(xv[it].z, hi.z, lo.z);
            split_tf32(xv[it].w, hi.w, lo.w);
            const uint32_t o = (c4 >> 3) * 16384 + sw128_off(m, c4 & 7);
            *reinterpret_cast<float4*>(sm + OFF_X1H + o) = hi;
            *reinterpret_cast<float4*>(sm + OFF_X1L + o) = lo;
        }
    }
    __syncthreads();  // Gm visible
#pragma unroll
    for (int it = 0; it < NX; ++it) {
        const int idx = tid + NTP * it;  // 0 .. 2047
        const int r = idx >> 5, c4 = idx & 31;
        float4 ki = make_float4(0.f, 0.f, 0.f, 0.f);
        kev[it] = qev[it] = ki;
        if (r < L) {
            const size_t gi = base + r * rowH + 4 * c4;
            const float4 kv = load4_f32<TIn>(Kg + gi);
            const float4 qv = load4_f32<TIn>(Qg + gi);
            const float4 gv = __ldg(reinterpret_cast<const float4*>(a.G + gi));
            const float4 gm = *reinterpret_cast<const float4*>(sGm + 4 * c4);
            const float x0 = gv.x - gm.x, x1 = gv.y - gm.y, x2 = gv.z - gm.z, x3 = gv.w - gm.w;
            const float e0 = __expf(x0), e1 = __expf(x1), e2 = __expf(x2), e3 = __expf(x3);
            kev[it] = make_float4(kv.x * e0, kv.y * e1, kv.z * e2, kv.w * e3);
            qev[it] = make_float4(qv.x * e0, qv.y * e1, qv.z * e2, qv.w * e3);
            ki = make_float4(kv.x * __expf(-x0), kv.y * __expf(-x1), kv.z * __expf(-x2),
                             kv.w * __expf(-x3));
        }
        float4 hi, lo;
        split_tf32(ki.x, hi.x, lo.x);
        split_tf32(ki.y, hi.y, lo.y);
        split_tf32(ki.z, hi.z, lo.z);
        split_tf32(ki.w, hi.w, lo.w);
        const uint32_t o = (c4 >> 3) * 8192 + sw128_32b_off(r, c4 & 7);
        *reinterpret_cast<float4*>(sm + OFF_B1H + o) = hi;
        *reinterpret_cast<float4*>(sm + OFF_B1L + o) = lo;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = s_tmem;
    // 3. the first product: [rowA ; dQp] before scaling (M = 128, N = 128, K = 64)
    if (tid == 0) {
        constexpr uint32_t id1 = idesc_tf32(128, 128, false, true);
        const uint32_t As[3] = {OFF_X1H, OFF_X1H, OFF_X1L}, Bs[3] = {OFF_B1H, OFF_B1L, OFF_B1H};
#pragma unroll
        for (int pass = 0; pass < 3; ++pass)
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int kb = ks >> 2, kk = ks & 3;
                mma_tf32_tc(tbase + TM_1, sdesc_sw128(sbase + As[pass] + kb * 16384 + kk * 32, 16, 1024),
                            sdesc_sw128_32b(sbase + Bs[pass] + ks * 1024, 8192, 512), id1,
                            (pass | ks) > 0);
            }
        mma_commit(bar_mma);
    }
    bool ok = mbar_wait(bar_mma, 0, kWaitNs);
    if (__syncthreads_or(!ok)) {
        if (tid == 0) {
            mbar_wait(bar_mma, 0, kWaitNs);  // bounded: the products still in flight
            atomicOr(a.status_out, STATUS_TIMEOUT);
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 0) tmem_dealloc(tbase, 256);
        return;
    }
    tc_fence_after();
    // 4. the second product's operands over the first's (all read)
#pragma unroll
    for (int it = 0; it < NX; ++it) {
        const int idx = tid + NTP * it;
        {
            const int m = idx >> 4, c4 = idx & 15;
            float4 hi, lo;
            split_tf32(xv[it].x, hi.x, lo.x);
            split_tf32(xv[it].y, hi.y, lo.y);
            split_tf32(xv[it].z, hi.z, lo.z);
            split_tf32(xv[it].w, hi.w, lo.w);
            const uint32_t o = (c4 >> 3) * 16384 + sw128_32b_off(m, c4 & 7);
            *reinterpret_cast<float4*>(sm + OFF_X2H + o) = hi;
            *reinterpret_cast<float4*>(sm + OFF_X2L + o) = lo;
        }
        {
            const int r = idx >> 5, c4 = idx & 31;
            const uint32_t o = (c4 >> 3) * 16384 + sw128_32b_off(r, c4 & 7);
            const uint32_t oq = (c4 >> 3) * 16384 + sw128_32b_off(64 + r, c4 & 7);
            float4 hi, lo;
            split_tf32(kev[it].x, hi.x, lo.x);
            split_tf32(kev[it].y, hi.y, lo.y);
            split_tf32(kev[it].z, hi.z, lo.z);
            split_tf32(kev[it].w, hi.w, lo.w);
            *reinterpret_cast<float4*>(sm + OFF_B2H + o) = hi;
            *reinterpret_cast<float4*>(sm + OFF_B2L + o) = lo;
            split_tf32(qev[it].x, hi.x, lo.x);
            split_tf32(qev[it].y, hi.y, lo.y);
            split_tf32(qev[it].z, hi.z, lo.z);
            split_tf32(qev[it].w, hi.w, lo.w);
            *reinterpret_cast<float4*>(sm + OFF_B2H + oq) = hi;
            *reinterpret_cast<float4*>(sm + OFF_B2L + oq) = lo;
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // 5. the second product: col before scaling (M = 64 padded to 128, N = 128, K = 128)
    if (tid == 0) {
        constexpr uint32_t id2 = idesc_tf32(128, 128, true, true);
        const uint32_t As[3] = {OFF_X2H, OFF_X2H, OFF_X2L}, Bs[3] = {OFF_B2H, OFF_B2L, OFF_B2H};
#pragma unroll
        for (int pass = 0; pass < 3; ++pass)
#pragma unroll
            for (int ks = 0; ks < 16; ++ks)
                mma_tf32_tc(tbase + TM_2, sdesc_sw128_32b(sbase + As[pass] + ks * 1024, 16384, 512),
                            sdesc_sw128_32b(sbase + Bs[pass] + ks * 1024, 16384, 512), id2,
                            (pass | ks) > 0);
        mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, 1, kWaitNs);
    if (__syncthreads_or(!ok)) {
        if (tid == 0) {
            mbar_wait(bar_mma, 1, kWaitNs);
            atomicOr(a.status_out, STATUS_TIMEOUT);
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 0) tmem_dealloc(tbase, 256);
        return;
    }
    tc_fence_after();
    // 4. the accumulators to shared memory (over the operands, all read):
    // warp (lane quarter, 32-column group cg)
    {
        float* D1 = reinterpret_cast<float*>(sm + OFF_D1);
        float* D2 = reinterpret_cast<float*>(sm + OFF_D2);
        const int row = 32 * quarter + lane;
        const uint32_t tl = static_cast<uint32_t>(32 * quarter) << 16;
        uint32_t v[32];
        tmem_ld32(tbase + tl + TM_1 + 32 * cg, v);
        tmem_wait_ld();
#pragma unroll
        for (int y = 0; y < 32; y += 4)
            *reinterpret_cast<float4*>(D1 + row * LDD + 32 * cg + y) =
                make_float4(__uint_as_float(v[y]), __uint_as_float(v[y + 1]),
                            __uint_as_float(v[y + 2]), __uint_as_float(v[y + 3]));
        if (quarter < 2) {
            tmem_ld32(tbase + tl + TM_2 + 32 * cg, v);
            tmem_wait_ld();
#pragma unroll
            for (int y = 0; y < 32; y += 4)
                *reinterpret_cast<float4*>(D2 + row * LDD + 32 * cg + y) =
                    make_float4(__uint_as_float(v[y]), __uint_as_float(v[y + 1]),
                                __uint_as_float(v[y + 2]), __uint_as_float(v[y + 3]));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 256);
    // 5. the epilogue of the exact kernel, channel c, rows 16 part .. + 15
    {
        const float* D1 = reinterpret_cast<const float*>(sm + OFF_D1);
        const float* D2 = reinterpret_cast<const float*>(sm + OFF_D2);
        const float gm = sGm[c];
        const float glast = __ldg(a.G + base + (L - 1) * rowH + c);
        float dG[16];
        float tot = 0.f, last = 0.f;
        // eight rows at a time: their loads (read-only path) issued together,
        // then their arithmetic and stores
#pragma unroll
        for (int b8 = 0; b8 < 2; ++b8) {
            float gr[8], qr[8], kr[8], x[8], y[8], z[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int r = 16 * part + 8 * b8 + j;
                if (r < L) {
                    const size_t gi = base + r * rowH + c;
                    gr[j] = __ldg(a.G + gi);
                    qr[j] = to_f32(__ldg(Qg + gi));
                    kr[j] = to_f32(__ldg(Kg + gi));
                    x[j] = __ldg(a.dQt + gi);
                    y[j] = __ldg(a.dKt + gi);
                    z[j] = __ldg(a.dKb + gi);
                } else {
                    gr[j] = qr[j] = kr[j] = x[j] = y[j] = z[j] = 0.f;
                }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int r = 16 * part + 8 * b8 + j;
                dG[8 * b8 + j] = 0.f;
                if (r < L) {
                    const size_t gi = base + r * rowH + c;
                    const float e = __expf(gr[j] - gm), ei = __expf(gm - gr[j]);
                    const float rowA = D1[r * LDD + c] * e, dQp = D1[(64 + r) * LDD + c] * e;
                    const float col = D2[r * LDD + c] * ei;
                    const float eg = expf(gr[j]), eb = expf(glast - gr[j]);
                    a.dq[gi] = dQp + x[j] * eg;
                    a.dk[gi] = rowA + col + y[j] * eg + z[j] * eb;
                    const float d = kr[j] * (rowA - col) + qr[j] * dQp + x[j] * qr[j] * eg +
                                    y[j] * kr[j] * eg - z[j] * kr[j] * eb;
                    dG[8 * b8 + j] = d;
                    tot += d;
                    last += z[j] * kr[j] * eb;
                }
            }
        }
        // [4][128] row-sum totals, [4][128] last-row terms, over the max / min
        // partials of step 1 (read before the range test's barrier)
        float* xch = sRed;
        xch[part * 128 + c] = tot;
        xch[512 + part * 128 + c] = last;
        __syncthreads();
        float acc = expf(glast) * a.dGam[((size_t)cidx * a.H + h) * DD + c] + xch[512 + c] +
                    xch[640 + c] + xch[768 + c] + xch[896 + c];
        for (int p2 = part + 1; p2 < 4; ++p2) acc += xch[p2 * 128 + c];  // rows after this part
#pragma unroll
        for (int j = 15; j >= 0; --j) {
            const int r = 16 * part + j;
            if (r < L) {
                acc += dG[j];
                a.dg[base + r * rowH + c] = acc;
            }
        }
    }
}

// ------------------------------------------------------------ A and P
// The recompute's first step per (chunk, head): G (the in-chunk inclusive sum
// of g), Kb = K exp(G_last - G), the right-hand sides b K exp(G), and
//   A[r][i] = sum_c k_rc k_ic exp(G_rc - G_ic)  (i < r; without b),
//   P[r][i] = sum_c q_rc k_ic exp(G_rc - G_ic)  (i <= r)
// as one M = 128 product [K * E ; Q * E] (K * E^-1)^T under the per-channel
// reference of the pair kernel.  A feeds the triangular solves, so the
// product is taken in three tf32 passes (each operand split into a rounded
// high part and the rounded remainder: hi hi + hi lo + lo hi), which keeps it
// close to fp32.  A chunk outside the reference's range sets slow = 1; the
// exact kernel then recomputes that chunk.
namespace ap {
constexpr uint32_t OFF_AH = 0;        // [K*E ; Q*E] high: 4 blocks [128][32] (K-major)
constexpr uint32_t OFF_AL = 65536;    // low
constexpr uint32_t OFF_BH = 131072;   // K*E^-1 [64 i][128 c] high: 4 blocks [64][32]
constexpr uint32_t OFF_BL = 163840;   // low
constexpr uint32_t OFF_RED = 196608;  // [4][128] totals, max, min
constexpr uint32_t OFF_BAR = OFF_RED + 6144;
constexpr uint32_t SMEM = OFF_BAR + 64 + 1024;
constexpr int NT = 512;
}  // namespace ap

struct ApArgs {
    const void* q;
    const void* k;
    const float* g;
    const float* beta;
    const int4* info;
    int H;
    const uint32_t* status;
    uint32_t* status_out;
    int* slow;
    float* G;
    float* Ar;
    float* P;
    float* Kb;
    float* Rk;
};

template <typename TIn>
__global__ void __launch_bounds__(ap::NT, 1) apkb_tc_kernel(const ApArgs a) {
    using namespace ap;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t s_tmem;
    __shared__ int s_skip;
    const int cidx = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int4 ci = a.info[cidx];
    const int t0 = ci.y, L = ci.z;
    if (tid == 0) s_skip = status_bad(a.status) || L <= 0;
    __syncthreads();
    if (s_skip) return;
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    float* sRed = reinterpret_cast<float*>(sm + OFF_RED);  // tot [4][128], mx [4][128], mn [4][128]
    uint64_t* bar_mma = reinterpret_cast<uint64_t*>(sm + ap::OFF_BAR);
    const TIn* Qg = static_cast<const TIn*>(a.q);
    const TIn* Kg = static_cast<const TIn*>(a.k);
    const int c = tid & 127, part = tid >> 7;  // channel, rows 16 part .. + 15
    const size_t rowH = (size_t)a.H * DD;
    const size_t base = ((size_t)t0 * a.H + h) * DD;
    // 1. G: each part's inclusive prefix over its 16 rows, then the totals of
    // the parts above it; per-channel max / min
    float gv[16], kv[16], qv[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int r = 16 * part + j;
        const bool in = r < L;
        gv[j] = in ? __ldg(a.g + base + r * rowH + c) : 0.f;
        kv[j] = in ? to_f32(__ldg(Kg + base + r * rowH + c)) : 0.f;
        qv[j] = in ? to_f32(__ldg(Qg + base + r * rowH + c)) : 0.f;
    }
    float run = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        run += gv[j];
        gv[j] = run;
    }
    sRed[part * 128 + c] = run;
    __syncthreads();
    float off = 0.f, glast = 0.f;
#pragma unroll
    for (int p2 = 0; p2 < 4; ++p2) {
        const float t = sRed[p2 * 128 + c];
        if (p2 < part) off += t;
        glast += t;  // the sum of every row < L
    }
    float mx = -INFINITY, mn = INFINITY;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        gv[j] += off;
        if (16 * part + j < L) {
            mx = fmaxf(mx, gv[j]);
            mn = fminf(mn, gv[j]);
        }
    }
    sRed[512 + part * 128 + c] = mx;
    sRed[1024 + part * 128 + c] = mn;
    // G, Kb and the right-hand sides: exact, whatever the range
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int r = 16 * part + j;
        if (r < L) {
            const size_t gi = base + r * rowH + c;
            a.G[gi] = gv[j];
            const float kb = kv[j] * __expf(glast - gv[j]);
            a.Kb[gi] = round_tf32(kb);
            a.Rk[gi] = __ldg(a.beta + (size_t)(t0 + r) * a.H + h) * kv[j] * __expf(gv[j]);
        }
    }
    __syncthreads();
    const float gmx = fmaxf(fmaxf(sRed[512 + c], sRed[640 + c]), fmaxf(sRed[768 + c], sRed[896 + c]));
    const float gmn = fminf(fminf(sRed[1024 + c], sRed[1152 + c]), fminf(sRed[1280 + c], sRed[1408 + c]));
    const bool bad = !(gmx - gmn <= 160.f) || !(gmx <= 60.f);
    const bool slow = __syncthreads_or(bad);
    if (tid == 0) a.slow[(size_t)cidx * a.H + h] = slow ? 1 : 0;
    if (slow) return;
    const float gm = gmx - 80.f;
    const int warp = tid >> 5, lane = tid & 31, quarter = warp & 3, cg = warp >> 2;
    if (warp == 0) {
        tmem_alloc(&s_tmem, 64);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    // 2. the operands, split into tf32 high and low parts; element (r, c) of
    // a K-major [rows][128] tile: block c / 32, 16-byte chunk (c % 32) / 4
    {
        const int blk = c >> 5, q16 = (c & 31) >> 2, w4 = (c & 3) * 4;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const int r = 16 * part + j;
            float ke = 0.f, qe = 0.f, ki = 0.f;
            if (r < L) {
                const float x = gv[j] - gm;
                const float e = __expf(x), ei = __expf(-x);
                ke = kv[j] * e;
                qe = qv[j] * e;
                ki = kv[j] * ei;
            }
            const float keh = round_tf32(ke), qeh = round_tf32(qe), kih = round_tf32(ki);
            const uint32_t oa = blk * 16384 + sw128_off(r, q16) + w4;
            const uint32_t oq = blk * 16384 + sw128_off(64 + r, q16) + w4;
            const uint32_t ob = blk * 8192 + sw128_off(r, q16) + w4;
            *reinterpret_cast<float*>(sm + OFF_AH + oa) = keh;
            *reinterpret_cast<float*>(sm + OFF_AL + oa) = round_tf32(ke - keh);
            *reinterpret_cast<float*>(sm + OFF_AH + oq) = qeh;
            *reinterpret_cast<float*>(sm + OFF_AL + oq) = round_tf32(qe - qeh);
            *reinterpret_cast<float*>(sm + OFF_BH + ob) = kih;
            *reinterpret_cast<float*>(sm + OFF_BL + ob) = round_tf32(ki - kih);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = s_tmem;
    // 3. D = Ah Bh^T + Ah Bl^T + Al Bh^T (M = 128, N = 64, K = 128)
    if (tid == 0) {
        constexpr uint32_t id = idesc_tf32(128, 64, false, false);
        const uint32_t As[3] = {OFF_AH, OFF_AH, OFF_AL}, Bs[3] = {OFF_BH, OFF_BL, OFF_BH};
#pragma unroll
        for (int pass = 0; pass < 3; ++pass)
#pragma unroll
            for (int ks = 0; ks < 16; ++ks) {
                const int kb = ks >> 2, kk = ks & 3;
                mma_tf32_tc(tbase, sdesc_sw128(sbase + As[pass] + kb * 16384 + kk * 32, 16, 1024),
                            sdesc_sw128(sbase + Bs[pass] + kb * 8192 + kk * 32, 16, 1024), id,
                            (pass | ks) > 0);
            }
        mma_commit(bar_mma);
    }
    const bool ok = mbar_wait(bar_mma, 0, kWaitNs);
    if (__syncthreads_or(!ok)) {
        if (tid == 0) {
            mbar_wait(bar_mma, 0, kWaitNs);
            atomicOr(a.status_out, STATUS_TIMEOUT);
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 0) tmem_dealloc(tbase, 64);
        return;
    }
    tc_fence_after();
    // 4. masked rows out: lane m of quarter (m < 64: A row m; else P row m - 64),
    // 32 columns per warp (cg 0, 1)
    if (cg < 2) {
        const int m = 32 * quarter + lane;
        const int r = m & 63, i0 = 32 * cg;
        uint32_t v[32];
        tmem_ld32(tbase + (static_cast<uint32_t>(32 * quarter) << 16) + i0, v);
        tmem_wait_ld();
        const bool isP = m >= 64;
        float* dst = (isP ? a.P : a.Ar) + ((size_t)cidx * a.H + h) * 64 * 64 + r * 64 + i0;
#pragma unroll
        for (int y = 0; y < 32; y += 4) {
            float o[4];
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                const int i = i0 + y + z;
                const bool keep = r < L && (isP ? i <= r : i < r);
                const float x = __uint_as_float(v[y + z]);
                o[z] = keep ? (isP ? round_tf32(x) : x) : 0.f;
            }
            *reinterpret_cast<float4*>(dst + y) = make_float4(o[0], o[1], o[2], o[3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 64);
}

// ------------------------------------------------------------ T = (I + A)^-1
// T = (I + diag(b) Ar)^-1 of one chunk in fp32, in shared memory ([64][LDT]):
// the four 16 x 16 diagonal blocks by forward substitution (one column per
// thread), then the blocks below them a diagonal at a time, T_IJ = -T_II
// sum_{K=J}^{I-1} A_IK T_KJ (the lower-triangular block inverse).  Ar rows
// past the chunk are zero and b there is zero, so T is the identity there.
constexpr int LDT = 65;
__device__ void tri_inverse(const float* Ar, const float* bs, float* Tm, float* Msc, int tid,
                            int nt) {
    for (int e = tid; e < 64 * LDT; e += nt) Tm[e] = 0.f;
    __syncthreads();
    if (tid < 64) {  // diagonal block I, column j
        const int I = tid >> 4, j = tid & 15, o = 16 * I;
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) t[r] = r == j ? 1.f : 0.f;
#pragma unroll
        for (int r = 1; r < 16; ++r) {
            if (r > j) {
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < r; ++i)
                    if (i >= j) acc += Ar[(o + r) * LDT + o + i] * t[i];
                t[r] = -bs[o + r] * acc;
            }
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tm[(o + r) * LDT + o + j] = t[r];
    }
    __syncthreads();
    for (int d = 1; d < 4; ++d) {
        const int nb = 4 - d;  // blocks (J + d, J), J = 0 .. nb - 1
        for (int e = tid; e < nb * 256; e += nt) {  // M_IJ = sum_K A_IK T_KJ
            const int J = e >> 8, r = (e >> 4) & 15, c = e & 15, I = J + d;
            float acc = 0.f;
            for (int K = J; K < I; ++K)
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    acc += Ar[(16 * I + r) * LDT + 16 * K + i] * Tm[(16 * K + i) * LDT + 16 * J + c];
            Msc[e] = bs[16 * I + r] * acc;
        }
        __syncthreads();
        for (int e = tid; e < nb * 256; e += nt) {  // T_IJ = -T_II M_IJ
            const int J = e >> 8, r = (e >> 4) & 15, c = e & 15, I = J + d;
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < 16; ++k)
                if (k <= r) acc += Tm[(16 * I + r) * LDT + 16 * I + k] * Msc[J * 256 + k * 16 + c];
            Tm[(16 * I + r) * LDT + 16 * J + c] = -acc;
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------ [W | Ut]
// (I + A) [W | Ut] = [b Kt | b V] as [W | Ut] = T [b Kt | b V]: T in fp32 by
// tri_inverse (also written out for the back substitution), the product in
// three tf32 passes (M = 64 padded to 128, N = 256, K = 64).
namespace sb {
constexpr int NT = 512;
constexpr uint32_t OFF_AH = 0;        // T high: 2 blocks [128][32], K-major (rows 64-127 zero)
constexpr uint32_t OFF_AL = 32768;    // T low
constexpr uint32_t OFF_BH = 65536;    // [b Kt | b V] high: 8 blocks [64 i][32 n], MN-major
constexpr uint32_t OFF_BL = 131072;   // low; before it is built: Ar, T, the block scratch
constexpr uint32_t OFF_BS = 196608;   // b [64]
constexpr uint32_t OFF_BAR = OFF_BS + 256;
constexpr uint32_t SMEM = OFF_BAR + 64 + 1024;
}  // namespace sb

struct SubstArgs {
    const void* v;
    const float* beta;
    const float* Ar;
    const int4* info;
    int H;
    const uint32_t* status;
    uint32_t* status_out;
    float* W;   // in: b Kt; out: W (rounded to tf32)
    float* Ut;  // out
    float* Tout;  // [chunks, H, 64, 64]
};

template <typename TIn>
__global__ void __launch_bounds__(sb::NT, 1) subst_tc_kernel(const SubstArgs a) {
    using namespace sb;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t s_tmem;
    __shared__ int s_skip;
    const int cidx = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int4 ci = a.info[cidx];
    const int t0 = ci.y, L = ci.z;
    if (tid == 0) s_skip = status_bad(a.status) || L <= 0;
    __syncthreads();
    if (s_skip) return;
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    float* Ar = reinterpret_cast<float*>(sm + OFF_BL);
    float* Tm = Ar + 64 * LDT;
    float* Msc = Tm + 64 * LDT;
    float* bs = reinterpret_cast<float*>(sm + OFF_BS);
    uint64_t* bar_mma = reinterpret_cast<uint64_t*>(sm + sb::OFF_BAR);
    const int warp = tid >> 5, lane = tid & 31, quarter = warp & 3, cg = warp >> 2;
    if (warp == 0) {
        tmem_alloc(&s_tmem, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    const size_t cc = ((size_t)cidx * a.H + h) * 64 * 64;
    for (int e = tid; e < 64 * 64; e += NT) Ar[(e >> 6) * LDT + (e & 63)] = __ldg(a.Ar + cc + e);
    if (tid < 64) bs[tid] = tid < L ? __ldg(a.beta + (size_t)(t0 + tid) * a.H + h) : 0.f;
    // the right-hand sides' rows i < L, requested now so that their latency
    // overlaps the inverse: b Kt (W on entry) and v (b applied later)
    constexpr int NB = 4096 / NT;
    float4 rhs[NB];
    {
        const size_t base = ((size_t)t0 * a.H + h) * DD;
        const size_t rowH = (size_t)a.H * DD;
        const TIn* Vg = static_cast<const TIn*>(a.v);
#pragma unroll
        for (int it = 0; it < NB; ++it) {
            const int idx = tid + NT * it;
            const int i = idx >> 6, n4 = idx & 63;
            rhs[it] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < L)
                rhs[it] = n4 < 32
                              ? __ldg(reinterpret_cast<const float4*>(a.W + base + i * rowH + 4 * n4))
                              : load4_f32<TIn>(Vg + base + i * rowH + 4 * (n4 - 32));
        }
    }
    __syncthreads();
    tri_inverse(Ar, bs, Tm, Msc, tid, NT);
    // T out (fp32) and T's tf32 split as the K-major A operand
    for (int e = tid; e < 128 * 64; e += NT) {
        const int r = e >> 6, i = e & 63;
        const float x = r < 64 ? Tm[r * LDT + i] : 0.f;
        if (r < 64) a.Tout[cc + e] = x;
        float hi, lo;
        split_tf32(x, hi, lo);
        const uint32_t o = (i >> 5) * 16384 + sw128_off(r, (i & 31) >> 2) + 4 * (i & 3);
        *reinterpret_cast<float*>(sm + OFF_AH + o) = hi;
        *reinterpret_cast<float*>(sm + OFF_AL + o) = lo;
    }
    __syncthreads();  // T, Ar read: the low half of B may overwrite them
    // [b Kt | b V] rows i < L (zeros after), four columns per float4
    {
#pragma unroll
        for (int it = 0; it < NB; ++it) {
            const int idx = tid + NT * it;
            const int i = idx >> 6, n4 = idx & 63;
            float4 x = rhs[it];
            if (n4 >= 32) {
                const float b = bs[i];
                x = make_float4(b * x.x, b * x.y, b * x.z, b * x.w);
            }
            float4 hi, lo;
            split_tf32(x.x, hi.x, lo.x);
            split_tf32(x.y, hi.y, lo.y);
            split_tf32(x.z, hi.z, lo.z);
            split_tf32(x.w, hi.w, lo.w);
            const uint32_t o = (n4 >> 3) * 8192 + sw128_32b_off(i, n4 & 7);
            *reinterpret_cast<float4*>(sm + OFF_BH + o) = hi;
            *reinterpret_cast<float4*>(sm + OFF_BL + o) = lo;
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = s_tmem;
    if (tid == 0) {
        constexpr uint32_t id = idesc_tf32(128, 256, false, true);
        const uint32_t As[3] = {OFF_AH, OFF_AH, OFF_AL}, Bs[3] = {OFF_BH, OFF_BL, OFF_BH};
#pragma unroll
        for (int pass = 0; pass < 3; ++pass)
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int kb = ks >> 2, kk = ks & 3;
                mma_tf32_tc(tbase, sdesc_sw128(sbase + As[pass] + kb * 16384 + kk * 32, 16, 1024),
                            sdesc_sw128_32b(sbase + Bs[pass] + ks * 1024, 8192, 512), id,
                            (pass | ks) > 0);
            }
        mma_commit(bar_mma);
    }
    const bool ok = mbar_wait(bar_mma, 0, kWaitNs);
    if (__syncthreads_or(!ok)) {
        if (tid == 0) {
            mbar_wait(bar_mma, 0, kWaitNs);
            atomicOr(a.status_out, STATUS_TIMEOUT);
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 0) tmem_dealloc(tbase, 256);
        return;
    }
    tc_fence_after();
    // rows r < L (lanes 0-63): columns 64 cg .. + 63 (cg 0, 1: W; 2, 3: Ut)
    if (quarter < 2) {
        const int r = 32 * quarter + lane;
        const size_t row = ((size_t)(t0 + r) * a.H + h) * DD;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            uint32_t v[32];
            tmem_ld32(tbase + (static_cast<uint32_t>(32 * quarter) << 16) + 64 * cg + 32 * x, v);
            tmem_wait_ld();
            if (r < L) {
                const int col = 64 * cg + 32 * x;
                float* dst = col < 128 ? a.W + row + col : a.Ut + row + col - 128;
#pragma unroll
                for (int y = 0; y < 32; y += 4) {
                    float4 o4 = make_float4(__uint_as_float(v[y]), __uint_as_float(v[y + 1]),
                                            __uint_as_float(v[y + 2]), __uint_as_float(v[y + 3]));
                    if (col < 128) o4 = round4_tf32(o4);
                    *reinterpret_cast<float4*>(dst + y) = o4;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 256);
}

// ------------------------------------------------------------ the solve
// (I + A)^T Y = dU as Y = T^T dU (T from the substitution kernel), then
// dA = -strict_lower(Y U^T) and dP = lower(dO U^T) as one M = 128 product
// [Y ; dO] U^T, both in three tf32 passes; dv = b Y, and the partial
// gradient of b, Y.V + sum_i dA[r][i] Ar[r][i].
namespace sv {
constexpr int NT = 512;
constexpr uint32_t OFF_TH = 0;        // T high: 2 blocks [64 i][32 r] (MN-major A; M padded)
constexpr uint32_t OFF_TL = 16384;    // T low
constexpr uint32_t OFF_DH = 32768;    // dU high: 4 blocks [64 i][32 j] (MN-major B)
constexpr uint32_t OFF_DL = 65536;    // dU low
constexpr uint32_t OFF_YH = 0;        // (second product) [Y ; dO] high: 4 blocks [128][32] (K-major)
constexpr uint32_t OFF_YL = 65536;    // low
constexpr uint32_t OFF_UH = 131072;   // U high: 4 blocks [64][32] (K-major B)
constexpr uint32_t OFF_UL = 163840;   // low
constexpr uint32_t OFF_RED = 196608;  // Y.V partials [4][64], dA.Ar partials [2][64]
constexpr uint32_t OFF_BS = OFF_RED + 1536;
constexpr uint32_t OFF_BAR = OFF_BS + 256;
constexpr uint32_t SMEM = OFF_BAR + 64 + 1024;
constexpr uint32_t TM_Y = 0, TM_2 = 128;
}  // namespace sv

struct SolveArgs {
    const void* v;
    const void* dout;
    const float* Ar;
    const float* beta;
    const float* U;
    const float* dU;
    const float* Tm;
    const int4* info;
    int H;
    const uint32_t* status;
    uint32_t* status_out;
    float* Y;
    float* dv;
    float* dAr;
    float* dP;
    float* dbB;
};

template <typename TIn>
__global__ void __launch_bounds__(sv::NT, 1) solve_tc_kernel(const SolveArgs a) {
    using namespace sv;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t s_tmem;
    __shared__ int s_skip;
    const int cidx = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const int4 ci = a.info[cidx];
    const int t0 = ci.y, L = ci.z;
    if (tid == 0) s_skip = status_bad(a.status) || L <= 0;
    __syncthreads();
    if (s_skip) return;
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    float* sRed = reinterpret_cast<float*>(sm + OFF_RED);
    float* bs = reinterpret_cast<float*>(sm + OFF_BS);
    uint64_t* bar_mma = reinterpret_cast<uint64_t*>(sm + sv::OFF_BAR);
    const int warp = tid >> 5, lane = tid & 31, quarter = warp & 3, cg = warp >> 2;
    const TIn* Vg = static_cast<const TIn*>(a.v);
    const TIn* Dg = static_cast<const TIn*>(a.dout);
    if (warp == 0) {
        tmem_alloc(&s_tmem, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    const size_t cc = ((size_t)cidx * a.H + h) * 64 * 64;
    const size_t base = ((size_t)t0 * a.H + h) * DD;
    const size_t rowH = (size_t)a.H * DD;
    if (tid < 64) bs[tid] = tid < L ? __ldg(a.beta + (size_t)(t0 + tid) * a.H + h) : 0.f;
    // dO and U of the second product, requested now (their latency overlaps
    // the first product)
    constexpr int NP2 = 2048 / NT;
    float4 dpre[NP2], upre[NP2];
#pragma unroll
    for (int it = 0; it < NP2; ++it) {
        const int idx = tid + NT * it;
        const int r = idx >> 5, j4 = idx & 31;
        dpre[it] = upre[it] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < L) {
            dpre[it] = load4_f32<TIn>(Dg + base + r * rowH + 4 * j4);
            upre[it] = __ldg(reinterpret_cast<const float4*>(a.U + base + r * rowH + 4 * j4));
        }
    }
    // T (rows i, columns r contiguous: the MN-major A of T^T) and dU (rows i)
#pragma unroll
    for (int it = 0; it < 1024 / NT; ++it) {
        const int idx = tid + NT * it;  // 0 .. 1023: (i, r4)
        const int i = idx >> 4, r4 = idx & 15;
        const float4 x = __ldg(reinterpret_cast<const float4*>(a.Tm + cc + i * 64 + 4 * r4));
        float4 hi, lo;
        split_tf32(x.x, hi.x, lo.x);
        split_tf32(x.y, hi.y, lo.y);
        split_tf32(x.z, hi.z, lo.z);
        split_tf32(x.w, hi.w, lo.w);
        const uint32_t o = (r4 >> 3) * 8192 + sw128_32b_off(i, r4 & 7);
        *reinterpret_cast<float4*>(sm + OFF_TH + o) = hi;
        *reinterpret_cast<float4*>(sm + OFF_TL + o) = lo;
    }
#pragma unroll
    for (int it = 0; it < 2048 / NT; ++it) {
        const int idx = tid + NT * it;  // 0 .. 2047: (i, j4)
        const int i = idx >> 5, j4 = idx & 31;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < L) x = __ldg(reinterpret_cast<const float4*>(a.dU + base + i * rowH + 4 * j4));
        float4 hi, lo;
        split_tf32(x.x, hi.x, lo.x);
        split_tf32(x.y, hi.y, lo.y);
        split_tf32(x.z, hi.z, lo.z);
        split_tf32(x.w, hi.w, lo.w);
        const uint32_t o = (j4 >> 3) * 8192 + sw128_32b_off(i, j4 & 7);
        *reinterpret_cast<float4*>(sm + OFF_DH + o) = hi;
        *reinterpret_cast<float4*>(sm + OFF_DL + o) = lo;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = s_tmem;
    if (tid == 0) {  // Y = T^T dU: M = 64 padded to 128, N = 128, K = 64
        constexpr uint32_t id = idesc_tf32(128, 128, true, true);
        const uint32_t As[3] = {OFF_TH, OFF_TH, OFF_TL}, Bs[3] = {OFF_DH, OFF_DL, OFF_DH};
#pragma unroll
        for (int pass = 0; pass < 3; ++pass)
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_tf32_tc(tbase + TM_Y, sdesc_sw128_32b(sbase + As[pass] + ks * 1024, 8192, 512),
                            sdesc_sw128_32b(sbase + Bs[pass] + ks * 1024, 8192, 512), id,
                            (pass | ks) > 0);
        mma_commit(bar_mma);
    }
    bool ok = mbar_wait(bar_mma, 0, kWaitNs);
    if (__syncthreads_or(!ok)) {
        if (tid == 0) {
            mbar_wait(bar_mma, 0, kWaitNs);
            atomicOr(a.status_out, STATUS_TIMEOUT);
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 0) tmem_dealloc(tbase, 256);
        return;
    }
    tc_fence_after();
    // Y rows (lanes 0-63), 32 columns per warp: Y, dv out, Y.V, and the split
    // of Y as rows 0-63 of the second product's A
    if (quarter < 2) {
        const int r = 32 * quarter + lane;
        uint32_t v[32];
        tmem_ld32(tbase + TM_Y + (static_cast<uint32_t>(32 * quarter) << 16) + 32 * cg, v);
        tmem_wait_ld();
        float yv = 0.f;
        const size_t row = base + r * rowH + 32 * cg;
        const bool in = r < L;
#pragma unroll
        for (int y = 0; y < 32; y += 4) {
            float4 y4 = make_float4(__uint_as_float(v[y]), __uint_as_float(v[y + 1]),
                                    __uint_as_float(v[y + 2]), __uint_as_float(v[y + 3]));
            if (!in) y4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (in) {
                const float b = bs[r];
                *reinterpret_cast<float4*>(a.Y + row + y) = round4_tf32(y4);
                *reinterpret_cast<float4*>(a.dv + row + y) =
                    make_float4(b * y4.x, b * y4.y, b * y4.z, b * y4.w);
                const float4 vv = load4_f32<TIn>(Vg + row + y);
                yv += y4.x * vv.x + y4.y * vv.y + y4.z * vv.z + y4.w * vv.w;
            }
            float4 hi, lo;
            split_tf32(y4.x, hi.x, lo.x);
            split_tf32(y4.y, hi.y, lo.y);
            split_tf32(y4.z, hi.z, lo.z);
            split_tf32(y4.w, hi.w, lo.w);
            const uint32_t o = cg * 16384 + sw128_off(r, y >> 2);
            // the first product's operands are all read: the A region is free
            *reinterpret_cast<float4*>(sm + OFF_YH + o) = hi;
            *reinterpret_cast<float4*>(sm + OFF_YL + o) = lo;
        }
        sRed[cg * 64 + r] = yv;
    }
    // dO (rows 64-127 of the A operand) and U (the B operand), rows < L
#pragma unroll
    for (int it = 0; it < NP2; ++it) {
        const int idx = tid + NT * it;  // (r, j4)
        const int r = idx >> 5, j4 = idx & 31;
        const float4 dd = dpre[it], uu = upre[it];
        float4 hi, lo;
        const uint32_t oa = (j4 >> 3) * 16384 + sw128_off(64 + r, j4 & 7);
        split_tf32(dd.x, hi.x, lo.x);
        split_tf32(dd.y, hi.y, lo.y);
        split_tf32(dd.z, hi.z, lo.z);
        split_tf32(dd.w, hi.w, lo.w);
        *reinterpret_cast<float4*>(sm + OFF_YH + oa) = hi;
        *reinterpret_cast<float4*>(sm + OFF_YL + oa) = lo;
        const uint32_t ob = (j4 >> 3) * 8192 + sw128_off(r, j4 & 7);
        split_tf32(uu.x, hi.x, lo.x);
        split_tf32(uu.y, hi.y, lo.y);
        split_tf32(uu.z, hi.z, lo.z);
        split_tf32(uu.w, hi.w, lo.w);
        *reinterpret_cast<float4*>(sm + OFF_UH + ob) = hi;
        *reinterpret_cast<float4*>(sm + OFF_UL + ob) = lo;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {  // [Y ; dO] U^T: M = 128, N = 64, K = 128
        constexpr uint32_t id = idesc_tf32(128, 64, false, false);
        const uint32_t As[3] = {OFF_YH, OFF_YH, OFF_YL}, Bs[3] = {OFF_UH, OFF_UL, OFF_UH};
#pragma unroll
        for (int pass = 0; pass < 3; ++pass)
#pragma unroll
            for (int ks = 0; ks < 16; ++ks) {
                const int kb = ks >> 2, kk = ks & 3;
                mma_tf32_tc(tbase + TM_2, sdesc_sw128(sbase + As[pass] + kb * 16384 + kk * 32, 16, 1024),
                            sdesc_sw128(sbase + Bs[pass] + kb * 8192 + kk * 32, 16, 1024), id,
                            (pass | ks) > 0);
            }
        mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, 1, kWaitNs);
    if (__syncthreads_or(!ok)) {
        if (tid == 0) {
            mbar_wait(bar_mma, 1, kWaitNs);
            atomicOr(a.status_out, STATUS_TIMEOUT);
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 0) tmem_dealloc(tbase, 256);
        return;
    }
    tc_fence_after();
    // lanes 0-63: Y U^T row r -> dA; lanes 64-127: dO U^T row r -> dP; 32
    // columns per warp (cg 0, 1)
    if (cg < 2) {
        const int m = 32 * quarter + lane, r = m & 63, i0 = 32 * cg;
        uint32_t v[32];
        tmem_ld32(tbase + TM_2 + (static_cast<uint32_t>(32 * quarter) << 16) + i0, v);
        tmem_wait_ld();
        if (m < 64) {
            float part = 0.f;
            if (r < L) {
                const float b = bs[r];
                const float* arow = a.Ar + cc + r * 64 + i0;
#pragma unroll
                for (int y = 0; y < 32; y += 4) {
                    const float4 ar = __ldg(reinterpret_cast<const float4*>(arow + y));
                    float da[4];
#pragma unroll
                    for (int z = 0; z < 4; ++z) da[z] = i0 + y + z < r ? -__uint_as_float(v[y + z]) : 0.f;
                    part += da[0] * ar.x + da[1] * ar.y + da[2] * ar.z + da[3] * ar.w;
                    *reinterpret_cast<float4*>(a.dAr + cc + r * 64 + i0 + y) =
                        make_float4(b * da[0], b * da[1], b * da[2], b * da[3]);
                }
            }
            sRed[256 + cg * 64 + r] = part;
        } else if (r < L) {
#pragma unroll
            for (int y = 0; y < 32; y += 4) {
                float p4[4];
#pragma unroll
                for (int z = 0; z < 4; ++z) p4[z] = i0 + y + z <= r ? __uint_as_float(v[y + z]) : 0.f;
                *reinterpret_cast<float4*>(a.dP + cc + r * 64 + i0 + y) =
                    make_float4(p4[0], p4[1], p4[2], p4[3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 256);
    if (tid < 64 && tid < L)
        a.dbB[(size_t)(t0 + tid) * a.H + h] = sRed[tid] + sRed[64 + tid] + sRed[128 + tid] +
                                              sRed[192 + tid] + sRed[256 + tid] + sRed[320 + tid];
}

PFN_cuTensorMapEncodeTiled_v12000 bwd_encode_fn() {
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

// fp32 [total, H, 128] read as boxes of 32 channels x 64 tokens, 128-byte
// swizzle with 16-byte (K-major use) or 32-byte (MN-major use) granules.
bool map_f32_rows(CUtensorMap* m, const float* base, int total, int H, bool mn_major) {
    auto fn = bwd_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)DD, (cuuint64_t)H, (cuuint64_t)total};
    cuuint64_t strides[2] = {(cuuint64_t)DD * 4, (cuuint64_t)DD * 4 * H};
    cuuint32_t box[3] = {32, 1, (cuuint32_t)CB};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              mn_major ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 [count][rows][cols] per-chunk matrices read as boxes of 32 columns x
// all rows of one matrix, in either swizzle.
bool map_f32_mats(CUtensorMap* m, const float* base, int count, int rows, int cols,
                  bool mn_major) {
    auto fn = bwd_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)count};
    cuuint64_t strides[2] = {(cuuint64_t)cols * 4, (cuuint64_t)cols * rows * 4};
    cuuint32_t box[3] = {32, (cuuint32_t)rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              mn_major ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool bwd_tc_available() { return bwd_encode_fn() != nullptr; }

cudaError_t launch_bwd_chains_tc(const float* W, const float* Kb, const float* G, const float* S0,
                                 const float* dS_end, float* U_in_out, const float* E,
                                 const float* F, const int32_t* cu, int T, int N, int H,
                                 const int* chunk_start, uint32_t* status, float* states,
                                 float* dU, float* dSx, float* dS0, cudaStream_t st) {
    const int total = cu ? T : N * T;
    if (N == 0) return cudaSuccess;
    // forward: W is A1 (K-major), Kb is A2 (MN-major); backward: the reverse
    CUtensorMap mw_k, mw_mn, mkb_k, mkb_mn;
    if (total > 0) {
        if (!map_f32_rows(&mw_k, W, total, H, false) || !map_f32_rows(&mw_mn, W, total, H, true) ||
            !map_f32_rows(&mkb_k, Kb, total, H, false) || !map_f32_rows(&mkb_mn, Kb, total, H, true))
            return cudaErrorInvalidValue;
    } else {
        memset(&mw_k, 0, sizeof(mw_k));
        memset(&mw_mn, 0, sizeof(mw_mn));
        memset(&mkb_k, 0, sizeof(mkb_k));
        memset(&mkb_mn, 0, sizeof(mkb_mn));
    }
    cudaError_t e = cudaFuncSetAttribute(chain_tc_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(chain_tc_kernel<true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
    if (e != cudaSuccess) return e;
    const dim3 grid(N, H, DD / NS);
    const ChainArgs fa{G, S0, U_in_out, nullptr, cu, T, chunk_start, H, status, status, U_in_out,
                       states, nullptr};
    chain_tc_kernel<false><<<grid, NTB, SMEM, st>>>(mw_k, mkb_mn, fa);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const ChainArgs ba{G, dS_end, E, F, cu, T, chunk_start, H, status, status, dU, dSx, dS0};
    chain_tc_kernel<true><<<grid, NTB, SMEM, st>>>(mw_mn, mkb_k, ba);
    return cudaGetLastError();
}

}  // namespace kda

namespace kda {

template <typename TIn>
cudaError_t launch_bwd_ef_tc(const TIn* q, const TIn* dout, const float* G, const float* P,
                             const float* W, const int4* info, int total, int maxc, int H,
                             uint32_t* status, float* E, float* F, cudaStream_t st) {
    if (maxc == 0 || total == 0) return cudaSuccess;
    CUtensorMap mp, mw;
    if (!map_f32_mats(&mp, P, maxc * H, 64, 64, true) || !map_f32_rows(&mw, W, total, H, true))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(ef_tc_kernel<TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ef::SMEM);
    if (e != cudaSuccess) return e;
    const EfArgs a{q, dout, G, info, H, status, status, E, F};
    ef_tc_kernel<TIn><<<dim3(maxc, H), NTB, ef::SMEM, st>>>(mp, mw, a);
    return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_bwd_dense_tc(const TIn* k, const TIn* dout, const float* G, const float* beta,
                                const float* U, const float* Y, const float* states,
                                const float* dSx, const float* dbB, const int4* info, int total,
                                int maxc, int H, uint32_t* status, float* dQt, float* dKt,
                                float* dKb, float* dGam, float* dbeta, cudaStream_t st) {
    if (maxc == 0 || total == 0) return cudaSuccess;
    CUtensorMap my, mu, ms, mx;
    if (!map_f32_rows(&my, Y, total, H, false) || !map_f32_rows(&mu, U, total, H, false) ||
        !map_f32_mats(&ms, states, maxc * H, 128, 128, false) ||
        !map_f32_mats(&mx, dSx, maxc * H, 128, 128, false))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(dense_tc_kernel<TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dn::SMEM);
    if (e != cudaSuccess) return e;
    const DenseArgs a{k, dout, G, beta, dbB, info, H, status, status, dQt, dKt, dKb, dGam, dbeta};
    dense_tc_kernel<TIn><<<dim3(maxc, H), NTB, dn::SMEM, st>>>(my, mu, ms, mx, a);
    return cudaGetLastError();
}

template cudaError_t launch_bwd_ef_tc<float>(const float*, const float*, const float*,
                                             const float*, const float*, const int4*, int, int,
                                             int, uint32_t*, float*, float*, cudaStream_t);
template cudaError_t launch_bwd_ef_tc<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                                     const float*, const float*, const float*,
                                                     const int4*, int, int, int, uint32_t*,
                                                     float*, float*, cudaStream_t);
template cudaError_t launch_bwd_dense_tc<float>(const float*, const float*, const float*,
                                                const float*, const float*, const float*,
                                                const float*, const float*, const float*,
                                                const int4*, int, int, int, uint32_t*, float*,
                                                float*, float*, float*, float*, cudaStream_t);
template cudaError_t launch_bwd_dense_tc<__nv_bfloat16>(
    const __nv_bfloat16*, const __nv_bfloat16*, const float*, const float*, const float*,
    const float*, const float*, const float*, const float*, const int4*, int, int, int,
    uint32_t*, float*, float*, float*, float*, float*, cudaStream_t);

}  // namespace kda

namespace kda {

template <typename TIn>
cudaError_t launch_bwd_pair_tc(const TIn* q, const TIn* k, const float* G, const float* dAr,
                               const float* dP, const float* dQt, const float* dKt,
                               const float* dKb, const float* dGam, const int4* info, int total,
                               int maxc, int H, uint32_t* status, int* slow, float* dq,
                               float* dk, float* dg, cudaStream_t st) {
    if (maxc == 0 || total == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(pair_tc_kernel<TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pr::SMEM);
    if (e != cudaSuccess) return e;
    const PairArgs a{q, k, G, dAr, dP, dQt, dKt, dKb, dGam, info, H, status, status, slow, dq, dk,
                     dg};
    pair_tc_kernel<TIn><<<dim3(maxc, H), pr::NTP, pr::SMEM, st>>>(a);
    return cudaGetLastError();
}

template cudaError_t launch_bwd_pair_tc<float>(const float*, const float*, const float*,
                                               const float*, const float*, const float*,
                                               const float*, const float*, const float*,
                                               const int4*, int, int, int, uint32_t*, int*,
                                               float*, float*, float*, cudaStream_t);
template cudaError_t launch_bwd_pair_tc<__nv_bfloat16>(
    const __nv_bfloat16*, const __nv_bfloat16*, const float*, const float*, const float*,
    const float*, const float*, const float*, const float*, const int4*, int, int, int,
    uint32_t*, int*, float*, float*, float*, cudaStream_t);

}  // namespace kda

namespace kda {

template <typename TIn>
cudaError_t launch_bwd_apkb_tc(const TIn* q, const TIn* k, const float* g, const float* beta,
                               const int4* info, int total, int maxc, int H, uint32_t* status,
                               int* slow, float* G, float* Ar, float* P, float* Kb, float* Rk,
                               cudaStream_t st) {
    if (maxc == 0 || total == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(apkb_tc_kernel<TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ap::SMEM);
    if (e != cudaSuccess) return e;
    const ApArgs a{q, k, g, beta, info, H, status, status, slow, G, Ar, P, Kb, Rk};
    apkb_tc_kernel<TIn><<<dim3(maxc, H), ap::NT, ap::SMEM, st>>>(a);
    return cudaGetLastError();
}

template cudaError_t launch_bwd_apkb_tc<float>(const float*, const float*, const float*,
                                               const float*, const int4*, int, int, int,
                                               uint32_t*, int*, float*, float*, float*, float*,
                                               float*, cudaStream_t);
template cudaError_t launch_bwd_apkb_tc<__nv_bfloat16>(const __nv_bfloat16*,
                                                       const __nv_bfloat16*, const float*,
                                                       const float*, const int4*, int, int, int,
                                                       uint32_t*, int*, float*, float*, float*,
                                                       float*, float*, cudaStream_t);

}  // namespace kda

namespace kda {

template <typename TIn>
cudaError_t launch_bwd_subst_tc(const TIn* v, const float* beta, const float* Ar,
                                const int4* info, int total, int maxc, int H, uint32_t* status,
                                float* W, float* Ut, float* Tm, cudaStream_t st) {
    if (maxc == 0 || total == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(subst_tc_kernel<TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb::SMEM);
    if (e != cudaSuccess) return e;
    const SubstArgs a{v, beta, Ar, info, H, status, status, W, Ut, Tm};
    subst_tc_kernel<TIn><<<dim3(maxc, H), sb::NT, sb::SMEM, st>>>(a);
    return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_bwd_solve_tc(const TIn* v, const TIn* dout, const float* Ar,
                                const float* beta, const float* U, const float* dU,
                                const float* Tm, const int4* info, int total, int maxc, int H,
                                uint32_t* status, float* Y, float* dv, float* dAr, float* dP,
                                float* dbB, cudaStream_t st) {
    if (maxc == 0 || total == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(solve_tc_kernel<TIn>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sv::SMEM);
    if (e != cudaSuccess) return e;
    const SolveArgs a{v, dout, Ar, beta, U, dU, Tm, info, H, status, status, Y, dv, dAr, dP, dbB};
    solve_tc_kernel<TIn><<<dim3(maxc, H), sv::NT, sv::SMEM, st>>>(a);
    return cudaGetLastError();
}

#define KDA_BWD_ST_INST(TIn)                                                                  \
    template cudaError_t launch_bwd_subst_tc<TIn>(const TIn*, const float*, const float*,      \
                                                  const int4*, int, int, int, uint32_t*,       \
                                                  float*, float*, float*, cudaStream_t);       \
    template cudaError_t launch_bwd_solve_tc<TIn>(                                             \
        const TIn*, const TIn*, const float*, const float*, const float*, const float*,        \
        const float*, const int4*, int, int, int, uint32_t*, float*, float*, float*, float*,   \
        float*, cudaStream_t);
KDA_BWD_ST_INST(float)
KDA_BWD_ST_INST(__nv_bfloat16)
#undef KDA_BWD_ST_INST

}  // namespace kda
