// The two serial chains of the chunked KDA backward on the 5th-generation
// tensor cores (tcgen05, kind::tf32, accumulators in tensor memory), for
// dk = dv = 128 and chunks of 64 tokens.  See kda_bwd.cu for the derivation
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

__device__ __forceinline__ void store_row32(uint8_t* blk, int row, const float (&x)[32]) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
        *reinterpret_cast<float4*>(blk + sw128_32b_off(row, q)) =
            make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
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
        {  // the state entering this step
            float* dst = a.per_chunk + cbase + (size_t)trow * DD + j0 + 32 * cq;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4*>(dst + i) =
                    make_float4(st[i], st[i + 1], st[i + 2], st[i + 3]);
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
                m[i] = row_ok ? (kBack ? x : base[i] - x) : 0.f;
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
