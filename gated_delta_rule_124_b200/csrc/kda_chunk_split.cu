// KDA chunkwise prefill on the 5th-generation tensor cores (tcgen05 + TMEM,
// operands staged by TMA and bulk copies), bf16 q/k/v/o, fp32 g/beta/state,
// dk = dv = 128, chunk C = 64 -- the default plan of kda_chunk_fwd for these
// shapes.
//
// Kimi Linear (aiwiki.ai), "The constrained DPLR form and the chunkwise
// algorithm": inside a chunk the per-token corrections are gathered into a WY
// form and the unit-triangular system is solved once (UT transform); between
// chunks the state is carried recurrently.  Per chunk (rows r, i; G = in-chunk
// inclusive cumsum of g; Gam = exp(G)):
//
//   A[r,i] = b_r sum_c k_rc k_ic exp(G_rc - G_ic)  (i < r)
//   P[r,i] = sum_c q_rc k_ic exp(G_rc - G_ic)      (i <= r)
//   Tb     = (I + A)^{-1} diag(b)                  (UT transform, blocked 16 x 16)
//   W = Tb (K * Gam)                               (MMA, N = 128)
//   X      = [Tb ; 0] V + [-W ; Q * Gam] S         (one accumulator, M = 128)
//          = [U ; (Q * Gam) S],  U = Tb V - W S
//   O      = X[64:128] + [. ; P] U                 (MMA accumulate)
//   S     <- Diag(Gam_last) S + (K * exp(G_last - G))^T U
//
// A and P come from one M = 128 MMA [K * E ; Q * E] (K * E^-1)^T with
// E = exp(G - Gm) and a per-channel reference Gm = max_r G - 80 (b_r is applied
// to the A rows afterwards): every factor is then within exp(+-80) whenever
// the chunk's per-channel log-decay range is at most 160 and max G <= 60 (for
// the gates of all benchmark configurations the range is below 100).  The same
// tiles give K * Gam = (K * E) exp(Gm) and K * exp(G_last - G) =
// (K * E^-1) exp(G_last - Gm), with the per-channel factors applied in fp32 in
// the epilogues.  A chunk outside that range is evaluated exactly instead
// (A and P on CUDA cores with an exp per pair, Gam and exp(G_last - G) taken
// directly), so any finite g is handled.
//
// Shared-memory operand tiles use the 128-byte swizzle; a [rows][128] tile of
// bf16 is two 64-column halves, each rows x 128 B, and serves as a K-major
// operand (contraction over its 128 columns) or as an MN-major one
// (contraction over its rows).
//
// Kernels:
//   chunk_intra_kernel  persistent, two 256-thread CTAs per SM over all
//                       (chunk, head) items: the in-chunk cumulative
//                       log-gate, the operand tiles, A and P, the UT transform
//                       and W; it writes the chain's operands for that chunk
//                       to the workspace as one blob laid out exactly as the
//                       chain kernel's shared memory wants it.
//   chunk_chain_kernel  two CTAs per (sequence, head) -- one per half of the
//                       value columns -- chunks in order: bulk copies of each
//                       chunk's blob and that half of V, then X, O and S as
//                       above, with S carried in fp32 in tensor memory.
//   chunk_overlap_kernel the same two bodies co-scheduled in one cooperative
//                       launch (one 512-thread CTA of two units per SM; chain
//                       units alone on their SMs), chains waiting on per-blob
//                       ready flags.
// Parallel inside a chunk, recurrent between chunks: the split runs the first
// part on every SM and keeps only the second on the per-chain critical path.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "kda_chunk_tc.cuh"
#include "kda_common.cuh"
#include "kda_sm100.cuh"
#include "kda_tc_util.cuh"

namespace kda {
namespace {

using namespace sm100;
using namespace tc;

constexpr float kRef = 80.f;
constexpr uint64_t kWaitNs = 2000000000ull;

// ---- per (chunk, head) blob in the workspace (each part 1024-byte aligned)
constexpr uint32_t BL_WQ = 0;        // [-W kb0 | Q*Gam kb0 | -W kb1 | Q*Gam kb1] 32 KB
constexpr uint32_t BL_RAP = 32768;   // K * E^-1 (or K * exp(G_last - G))         16 KB
constexpr uint32_t BL_PM = 49152;    // P (masked), rows 64-127 of its operand      8 KB
constexpr uint32_t BL_TB = 57344;    // T diag(b), rows 0-63 of its operand         8 KB
constexpr uint32_t BL_SC = 65536;    // exp(G_last)[128], row scale of K~^T U [128]  1 KB
constexpr uint32_t BLOB = 66560;

}  // namespace

size_t split_blob_bytes() { return BLOB; }

namespace {

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) &
                                      ~static_cast<uintptr_t>(1023));
}

// ===================================================================== intra
// Persistent, two CTAs of 256 threads per SM (about 100 KB of shared memory
// each): every CTA walks the (chunk slot, head) items with a stride of the
// grid.  Operand tiles are built in place over the loaded K and Q; everything
// that only the chain kernel needs (Q * Gam, P, Tb, -W, the row scales) goes
// straight from registers to the item's blob in the workspace.  The next
// item's inputs are fetched as soon as their shared-memory regions are free;
// the other CTA on the SM covers the wait.
namespace intra {
constexpr int NTI = 256;
// [K kb0 | Q kb0 | K kb1 | Q kb1] as loaded; E2 turns it in place into the
// 128-row operand [K * E ; Q * E] (exact path: K * Gam in the K rows).
constexpr uint32_t OFF_KQ = 0;
constexpr uint32_t OFF_G = 32768;      // g (TMA) -> G -> A fp32 | T fp32
constexpr uint32_t OFF_RAP = 65536;    // K * E^-1 (exact path: K * exp(G_last - G))
// T diag(b) rows 0-63, then the garbage rows of its 128-row operand (also the
// inverse's scratch); before that: the scan's partial results (E1) and, on
// the exact path, A in fp32 (16 KB).
constexpr uint32_t OFF_TB = 81920;
constexpr uint32_t OFF_MID = 90112;
constexpr uint32_t OFF_BETA = 98304;
constexpr uint32_t OFF_GM = OFF_BETA + 256;
constexpr uint32_t OFF_EGM = OFF_GM + 512;
constexpr uint32_t OFF_GL = OFF_EGM + 512;
constexpr uint32_t OFF_WSC = OFF_GL + 512;
// head-uniform gate: g of the chunk's rows -> their G (64 floats), then
// {Gm, exp(Gm), G_last}
constexpr uint32_t OFF_GS = OFF_WSC + 512;
constexpr uint32_t OFF_GSC = OFF_GS + 256;
constexpr uint32_t OFF_BAR = OFF_GSC + 64;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;
// (layer variant) the 3 raw rows before the chunk of xk, xq [2][3][128] bf16,
// and the head's convolution filters of k, q [2][128][4] fp32 (slot 0: k,
// slot 1: q, the order of the K and Q tiles)
constexpr uint32_t OFF_HALO = OFF_BAR + 64;
constexpr uint32_t OFF_CW = OFF_HALO + 1536;
constexpr uint32_t SMEM_BYTES_CONV = OFF_CW + 4096 + 1024;
static_assert(OFF_MID == OFF_TB + 8192, "Tb garbage rows follow Tb");
static_assert(2 * (SMEM_BYTES_CONV + 1024) <= 233472, "two CTAs per SM");
constexpr uint32_t TM_X = 0;     // [A ; P] accumulator, 64 columns
constexpr uint32_t TM_W = 128;   // W accumulator, 128 columns
constexpr uint32_t TX_K = 16384, TX_Q = 16384, TX_G = 32768;

struct Params {
    const float* beta;
    const int4* info;
    int maxc;
    int H;
    const uint32_t* status;
    uint32_t* status_out;
    uint8_t* blobs;
    // co-scheduled with the chain kernel only:
    int N;
    const int* chunk_start;
    const uint32_t* rounds;  // largest number of chunks of one sequence
    uint32_t* flags;         // [slot, head]: set once that blob is complete
    const float* gh;         // head-uniform gate [total, H] (kScalar)
    // (testing the bounded-wait error path only) the flag index slot * H + h
    // that is never released, or -1
    long long withheld;
    // (layer variant) raw xq, xk [total, H, 128] (the tensor maps read them
    // too), their filters [H * 128, 4] and the L2-norm epsilon
    const __nv_bfloat16* xq;
    const __nv_bfloat16* xk;
    const float* wq;
    const float* wk;
    float l2_eps;
};

// (layer variant) q and k of the chunk from the raw inputs in place: the
// depthwise causal convolution of kernel 4 (the 3 rows before the chunk come
// from the halo buffer: the previous chunk's rows, or zeros at a sequence
// start), Swish, then each row divided by sqrt(sum of squares + eps) over its
// 128 channels.  Thread (row block b = tid / 16, channel chunk j = tid % 16)
// owns rows 4 b .. 4 b + 3, channels 8 j .. 8 j + 7: it reads its raw rows
// (and the three above them), waits at the barrier until every thread has
// read, then writes its rows.  The 16 threads of a row block are 16
// consecutive lanes, so the row sums are shuffles.
__device__ __forceinline__ void conv_qk_tile(uint8_t* sm, const Params& p, int tid, uint32_t bar,
                                             int nthreads) {
    const int j = tid & 15, kb = j >> 3, ch = j & 7, b = tid >> 4;
    uint4 out[2][4];
#pragma unroll
    for (int tensor = 0; tensor < 2; ++tensor) {
        const uint8_t* tile = sm + OFF_KQ + kb * 16384 + tensor * 8192;
        const float4* w = reinterpret_cast<const float4*>(sm + OFF_CW) + tensor * 128 + 8 * j;
        float x[7][8];
#pragma unroll
        for (int rr = 0; rr < 7; ++rr) {
            const int row = 4 * b - 3 + rr;
            const uint4 u = row >= 0 ? *reinterpret_cast<const uint4*>(tile + sw128_off(row, ch))
                                     : *reinterpret_cast<const uint4*>(
                                           sm + OFF_HALO + (tensor * 3 + row + 3) * 256 + 16 * j);
            unpack8(u, x[rr]);
        }
        float ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 wc = w[c];  // taps 0..3, tap 3 on the current row
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // x[i] is not read again after row i
                const float a = wc.x * x[i][c] + wc.y * x[i + 1][c] + wc.z * x[i + 2][c] +
                                wc.w * x[i + 3][c];
                const float y = fast_swish(a);
                x[i][c] = y;
                ss[i] += y * y;
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) ss[i] += __shfl_xor_sync(0xffffffffu, ss[i], o);
            const float inv = rsqrtf(ss[i] + p.l2_eps);
            float y[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) y[c] = x[i][c] * inv;
            out[tensor][i] = pack8(y);
        }
    }
    group_sync(bar, nthreads);
#pragma unroll
    for (int tensor = 0; tensor < 2; ++tensor) {
        uint8_t* tile = sm + OFF_KQ + kb * 16384 + tensor * 8192;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4*>(tile + sw128_off(4 * b + i, ch)) = out[tensor][i];
    }
}

// One worker (CTA) of the intra-chunk kernel.  Items are (chunk slot, head)
// pairs taken with a stride of `nworkers`: alone, in slot order; co-scheduled
// with the chains (kOverlap), round by round -- chunk n of every (sequence,
// head) before chunk n + 1 of any -- and each finished blob is flagged.
// The unit is a group of NTI threads (a whole CTA, or half of one) that
// synchronises on named barrier `bar`; `tbase` is its 256 TMEM columns.
// kScalar: the gate is one value per (token, head) (Gated DeltaNet; Kimi
// Linear (aiwiki.ai), "Background: from the delta rule to gated DeltaNet"):
// read from p.gh by plain loads, scanned by one warp, and every per-channel
// factor of a row is that row's one factor.
// kConv (layer variant, not with kOverlap or kScalar): the tensor maps read
// the raw inputs xq, xk, and conv_qk_tile makes q and k of them in place.
template <bool kOverlap, bool kScalar = false, bool kConv = false>
__device__ __forceinline__ void run(const CUtensorMap* tmq, const CUtensorMap* tmk,
                                    const CUtensorMap* tmg, const Params& p, uint8_t* sm,
                                    uint32_t tbase, uint32_t bar, int worker, int nworkers) {
    const int maxc = p.maxc, NH = kOverlap ? p.N * p.H : 1;
    const int nitems = kOverlap ? static_cast<int>(*p.rounds) * NH : maxc * p.H;
    const uint32_t sbase = smem_u32(sm);
    float* sbeta = reinterpret_cast<float*>(sm + OFF_BETA);
    float* sGm = reinterpret_cast<float*>(sm + OFF_GM);
    float* seGm = reinterpret_cast<float*>(sm + OFF_EGM);
    float* sGL = reinterpret_cast<float*>(sm + OFF_GL);
    float* sWsc = reinterpret_cast<float*>(sm + OFF_WSC);
    uint64_t* bar_k = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint64_t* bar_q = bar_k + 1;
    uint64_t* bar_g = bar_k + 2;
    uint64_t* bar_mma = bar_k + 3;
    const int tid = threadIdx.x & (NTI - 1), warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, cq = warp >> 2;  // TMEM lanes 32 quarter.., columns 32 cq..
    const int trow = 32 * quarter + lane;
    const uint32_t tlane = static_cast<uint32_t>(32 * quarter) << 16;
    // item -> (chunk slot, head); items of empty slots (varlen upper bound)
    // or past the end of a sequence are skipped
    auto slot_of = [&](int it) {
        return kOverlap ? p.chunk_start[(it % NH) / p.H] + it / NH : it % maxc;
    };
    auto head_of = [&](int it) { return kOverlap ? (it % NH) % p.H : it / maxc; };
    auto valid = [&](int it) {
        if (!kOverlap) return p.info[it % maxc].z > 0;
        const int s = (it % NH) / p.H;
        return p.chunk_start[s] + it / NH < p.chunk_start[s + 1];
    };
    auto advance = [&](int it) {
        while (it < nitems && !valid(it)) it += nworkers;
        return it;
    };
    // everything the loop needs of an item, fetched (global loads) one item
    // ahead of its use: {item, chunk slot, head, rows, first token}
    struct Item {
        int it, slot, h, L, t0, cs;  // cs: the chunk's index in its sequence
    };
    auto describe = [&](int it) {
        Item d{it, 0, 0, 0, 0, 0};
        if (it < nitems) {
            d.slot = slot_of(it);
            d.h = head_of(it);
            const int4 c = p.info[d.slot];
            d.L = c.z;
            d.t0 = c.y;
            d.cs = c.w;
        }
        return d;
    };
    int* s_ahead = reinterpret_cast<int*>(sm + OFF_BAR + 32);  // the item after the next
    // loads of an item's inputs (thread 0), each on its own barrier
    auto load_k = [&](const Item& d) {
        mbar_arrive_expect_tx(bar_k, TX_K);
        tma_load_3d(sm + OFF_KQ, tmk, bar_k, 0, d.h, d.t0);
        tma_load_3d(sm + OFF_KQ + 16384, tmk, bar_k, 64, d.h, d.t0);
    };
    auto load_q = [&](const Item& d) {
        mbar_arrive_expect_tx(bar_q, TX_Q);
        tma_load_3d(sm + OFF_KQ + 8192, tmq, bar_q, 0, d.h, d.t0);
        tma_load_3d(sm + OFF_KQ + 24576, tmq, bar_q, 64, d.h, d.t0);
    };
    auto load_g = [&](const Item& d) {
        mbar_arrive_expect_tx(bar_g, TX_G);
        tma_load_3d(sm + OFF_G, tmg, bar_g, 0, d.h, d.t0);
    };

    if (tid == 0) {
        mbar_init(bar_k, 1);
        mbar_init(bar_q, 1);
        mbar_init(bar_g, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    group_sync(bar, NTI);
    tc_fence_after();
    bool failed = false;
    uint32_t mma_phase = 0;
    // loads issued (thread 0's count; for the exit path)
    int k_issued = 0, q_issued = 0, g_issued = 0;
    Item cur = describe(advance(worker));
    Item nxt = describe(cur.it < nitems ? advance(cur.it + nworkers) : nitems);
    long long flag_pending = -1;  // (kOverlap) finished blob not yet released
    float beta_next = 0.f;  // (tid < C) this thread's beta of the next item
    auto fetch_beta = [&](const Item& d) {
        return tid < d.L ? p.beta[(size_t)(d.t0 + tid) * p.H + d.h] : 0.f;
    };
    float* sGs = reinterpret_cast<float*>(sm + OFF_GS);
    float* sGsc = reinterpret_cast<float*>(sm + OFF_GSC);
    float gs_next = 0.f;  // (kScalar, tid < C) this thread's g of the next item
    auto fetch_gs = [&](const Item& d) {
        return tid < d.L ? p.gh[(size_t)(d.t0 + tid) * p.H + d.h] : 0.f;
    };
    if (cur.it < nitems) {
        if (tid == 0) {
            load_k(cur);
            load_q(cur);
            if (!kScalar) load_g(cur);
            k_issued = q_issued = 1;
            g_issued = kScalar ? 0 : 1;
        }
        if (tid < C) beta_next = fetch_beta(cur);
        if (kScalar && tid < C) gs_next = fetch_gs(cur);
    }
    int n = 0;
    for (; cur.it < nitems && !failed; ++n) {
        const int slot = cur.slot, h = cur.h, L = cur.L;
        const bool more = nxt.it < nitems;
        uint8_t* blob = p.blobs + ((size_t)slot * p.H + h) * BLOB;
        if (kConv) {
            // the 3 raw rows of xq, xk before the chunk (zeros at a sequence
            // start) and the head's filters, waited for before the convolution
            for (int e = tid; e < 96 + 256; e += NTI) {
                if (e < 96) {
                    const int tensor = e / 48, row = (e % 48) / 16, j = e % 16;
                    uint8_t* dst = sm + OFF_HALO + (tensor * 3 + row) * 256 + 16 * j;
                    if (cur.cs > 0)  // slot 0: k, slot 1: q (the order of the tiles)
                        cp_async16(dst, (tensor ? p.xq : p.xk) +
                                            ((size_t)(cur.t0 - 3 + row) * p.H + h) * D + 8 * j);
                    else
                        *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
                } else {
                    const int tensor = (e - 96) >> 7, c = (e - 96) & 127;
                    cp_async16(sm + OFF_CW + (tensor * 128 + c) * 16,
                               (tensor ? p.wq : p.wk) + ((size_t)h * D + c) * 4);
                }
            }
            cp_async_commit();
        }
        if (tid < C) sbeta[tid] = beta_next;
        if (kScalar && tid < C) sGs[tid] = gs_next;
        if (tid == 0) {
            // the previous item's bulk write-out has read its tiles (and, when
            // a chain waits for it, has completed)
            if (kOverlap)
                bulk_wait_all();
            else
                bulk_wait_read();
        }
        bool ok = kScalar || mbar_wait(bar_g, n & 1, kWaitNs);  // K, Q: after E1
        if (group_sync_or(bar, NTI, !ok)) {
            failed = true;
            break;
        }
        // ------------- E1: in-chunk cumulative log-gate, per channel.  Thread
        // (row group grp = 8 rows, channels 4 c4 ..): scan of its 8 rows, then
        // the totals of the groups above it added; per-channel max / min.
        bool slow_local = false;
        if (kScalar) {
            // one warp: lane l holds rows 2l, 2l + 1; inclusive scan by shuffles
            if (warp == 0) {
                const int r0 = 2 * lane;
                const float v0 = r0 < L ? sGs[r0] : 0.f, v1 = r0 + 1 < L ? sGs[r0 + 1] : 0.f;
                float pre = v0 + v1;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, pre, o);
                    if (lane >= o) pre += y;
                }
                const float G0 = pre - v1, G1 = pre;
                float mx = -INFINITY, mn = INFINITY;
                if (r0 < L) { mx = G0; mn = G0; }
                if (r0 + 1 < L) { mx = fmaxf(mx, G1); mn = fminf(mn, G1); }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                }
                __syncwarp();
                sGs[r0] = G0;
                sGs[r0 + 1] = G1;
                __syncwarp();
                if (lane == 0) {
                    const float Gm = mx - kRef;
                    sGsc[0] = Gm;
                    sGsc[1] = expf(Gm);
                    sGsc[2] = sGs[L - 1];
                }
                slow_local = !(mx - mn <= 2.f * kRef) || !(mx <= 60.f);
            }
            group_sync(bar, NTI);
            if (tid < D) {  // the per-channel arrays all hold the row-uniform values
                sGm[tid] = sGsc[0];
                seGm[tid] = sGsc[1];
                sGL[tid] = sGsc[2];
            }
        } else {
            float* g = reinterpret_cast<float*>(sm + OFF_G);
            float4* tot = reinterpret_cast<float4*>(sm + OFF_TB);           // [8][32]
            float4* gmx = reinterpret_cast<float4*>(sm + OFF_TB + 4096);    // [8][32]
            float4* gmn = reinterpret_cast<float4*>(sm + OFF_TB + 8192);    // [8][32]
            const int c4 = tid & 31, grp = tid >> 5, r0 = 8 * grp;
            float4 x[8];
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float4 v = *reinterpret_cast<const float4*>(g + (r0 + i) * D + 4 * c4);
                if (r0 + i >= L) v = make_float4(0.f, 0.f, 0.f, 0.f);
                acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
                x[i] = acc;
            }
            tot[grp * 32 + c4] = acc;
            group_sync(bar, NTI);
            float4 off = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int j = 0; j < grp; ++j) {
                const float4 t = tot[j * 32 + c4];
                off.x += t.x; off.y += t.y; off.z += t.z; off.w += t.w;
            }
            float4 mx = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            float4 mn = make_float4(INFINITY, INFINITY, INFINITY, INFINITY);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float4 v = x[i];
                v.x += off.x; v.y += off.y; v.z += off.z; v.w += off.w;
                *reinterpret_cast<float4*>(g + (r0 + i) * D + 4 * c4) = v;
                if (r0 + i < L) {
                    mx.x = fmaxf(mx.x, v.x); mx.y = fmaxf(mx.y, v.y);
                    mx.z = fmaxf(mx.z, v.z); mx.w = fmaxf(mx.w, v.w);
                    mn.x = fminf(mn.x, v.x); mn.y = fminf(mn.y, v.y);
                    mn.z = fminf(mn.z, v.z); mn.w = fminf(mn.w, v.w);
                }
            }
            gmx[grp * 32 + c4] = mx;
            gmn[grp * 32 + c4] = mn;
            group_sync(bar, NTI);
            if (tid < D) {
                const int c = tid;
                const float* fx = reinterpret_cast<const float*>(gmx);
                const float* fn = reinterpret_cast<const float*>(gmn);
                float gmax = -INFINITY, gmin = INFINITY;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    gmax = fmaxf(gmax, fx[j * D + c]);
                    gmin = fminf(gmin, fn[j * D + c]);
                }
                const float Gm = gmax - kRef;
                const float gl = g[(L - 1) * D + c];
                sGm[c] = Gm;
                seGm[c] = expf(Gm);
                sGL[c] = gl;
                slow_local = !(gmax - gmin <= 2.f * kRef) || !(gmax <= 60.f);
            }
        }
        ok = mbar_wait(bar_k, n & 1, kWaitNs) && mbar_wait(bar_q, n & 1, kWaitNs);
        if (kConv) cp_async_wait_all();
        if (group_sync_or(bar, NTI, !ok)) {
            failed = true;
            break;
        }
        if (kConv) conv_qk_tile(sm, p, tid, bar, NTI);  // its writes: visible after the next barrier
        const bool slow = group_sync_or(bar, NTI, slow_local);
        if (tid < D) {  // row scales of the chain kernel; -W column scale
            const float gl = sGL[tid];
            sWsc[tid] = slow ? -1.f : -seGm[tid];
            float* sc = reinterpret_cast<float*>(blob + BL_SC);
            sc[tid] = expf(gl);
            sc[D + tid] = slow ? 1.f : expf(gl - sGm[tid]);
        }
        // -------- exact A (fp32, into the Tb region) and P (straight to the
        // blob) on CUDA cores (rare: extreme decay)
        if (slow) {
            const float* G = reinterpret_cast<const float*>(sm + OFF_G);
            float* Af = reinterpret_cast<float*>(sm + OFF_TB);
            for (int task = tid; task < C * 8; task += NTI) {
                const int r = task >> 3, i0 = 8 * (task & 7);
                float a[8], pp[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) a[j] = pp[j] = 0.f;
                if (r < L && kScalar) {  // one factor per pair, outside the dot products
                    for (int c = 0; c < D; ++c) {
                        const float kr = tile_elem(sm + OFF_KQ, 16384, r, c);
                        const float qr = tile_elem(sm + OFF_KQ + 8192, 16384, r, c);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float ki = tile_elem(sm + OFF_KQ, 16384, i0 + j, c);
                            a[j] += kr * ki;
                            pp[j] += qr * ki;
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int i = i0 + j;
                        const float e = i <= r ? expf(sGs[r] - sGs[i]) : 0.f;
                        a[j] *= e;
                        pp[j] *= e;
                    }
                } else if (r < L) {
                    for (int c = 0; c < D; ++c) {
                        const float kr = tile_elem(sm + OFF_KQ, 16384, r, c);
                        const float qr = tile_elem(sm + OFF_KQ + 8192, 16384, r, c);
                        const float gr = G[r * D + c];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int i = i0 + j;
                            if (i <= r) {
                                const float e = expf(gr - G[i * D + c]);
                                const float ki = tile_elem(sm + OFF_KQ, 16384, i, c) * e;
                                a[j] += kr * ki;
                                pp[j] += qr * ki;
                            }
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int i = i0 + j;
                    Af[a_idx(r, i)] = (i < r) ? sbeta[r] * a[j] : 0.f;
                    if (i > r) pp[j] = 0.f;
                }
                *reinterpret_cast<uint4*>(blob + BL_PM + sw128_off(r, task & 7)) = pack8(pp);
            }
            group_sync(bar, NTI);
        }
        // ------------------------------ E2: operand tiles, row-parallel; each
        // thread keeps one 8-channel group (j = tid & 15) for all its rows
        {
            const float* G = reinterpret_cast<const float*>(sm + OFF_G);
            const int j = tid & 15, kb = j >> 3, ch = j & 7, c0 = 8 * j;
            float m8[8], e8[8];
            load8(slow ? sGL + c0 : sGm + c0, m8);
            load8(seGm + c0, e8);
#pragma unroll
            for (int s = 0; s < (C * 16) / NTI; ++s) {
                const int r = (tid + NTI * s) >> 4;
                const uint32_t o64 = sw128_off(r, ch);
                uint8_t* pk = sm + OFF_KQ + kb * 16384 + o64;
                uint8_t* pq = pk + 8192;
                float lk[8], lq[8], rk[8], qg[8];
                if (r < L && kScalar) {  // the row's factors, once
                    float k8[8], q8[8];
                    unpack8(*reinterpret_cast<const uint4*>(pk), k8);
                    unpack8(*reinterpret_cast<const uint4*>(pq), q8);
                    const float gr = sGs[r];
                    if (!slow) {
                        const float x = gr - m8[0];
                        const float E = __expf(x), Ei = __expf(-x), eg = e8[0];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            lk[i] = k8[i] * E;
                            lq[i] = q8[i] * E;
                            rk[i] = k8[i] * Ei;
                            qg[i] = lq[i] * eg;
                        }
                    } else {  // m8 holds G_last here
                        const float gam = expf(gr), back = expf(m8[0] - gr);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            lk[i] = k8[i] * gam;
                            lq[i] = 0.f;
                            rk[i] = k8[i] * back;
                            qg[i] = q8[i] * gam;
                        }
                    }
                } else if (r < L) {
                    float k8[8], q8[8], g8[8];
                    unpack8(*reinterpret_cast<const uint4*>(pk), k8);
                    unpack8(*reinterpret_cast<const uint4*>(pq), q8);
                    load8(G + r * D + c0, g8);
                    if (!slow) {
                        // factors within exp(+-80), rounded to bf16 right after
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float x = g8[i] - m8[i];
                            const float E = __expf(x), Ei = __expf(-x);
                            lk[i] = k8[i] * E;
                            lq[i] = q8[i] * E;
                            rk[i] = k8[i] * Ei;
                            qg[i] = lq[i] * e8[i];
                        }
                    } else {  // m8 holds G_last here
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float gam = expf(g8[i]);
                            lk[i] = k8[i] * gam;  // K * Gam, in place of K
                            lq[i] = 0.f;
                            rk[i] = k8[i] * expf(m8[i] - g8[i]);
                            qg[i] = q8[i] * gam;
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) lk[i] = lq[i] = rk[i] = qg[i] = 0.f;
                }
                *reinterpret_cast<uint4*>(pk) = pack8(lk);
                *reinterpret_cast<uint4*>(pq) = pack8(lq);
                *reinterpret_cast<uint4*>(sm + OFF_RAP + kb * 8192 + o64) = pack8(rk);
                *reinterpret_cast<uint4*>(blob + BL_WQ + kb * 16384 + 8192 + o64) = pack8(qg);
            }
        }
        fence_async_smem();
        tc_fence_before();
        group_sync(bar, NTI);
        tc_fence_after();
        if (tid < C && more) {
            beta_next = fetch_beta(nxt);
            if (kScalar) gs_next = fetch_gs(nxt);
        }
        if (tid == 0) {
            bulk_s2g(blob + BL_RAP, sm + OFF_RAP, 16384);  // the chain's K E^-1
            bulk_commit();
            if (slow && more) {  // exact path: Q is consumed already
                load_q(nxt);
                ++q_issued;
            }
        }
        // ------------------------------------------------ A, P (M=128, N=64)
        if (!slow) {
            if (tid == 0) {
                constexpr uint32_t id = idesc_bf16_f32(128, 64, false, false);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const int kb = ks >> 2, kk = ks & 3;
                    mma_bf16(tbase + TM_X,
                             sdesc_sw128(sbase + OFF_KQ + kb * 16384 + kk * 32, 16, 1024),
                             sdesc_sw128(sbase + OFF_RAP + kb * 8192 + kk * 32, 16, 1024), id,
                             ks > 0);
                }
                mma_commit(bar_mma);
            }
            ok = mbar_wait(bar_mma, mma_phase & 1, kWaitNs);
            ++mma_phase;
            if (group_sync_or(bar, NTI, !ok)) {
                failed = true;
                break;
            }
            tc_fence_after();
            if (tid == 0 && more) {  // the Q * E rows are consumed
                load_q(nxt);
                ++q_issued;
            }
        }
        // ------ A -> fp32 (swizzled, in the G region); P -> bf16, to the blob
        {
            float* Af = reinterpret_cast<float*>(sm + OFF_G);
            const int m = trow;  // TMEM lane == row of the 128-row result
            // (warp 4 holds the block of A above the diagonal: never read)
            if (!slow && !(quarter == 0 && cq == 1)) {
                uint32_t v[32];
                tmem_ld32(tbase + tlane + TM_X + cq * 32, v);
                tmem_wait_ld();
                if (m < C) {
                    const float b = sbeta[m];
#pragma unroll
                    for (int i4 = 0; i4 < 8; ++i4) {
                        const int col = cq * 32 + 4 * i4;
                        float y[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            y[i] = (m < L && col + i < m) ? b * __uint_as_float(v[4 * i4 + i])
                                                          : 0.f;
                        *reinterpret_cast<float4*>(Af + a_idx(m, col)) =
                            make_float4(y[0], y[1], y[2], y[3]);
                    }
                } else {
                    const int r = m - C;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        float y[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int col = cq * 32 + q4 * 8 + i;
                            y[i] = (r < L && col <= r) ? __uint_as_float(v[q4 * 8 + i]) : 0.f;
                        }
                        *reinterpret_cast<uint4*>(blob + BL_PM +
                                                  sw128_off(r, (cq * 32 + q4 * 8) >> 3)) =
                            pack8(y);
                    }
                }
            } else if (slow) {
                const float4* srcA = reinterpret_cast<const float4*>(sm + OFF_TB);
                float4* dstA = reinterpret_cast<float4*>(Af);
                for (int i = tid; i < C * C / 4; i += NTI) dstA[i] = srcA[i];
                group_sync(bar, NTI);  // (slow is the same on every thread)
            }
        }
        // ------------------ UT transform: T = (I + A)^{-1}, blocked 16 x 16,
        // written as T (fp32) and Tb = T diag(b) (bf16, rows 0-63 of the W
        // product's operand).  The warps that hold A's diagonal blocks (warp
        // 0: rows and columns 0-31, warp 5: 32-63) invert them and form the
        // off-diagonal block between them right after their read-out; warp 4
        // zeroes Tb above the diagonal; then the lower-left 32 x 32 block.
        {
            const float* __restrict__ Af = reinterpret_cast<const float*>(sm + OFF_G);
            float* Tf = reinterpret_cast<float*>(sm + OFF_G + 16384);
            float* Mf = reinterpret_cast<float*>(sm + OFF_MID);
            uint8_t* tb = sm + OFF_TB;
            if (warp == 0 || warp == 5) {
                const int J = warp == 0 ? 0 : 2;
                __syncwarp();
                diag_inverse(Af, Tf, tb, sbeta, J, lane);
                __syncwarp();
                inverse_pair(Af, Tf, Mf + J * 128, tb, sbeta, J, lane);
            } else if (warp == 4) {
                tb_zero_upper(tb, lane);
            }
            if (tid == NTI - 32) {
                // the previous item's blob is complete (all of its writes came
                // before this item's first barrier): release it to its chain
                if (kOverlap && flag_pending >= 0 && flag_pending != p.withheld) {
                    fence_proxy_async_global();
                    flag_release(p.flags + flag_pending, 1u);
                }
                // look up the item after the next
                const Item d = describe(more ? advance(nxt.it + nworkers) : nitems);
                s_ahead[0] = d.it;
                s_ahead[1] = d.slot;
                s_ahead[2] = d.h;
                s_ahead[3] = d.L;
                s_ahead[4] = d.t0;
                s_ahead[5] = d.cs;
            }
            group_sync(bar, NTI);
            inverse_lower_left(Af, Tf, Mf, tb, sbeta, warp, lane, bar + 2);
        }
        fence_async_smem();
        tc_fence_before();
        group_sync(bar, NTI);
        tc_fence_after();
        // ---------------------------------- W = Tb (K*E) [*exp(Gm)]  (N=128)
        if (tid == 0) {
            bulk_s2g(blob + BL_TB, sm + OFF_TB, 8192);  // the chain's Tb
            bulk_commit();
            if (more && !kScalar) {  // the G region is free: fetch the next g
                load_g(nxt);
                ++g_issued;
            }
            constexpr uint32_t id = idesc_bf16_f32(128, 128, false, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tbase + TM_W, sdesc_sw128(sbase + OFF_TB + ks * 32, 16, 1024),
                         sdesc_sw128(sbase + OFF_KQ + ks * 2048, 16384, 1024), id, ks > 0);
            mma_commit(bar_mma);
        }
        ok = mbar_wait(bar_mma, mma_phase & 1, kWaitNs);
        ++mma_phase;
        if (group_sync_or(bar, NTI, !ok)) {
            failed = true;
            break;
        }
        tc_fence_after();
        if (tid == 0 && more) {  // the K rows are consumed: fetch the next K
            load_k(nxt);
            ++k_issued;
        }
        // -W (rows 0-63), column-scaled -> bf16, to the blob's [-W ; Q*Gam]
        if (quarter < 2) {
            const int r = trow;
#pragma unroll
            for (int hcol = 0; hcol < 2; ++hcol) {
                const int cbase = 64 * cq + 32 * hcol;
                uint32_t v[32];
                tmem_ld32(tbase + tlane + TM_W + cbase, v);
                tmem_wait_ld();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int col = cbase + q4 * 8;
                    float sc[8], y[8];
                    load8(sWsc + col, sc);
#pragma unroll
                    for (int i = 0; i < 8; ++i) y[i] = __uint_as_float(v[q4 * 8 + i]) * sc[i];
                    *reinterpret_cast<uint4*>(blob + BL_WQ + (col >> 6) * 16384 +
                                              sw128_off(r, (col & 63) >> 3)) = pack8(y);
                }
            }
        }
        if (kOverlap) flag_pending = static_cast<long long>(slot) * p.H + h;
        cur = nxt;
        nxt = Item{s_ahead[0], s_ahead[1], s_ahead[2], s_ahead[3], s_ahead[4], s_ahead[5]};
    }
    if (tid == 0) bulk_wait_all();
    if (failed && tid == 0) {
        // wait (bounded) for this CTA's copies and products still in flight
        // (a wait on a phase that has already completed returns at once)
        if (mma_phase > 0) mbar_wait(bar_mma, (mma_phase - 1) & 1, kWaitNs);
        if (k_issued > 0) mbar_wait(bar_k, (k_issued - 1) & 1, kWaitNs);
        if (q_issued > 0) mbar_wait(bar_q, (q_issued - 1) & 1, kWaitNs);
        if (g_issued > 0) mbar_wait(bar_g, (g_issued - 1) & 1, kWaitNs);
        atomicOr(p.status_out, STATUS_TIMEOUT);
    }
    tc_fence_before();
    group_sync(bar, NTI);
    if (kOverlap && flag_pending >= 0 && flag_pending != p.withheld && tid == NTI - 32) {
        fence_proxy_async_global();
        flag_release(p.flags + flag_pending, 1u);
    }
}

template <bool kScalar, bool kConv>
__global__ void __launch_bounds__(NTI, 2)
    chunk_intra_kernel(const __grid_constant__ CUtensorMap tmq,
                       const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmg, const Params p) {
    if (status_bad(p.status)) return;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t s_tmem;
    if (threadIdx.x < 32) {
        tmem_alloc(&s_tmem, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    run<false, kScalar, kConv>(&tmq, &tmk, &tmg, p, align1024(smem_raw), s_tmem, 1, blockIdx.x,
                               gridDim.x);
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) tmem_dealloc(s_tmem, 256);
}
}  // namespace intra

// ===================================================================== chain
// One CTA per (sequence, head, half of the value columns): the two halves of a
// state evolve independently (the transition acts on the key side only), so a
// chain runs on two SMs with N = 64 products, and two such CTAs fit on one SM.
namespace chain {
constexpr int NTC = 256;         // threads (8 warps: 4 lane quarters x 2 column pieces)
constexpr int DVS = 64;          // value columns per CTA
constexpr uint32_t OFF_WQ = 0;         // [W | Q*Gam] (blob part)
constexpr uint32_t OFF_RAP = 32768;    // K E^-1
constexpr uint32_t OFF_PM = 49152;     // P rows 64-127; operand starts 8 KB earlier (RAP tail)
constexpr uint32_t OFF_TB = 57344;     // Tb rows 0-63 of a 128-row operand ...
constexpr uint32_t OFF_ZERO = 65536;   // ... whose rows 64-127 are zeros (set once)
constexpr uint32_t OFF_V = 73728;      // V [64 tokens][64 columns of this half] (TMA)
constexpr uint32_t OFF_SB = 81920;     // S bf16 [dk][64], MN-major
constexpr uint32_t OFF_UB = 98304;     // U bf16 [token][64], MN-major
constexpr uint32_t OFF_SC0 = 106496;   // exp(G_last), row scale: two buffers of 1 KB
constexpr uint32_t OFF_SC1 = 107520;
constexpr uint32_t OFF_BAR = 108544;
// (co-scheduled) number of leading chunks whose blobs are ready, or -1 if the
// wait for one gave up; written by the watcher thread, read by thread 0
constexpr uint32_t OFF_RDY = OFF_BAR + 32;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;
// (layer variant) raw V rows 61-63 of the previous chunk [3][64] bf16 (zeros
// before a sequence's first chunk); this half's v filters [64][4] fp32 and
// RMSNorm weights [64] fp32; the partner half's row sums of o^2 written into
// this unit by the partner unit [2 chunk parities][64]; this unit's two
// column pieces' row sums [2][64]; two mbarriers (one per parity) on which
// the partner's 64 row threads arrive
constexpr uint32_t OFF_VH = OFF_BAR + 64;
constexpr uint32_t OFF_WV = OFF_VH + 384;
constexpr uint32_t OFF_WN = OFF_WV + 1024;
constexpr uint32_t OFF_SSX = OFF_WN + 256;
constexpr uint32_t OFF_SSL = OFF_SSX + 512;
constexpr uint32_t OFF_NBAR = OFF_SSL + 512;
static_assert(OFF_ZERO == OFF_TB + 8192, "Tb zero rows");
static_assert(OFF_PM == OFF_RAP + 16384, "P garbage rows");
static_assert(2 * SMEM_BYTES <= 228 * 1024, "two CTAs per SM");
constexpr uint32_t TM_W = 0;     // (K E^-1)^T U   [128 x 64]
// [Ut ; 0] + [-W ; Q*Gam] S = [U ; Q*Gam S], then O in rows 64-127; two
// buffers (even / odd chunks), so that a chunk's O is read out while the next
// chunk's first products run
constexpr uint32_t TM_X = 64;
constexpr uint32_t TM_S = 128;   // fp32 state [128 x 64]
constexpr uint32_t TM_X1 = 192;
// loads of one chunk: groups 1 and 2 on one barrier, group 3 (needed only by
// the second round of products) on another
constexpr uint32_t TX_A = 1024 + 8192 + 8192 + 32768, TX_B = 16384 + 8192;

struct Params {
    const float* h0;
    const int32_t* cu;
    int T;
    int H;
    const int* chunk_start;
    const uint32_t* status;
    uint32_t* status_out;
    const uint8_t* blobs;
    __nv_bfloat16* o;
    float* hN;
    const uint32_t* flags;  // co-scheduled with the intra kernel: blob ready flags
    uint64_t flag_wait_ns;  // bound of the watcher's wait on one flag
    const int* order;       // (split plan) sequences, longest first, or NULL
    // (layer variant) the tensor map reads raw xv; its filters [H * 128, 4];
    // y = RMSNorm(o) * w_norm * sigmoid(gate) is written instead of o
    const float* wv;
    const __nv_bfloat16* gate;
    const float* w_norm;
    float rms_eps;
    __nv_bfloat16* y;
    // (state maps only) v taken as zero (V is not read, the Tb V product is
    // not formed) and the entry state as the identity (h0 is not read)
    bool zero_v;
    bool identity_h0;
};

// (layer variant) V of the chunk from the raw inputs in place: the depthwise
// causal convolution of kernel 4 and Swish.  Thread (row pair b = tid / 8,
// column chunk j = tid % 8) owns rows 2 b, 2 b + 1 and columns 8 j .. 8 j + 7;
// the 3 rows above the tile come from the halo (the previous chunk's raw rows
// 61-63), which the owners of rows 61-63 then refill from this chunk.  Reads,
// barrier, writes.
__device__ __forceinline__ void conv_v_tile(uint8_t* sm, int tid, uint32_t bar, int nthreads) {
    const int j = tid & 7, b = tid >> 3;
    const float4* w = reinterpret_cast<const float4*>(sm + OFF_WV) + 8 * j;
    float x[5][8];
#pragma unroll
    for (int rr = 0; rr < 5; ++rr) {
        const int row = 2 * b - 3 + rr;
        const uint4 u = row >= 0
                            ? *reinterpret_cast<const uint4*>(sm + OFF_V + sw128_off(row, j))
                            : *reinterpret_cast<const uint4*>(sm + OFF_VH + (row + 3) * 128 + 16 * j);
        unpack8(u, x[rr]);
    }
    // raw rows 61, 62, 63 for the next chunk's halo: rows 2b+1 (b = 30) and 2b,
    // 2b+1 (b = 31) are x[4] (b = 30), x[3], x[4] (b = 31)
    const uint4 raw_a = pack8(x[3]), raw_b = pack8(x[4]);
    uint4 out[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        float y[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 wc = w[c];
            const float a = wc.x * x[i][c] + wc.y * x[i + 1][c] + wc.z * x[i + 2][c] +
                            wc.w * x[i + 3][c];
            y[c] = fast_swish(a);
        }
        out[i] = pack8(y);
    }
    group_sync(bar, nthreads);
#pragma unroll
    for (int i = 0; i < 2; ++i)
        *reinterpret_cast<uint4*>(sm + OFF_V + sw128_off(2 * b + i, j)) = out[i];
    uint4* vh = reinterpret_cast<uint4*>(sm + OFF_VH);
    if (b == 30) vh[0 * 8 + j] = raw_b;  // row 61
    if (b == 31) {
        vh[1 * 8 + j] = raw_a;  // row 62
        vh[2 * 8 + j] = raw_b;  // row 63
    }
}

// One chain CTA: (sequence, head) `chain_id`, value columns [64 half, +64).
// Each chunk's loads come in three groups, issued as soon as their regions
// are free (1: row scales; 2: Tb, V, [-W ; Q*Gam]; 3: K E^-1, P).  When
// co-scheduled with the intra kernel (kOverlap) a chunk's groups wait until
// the watcher (another thread of the CTA, below) has seen that chunk's blob
// flag: checked at each issue point, waited for (bounded) only when the chunk
// is next.
// The unit is a group of NTC threads synchronising on named barrier `bar`;
// `tbase` is its 256 TMEM columns.
// kLayer (layer variant, split plan only, the two halves of a chain as the two
// units of one CTA): V is convolved in place (conv_v_tile) -- the first
// chunk's between the two parts of its first product, later ones' during the
// previous chunk's second products -- and the O read-out writes y =
// RMSNorm(o) * w_norm * sigmoid(gate), the row sums of o^2 over all 128
// columns combined with the partner unit's through shared memory
// (sm_partner: the partner unit's region).
template <bool kOverlap, bool kLayer = false>
__device__ __forceinline__ void run(const CUtensorMap* tmv, const Params& p, uint8_t* sm,
                                    uint32_t tbase, uint32_t bar, int chain_id, int half,
                                    const CUtensorMap* tmgate = nullptr,
                                    uint8_t* sm_partner = nullptr) {
    const uint32_t sbase = smem_u32(sm);
    uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint64_t* bar_mma = bar_ld + 1;
    uint64_t* bar_ld3 = bar_ld + 2;
    uint64_t* bar_gt = bar_ld + 3;  // (layer variant) the output gate tile of a chunk
    const int tid = threadIdx.x & (NTC - 1), warp = tid >> 5;
    const int quarter = warp & 3, cq = warp >> 2;  // rows 32 quarter + lane, columns 32 cq ..
    const int trow = 32 * quarter + (tid & 31);
    const uint32_t tlane = static_cast<uint32_t>(32 * quarter) << 16;
    const int j0 = DVS * half;
    const int seq = chain_id / p.H, h = chain_id % p.H;
    const int t_begin = p.cu ? p.cu[seq] : seq * p.T;
    const int t_end = p.cu ? p.cu[seq + 1] : (seq + 1) * p.T;
    const int cbase = p.chunk_start[seq];
    auto blob = [&](int n) { return p.blobs + ((size_t)(cbase + n) * p.H + h) * BLOB; };
    auto tx = [](int n) { return (n & 1) ? TM_X1 : TM_X; };

    if (tid == 0) {
        mbar_init(bar_ld, 1);
        if (kLayer) mbar_init(bar_gt, 1);
        mbar_init(bar_ld3, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    group_sync(bar, NTC);
    tc_fence_after();
    bool failed = false;
    uint32_t mma_phase = 0;
    // thread 0: load groups of the coming chunk not issued yet, whether its
    // transaction count is registered, whether its blob was seen ready
    int pend = 0, coming = 0;
    int ld3_chunk = -1;  // chunk whose group 3 is in flight and not yet waited for
    int gt_issued = 0;   // (layer variant, thread 0) gate tiles requested
    bool armed = false, armed3 = false, rdy = false;
    const int* s_rdy = reinterpret_cast<const int*>(sm + OFF_RDY);
    auto issue = [&](int n, int groups) {
        const uint8_t* b = blob(n);
        if (groups & 1) bulk_g2s(sm + ((n & 1) ? OFF_SC1 : OFF_SC0), b + BL_SC, 1024, bar_ld);
        if (groups & 2) {
            bulk_g2s(sm + OFF_TB, b + BL_TB, 8192, bar_ld);
            if (!p.zero_v) tma_load_3d(sm + OFF_V, tmv, bar_ld, j0, h, t_begin + n * C);
            bulk_g2s(sm + OFF_WQ, b + BL_WQ, 32768, bar_ld);
        }
        if (groups & 4) {
            bulk_g2s(sm + OFF_RAP, b + BL_RAP, 16384, bar_ld3);
            bulk_g2s(sm + OFF_PM, b + BL_PM, 8192, bar_ld3);
            ld3_chunk = n;
        }
    };
    auto issue_ready = [&](int n, int groups) {  // thread 0
        groups &= pend;
        if (!groups) return;
        if ((groups & 3) && !armed) {
            mbar_arrive_expect_tx(bar_ld, p.zero_v ? TX_A - 8192 : TX_A);
            armed = true;
        }
        if ((groups & 4) && !armed3) {
            mbar_arrive_expect_tx(bar_ld3, TX_B);
            armed3 = true;
        }
        issue(n, groups);
        pend &= ~groups;
    };
    // gate(): issue `groups` of chunk n if the watcher has seen its blob ready
    auto gate = [&](int n, int groups) {  // thread 0: non-blocking
        if (kOverlap && !rdy) {
            if (smem_acquire(s_rdy) <= n) return;
            rdy = true;
            fence_proxy_async_global();
        }
        issue_ready(n, groups);
    };
    auto gate_wait = [&](int n) -> bool {  // thread 0: bounded wait, then all groups
        if (kOverlap && !rdy) {
            const uint64_t t0 = global_timer_ns();
            while (true) {
                const int r = smem_acquire(s_rdy);
                if (r > n) break;
                if (r < 0 || global_timer_ns() - t0 > kWaitNs) return false;
                __nanosleep(32);
            }
            rdy = true;
            fence_proxy_async_global();
        }
        issue_ready(n, 7);
        return true;
    };

    if (tid == 0 && t_begin < t_end) {
        pend = 7;
        gate(0, 7);
    }
    // ---- initial state (this half): fp32 into TMEM (row c = lane), bf16 into Sb
    {
        const int c = trow;
        const float* src =
            p.h0 ? p.h0 + (((size_t)seq * p.H + h) * D + c) * D + j0 + cq * 32 : nullptr;
        uint32_t r[32];
        float x[32];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            float4 v = src ? *reinterpret_cast<const float4*>(src + i)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
        }
        if (p.identity_h0) {  // row c of the identity, this half's columns
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] = (c == j0 + cq * 32 + i) ? 1.f : 0.f;
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(x[i]);
        tmem_st32(tbase + tlane + TM_S + cq * 32, r);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            float y[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = x[q4 * 8 + i];
            *reinterpret_cast<uint4*>(sm + OFF_SB + sw128_off(c, cq * 4 + q4)) = pack8(y);
        }
        tmem_wait_st();
    }
    for (int i = tid; i < 8192 / 16; i += NTC)
        reinterpret_cast<uint4*>(sm + OFF_ZERO)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (kLayer) {  // this half's filters and norm weights; no rows before the sequence
        for (int i = tid; i < DVS; i += NTC) {
            reinterpret_cast<float4*>(sm + OFF_WV)[i] =
                reinterpret_cast<const float4*>(p.wv)[(size_t)h * D + j0 + i];
            reinterpret_cast<float*>(sm + OFF_WN)[i] = p.w_norm[j0 + i];
        }
        for (int i = tid; i < 24; i += NTC)
            reinterpret_cast<uint4*>(sm + OFF_VH)[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_async_smem();
    tc_fence_before();
    group_sync(bar, NTC);
    tc_fence_after();

    // O rows of chunk m (rows 64-127 of its X buffer; warps of lane quarters 2,
    // 3); false if (layer variant) the wait for the partner's row sums gave up
    uint64_t* nbar = reinterpret_cast<uint64_t*>(sm + OFF_NBAR);
    auto o_out = [&](int m, int tt0, int LL) -> bool {
        const int r = trow - C;
        uint32_t v[32];
        tmem_ld32(tbase + tlane + tx(m) + cq * 32, v);
        tmem_wait_ld();
        if (!kLayer) {
            if (p.o && r < LL) {
                __nv_bfloat16* dst = p.o + ((size_t)(tt0 + r) * p.H + h) * D + j0 + cq * 32;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float y[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) y[i] = __uint_as_float(v[q4 * 8 + i]);
                    *reinterpret_cast<uint4*>(dst + q4 * 8) = pack8(y);
                }
            }
            return true;
        }
        // y = o / sqrt(mean o^2 + eps) * w_norm * sigmoid(gate): the row sum of
        // o^2 is this thread's 32 columns + the other column piece's (shared
        // memory) + the partner half's 64 (written into this unit's buffer by
        // the partner unit, with an arrival on nbar[m & 1] per row)
        const size_t grow = ((size_t)(tt0 + min(r, LL - 1)) * p.H + h) * D + j0 + cq * 32;
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) ss += __uint_as_float(v[i]) * __uint_as_float(v[i]);
        float* ssl = reinterpret_cast<float*>(sm + OFF_SSL);
        float* ssx = reinterpret_cast<float*>(sm + OFF_SSX) + (m & 1) * C;
        ssl[cq * C + r] = ss;
        group_sync(bar + 2, 128);  // the four read-out warps of this unit
        if (cq == 0) {  // into the partner unit's buffer, then arrive on its barrier
            float* pssx = reinterpret_cast<float*>(sm_partner + OFF_SSX) + (m & 1) * C;
            pssx[r] = ssl[r] + ssl[C + r];
            mbar_arrive(reinterpret_cast<uint64_t*>(sm_partner + OFF_NBAR) + (m & 1));
        }
        if (!mbar_wait(nbar + (m & 1), (m >> 1) & 1, kWaitNs)) return false;
        // the chunk's gate tile, brought into the (then idle) U buffer by TMA
        if (!mbar_wait(bar_gt, m & 1, kWaitNs)) return false;
        const float inv = rsqrtf((ssl[r] + ssl[C + r] + ssx[r]) / D + p.rms_eps);
        if (r < LL) {
            const float* wn = reinterpret_cast<const float*>(sm + OFF_WN) + cq * 32;
            __nv_bfloat16* dst = p.y + grow;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                float gt[8], y[8];
                unpack8(*reinterpret_cast<const uint4*>(sm + OFF_UB + sw128_off(r, cq * 4 + q4)),
                        gt);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    y[i] = __uint_as_float(v[q4 * 8 + i]) * inv * wn[q4 * 8 + i] *
                           fast_sigmoid(gt[i]);
                *reinterpret_cast<uint4*>(dst + 8 * q4) = pack8(y);
            }
        }
        return true;
    };
    int prev_t0 = 0, prev_L = 0;
    int n = 0;
    for (int t0 = t_begin; t0 < t_end && !failed; t0 += C, ++n) {
        const int L = min(C, t_end - t0);
        const int tn = t0 + C;
        const bool has_next = tn < t_end;
        const float* ssc = reinterpret_cast<const float*>(sm + ((n & 1) ? OFF_SC1 : OFF_SC0));
        bool ok = true;
        if (tid == 0 && pend) ok = gate_wait(n);
        ok = ok && mbar_wait(bar_ld, n & 1, kWaitNs);
        if (group_sync_or(bar, NTC, !ok)) {
            failed = true;
            break;
        }
        if (has_next && tid == 0) {  // the other row-scale buffer is free
            pend = 7;
            coming = n + 1;
            armed = armed3 = rdy = false;
            gate(n + 1, 1);
        }
        // ---- [Ut ; 0] = [Tb ; 0] V, then += [-W ; Q*Gam] S  (one accumulator, N=64)
        constexpr uint32_t id1 = idesc_bf16_f32(128, DVS, false, true);
        if ((!kLayer || n > 0) && tid == 0) {  // (layer: V already convolved, below)
            if (!p.zero_v) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tbase + tx(n), sdesc_sw128(sbase + OFF_TB + ks * 32, 16, 1024),
                             sdesc_sw128(sbase + OFF_V + ks * 2048, 8192, 1024), id1, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int kb = ks >> 2, kk = ks & 3;
                mma_bf16(tbase + tx(n), sdesc_sw128(sbase + OFF_WQ + kb * 16384 + kk * 32, 16, 1024),
                         sdesc_sw128(sbase + OFF_SB + ks * 2048, 16384, 1024), id1,
                         (p.zero_v && ks == 0) ? 0u : 1u);
            }
            mma_commit(bar_mma);
        }
        if (kLayer && n == 0) {
            // the S part first; V is convolved in place meanwhile, then its part
            // (later chunks' V is convolved during the previous chunk)
            if (tid == 0) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const int kb = ks >> 2, kk = ks & 3;
                    mma_bf16(tbase + tx(n),
                             sdesc_sw128(sbase + OFF_WQ + kb * 16384 + kk * 32, 16, 1024),
                             sdesc_sw128(sbase + OFF_SB + ks * 2048, 16384, 1024), id1, ks > 0);
                }
            }
            conv_v_tile(sm, tid, bar, NTC);
            fence_async_smem();
            group_sync(bar, NTC);
            if (tid == 0) {
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tbase + tx(n), sdesc_sw128(sbase + OFF_TB + ks * 32, 16, 1024),
                             sdesc_sw128(sbase + OFF_V + ks * 2048, 8192, 1024), id1, 1);
                mma_commit(bar_mma);
            }
        }
        // the previous chunk's O rows, read out while these products run
        bool ook = true;
        if (n > 0 && quarter >= 2) ook = o_out(n - 1, prev_t0, prev_L);
        ok = mbar_wait(bar_mma, mma_phase & 1, kWaitNs);
        ok = ok && ook;
        ++mma_phase;
        if (group_sync_or(bar, NTC, !ok)) {
            failed = true;
            break;
        }
        tc_fence_after();
        if (has_next && tid == 0) gate(n + 1, 3);  // V, Tb, [-W ; Q*Gam] regions free
        // U (rows 0-63 of the accumulator) -> bf16 Ub
        if (quarter < 2) {
            const int r = trow;
            uint32_t a[32];
            tmem_ld32(tbase + tlane + tx(n) + cq * 32, a);
            tmem_wait_ld();
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                float y[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) y[i] = __uint_as_float(a[q4 * 8 + i]);
                *reinterpret_cast<uint4*>(sm + OFF_UB + sw128_off(r, cq * 4 + q4)) = pack8(y);
            }
        }
        fence_async_smem();
        tc_fence_before();
        group_sync(bar, NTC);
        tc_fence_after();
        // ---- O = X[64:] + [. ; P] U  (accumulate);  (K E^-1)^T U -> TM_W   (N=64)
        bool ok3 = true;
        if (tid == 0) {  // K E^-1, P of this chunk
            ok3 = mbar_wait(bar_ld3, n & 1, kWaitNs);
            if (ok3) ld3_chunk = -1;
        }
        if (tid == 0 && ok3) {
            constexpr uint32_t idP = idesc_bf16_f32(128, DVS, false, true);
            constexpr uint32_t idK = idesc_bf16_f32(128, DVS, true, true);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tbase + tx(n), sdesc_sw128(sbase + OFF_PM - 8192 + ks * 32, 16, 1024),
                         sdesc_sw128(sbase + OFF_UB + ks * 2048, 8192, 1024), idP, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tbase + TM_W, sdesc_sw128(sbase + OFF_RAP + ks * 2048, 8192, 1024),
                         sdesc_sw128(sbase + OFF_UB + ks * 2048, 8192, 1024), idK, ks > 0);
            mma_commit(bar_mma);
        }
        if (kLayer && has_next) {
            // while these products run: the next chunk's V (loaded since the
            // first products completed) convolved in place
            const bool okv = mbar_wait(bar_ld, (n + 1) & 1, kWaitNs);
            if (group_sync_or(bar, NTC, !okv)) {
                ++mma_phase;  // the drain below then waits for these products too
                failed = true;
                break;
            }
            conv_v_tile(sm, tid, bar, NTC);
            fence_async_smem();
        }
        ok = ok3 && mbar_wait(bar_mma, mma_phase & 1, kWaitNs);
        ++mma_phase;
        if (group_sync_or(bar, NTC, !ok)) {
            failed = true;
            break;
        }
        tc_fence_after();
        if (has_next && tid == 0) gate(n + 1, 7);  // K E^-1 and P regions free
        if (kLayer && tid == 0) {  // U is consumed: this chunk's gate tile into its buffer
            fence_async_smem();
            mbar_arrive_expect_tx(bar_gt, 8192);
            tma_load_3d(sm + OFF_UB, tmgate, bar_gt, j0, h, t0);
            ++gt_issued;
        }
        // S <- Gam_last * S + ksc * (K E^-1)^T U   (lane = state row c)
        {
            const int c = trow;
            const float gc = ssc[c], ks = ssc[D + c];
            uint32_t a[32], sv[32];
            tmem_ld32(tbase + tlane + TM_W + cq * 32, a);
            tmem_ld32(tbase + tlane + TM_S + cq * 32, sv);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i)
                sv[i] = __float_as_uint(fmaf(gc, __uint_as_float(sv[i]), ks * __uint_as_float(a[i])));
            tmem_st32(tbase + tlane + TM_S + cq * 32, sv);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                float y[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) y[i] = __uint_as_float(sv[q4 * 8 + i]);
                *reinterpret_cast<uint4*>(sm + OFF_SB + sw128_off(c, cq * 4 + q4)) = pack8(y);
            }
            tmem_wait_st();
        }
        fence_async_smem();
        tc_fence_before();
        group_sync(bar, NTC);
        tc_fence_after();
        prev_t0 = t0;
        prev_L = L;
    }
    bool last_ok = true;
    if (!failed && n > 0 && quarter >= 2) last_ok = o_out(n - 1, prev_t0, prev_L);
    if (group_sync_or(bar, NTC, !last_ok)) failed = true;

    if (!failed && p.hN) {
        const int c = trow;
        float* dst = p.hN + (((size_t)seq * p.H + h) * D + c) * D + j0 + cq * 32;
        uint32_t s[32];
        tmem_ld32(tbase + tlane + TM_S + cq * 32, s);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + i) =
                make_float4(__uint_as_float(s[i]), __uint_as_float(s[i + 1]),
                            __uint_as_float(s[i + 2]), __uint_as_float(s[i + 3]));
    }
    if (failed && tid == 0) {
        // wait (bounded) for products and copies still in flight
        if (mma_phase > 0) mbar_wait(bar_mma, (mma_phase - 1) & 1, kWaitNs);
        if (armed) mbar_wait(bar_ld, coming & 1, kWaitNs);  // at once if complete
        if (ld3_chunk >= 0) mbar_wait(bar_ld3, ld3_chunk & 1, kWaitNs);
        if (kLayer && gt_issued > 0) mbar_wait(bar_gt, (gt_issued - 1) & 1, kWaitNs);
        atomicOr(p.status_out, STATUS_TIMEOUT);
    }
    tc_fence_before();
    group_sync(bar, NTC);
}

// The watcher of a co-scheduled chain CTA (one thread of its other unit):
// follows the blob flags of the chain's chunks in order (acquire, bounded
// waits) and publishes how many are ready in the chain unit's shared memory,
// so that the chain's issuing thread never waits on a global read.
__device__ __forceinline__ void watch(const Params& p, uint8_t* sm_chain, int chain_id) {
    const int seq = chain_id / p.H, h = chain_id % p.H;
    const int cbase = p.chunk_start[seq], nch = p.chunk_start[seq + 1] - cbase;
    int* s_rdy = reinterpret_cast<int*>(sm_chain + OFF_RDY);
    const uint32_t* f = p.flags + (size_t)cbase * p.H + h;
    for (int n = 0; n < nch; ++n) {
        const uint64_t t0 = global_timer_ns();
        while (flag_acquire(f + (size_t)n * p.H) == 0u) {
            if (status_bad(p.status) || global_timer_ns() - t0 > p.flag_wait_ns) {
                smem_release(s_rdy, -1);
                return;
            }
            __nanosleep(64);
        }
        smem_release(s_rdy, n + 1);
    }
}

__global__ void __launch_bounds__(NTC, 2)
    chunk_chain_kernel(const __grid_constant__ CUtensorMap tmv, const Params p) {
    if (status_bad(p.status)) return;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t s_tmem;
    if (threadIdx.x < 32) {
        tmem_alloc(&s_tmem, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // CTA pairs take the (sequence, head) chains longest sequence first
    const int r = static_cast<int>(blockIdx.x >> 1);
    const int chain_id = p.order ? p.order[r / p.H] * p.H + r % p.H : r;
    run<false>(&tmv, p, align1024(smem_raw), s_tmem, 1, chain_id, blockIdx.x & 1);
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) tmem_dealloc(s_tmem, 256);
}

// The layer variant: one CTA of two 256-thread units per (sequence, head),
// unit u running the chain on value half u with named barriers 1 + u (and
// 3 + u for its read-out warps), its own shared-memory region and 256 TMEM
// columns.  The units add their row sums of o^2 through each other's shared
// memory (the partner's buffer, then an arrival on the partner's mbarrier;
// every wait bounded), so the RMSNorm over all 128 columns needs no cluster:
// a cluster launch of kernels that allocate tensor memory is placed one CTA
// per SM.
constexpr uint32_t LAYER_UNIT = (OFF_NBAR + 16 + 1023) / 1024 * 1024;
constexpr uint32_t LAYER_SMEM = 2 * LAYER_UNIT + 1024;
static_assert(LAYER_SMEM + 1024 <= 232448, "one 512-thread CTA per SM");
__global__ void __launch_bounds__(2 * NTC, 1)
    chunk_chain_layer_kernel(const __grid_constant__ CUtensorMap tmv,
                             const __grid_constant__ CUtensorMap tmgate, const Params p) {
    if (status_bad(p.status)) return;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t s_tmem;
    uint8_t* base = align1024(smem_raw);
    const int unit = static_cast<int>(threadIdx.x) >> 8;
    if (threadIdx.x < 32) {
        tmem_alloc(&s_tmem, 512);
        tmem_relinquish();
    }
    if (threadIdx.x < 2) {  // the row-sum barriers of unit threadIdx.x
        uint64_t* nbar = reinterpret_cast<uint64_t*>(base + threadIdx.x * LAYER_UNIT + OFF_NBAR);
        mbar_init(nbar, C);
        mbar_init(nbar + 1, C);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int r = static_cast<int>(blockIdx.x);
    const int chain_id = p.order ? p.order[r / p.H] * p.H + r % p.H : r;
    run<false, true>(&tmv, p, base + unit * LAYER_UNIT, s_tmem + 256u * unit, 1 + unit, chain_id,
                     unit, &tmgate, base + (1 - unit) * LAYER_UNIT);
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) tmem_dealloc(s_tmem, 512);
}
}  // namespace chain

// =================================================================== overlap
// Both kernels in one cooperative launch of one 512-thread CTA per SM; each
// CTA is two independent 256-thread units (named barriers 1 and 2, 256 TMEM
// columns and one shared-memory region each).  The first 2 N H CTAs run one
// chain unit each (one value-column half of one (sequence, head)) with the
// SM to itself -- a chain step is a short dependent sequence of products and
// epilogues that slows down by more than half when another unit shares its
// SM; one thread of the idle unit watches the chain's blob flags -- and the
// others run two intra-chunk units each, round by round.  A
// chain waits only for the blobs of its own chunks and an intra unit never
// waits for a chain; every CTA is resident (cooperative launch), so every
// wait ends (each is also bounded).
constexpr int NTO = 512;
static_assert(intra::NTI == 256 && chain::NTC == 256, "two 256-thread units per CTA");
constexpr uint32_t unit_bytes() {
    const uint32_t a = intra::OFF_BAR + 64, b = chain::OFF_BAR + 64;
    return ((a > b ? a : b) + 1023) / 1024 * 1024;
}
constexpr uint32_t UNIT_BYTES = unit_bytes();
constexpr uint32_t OVERLAP_SMEM = 2 * UNIT_BYTES + 1024;
static_assert(OVERLAP_SMEM + 1024 <= 232448, "one CTA per SM");

template <bool kScalar>
__global__ void __launch_bounds__(NTO, 1)
    chunk_overlap_kernel(const __grid_constant__ CUtensorMap tmq,
                         const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmg,
                         const __grid_constant__ CUtensorMap tmv, const intra::Params pi,
                         const chain::Params pc, int nchain) {
    if (status_bad(pi.status)) return;
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t s_tmem;
    const int b = static_cast<int>(blockIdx.x);
    if (threadIdx.x < 32) {
        tmem_alloc(&s_tmem, 512);
        tmem_relinquish();
    }
    if (b < nchain && threadIdx.x == 0)
        *reinterpret_cast<int*>(align1024(smem_raw) + chain::OFF_RDY) = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int unit = static_cast<int>(threadIdx.x) >> 8;
    uint8_t* sm = align1024(smem_raw) + unit * UNIT_BYTES;
    const uint32_t tb = s_tmem + 256u * unit;
    if (b < nchain) {
        if (unit == 0)
            chain::run<true, false>(&tmv, pc, sm, tb, 1, b >> 1, b & 1);
        else if (threadIdx.x == 256)
            chain::watch(pc, align1024(smem_raw), b >> 1);
    } else
        intra::run<true, kScalar>(&tmq, &tmk, &tmg, pi, sm, tb, 1 + unit,
                                  2 * (b - nchain) + unit,
                                  2 * (static_cast<int>(gridDim.x) - nchain));
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) tmem_dealloc(s_tmem, 512);
}

PFN_cuTensorMapEncodeTiled_v12000 split_encode_fn() {
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

bool split_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int total,
               int H, int box0, CUtensorMapSwizzle sw) {
    auto fn = split_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)total};
    cuuint64_t strides[2] = {(cuuint64_t)D * esize, (cuuint64_t)D * esize * H};
    cuuint32_t box[3] = {(cuuint32_t)box0, 1, (cuuint32_t)C};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_path_available() { return split_encode_fn() != nullptr; }

namespace {
// Dynamic shared memory of `smem` bytes and the largest shared-memory carveout
// (two of these CTAs, about 100 KB each, share an SM).
template <typename F>
cudaError_t set_smem_max_carveout(F* fn, uint32_t smem) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
    return e;
}
}  // namespace

cudaError_t launch_split_intra(const void* q, const void* k, const float* g, const float* beta,
                               int total, int H, const int4* chunk_info, int maxc,
                               uint32_t* status, void* blobs, cudaStream_t st, const float* gh,
                               const LayerArgs* layer) {
    if (total == 0 || maxc == 0) return cudaSuccess;
    if (layer && gh) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mg;
    if (!split_map(&mq, layer ? layer->xq : q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, total, H, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
        !split_map(&mk, layer ? layer->xk : k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, total, H, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (gh) {
        mg = mq;  // not read: the head-uniform gate comes by plain loads
    } else if (!split_map(&mg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, total, H, 128,
                          CU_TENSOR_MAP_SWIZZLE_NONE)) {
        return cudaErrorInvalidValue;
    }
    cudaError_t e = set_smem_max_carveout(intra::chunk_intra_kernel<false, false>,
                                          intra::SMEM_BYTES);
    if (e == cudaSuccess)
        e = set_smem_max_carveout(intra::chunk_intra_kernel<true, false>, intra::SMEM_BYTES);
    if (e == cudaSuccess)
        e = set_smem_max_carveout(intra::chunk_intra_kernel<false, true>, intra::SMEM_BYTES_CONV);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long items = (long long)maxc * H;
    const int grid = (int)(items < 2 * sms ? items : 2 * sms);
    intra::Params pa{beta, chunk_info, maxc, H, status, status, static_cast<uint8_t*>(blobs)};
    pa.gh = gh;
    pa.withheld = -1;
    if (layer) {
        pa.xq = static_cast<const __nv_bfloat16*>(layer->xq);
        pa.xk = static_cast<const __nv_bfloat16*>(layer->xk);
        pa.wq = layer->wq;
        pa.wk = layer->wk;
        pa.l2_eps = layer->l2_eps;
        intra::chunk_intra_kernel<false, true>
            <<<grid, intra::NTI, intra::SMEM_BYTES_CONV, st>>>(mq, mk, mg, pa);
    } else if (gh) {
        intra::chunk_intra_kernel<true, false><<<grid, intra::NTI, intra::SMEM_BYTES, st>>>(
            mq, mk, mg, pa);
    } else {
        intra::chunk_intra_kernel<false, false><<<grid, intra::NTI, intra::SMEM_BYTES, st>>>(
            mq, mk, mg, pa);
    }
    return cudaGetLastError();
}

cudaError_t launch_split_chain(const void* v, const float* h0, const int32_t* cu_seqlens, int T,
                               int N, int H, const int* chunk_start, uint32_t* status,
                               const void* blobs, void* o, float* hN, cudaStream_t st,
                               const int* seq_order, const LayerArgs* layer) {
    const int total = cu_seqlens ? T : N * T;
    if (total == 0) {
        if (hN) {
            if (h0) return cudaMemcpyAsync(hN, h0, sizeof(float) * (size_t)N * H * D * D,
                                           cudaMemcpyDeviceToDevice, st);
            return cudaMemsetAsync(hN, 0, sizeof(float) * (size_t)N * H * D * D, st);
        }
        return cudaSuccess;
    }
    CUtensorMap mv;
    if (!split_map(&mv, layer ? layer->xv : v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, total, H, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    chain::Params pb{h0, cu_seqlens, T, H, chunk_start, status, status,
                     static_cast<const uint8_t*>(blobs), (__nv_bfloat16*)o, hN};
    pb.order = seq_order;
    if (!layer) {
        cudaError_t e = set_smem_max_carveout(chain::chunk_chain_kernel, chain::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        chain::chunk_chain_kernel<<<2 * N * H, chain::NTC, chain::SMEM_BYTES, st>>>(mv, pb);
        return cudaGetLastError();
    }
    cudaError_t e = set_smem_max_carveout(chain::chunk_chain_layer_kernel, chain::LAYER_SMEM);
    if (e != cudaSuccess) return e;
    pb.wv = layer->wv;
    pb.gate = static_cast<const __nv_bfloat16*>(layer->gate);
    pb.w_norm = layer->w_norm;
    pb.rms_eps = layer->rms_eps;
    pb.y = static_cast<__nv_bfloat16*>(layer->y);
    CUtensorMap mgt;
    if (!split_map(&mgt, layer->gate, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, total, H, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    chain::chunk_chain_layer_kernel<<<N * H, 2 * chain::NTC, chain::LAYER_SMEM, st>>>(mv, mgt,
                                                                                      pb);
    return cudaGetLastError();
}

namespace {
// dst[n, h] = I (dk = dv = 128): the state map of sequences without tokens.
__global__ void identity_fill_kernel(float* dst, long long mats) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= mats * D * D) return;
    const int e = static_cast<int>(i % (D * D));
    dst[i] = (e / D == e % D) ? 1.f : 0.f;
}
}  // namespace

cudaError_t launch_split_state_maps(const void* q, const void* k, const void* v, const float* g,
                                    const float* beta, const int32_t* cu_seqlens, int T, int N,
                                    int H, const int4* chunk_info, int maxc,
                                    const int* chunk_start, uint32_t* status, void* blobs,
                                    float* M, float* Bm, cudaStream_t st, const int* seq_order) {
    const int total = cu_seqlens ? T : N * T;
    if (total == 0) {
        const long long mats = (long long)N * H;
        cudaError_t e = cudaMemsetAsync(Bm, 0, sizeof(float) * (size_t)mats * D * D, st);
        if (e != cudaSuccess) return e;
        identity_fill_kernel<<<(unsigned)((mats * D * D + 255) / 256), 256, 0, st>>>(M, mats);
        return cudaGetLastError();
    }
    cudaError_t e = launch_split_intra(q, k, g, beta, total, H, chunk_info, maxc, status, blobs,
                                       st);
    if (e != cudaSuccess) return e;
    CUtensorMap mv;
    if (!split_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, total, H, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if ((e = set_smem_max_carveout(chain::chunk_chain_kernel, chain::SMEM_BYTES)) != cudaSuccess)
        return e;
    // B: from a zero state with the values; M: from the identity with zero values
    chain::Params pb{nullptr, cu_seqlens, T, H, chunk_start, status, status,
                     static_cast<const uint8_t*>(blobs), nullptr, Bm};
    pb.order = seq_order;
    chain::chunk_chain_kernel<<<2 * N * H, chain::NTC, chain::SMEM_BYTES, st>>>(mv, pb);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    chain::Params pm = pb;
    pm.hN = M;
    pm.zero_v = true;
    pm.identity_h0 = true;
    chain::chunk_chain_kernel<<<2 * N * H, chain::NTC, chain::SMEM_BYTES, st>>>(mv, pm);
    return cudaGetLastError();
}

// Grid of the co-scheduled launch (one CTA per SM), or 0 when it does not
// apply: the device must support cooperative launches and keep one such CTA
// per SM resident, and at least one SM must be left for the intra-chunk work
// after one SM per chain unit.
int overlap_grid(int N, int H) {
    int dev = 0, sms = 0, nb = 0, coop = 0;
    int nb_scalar = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess ||
        set_smem_max_carveout(chunk_overlap_kernel<false>, OVERLAP_SMEM) != cudaSuccess ||
        set_smem_max_carveout(chunk_overlap_kernel<true>, OVERLAP_SMEM) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, chunk_overlap_kernel<false>, NTO,
                                                      OVERLAP_SMEM) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb_scalar, chunk_overlap_kernel<true>,
                                                      NTO, OVERLAP_SMEM) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    if (!coop || nb < 1 || nb_scalar < 1 || sms <= 0) return 0;
    if (2LL * N * H >= sms) return 0;
    return sms;
}

cudaError_t launch_chunk_fwd_overlap(const void* q, const void* k, const void* v, const float* g,
                                     const float* beta, const float* h0,
                                     const int32_t* cu_seqlens, int T, int N, int H,
                                     const int4* chunk_info, int maxc, const int* chunk_start,
                                     uint32_t* status, void* blobs, uint32_t* flags, void* o,
                                     float* hN, cudaStream_t st, long long withheld_flag,
                                     unsigned long long flag_wait_ns, const float* gh) {
    const int total = cu_seqlens ? T : N * T;
    if (total == 0)
        return launch_split_chain(v, h0, cu_seqlens, T, N, H, chunk_start, status, blobs, o, hN,
                                  st);
    const int grid = overlap_grid(N, H);
    if (grid == 0) return cudaErrorInvalidConfiguration;
    CUtensorMap mq, mk, mg, mv;
    if (!split_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, total, H, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
        !split_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, total, H, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
        !split_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, total, H, 64,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (gh) {
        mg = mq;  // not read: the head-uniform gate comes by plain loads
    } else if (!split_map(&mg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, total, H, 128,
                          CU_TENSOR_MAP_SWIZZLE_NONE)) {
        return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaMemsetAsync(flags, 0, sizeof(uint32_t) * (size_t)maxc * H, st);
    if (e != cudaSuccess) return e;
    uint8_t* bl = static_cast<uint8_t*>(blobs);
    intra::Params pi{beta, chunk_info, maxc, H, status, status, bl,
                     N, chunk_start, status + 1, flags};
    pi.withheld = withheld_flag;
    pi.gh = gh;
    chain::Params pc{h0, cu_seqlens, T, H, chunk_start, status, status, bl,
                     (__nv_bfloat16*)o, hN, flags};
    pc.flag_wait_ns = flag_wait_ns ? flag_wait_ns : kWaitNs;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NTO);
    cfg.dynamicSmemBytes = OVERLAP_SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (gh)
        return cudaLaunchKernelEx(&cfg, chunk_overlap_kernel<true>, mq, mk, mg, mv, pi, pc,
                                  2 * N * H);
    return cudaLaunchKernelEx(&cfg, chunk_overlap_kernel<false>, mq, mk, mg, mv, pi, pc,
                              2 * N * H);
}

cudaError_t launch_chunk_fwd_split(const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, const float* h0,
                                   const int32_t* cu_seqlens, int T, int N, int H,
                                   const int4* chunk_info, int maxc, const int* chunk_start,
                                   uint32_t* status, void* blobs, void* o, float* hN,
                                   cudaStream_t st, const float* gh, const int* seq_order,
                                   const LayerArgs* layer) {
    const int total = cu_seqlens ? T : N * T;
    cudaError_t e = launch_split_intra(q, k, g, beta, total, H, chunk_info, maxc, status, blobs,
                                       st, gh, layer);
    if (e != cudaSuccess) return e;
    return launch_split_chain(v, h0, cu_seqlens, T, N, H, chunk_start, status, blobs, o, hN, st,
                              seq_order, layer);
}

}  // namespace kda
