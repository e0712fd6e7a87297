/*
 * kda.h -- C ABI of libkda.so: Kimi Delta Attention (KDA) on one NVIDIA B200.
 *
 * KDA (Kimi Linear, aiwiki.ai, section "Kimi Delta Attention") is the gated
 * delta rule with the scalar forget gate replaced by a diagonal, per-channel
 * gate.  Per (sequence, head) it carries a state S of dk x dv floats and, for
 * each token t,
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t,            alpha_t = exp(g_t) per key channel.
 *
 * In the diagonal-plus-low-rank reading (section "The constrained DPLR form
 * and the chunkwise algorithm") the transition is Diag(alpha) - a b^T with
 * a = beta k and b = alpha * k.  Prefill evaluates this chunk by chunk (WY
 * representation + UT transform inside a chunk, a carried state between
 * chunks); decode applies one token to a resident state.
 *
 * ---------------------------------------------------------------- conventions
 * Pointers:   every tensor pointer is a DEVICE pointer unless stated, must be
 *             16-byte aligned, and is owned by the caller.  The library never
 *             allocates, frees or keeps memory, never synchronises a stream
 *             (except kda_get_device_status) and keeps no global state.
 * Streams:    `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *             stream).  All work is enqueued asynchronously on it.
 * Layouts:    row-major (C order), token-major:
 *               q, k, g     [total_tokens, H, dk]
 *               v, o        [total_tokens, H, dv]
 *               beta        [total_tokens, H]
 *               states      [num_seqs, H, dk, dv]  -- S[c][j] is key channel c,
 *                           value channel j (dv contiguous); this one layout is
 *                           used by prefill, decode and every state argument.
 * Sequences:  cu_seqlens == NULL: B sequences of T tokens each, total = B*T,
 *             num_seqs must equal B.  cu_seqlens != NULL: int32 device array
 *             [num_seqs + 1] of packed-sequence offsets (cu[0] = 0,
 *             non-decreasing, cu[num_seqs] = T); B must be 1 and T is the
 *             total token count.  Chunks start at each sequence's first token
 *             and never straddle sequences; a sequence's last chunk may be
 *             short.  A zero-length sequence passes its initial state through.
 * Gates:      g = log(alpha) in fp32, any finite value; beta in fp32.
 * dtype:      the type of q, k, v and o (KDA_DTYPE_F32 or KDA_DTYPE_BF16).
 *             g, beta and every state are always fp32; arithmetic is fp32.
 * Errors:     a return other than KDA_OK means nothing was enqueued.  Checks
 *             that need device data (cu_seqlens contents) run on the device
 *             and are reported by kda_get_device_status().
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,  /* NULL / misaligned pointer, bad size or shape combination */
    KDA_ERR_UNSUPPORTED = 2,  /* valid arguments, but no kernel for this shape / dtype */
    KDA_ERR_CUDA = 3,         /* a CUDA runtime call failed (launch error, ...) */
    KDA_ERR_TIMEOUT = 4,      /* device side: a bounded wait gave up (set in the status word) */
    KDA_ERR_WORKSPACE = 5,    /* workspace NULL or smaller than *_workspace_size() */
    KDA_ERR_BAD_SEQLENS = 6   /* device side: cu_seqlens not 0 .. T non-decreasing */
} kda_status_t;

typedef enum { KDA_DTYPE_F32 = 0, KDA_DTYPE_BF16 = 1 } kda_dtype_t;

/* Human-readable name of a status code (static storage; never NULL). */
const char* kda_status_string(kda_status_t status);

/* ------------------------------------------------------------------ prefill
 * kda_chunk_fwd: chunkwise KDA forward over B x T tokens or packed sequences.
 *   Defining passage: Kimi Linear (aiwiki.ai), "The constrained DPLR form and
 *   the chunkwise algorithm" (chunks of C tokens, WY representation, UT
 *   transform, recurrent between chunks, parallel inside a chunk).
 * In:  q, k [total, H, dk], v [total, H, dv] (dtype); g [total, H, dk] fp32;
 *      beta [total, H] fp32; initial_state [num_seqs, H, dk, dv] fp32 or NULL
 *      (zeros); cu_seqlens as above or NULL.
 * Out: o [total, H, dv] (dtype), every token written; final_state
 *      [num_seqs, H, dk, dv] fp32 or NULL (not written).  initial_state and
 *      final_state may be the same buffer.
 * Workspace: device scratch of at least kda_chunk_fwd_workspace_size() bytes,
 *      256-byte aligned, owned by the caller, reusable across calls on the same
 *      stream; it also holds the device status word.
 * Shapes: dk, dv in {32, 64, 128}; chunk in {16, 32, 64}; anything else is
 *      KDA_ERR_UNSUPPORTED.  Which kernels run is the call's plan (see
 *      kda_chunk_fwd_plan below): bf16 with dk = dv = 128 and chunk = 64 runs
 *      on the tensor cores (tcgen05 / TMEM / TMA) as the split plan, other
 *      supported shapes on the CUDA-core kernels (the four step calls below,
 *      in order).  kda_chunk_fwd_workspace_size() follows the plan.
 */
size_t kda_chunk_fwd_workspace_size(int total_tokens, int num_seqs, int H, int dk, int dv,
                                    int chunk, kda_dtype_t dtype);

/* Plans of kda_chunk_fwd (which kernels one call runs):
 *   KDA_PLAN_SIMT     the CUDA-core kernels: gate cumsum, intra, inter, output;
 *   KDA_PLAN_SPLIT    kda_chunk_split_intra then kda_chunk_split_chain (below):
 *                     the chunk-parallel part on every SM, then the chains;
 *   KDA_PLAN_OVERLAP  the same two kernels co-scheduled in one cooperative
 *                     launch, chains and intra-chunk work on disjoint SMs,
 *                     each chain starting on a chunk as soon as that chunk's
 *                     operands are ready.  Runs only where 2 * num_seqs * H is
 *                     below the number of SMs (one SM per chain half).
 * The default plan depends only on the arguments and the device: SIMT for
 * every shape other than bf16, dk = dv = 128, chunk = 64; for that shape
 * OVERLAP when the chain length is known on the host (no cu_seqlens, or a
 * single packed sequence), the launch applies, and a cost model says that the
 * chains, not the intra-chunk work, are the longer part (long sequences, few
 * heads); SPLIT otherwise.  kda_chunk_fwd_plan returns it (`packed` != 0: the
 * call passes cu_seqlens), or -1 for arguments kda_chunk_fwd_workspace_size()
 * rejects.  The split and overlap plans share one workspace layout.  (The
 * value 1 is not a plan.) */
enum {
    KDA_PLAN_SIMT = 0,
    KDA_PLAN_SPLIT = 2,
    KDA_PLAN_OVERLAP = 3
};
int kda_chunk_fwd_plan(int total_tokens, int num_seqs, int packed, int H, int dk, int dv,
                       int chunk, kda_dtype_t dtype);

kda_status_t kda_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, const float* initial_state,
                           const int32_t* cu_seqlens, int B, int T, int num_seqs, int H,
                           int dk, int dv, int chunk, kda_dtype_t dtype, void* o,
                           float* final_state, void* workspace, size_t workspace_bytes,
                           void* stream);

/* kda_chunk_fwd_with_plan: kda_chunk_fwd on an explicitly chosen plan (for
 * testing one plan against another, and for measuring each), with the same
 * arguments, results and error behaviour.  A plan that cannot run these
 * shapes on this device (a tensor-core plan for another shape or dtype, the
 * overlap plan where its launch does not apply) returns KDA_ERR_UNSUPPORTED;
 * an unknown plan KDA_ERR_INVALID_ARG.  Its workspace is
 * kda_chunk_fwd_plan_workspace_size(plan, ...) bytes, which is 0 exactly when
 * the plan does not apply (or the arguments are invalid). */
size_t kda_chunk_fwd_plan_workspace_size(int plan, int total_tokens, int num_seqs, int H, int dk,
                                         int dv, int chunk, kda_dtype_t dtype);

kda_status_t kda_chunk_fwd_with_plan(int plan, const void* q, const void* k, const void* v,
                                     const float* g, const float* beta,
                                     const float* initial_state, const int32_t* cu_seqlens, int B,
                                     int T, int num_seqs, int H, int dk, int dv, int chunk,
                                     kda_dtype_t dtype, void* o, float* final_state,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* --------------------------------------------- prefill, one step per call
 * The four steps of the chunkwise form as separate calls, with the
 * intermediates in caller-owned buffers.  kda_chunk_fwd computes the same
 * result; these exist so that each step can be checked and timed on its own.
 * Notation, per (sequence, head, chunk) with rows r, i of the chunk:
 *   G_r = sum_{j <= r in chunk} g_j (inclusive, per channel), Gam = exp(G);
 *   A[r,i] = beta_r sum_c k[r,c] k[i,c] exp(G[r,c] - G[i,c])   (i < r);
 *   Tm = (I + A)^{-1};  W = Tm diag(beta) (K * Gam);  Ut = Tm diag(beta) V;
 *   S_n = state at the start of chunk n;  U_n = Ut - W S_n;
 *   S_{n+1} = Diag(Gam_last) S_n + (K * exp(G_last - G))^T U_n;
 *   O_n = (Q * Gam) S_n + (P masked to i <= r) U_n,
 *         P[r,i] = sum_c q[r,c] k[i,c] exp(G[r,c] - G[i,c]).
 * (Derived from the recurrence above: one step is S_r = Diag(alpha_r)
 * S_{r-1} + k_r u_r^T with u_r = beta_r (v_r - (Diag(alpha_r) S_{r-1})^T k_r),
 * unrolled inside a chunk.)
 * All intermediates are fp32 and token-major where they have one row per
 * token.  Chunk states are numbered by global chunk index: sequences in
 * order, chunks in order within a sequence; there are
 * kda_num_chunks_upper_bound() slots, of which sum_s ceil(len_s / chunk) are
 * used.  Workspace: kda_chunk_fwd_workspace_size() bytes, as for
 * kda_chunk_fwd.  Any dtype / shape that kda_chunk_fwd accepts.
 */
int kda_num_chunks_upper_bound(int total_tokens, int num_seqs, int chunk);

/* a1: cumulative log-gate.  G [total, H, dk] fp32 = per-chunk inclusive
 * cumulative sum of g over tokens, per (head, channel): the logarithm of the
 * running decay product that section "The constrained DPLR form and the
 * chunkwise algorithm" identifies as the unstable divisor of general DPLR. */
kda_status_t kda_chunk_gate_cumsum(const float* g, const int32_t* cu_seqlens, int B, int T,
                                   int num_seqs, int H, int dk, int chunk, float* G,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* a2: intra-chunk WY / UT factors.  From k, v (dtype), G, beta: builds A,
 * solves the unit-lower-triangular system (UT transform) and writes
 * W [total, H, dk] fp32 and Ut [total, H, dv] fp32 (row r of a chunk at the
 * chunk's r-th token). */
kda_status_t kda_chunk_intra(const void* k, const void* v, const float* G, const float* beta,
                             const int32_t* cu_seqlens, int B, int T, int num_seqs, int H,
                             int dk, int dv, int chunk, kda_dtype_t dtype, float* W, float* Ut,
                             void* workspace, size_t workspace_bytes, void* stream);

/* a3: inter-chunk state propagation, serial over the chunks of each
 * sequence, state carried in fp32.  In: k (dtype), G, W, U (holding Ut on
 * entry; overwritten in place with U_n = Ut - W S_n), initial_state or NULL.
 * Out: chunk_states [num_chunks_upper_bound, H, dk, dv] fp32 (S_n per
 * chunk), final_state [num_seqs, H, dk, dv] or NULL. */
kda_status_t kda_chunk_inter(const void* k, const float* G, const float* W, float* U,
                             const float* initial_state, const int32_t* cu_seqlens, int B,
                             int T, int num_seqs, int H, int dk, int dv, int chunk,
                             kda_dtype_t dtype, float* chunk_states, float* final_state,
                             void* workspace, size_t workspace_bytes, void* stream);

/* a4: output.  O_n = (Q * Gam) S_n + (P masked) U_n for every chunk.
 * In: q, k (dtype), G, U (as left by kda_chunk_inter), chunk_states.
 * Out: o [total, H, dv] (dtype). */
kda_status_t kda_chunk_output(const void* q, const void* k, const float* G, const float* U,
                              const float* chunk_states, const int32_t* cu_seqlens, int B,
                              int T, int num_seqs, int H, int dk, int dv, int chunk,
                              kda_dtype_t dtype, void* o, void* workspace,
                              size_t workspace_bytes, void* stream);

/* --------------------------------- tensor-core split plan, one kernel per call
 * The two kernels of the split plan (see kda_chunk_fwd), callable one at a
 * time so that each can be checked and timed on its own.  q, k, v, o bf16;
 * dk = dv = 128; chunk = 64 (no other shape: the call returns
 * KDA_ERR_UNSUPPORTED when the tensor-core kernels are not in the library).
 *   kda_chunk_split_intra: chunk-parallel over (chunk, head).  Builds the
 *     chunk table, then per chunk computes G (a1), A, the UT-transform
 *     inverse and W (a2), and the chunk-local operands of a4 (Q * Gam, the
 *     masked P), and stores them, in bf16 tensor-core tile layout, in the
 *     workspace (an opaque format of this library version).
 *   kda_chunk_split_chain: two CTAs per (sequence, head), one per half of
 *     the value columns (the transition acts on the key side only, so the
 *     columns of S evolve independently).  Serial over the chunks of the
 *     sequence: Ut = Tm diag(beta) V, U_n = Ut - W S_n, O_n, S_{n+1} (a3, a4),
 *     S carried in fp32 in tensor memory.  Writes o and final_state (NULL:
 *     not written).  It must follow kda_chunk_split_intra on the same
 *     stream, with the same workspace, cu_seqlens and shapes; it does not
 *     reset the device status word, so a failure of either kernel is
 *     reported by kda_get_device_status().
 * Workspace: at least kda_chunk_split_workspace_size() bytes, 256-byte
 *   aligned (it is kda_chunk_fwd_workspace_size() when kda_chunk_fwd takes
 *   the split plan).  Defining passage: Kimi Linear (aiwiki.ai), "The
 *   constrained DPLR form and the chunkwise algorithm" (the intra-chunk part
 *   is parallel across chunks; only the state passes from chunk to chunk).
 */
size_t kda_chunk_split_workspace_size(int total_tokens, int num_seqs, int H);

kda_status_t kda_chunk_split_intra(const void* q, const void* k, const float* g,
                                   const float* beta, const int32_t* cu_seqlens, int B, int T,
                                   int num_seqs, int H, void* workspace, size_t workspace_bytes,
                                   void* stream);

kda_status_t kda_chunk_split_chain(const void* v, const float* initial_state,
                                   const int32_t* cu_seqlens, int B, int T, int num_seqs, int H,
                                   void* o, float* final_state, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* ------------------------------- affine state maps (context parallelism)
 * Kimi Linear (aiwiki.ai), "The constrained DPLR form and the chunkwise
 * algorithm": the state is carried recurrently between chunks, and over any
 * span of tokens that carry is affine in the entry state, S_out = M S_in + B.
 * A long sequence split over ranks by token ranges is therefore prefilled as:
 * every rank computes its segment's (M, B), the ranks exchange them, every
 * rank folds the maps before it into its entry state, and prefills its
 * segment from that state.
 *
 * kda_chunk_state_maps: (M, B) of every (sequence, head) of a prefill, without
 * its outputs: final_state = M initial_state + B, M [num_seqs, H, 128, 128]
 * (the product of the transitions (I - beta k k^T) Diag(alpha), acting on the
 * key side), B [num_seqs, H, 128, 128] (the final state from a zero initial
 * state).  bf16 q, k, v, dk = dv = 128, chunk 64 (the split plan's shapes;
 * otherwise KDA_ERR_UNSUPPORTED): the intra-chunk kernel once, then the chain
 * kernel twice without outputs (from zero with v, from the identity with v
 * taken as zero).  Other arguments and the workspace as kda_chunk_split_*.
 */
kda_status_t kda_chunk_state_maps(const void* q, const void* k, const void* v, const float* g,
                                  const float* beta, const int32_t* cu_seqlens, int B, int T,
                                  int num_seqs, int H, float* M, float* Bm, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* kda_fold_segment_states: composition of R segments' maps, per (sequence,
 * head), on the CUDA cores in fp32.
 *   reverse = 0: S_0 = S0 (NULL: zeros); each[r] = S_r (the entry state of
 *     segment r); S_{r+1} = M_r S_r + Bm_r; final_state = S_R.
 *   reverse != 0 (the backward): g_R = S0 (the final state's gradient; NULL:
 *     zeros); each[r] = g_{r+1} (the gradient of segment r's exit state);
 *     g_r = M_r^T g_{r+1} + Bm_r (Bm_r: the entry-state gradient segment r's
 *     own outputs produce); final_state = g_0 (the initial state's gradient).
 * In:  M [R, N, H, dk, dk], Bm [R, N, H, dk, dv], S0 [N, H, dk, dv] fp32.
 * Out: each [R, N, H, dk, dv], final_state [N, H, dk, dv] fp32.
 * Shapes: dk, dv in {32, 64, 128}; R >= 0 (R = 0: final_state = S0).
 */
kda_status_t kda_fold_segment_states(const float* M, const float* Bm, const float* S0, int R,
                                     int N, int H, int dk, int dv, int reverse, float* each,
                                     float* final_state, void* stream);

/* ------------------------------------------------------------------- decode
 * kda_decode_step: one token per (sequence, head), state updated in place.
 *   Defining passages: Kimi Linear (aiwiki.ai), "Why linear attention exists"
 *   (decoding is a recurrent update whose cost per token does not depend on
 *   the context read so far) and "The constrained DPLR form and the chunkwise
 *   algorithm" (a fixed 128 x 128 state per head).
 * In:  q, k [N, H, dk], v [N, H, dv] (dtype); g [N, H, dk] fp32; beta [N, H]
 *      fp32.  In/out: state [N, H, dk, dv] fp32 (the prefill state layout).
 * Out: o [N, H, dv] (dtype) = S_new^T q.
 * One read and one write of every state element.  No workspace.
 * Shapes: dk, dv in {32, 64, 128}; N >= 0 (N = 0 enqueues nothing).
 */
kda_status_t kda_decode_step(const void* q, const void* k, const void* v, const float* g,
                             const float* beta, float* state, void* o, int N, int H, int dk,
                             int dv, kda_dtype_t dtype, void* stream);

/* ------------------------------- Gated DeltaNet: one gate value per head
 * Kimi Linear (aiwiki.ai), "Background: from the delta rule to gated
 * DeltaNet": the recurrence with a head-uniform gate alpha_t (one value per
 * (token, head)) instead of KDA's per-channel one; DeltaNet is the case
 * g = 0.  Same arguments, layouts, plans' kernels and error behaviour as
 * kda_chunk_fwd / kda_decode_step, except:
 *   g [total, H] fp32 (prefill), [N, H] fp32 (decode) -- log alpha per (token,
 *   head); the workspace is kda_gdn_chunk_fwd_workspace_size() bytes.
 * bf16, dk = dv = 128, chunk 64 runs the tensor-core plan kda_chunk_fwd would
 * choose for the same shape (split, or co-scheduled for few long chains) with
 * the gate read per (token, head) (one exponential per row instead of per
 * element); other shapes spread g over the dk channels in the workspace and
 * run the CUDA-core plan.
 */
size_t kda_gdn_chunk_fwd_workspace_size(int total_tokens, int num_seqs, int H, int dk, int dv,
                                        int chunk, kda_dtype_t dtype);

kda_status_t kda_gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, const float* initial_state,
                               const int32_t* cu_seqlens, int B, int T, int num_seqs, int H,
                               int dk, int dv, int chunk, kda_dtype_t dtype, void* o,
                               float* final_state, void* workspace, size_t workspace_bytes,
                               void* stream);

kda_status_t kda_gdn_decode_step(const void* q, const void* k, const void* v, const float* g,
                                 const float* beta, float* state, void* o, int N, int H, int dk,
                                 int dv, kda_dtype_t dtype, void* stream);

/* ----------------------------------------------------------------- backward
 * kda_chunk_bwd: gradients of L = sum(o * dout) + sum(final_state *
 * dfinal_state) for the forward kda_chunk_fwd computes (same inputs, shapes
 * and sequence description), with respect to q, k, v, g, beta and the
 * initial state.  The pages give no backward equations; they are derived from
 * the chunk form (Kimi Linear (aiwiki.ai), "The constrained DPLR form and the
 * chunkwise algorithm"; chunks of 64 tokens): the forward's per-chunk
 * quantities and entry states are recomputed, a reverse pass over each
 * sequence's chunks carries the state gradient, and per-chunk kernels form
 * the token gradients.  Nine kernel launches on `stream`, fp32 arithmetic on
 * the CUDA cores.
 * In:  q, k [total, H, dk], v [total, H, dv], dout [total, H, dv] (dtype);
 *      g [total, H, dk], beta [total, H] fp32; initial_state [num_seqs, H, dk,
 *      dv] fp32 or NULL (zeros); dfinal_state likewise or NULL (zeros).
 * Out: dq, dk [total, H, dk], dv [total, H, dv], dg [total, H, dk], dbeta
 *      [total, H] -- all fp32; dinitial_state [num_seqs, H, dk, dv] fp32 or
 *      NULL (not written).
 * Workspace: kda_chunk_bwd_workspace_size() bytes, 256-byte aligned (the
 *      forward's intermediates and per-chunk states, the backward's per-token
 *      and per-chunk gradients: about 4 * (total * H * (6 dk + 4 dv + 1) +
 *      chunks * H * (3 dk dv + 4 * 64 * 64 + dk)) bytes, chunks <= (total +
 *      63 num_seqs) / 64).  It starts with the same status word as the
 *      prefill workspace: invalid device cu_seqlens (not 0 .. T, or
 *      decreasing) leave the outputs unwritten and are reported by
 *      kda_get_device_status(workspace).  Shapes: dk, dv in {32, 64, 128}.
 */
size_t kda_chunk_bwd_workspace_size(int total_tokens, int num_seqs, int H, int dk, int dv);

kda_status_t kda_chunk_bwd(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, const float* initial_state, const void* dout,
                           const float* dfinal_state, const int32_t* cu_seqlens, int B, int T,
                           int num_seqs, int H, int dk, int dv, kda_dtype_t dtype, float* dq,
                           float* dk_out, float* dv_out, float* dg, float* dbeta,
                           float* dinitial_state, void* workspace, size_t workspace_bytes,
                           void* stream);

/* kda_gdn_chunk_bwd: the same gradients for Gated DeltaNet (Kimi Linear
 * (aiwiki.ai), "Kimi Delta Attention": one gate value per token and head).
 * g and dg are [total, H] fp32; every other argument is as in kda_chunk_bwd.
 * The gate is spread over the dk channels, the per-channel backward runs, and
 * dg[t, h] is the sum of the channel gradients (the chain rule of the
 * spread).  Workspace: kda_gdn_chunk_bwd_workspace_size() bytes (the
 * kda_chunk_bwd workspace plus two [total, H, dk] fp32 arrays), 256-byte
 * aligned; the status word is read the same way.
 */
size_t kda_gdn_chunk_bwd_workspace_size(int total_tokens, int num_seqs, int H, int dk, int dv);

kda_status_t kda_gdn_chunk_bwd(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, const float* initial_state, const void* dout,
                               const float* dfinal_state, const int32_t* cu_seqlens, int B, int T,
                               int num_seqs, int H, int dk, int dv, kda_dtype_t dtype, float* dq,
                               float* dk_out, float* dv_out, float* dg, float* dbeta,
                               float* dinitial_state, void* workspace, size_t workspace_bytes,
                               void* stream);

/* ---------------------------------------- the steps around the operator
 * Kimi Linear (aiwiki.ai), "The constrained DPLR form and the chunkwise
 * algorithm" (the paragraph on what each KDA head applies): a short depthwise
 * convolution (kernel 4) with a Swish activation on q, k and v and the L2
 * normalisation of q and k before the operator; a head-wise RMSNorm and a
 * sigmoid output gate after it.  Arithmetic in fp32; both calls read and write
 * each tensor once.
 *
 * kda_qkv_conv_norm: for each of q, k, v: y[t, h, c] = Swish(sum_{i=0..3}
 * w[h*d + c][i] * x[t - 3 + i, h, c]) with Swish(x) = x * sigmoid(x), no bias,
 * tap 3 on the current token and tokens before the first token of t's
 * sequence counting as zero (a packed batch never convolves across
 * sequences); then q and k are scaled per (token, head) by
 * 1 / sqrt(sum_c y^2 + eps).
 * In:  xq, xk [total, H, dk], xv [total, H, dv] (dtype); wq, wk [H*dk, 4] and
 *      wv [H*dv, 4] fp32; cu_seqlens / B / T / num_seqs as for kda_chunk_fwd
 *      (cu_seqlens contents are not checked here; a malformed array cannot
 *      make a read leave the tensors); eps > 0.
 * Out: q, k [total, H, dk], v [total, H, dv] (dtype), not aliasing the inputs.
 * Shapes: dk, dv in {32, 64, 128}.
 */
kda_status_t kda_qkv_conv_norm(const void* xq, const void* xk, const void* xv, const float* wq,
                               const float* wk, const float* wv, const int32_t* cu_seqlens,
                               int B, int T, int num_seqs, int H, int dk, int dv,
                               kda_dtype_t dtype, float eps, void* q, void* k, void* v,
                               void* stream);

/* kda_qkv_conv_norm_step: the same for one decode token per sequence, with a
 * convolution state per tensor: conv_q, conv_k [N, 3, H, dk] and conv_v
 * [N, 3, H, dv] (dtype) hold each sequence's last three inputs, oldest first
 * (zeros: no history, as at the start of a prefill).  y = Swish(w0 c0 + w1 c1
 * + w2 c2 + w3 x), q and k L2-normalised; then each state drops its oldest
 * row and appends x (in place).  A prefill hands over by copying the last
 * three input rows of each sequence (zero rows before its start).
 * In:  xq, xk [N, H, dk], xv [N, H, dv] (dtype); weights as above; eps > 0.
 * Out: q, k [N, H, dk], v [N, H, dv] (dtype), not aliasing the inputs or the
 *      states.  Shapes: dk, dv in {32, 64, 128}; N == 0 does nothing.
 */
kda_status_t kda_qkv_conv_norm_step(const void* xq, const void* xk, const void* xv,
                                    const float* wq, const float* wk, const float* wv,
                                    void* conv_q, void* conv_k, void* conv_v, int N, int H,
                                    int dk, int dv, kda_dtype_t dtype, float eps, void* q,
                                    void* k, void* v, void* stream);

/* kda_output_norm_gate: y[t, h, :] = o[t, h, :] / sqrt(mean_j o[t, h, j]^2 +
 * eps) * w * sigmoid(gate[t, h, :]).
 * In:  o, gate [total_tokens, H, dv] (dtype); w [dv] fp32 (shared by the
 *      heads); eps > 0.  Out: y [total_tokens, H, dv] (dtype); y may be o.
 * Shapes: dv in {32, 64, 128}.
 */
kda_status_t kda_output_norm_gate(const void* o, const void* gate, const float* w,
                                  int total_tokens, int H, int dv, kda_dtype_t dtype, float eps,
                                  void* y, void* stream);

/* kda_layer_chunk_fwd: the prefill of a whole KDA layer core --
 * kda_qkv_conv_norm, kda_chunk_fwd and kda_output_norm_gate in one call:
 *   q, k = L2-normalised Swish(conv4) of xq, xk (eps l2_eps), v = Swish(conv4)
 *   of xv, per sequence (zero history at each sequence start);
 *   the chunkwise prefill on (q, k, v, g, beta, initial_state) -> o, S_final;
 *   y = o / sqrt(mean_j o_j^2 + rms_eps) * w_norm * sigmoid(gate).
 * Defining passages: those of the three calls (Kimi Linear (aiwiki.ai), "The
 * constrained DPLR form and the chunkwise algorithm").
 * bf16, dk = dv = 128, chunk 64 runs the split tensor-core plan with the steps
 * fused into its kernels: the intra-chunk kernel convolves and normalises the
 * q and k tiles it loads (the 3 rows before a chunk read from the previous
 * chunk), the chain kernel convolves its V tiles and writes y from the O
 * read-out (the two value-column halves of a chain are the two units of one
 * CTA and add their row sums of o^2 through its shared memory);
 * q, k, v and o never reach HBM.  Every other supported shape runs the three
 * steps one after another with q, k, v, o in the workspace.
 * In:  xq, xk [total, H, dk], xv [total, H, dv], gate [total, H, dv] (dtype);
 *      wq, wk [H*dk, 4], wv [H*dv, 4], w_norm [dv], g [total, H, dk], beta
 *      [total, H] fp32; initial_state and cu_seqlens as for kda_chunk_fwd.
 * Out: y [total, H, dv] (dtype), every token written; final_state as for
 *      kda_chunk_fwd.
 * Workspace: kda_layer_chunk_fwd_workspace_size() bytes, 256-byte aligned,
 *      with the status word read by kda_get_device_status().
 */
size_t kda_layer_chunk_fwd_workspace_size(int total_tokens, int num_seqs, int H, int dk, int dv,
                                          int chunk, kda_dtype_t dtype);

kda_status_t kda_layer_chunk_fwd(const void* xq, const void* xk, const void* xv, const float* wq,
                                 const float* wk, const float* wv, const float* g,
                                 const float* beta, const float* initial_state,
                                 const int32_t* cu_seqlens, int B, int T, int num_seqs, int H,
                                 int dk, int dv, int chunk, kda_dtype_t dtype, const void* gate,
                                 const float* w_norm, float l2_eps, float rms_eps, void* y,
                                 float* final_state, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* kda_layer_decode_step: one decode token of a whole KDA layer core in one
 * launch -- kda_qkv_conv_norm_step, kda_decode_step and kda_output_norm_gate
 * fused, so q, k, v and o never leave the chip:
 *   q, k = L2-normalised Swish(conv4) of xq, xk with the convolution states
 *   (eps l2_eps), v = Swish(conv4) of xv; the states shift in place;
 *   the decode step on (q, k, v, g, beta, state) -> o (fp32, not rounded);
 *   y = o / sqrt(mean_j o_j^2 + rms_eps) * w_norm * sigmoid(gate).
 * Defining passages: those of the three calls (Kimi Linear (aiwiki.ai), "The
 * constrained DPLR form and the chunkwise algorithm": the steps each KDA head
 * applies around the operator).
 * In:  xq, xk [N, H, dk], xv [N, H, dv], gate [N, H, dv] (dtype); wq, wk
 *      [H*dk, 4], wv [H*dv, 4], w_norm [dv], g [N, H, dk], beta [N, H] fp32.
 * In/out: conv_q, conv_k [N, 3, H, dk], conv_v [N, 3, H, dv] (dtype) as for
 *      kda_qkv_conv_norm_step; state [N, H, dk, dv] fp32 as for kda_decode_step.
 * Out: y [N, H, dv] (dtype), not aliasing any input.
 * One 256-thread CTA per (sequence, head) takes all dv value columns, so the
 * RMSNorm's sum over dv stays in its shared memory.  Shapes: dk, dv in
 * {32, 64, 128};
 * N == 0 does nothing.  No workspace.
 */
kda_status_t kda_layer_decode_step(const void* xq, const void* xk, const void* xv,
                                  const float* wq, const float* wk, const float* wv,
                                  void* conv_q, void* conv_k, void* conv_v, const float* g,
                                  const float* beta, float* state, const void* gate,
                                  const float* w_norm, int N, int H, int dk, int dv,
                                  kda_dtype_t dtype, float l2_eps, float rms_eps, void* y,
                                  void* stream);

/* ------------------------------------------------ prefill, no allocation
 * kda_chunk_fwd_noalloc: the same computation as kda_chunk_fwd, with no
 * workspace argument, for callers that may not obtain device memory: an
 * operator inside an engine or graph runtime whose interface passes only
 * inputs and outputs and whose planner owns all device memory, or a serving
 * loop that reserved nearly all HBM up front, where a cudaMalloc would fail,
 * fragment that reservation or stall other streams.  The pages have no
 * counterpart to this call; it is a packaging choice of this library.
 * Scratch: one static device array of KDA_NOALLOC_SCRATCH_BYTES inside the
 *      library, held on every GPU that loads it until the process exits.
 *      When it is committed is the CUDA driver's module-loading choice: with
 *      lazy loading (CUDA 12's default) it is the first call of this entry
 *      point on the device, with eager loading the creation of the context.
 *      So a caller that reserves nearly all HBM up front makes its first call
 *      (a tiny problem will do) before taking that reservation; later calls
 *      take no memory.  The first call on a device also looks up the array's
 *      address (with the device current) -- make it before any stream
 *      capture.  Calls share the array: results never depend on an earlier
 *      call, but calls whose work overlaps on the GPU race.
 * Limit: a problem fits when kda_chunk_fwd_workspace_size(total_tokens,
 *      num_seqs, H, dk, dv, chunk, KDA_DTYPE_F32) <= KDA_NOALLOC_SCRATCH_BYTES;
 *      otherwise KDA_ERR_WORKSPACE and nothing is enqueued.
 * Path: the CUDA-core kernels, for both dtypes.  Device-side cu_seqlens
 *      errors skip the work (o, final_state unwritten) and are not reported.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * Arguments and other errors: as kda_chunk_fwd.
 */
#define KDA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

kda_status_t kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g,
                                   const float* beta, const float* initial_state,
                                   const int32_t* cu_seqlens, int B, int T, int num_seqs, int H,
                                   int dk, int dv, int chunk, kda_dtype_t dtype, void* o,
                                   float* final_state, void* stream);

/* ------------------------------------------------- testing the error path
 * kda_test_overlap_flag_timeout: the overlap plan of kda_chunk_fwd (bf16,
 * dk = dv = 128, chunk 64; KDA_ERR_UNSUPPORTED where that plan does not apply)
 * with the ready flag of global chunk slot `withheld_chunk` of head
 * `withheld_head` never set, and every chain's wait on one flag bounded by
 * flag_wait_ns (1 ns .. 2 s) instead of 2 s.  It exists to exercise the
 * device-side bounded-wait error path without any fault: the chain that needs
 * the withheld chunk gives up after flag_wait_ns, waits for its own copies and
 * products in flight, records KDA_ERR_TIMEOUT in the status word and returns;
 * every other chain and every intra-chunk unit completes (none of them waits
 * on that flag).  kda_get_device_status(workspace) then returns
 * KDA_ERR_TIMEOUT; outputs are unspecified; the next prefill call on the same
 * workspace starts clean.  Arguments otherwise as kda_chunk_fwd_with_plan with
 * KDA_PLAN_OVERLAP (workspace: kda_chunk_fwd_plan_workspace_size of that plan).
 * Not a computation: no caller outside the tests needs it.
 */
kda_status_t kda_test_overlap_flag_timeout(const void* q, const void* k, const void* v,
                                           const float* g, const float* beta,
                                           const float* initial_state,
                                           const int32_t* cu_seqlens, int B, int T,
                                           int num_seqs, int H, void* o, float* final_state,
                                           void* workspace, size_t workspace_bytes,
                                           int withheld_chunk, int withheld_head,
                                           unsigned long long flag_wait_ns, void* stream);

/* ------------------------------------------------------------------ status
 * Synchronises `stream`, then reads the device status word kept at the start
 * of `workspace`.  Every prefill call (kda_chunk_fwd and the step calls)
 * clears that word on entry, so it describes the LAST prefill call enqueued
 * with this workspace.  Returns KDA_OK, the device-side error it recorded
 * (KDA_ERR_BAD_SEQLENS, KDA_ERR_TIMEOUT), or KDA_ERR_CUDA if the copy or the
 * stream reports an error.  The only blocking call in the library.  After a
 * device-side error the call's kernels skipped their work: outputs are
 * unspecified.
 */
kda_status_t kda_get_device_status(void* workspace, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* KDA_H_ */
