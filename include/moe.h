/*
 * moe.h -- C ABI of the B200 (sm_100a) MoE FFN layer library (libmoe.so).
 *
 * The layer is the fine-grained MoE FFN of dots.llm1 (dots.llm1 Technical
 * Report, §Architecture "Mixture of Experts layer" and "Load balancing";
 * §3.2 "Efficient implementation of Grouped GEMM"):
 *
 *   1. FP32 gate:        logit = X Wg^T in FP32                (moe_gate_topk)
 *   2. aux-loss-free top-k: p = softmax(logit), s = p + bias, top-k of s,
 *                        w = p renormalised over the chosen k  (moe_gate_topk)
 *   3. permute into per-expert segments padded to P rows       (moe_permute_align)
 *   4. grouped SwiGLU expert GEMMs, routed + shared experts    (grouped_gemm_fwd)
 *   5. weighted combine                                        (moe_combine)
 *   backward: combine bwd, dX and dW grouped GEMMs             (moe_combine_bwd,
 *             grouped_gemm_bwd_dx, grouped_gemm_bwd_dw, moe_combine)
 *   router backward: dlogits, gate dX and dWg                  (moe_router_bwd)
 *   sequence-wise balance loss and its router gradient         (moe_seq_balance_loss,
 *                                                               moe_router_bwd_seqbal)
 *   aux-loss-free bias step                                    (moe_bias_update)
 *   combine with the shared rows apart (expert parallelism)    (moe_combine_split)
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates or frees device memory.  Row-major, densely packed.
 *   - bf16 tensors are passed as `void*` holding IEEE bfloat16 values.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronise the host, except moe_get_device_status.
 *   - Argument and shape errors return a negative moe_status before anything is
 *     launched.  Errors found on the device (a bounded wait that ran out, an
 *     inconsistent group table) are written to a status word inside the
 *     workspace and read with moe_get_device_status.
 *
 * Shapes (struct moe_dims): T tokens, d hidden, E routed experts, k experts per
 * token, S shared experts, I expert intermediate size, P pad block.
 *   G  = E + S groups; group e < E is routed expert e, group E + s is shared s.
 *   Rr = routed row capacity = dims.rows_cap, or T*k + E*(P-1) when 0.
 *   Rt = Rr + S*T rows of the "grouped row space": routed expert e owns rows
 *        [off_e, off_e + roundup(c_e, P)); shared expert s owns rows
 *        [Rr + s*T, Rr + (s+1)*T) (one row per token, in token order).
 * Weights: W1 [G, 2I, d] bf16 (rows 0..I-1 gate projection, I..2I-1 up
 * projection), W2 [G, d, I] bf16, Wg [E, d] f32, bias [E] f32.
 * Supported: d % 64 == 0, I % 64 == 0, 1 <= k <= E <= 256 (E % 8 == 0 for the
 * gate), S <= 8, P % 8 == 0, P >= 8, Rt < 2^31, T*k < 2^31; the backward needs
 * P % 64 == 0.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,       /* null pointer, bad enum value, ws too small */
  MOE_ERR_UNSUPPORTED_SHAPE = -2, /* shape outside the supported set above */
  MOE_ERR_CUDA = -3,              /* a CUDA runtime/driver call failed */
  MOE_ERR_DEVICE_TIMEOUT = -4,    /* (device) a bounded wait in a kernel ran out */
  MOE_ERR_BAD_ROUTING = -5        /* (device) padded rows exceed Rr, or bad expert id */
} moe_status;

typedef struct moe_dims {
  int64_t T;        /* tokens */
  int32_t d;        /* hidden size */
  int32_t E;        /* routed experts */
  int32_t k;        /* routed experts per token */
  int32_t S;        /* shared experts */
  int32_t I;        /* expert intermediate size */
  int32_t P;        /* pad block of a routed segment (rows) */
  int64_t rows_cap; /* Rr, rows of the routed row space; 0 => T*k + E*(P-1) */
} moe_dims;

/* Which GEMM of the expert FFN a backward call works on. */
enum { MOE_GEMM1 = 1, /* gate|up projection  A1 = A W1^T  (N = 2I, K = d) */
       MOE_GEMM2 = 2  /* down projection     Y  = H W2^T  (N = d,  K = I) */ };

/* Rr and Rt as defined above (-1 for invalid dims).  Host-side sizes: the pages
 * have no counterpart. */
int64_t moe_rows_routed(const moe_dims* dims);
int64_t moe_rows_total(const moe_dims* dims);

/* Bytes of device workspace that the calls taking `ws` need (host-side, no
 * counterpart on the pages).  One workspace
 * serves a whole layer.  It starts with the routing tables (the status word,
 * the group table, tile prefixes, per-chunk histograms): moe_permute_align (or
 * grouped_gemm_set_groups) writes them, the GEMM and combine-backward calls
 * read them.  The routing header also holds one tile counter per grouped-GEMM
 * launch kind (forward GEMM1 and GEMM2, the two data-gradient and the two
 * weight-gradient GEMMs): the routing calls clear them, and every launch draws
 * its tiles from its counter and leaves it at 0, also when its waits ran out.
 * So two launches of the same kind on one workspace must not overlap on the GPU
 * (launches of different kinds may).  After the routing tables, 1024-byte
 * aligned, moe_gate_topk keeps the gate weights split into three bf16 planes,
 * 3 * E_pad * d * 2 bytes with E_pad = E rounded up to a multiple of 32. */
size_t moe_workspace_size(const moe_dims* dims);

/* Gate and aux-loss-free top-k routing.
 * Passage: dots.llm1 Technical Report, §Architecture "Mixture of Experts
 * layer" (the gating layer runs in FP32, top-6 of 128 routed experts) and
 * "Load balancing" (a per-expert bias is added to the affinity scores only to
 * decide the top-k routing).
 *   x     [T, d]  bf16          hidden states
 *   wg    [E, d]  f32           gate weights
 *   bias  [E]     f32           selection bias (may be NULL: zero)
 * Out:
 *   topk_idx [T, k] int32       chosen experts, biased score descending, equal
 *                               scores to the lower expert index
 *   topk_w   [T, k] f32         p[e_j] / sum_j p[e_j] (unbiased, renormalised)
 *   probs    [T, E] f32         softmax affinities (may be NULL)
 *   ws / ws_bytes               workspace of moe_workspace_size(dims) bytes: the
 *                               call rewrites its gate-weight planes and may set
 *                               its status word; the routing tables are untouched
 * The logits are FP32 sums of exact FP32 products: each FP32 weight is split
 * exactly into three bf16 terms (hi + mid + lo, exact to below 2^-24 |w|),
 * x is bf16, and the tensor cores accumulate the products in FP32.  p uses
 * expf.  Non-finite inputs cannot make an invalid choice: a NaN score ranks
 * last (ties by index), so every token still names k distinct experts in
 * [0, E).  Requires E % 8 == 0, E <= 256, d % 64 == 0.  A bounded wait that runs
 * out on the device sets MOE_ERR_DEVICE_TIMEOUT in the status word and leaves
 * the outputs of the affected tokens unwritten. */
int moe_gate_topk(const moe_dims* dims, const void* x, const float* wg, const float* bias,
                  int32_t* topk_idx, float* topk_w, float* probs, void* ws, size_t ws_bytes,
                  void* stream);

/* Permutation into per-expert segments padded to P rows, plus the group table.
 * Passage: dots.llm1 Technical Report, §3.2 "Efficient implementation of
 * Grouped GEMM" (each expert's token segment M_i is aligned to a fixed block,
 * so one tile belongs to one expert) and §Architecture "Load balancing" (no
 * token is dropped: segments grow with the load, there is no capacity).
 *   topk_idx [T, k] int32 (from moe_gate_topk or the caller), x [T, d] bf16
 * Out:
 *   counts     [E]      int32   c_e, tokens routed to expert e
 *   offsets    [E + 1]  int32   off_0 = 0, off_{e+1} = off_e + roundup(c_e, P)
 *   sorted_ids [Rr]     int32   token of each routed row (ascending inside a
 *                               segment), -1 on pad rows and rows >= off_E
 *   row_of     [T, k]   int32   routed row of (t, j)
 *   x_perm     [Rr, d]  bf16    x_perm[row_of[t, j]] = x[t]; pad rows zero;
 *                               rows >= off_E are not written.  May be NULL
 *                               (then x may be NULL too): only the routing
 *                               tables are written, for the *_gather GEMMs
 *                               below, which read x rows through sorted_ids
 *   ws / ws_bytes               workspace (group table written here)
 * Deterministic: the same input gives the same output bit for bit.  An expert
 * id outside [0, E) or off_E > Rr sets MOE_ERR_BAD_ROUTING in the device
 * status, leaves an empty group table and sets every row_of entry to -1, so
 * the combine calls below add nothing for those picks instead of following a
 * stale row. */
int moe_permute_align(const moe_dims* dims, const int32_t* topk_idx, const void* x,
                      int32_t* counts, int32_t* offsets, int32_t* sorted_ids, int32_t* row_of,
                      void* x_perm, void* ws, size_t ws_bytes, void* stream);

/* moe_permute_align without a workspace argument: the same outputs, with the
 * scratch (status header, group table, chunk histograms) held in a fixed
 * 1 MiB device array inside the library.  (The pages have no counterpart: this
 * is an allocation-free form of the call above.)  It serves callers that cannot
 * allocate device memory or keep a workspace alive between calls -- code inside
 * a host framework whose allocator owns every device buffer, foreign-function
 * callers that pass only inputs and outputs, paths where cudaMalloc is not
 * allowed.  It calls no cudaMalloc or cudaFree.
 *   - Limit: the call's scratch is the routing-table part of the workspace
 *     only (not the gate planes or router-backward scratch that
 *     moe_workspace_size also counts): a 64-byte header, 16 G bytes of group
 *     table, 4 (G + 1) of tile prefix, 4 G of group order and
 *     4 E max(1, ceil(T k / 1024)) of chunk histograms, each part starting on
 *     a 16-byte boundary and the sum rounded up to 256.  It must be at most
 *     1 MiB (1,048,576 bytes; about 2 million routed assignments at E = 128,
 *     1 million at E = 256); larger shapes return MOE_ERR_UNSUPPORTED_SHAPE
 *     before anything is launched.
 *   - The array is shared by every call in the process and keeps the last
 *     call's contents; each call clears what must start at zero.  Calls whose
 *     executions overlap on the GPU (other streams, other threads) race on it
 *     and must be serialised by the caller.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any stream
 *     capture.  The address is kept for the life of the process: it does not
 *     survive cudaDeviceReset, after which this call must not be used on that
 *     device again.
 *   - Routing errors (expert id outside [0, E), padded rows above Rr) leave
 *     sorted_ids and row_of at -1 and x_perm unwritten; no device status is
 *     kept. */
int moe_permute_align_static(const moe_dims* dims, const int32_t* topk_idx, const void* x,
                             int32_t* counts, int32_t* offsets, int32_t* sorted_ids,
                             int32_t* row_of, void* x_perm, void* stream);

/* Group table from given per-expert row counts, for callers that already hold
 * the permuted rows (the grouped GEMM used on its own).
 * Passage: dots.llm1 Technical Report, §3.2 "Efficient implementation of
 * Grouped GEMM" (g groups with per-group row counts M_i, each aligned to a
 * fixed block).  counts [E] int32
 * (device); writes offsets [E + 1] (device) and the group table in ws, with
 * segments padded to P as in moe_permute_align. */
int grouped_gemm_set_groups(const moe_dims* dims, const int32_t* counts, int32_t* offsets,
                            void* ws, size_t ws_bytes, void* stream);

/* Forward grouped GEMMs of the expert FFNs (routed + shared), SwiGLU fused.
 * Passage: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
 * (fine-grained two-layer SwiGLU experts; 2 shared experts see every token)
 * and §3.2 (one tile = one expert's aligned segment).
 *   ws       workspace holding the group table
 *   x_perm   [Rr, d] bf16  A rows of the routed groups
 *   x        [T, d]  bf16  A rows of the shared groups (may be NULL when S = 0 or T = 0)
 *   w1 [G, 2I, d] bf16, w2 [G, d, I] bf16
 * Out (grouped row space, rows of each group up to its padded size):
 *   h  [Rt, I]  bf16  H = silu(A W1g^T) * (A W1u^T), from the FP32 accumulator
 *   a1 [Rt, 2I] bf16  [A W1g^T | A W1u^T], saved for the backward (may be NULL)
 *   y  [Rt, d]  bf16  Y = H W2^T
 * bf16 operands, FP32 accumulation in tensor memory (tcgen05). */
int grouped_gemm_fwd(const moe_dims* dims, const void* ws, const void* x_perm, const void* x,
                     const void* w1, const void* w2, void* h, void* a1, void* y, void* stream);

/* grouped_gemm_fwd with the routed groups' A rows gathered from x itself: row
 * r of routed group e is x[sorted_ids[off_e + r]], loaded four rows at a time
 * by tile::gather4 tensor copies, so no permuted copy x_perm is written or
 * read.  (Passage: §3.2, as above; the row order inside a segment is the one
 * moe_permute_align gives.)
 *   sorted_ids [Rr] int32 (device), as written by moe_permute_align
 *   x          [T, d] bf16 (may be NULL only when T = 0)
 *   other arguments and outputs as in grouped_gemm_fwd.
 * Rows holding no token (pad rows, id -1) and ids outside [0, T) read the
 * group's first token instead of zeros: their h / a1 / y rows hold that
 * token's values (pad-row contents are unspecified; nothing reads them, and
 * with zero upstream gradients on pad rows they add nothing to dW).  No row
 * outside x is ever read. */
int grouped_gemm_fwd_gather(const moe_dims* dims, const void* ws, const int32_t* sorted_ids,
                            const void* x, const void* w1, const void* w2, void* h, void* a1,
                            void* y, void* stream);

/* Backward data-gradient grouped GEMMs.
 * Passage: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
 * (the SwiGLU expert FFN whose input gradient this is) and §3.2 "Performance
 * comparison" (the backward grouped GEMM, timed against Transformer Engine).
 *   which = MOE_GEMM2: dH = dY W2, then the SwiGLU backward with the saved a1:
 *       dG = dH * U * s * (1 + G (1 - s)), s = sigmoid(G);  dU = dH * silu(G)
 *     dy_routed [Rr, d] bf16 (from moe_combine_bwd), dy_shared [T, d] bf16 (the
 *     upstream gradient itself; may be NULL when S = 0 or T = 0), w = w2, a1 [Rt, 2I]
 *     -> out = dA [Rt, 2I] bf16 ([dG | dU])
 *   which = MOE_GEMM1: dX_perm = dA W1
 *     dy_routed = dA [Rt, 2I] bf16, dy_shared ignored, w = w1, a1 ignored
 *     -> out = dX rows [Rt, d] bf16 (reduce with moe_combine, topk_w = NULL) */
int grouped_gemm_bwd_dx(const moe_dims* dims, const void* ws, int which, const void* dy_routed,
                        const void* dy_shared, const void* w, const void* a1, void* out,
                        void* stream);

/* Backward weight-gradient grouped GEMMs; the reduction runs over each group's
 * (padded) rows.
 * Passage: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
 * (the expert weights being trained) and §3.2 "Performance comparison" (the
 * backward grouped GEMM); the aligned segments of §3.2 "Efficient
 * implementation of Grouped GEMM" keep every 64-row reduction block inside one
 * expert (hence P % 64 == 0).
 *   which = MOE_GEMM2: dW2_g = dY_g^T H_g
 *     lhs_routed = dY [Rr, d], lhs_shared = upstream gradient [T, d],
 *     rhs_routed = H [Rt, I], rhs_shared ignored  -> dw = dW2 [G, d, I] f32
 *   which = MOE_GEMM1: dW1_g = dA_g^T A_g
 *     lhs_routed = dA [Rt, 2I], lhs_shared ignored,
 *     rhs_routed = x_perm [Rr, d], rhs_shared = x [T, d] -> dw = dW1 [G, 2I, d] f32
 * accumulate = 0 overwrites dw (an expert with no rows gets zeros);
 * accumulate = 1 adds to it. */
int grouped_gemm_bwd_dw(const moe_dims* dims, const void* ws, int which, const void* lhs_routed,
                        const void* lhs_shared, const void* rhs_routed, const void* rhs_shared,
                        float* dw, int accumulate, void* stream);

/* Passage: as grouped_gemm_bwd_dw above (§Architecture "Mixture of Experts
 * layer"; §3.2 "Performance comparison").
 * dW1_g = dA_g^T X_g (grouped_gemm_bwd_dw with which = MOE_GEMM1) with the
 * routed groups' x rows gathered from x by sorted_ids as in
 * grouped_gemm_fwd_gather; no x_perm.
 *   sorted_ids [Rr] int32, da [Rt, 2I] bf16, x [T, d] bf16 (NULL only when T = 0)
 *   -> dw1 [G, 2I, d] f32; accumulate as in grouped_gemm_bwd_dw.
 * Pad rows of da must be zero (moe_combine_bwd zeroes the pad rows of dY, and
 * the SwiGLU backward keeps them zero), since their x rows are a real token's. */
int grouped_gemm_bwd_dw1_gather(const moe_dims* dims, const void* ws, const int32_t* sorted_ids,
                                const void* da, const void* x, float* dw1, int accumulate,
                                void* stream);

/* Weighted combine (un-permute).
 * Passage: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
 * (each token's output sums its 6 routed experts and the 2 shared experts).
 *   y [Rt, d] bf16 (grouped row space), row_of [T, k], topk_w [T, k] f32
 *   out[t] = sum_j topk_w[t, j] * y[row_of[t, j]] + sum_s y[Rr + s*T + t]
 * accumulated in FP32, stored bf16 into out [T, d].  topk_w = NULL uses weight 1
 * for every routed row: the un-permute-sum that turns dX rows into dX.  A pick
 * whose row_of is outside [0, Rr) (-1 after a refused permutation) adds
 * nothing. */
int moe_combine(const moe_dims* dims, const void* y, const int32_t* row_of, const float* topk_w,
                void* out, void* stream);

/* Passage: as moe_combine above; the expert-parallel layout it serves is the
 * pages' training setting (§3.1, all-to-all dispatch and combine of expert
 * parallelism overlapped with computation).
 * moe_combine with the shared experts' rows in a buffer of their own:
 *   out[t] = sum_j topk_w[t, j] * y_routed[row_of[t, j]] + sum_s y_shared[s*T + t]
 * y_routed [Rr, d] bf16 (the routed rows of the grouped row space), y_shared
 * [S, T, d] bf16 (NULL only when S = 0).  The sums, their order and the
 * rounding are moe_combine's; with y_shared = y_routed + Rr rows the result is
 * moe_combine's bit for bit.  Used under expert parallelism, where a rank's
 * routed rows come back from the experts' owners into one buffer while its
 * shared experts' rows stay in the buffer of its local grouped GEMM.
 * topk_w = NULL: the un-permute-sum, as in moe_combine. */
int moe_combine_split(const moe_dims* dims, const void* y_routed, const void* y_shared,
                      const int32_t* row_of, const float* topk_w, void* out, void* stream);

/* Passage: as moe_combine above (§Architecture "Mixture of Experts layer").
 * moe_combine with the FP32 sums stored as they are, out [T, d] f32, without the
 * final bf16 rounding (the same sums in the same order: rounding this output to
 * bf16 gives moe_combine's bits).  For callers that keep the layer output, or
 * dX before the router's term is added, in FP32. */
int moe_combine_f32(const moe_dims* dims, const void* y, const int32_t* row_of,
                    const float* topk_w, float* out, void* stream);

/* Backward of the weighted combine.
 * Passage: dots.llm1 Technical Report, §Architecture "Mixture of Experts layer"
 * (the output is the affinity-weighted sum of the routed experts plus the
 * shared experts; this is its gradient with respect to the routed rows and the
 * weights).
 *   dout [T, d] bf16, y [Rt, d] bf16 (forward output rows), row_of, topk_w
 * Out:
 *   dy_routed [Rr, d] bf16   dy[row_of[t, j]] = topk_w[t, j] * dout[t];
 *                            pad rows of every segment set to zero
 *   dw        [T, k]  f32    dw[t, j] = sum_c dout[t, c] * y[row_of[t, j], c]
 * The shared experts' dY is dout itself (no copy).  A pick whose row_of is
 * outside [0, Rr) scatters nothing and gets dw = 0. */
int moe_combine_bwd(const moe_dims* dims, const void* ws, const void* dout, const void* y,
                    const int32_t* row_of, const float* topk_w, void* dy_routed, float* dw,
                    void* stream);

/* Router backward: the gradient of the combine weights through their
 * renormalisation over the chosen k and the softmax, into the gate's input and
 * weights.
 * Passage: dots.llm1 Technical Report, §Architecture "Mixture of Experts
 * layer" (FP32 gate; the weights are the chosen experts' affinities) and "Load
 * balancing" (the bias only decides the selection, so it gets no gradient; the
 * selection itself is piecewise constant).  With Z = sum_{j chosen} p_j:
 *   dp_j = (dw_j - sum_i dw_i w_i) / Z  (chosen j; 0 elsewhere)
 *   dlogit_e = p_e (dp_e - sum_j p_j dp_j)
 *   dx += dlogit Wg                      dwg (+)= dlogit^T x
 *   x        [T, d] bf16             the gate's input
 *   wg       [E, d] f32              gate weights
 *   probs    [T, E] f32              softmax affinities (moe_gate_topk's probs)
 *   topk_idx, topk_w [T, k]          the forward's choice and combine weights
 *   dw       [T, k] f32              dL/dw (moe_combine_bwd's dw)
 * Out:
 *   dlogits  [T, E] f32              may be NULL
 *   dx       [T, d] bf16             read-modify-write: the gate's term is added
 *   dwg      [E, d] f32              written, or added to when accumulate != 0
 *   ws / ws_bytes                    workspace of moe_workspace_size(dims) bytes;
 *                                    the call overwrites its gate-weight planes and
 *                                    scratch, not its routing tables
 * Both GEMMs run on the tensor cores over exact three-term bf16 splits of the
 * FP32 operands (dlogit, Wg), accumulating in FP32.  Requires E % 8 == 0,
 * E <= 256, d % 64 == 0.  A bounded wait that runs out on the device sets
 * MOE_ERR_DEVICE_TIMEOUT in the status word. */
int moe_router_bwd(const moe_dims* dims, const void* x, const float* wg, const float* probs,
                   const int32_t* topk_idx, const float* topk_w, const float* dw, float* dlogits,
                   void* dx, float* dwg, int accumulate, void* ws, size_t ws_bytes, void* stream);

/* Sequence-wise balance loss and the gradient it sends into the router.
 * Passage: dots.llm1 Technical Report, §Architecture "Load balancing": besides
 * the aux-loss-free bias, a sequence-wise balance loss keeps a single sequence
 * from extreme imbalance.  The pages give no formula; this is the one of the
 * report they cite for their method (DeepSeek-V3), with this layer's softmax
 * affinities and the batch's loss the mean over its sequences.  The T tokens
 * form sequences of seq_len tokens (the last may be shorter); for sequence s
 * with L_s tokens and expert e:
 *   f[s, e] = E / (k L_s) * #{(t in s, j) : topk_idx[t, j] = e}
 *   P[s, e] = (1 / L_s) * sum_{t in s} probs[t, e]       (probs sum to 1 per token)
 *   loss    = alpha / n_seq * sum_s sum_e f[s, e] P[s, e]
 *   seq_grad[s, e] = alpha f[s, e] / (n_seq L_s) = dloss / dprobs[t, e], t in s
 * (the picks are piecewise constant: the gradient runs through P only).
 *   topk_idx [T, k] int32, probs [T, E] f32   (moe_gate_topk's outputs)
 * Out:
 *   loss     [1] f32 (device)
 *   seq_grad [ceil(T / seq_len), E] f32      for moe_router_bwd_seqbal
 *   ws / ws_bytes                            workspace of moe_workspace_size(dims)
 *                                            bytes (its balance-loss scratch is used)
 * Requires seq_len >= 128 (MOE_ERR_UNSUPPORTED_SHAPE otherwise).  FP32, in a
 * fixed order: the same inputs give the same bits.  T = 0 gives loss 0. */
int moe_seq_balance_loss(const moe_dims* dims, int64_t seq_len, float alpha,
                         const int32_t* topk_idx, const float* probs, float* loss,
                         float* seq_grad, void* ws, size_t ws_bytes, void* stream);

/* Passage: as moe_router_bwd and moe_seq_balance_loss above (§Architecture
 * "Mixture of Experts layer" and "Load balancing").
 * moe_router_bwd with the sequence-wise balance loss's gradient included: for a
 * token t of sequence s = t / seq_len, dp[e] += seq_grad[s, e] for every expert
 * before the softmax backward, so dlogits, the gate's dx term and dwg carry
 * both losses.  seq_grad and seq_len as written and used by
 * moe_seq_balance_loss (seq_len >= 128); other arguments as in moe_router_bwd. */
int moe_router_bwd_seqbal(const moe_dims* dims, const void* x, const float* wg,
                          const float* probs, const int32_t* topk_idx, const float* topk_w,
                          const float* dw, const float* seq_grad, int64_t seq_len,
                          float* dlogits, void* dx, float* dwg, int accumulate, void* ws,
                          size_t ws_bytes, void* stream);

/* Aux-loss-free bias step.
 * Passage: dots.llm1 Technical Report, §Architecture "Load balancing" (the
 * per-expert bias is adjusted during training to keep the loads balanced; the
 * pages give no rule, this is the plainest one of that kind):
 *   bias_out[e] = bias_in[e] + gamma * sign(T k / E - counts[e])   (sign(0) = 0)
 *   counts [E] int32   the step's routed load per expert (moe_permute_align's counts)
 * bias_in and bias_out may be the same buffer.  One FP32 addition per expert,
 * correctly rounded. */
int moe_bias_update(const moe_dims* dims, const int32_t* counts, float gamma,
                    const float* bias_in, float* bias_out, void* stream);

/* ---------------------------------------------------------------------------
 * Expert parallelism on the device.
 * Passage: dots.llm1 Technical Report, §3.1 "Interleaved-1F1B based
 * communication/computation overlap" (the all-to-all dispatch and combine of
 * expert parallelism, overlapped with computation) and §3.2 (expert-aligned
 * segments).
 *
 * W <= MOE_EP_MAX_WORLD ranks of one node; rank r owns the routed experts
 * r E_l .. (r + 1) E_l - 1 (E_l = E / W) and every rank keeps the S shared
 * experts for its own tokens.  Each rank routes and permutes its own T tokens
 * over all E experts (moe_gate_topk, moe_permute_align with x_perm = NULL); an
 * owner lays out what it receives expert-major: for each of its experts, the
 * P-padded segments of ranks 0 .. W-1.
 *
 * Rows move by kernels that write straight into other ranks' buffers through
 * peer pointers (device memory of the other GPUs mapped into this process, e.g.
 * symmetric memory; a rank's own entries are its own buffers).  Every sending
 * kernel ends with its last CTA adding 1 to a counter in each receiving rank's EP
 * workspace; every receiver waits on the device, bounded by the library's wait
 * budget, until its counter reaches W x (its step count).  No size or count
 * comes to the host, so a whole step can be captured in a CUDA graph.
 *
 * Order of one training step on every rank (one stream):
 *   moe_gate_topk, moe_permute_align (x_perm = NULL), an all-gather of every
 *   rank's counts into counts_all [W, E] (e.g. NCCL), moe_ep_plan,
 *   grouped_gemm_set_groups (local dims, counts_loc), moe_ep_zero_pads (the
 *   receive buffer of x rows), moe_ep_dispatch, grouped_gemm_fwd_ep,
 *   moe_ep_wait(MOE_EP_WAIT_Y), moe_combine_split;
 *   moe_ep_zero_pads (the receive buffer of dY), moe_ep_combine_bwd,
 *   grouped_gemm_bwd_dx_ep(MOE_GEMM2), grouped_gemm_bwd_dw (both), and only then
 *   grouped_gemm_bwd_dx_ep(MOE_GEMM1), moe_ep_wait(MOE_EP_WAIT_DX),
 *   moe_combine_split (topk_w = NULL) and the router backward.
 * The data-gradient return comes last on purpose: a source starts writing its
 * next step's rows into an owner's receive buffers only after every owner has
 * returned its dX rows, and by then that owner has finished reading them.
 * Every rank must run the same number of steps.  A receive buffer too small for
 * the rows a step sends it (recv_cap) is reported as MOE_ERR_BAD_ROUTING in the
 * EP workspace's status word and nothing is written into it.  A wait that runs
 * out sets MOE_ERR_DEVICE_TIMEOUT (in the EP workspace for moe_ep_wait, in the
 * layer workspace for the GEMMs) and the call returns without its rows.
 * Requires P % 32 == 0, E % W == 0 and k <= 32.
 * ------------------------------------------------------------------------- */
#define MOE_EP_MAX_WORLD 8

typedef struct moe_ep_peers {
  int32_t rank;   /* this process's rank */
  int32_t world;  /* W, 1 .. MOE_EP_MAX_WORLD */
  int64_t rows_cap;                /* rows of each buffer in rows[] */
  void* ep_ws[MOE_EP_MAX_WORLD];   /* every rank's EP workspace, as mapped here */
  void* rows[MOE_EP_MAX_WORLD];    /* every rank's buffer this call writes rows into
                                      (bf16 [rows_cap, d]); unused entries NULL */
} moe_ep_peers;

/* Which counter moe_ep_wait waits on. */
enum { MOE_EP_WAIT_Y = 3,  /* every owner has written its Y rows into this rank's buffer */
       MOE_EP_WAIT_DX = 5  /* every owner has written its dX rows into this rank's buffer */ };

/* Bytes of a rank's EP workspace (counters, status word and the step's plan;
 * host-side size, no counterpart on the pages).
 * It must be zeroed once before the first step and be reachable from every
 * rank; afterwards only the calls below touch it. */
size_t moe_ep_workspace_size(const moe_dims* dims, int32_t world);

/* The step's exchange plan from every rank's per-expert counts (Passage: §3.1
 * and §3.2, as above).
 *   dims        the layer's dims (all E experts, this rank's T tokens)
 *   counts_all  [W, E] int32 (device): row s = rank s's counts from moe_permute_align
 *   counts_loc  [E_l] int32 (device) out: rows of each local expert, all segments
 *               padded to P (for grouped_gemm_set_groups on the local dims)
 *   recv_cap    rows of every rank's receive buffers (the same on all ranks)
 * Also advances this rank's step count.  peers->rows is not used. */
int moe_ep_plan(const moe_dims* dims, const moe_ep_peers* peers, const int32_t* counts_all,
                int32_t* counts_loc, int64_t recv_cap, void* stream);

/* Dispatch (Passage: §3.1, the all-to-all dispatch): this rank's segment of each
 * expert g -- the rows of x that sorted_ids lists for it, in order -- into the
 * owner's receive buffer (peers->rows[o], [recv_cap, d] bf16) at the rows the
 * plan gives.  Segments go out local expert by local expert (every owner's first
 * expert, then every owner's second, ...), and as soon as a segment is written the
 * owner's arrival counter of that expert is raised, so the owner's grouped GEMM
 * starts on an expert while later ones are still arriving.
 *   sorted_ids [Rr], offsets [E + 1] as moe_permute_align wrote them for this
 *   rank; x [T, d] bf16. */
int moe_ep_dispatch(const moe_dims* dims, const moe_ep_peers* peers, const int32_t* sorted_ids,
                    const int32_t* offsets, const void* x, void* stream);

/* Owner (Passage: §3.2, segments padded to a fixed block): zero the pad rows
 * of every received segment of its receive buffer
 * recv [recv_cap, d] bf16 (x rows before the forward, dY rows before the
 * backward), as the plan lays them out. */
int moe_ep_zero_pads(const moe_dims* dims, const moe_ep_peers* peers, void* recv, void* stream);

/* Source: wait (bounded) until every owner has returned this step's rows
 * (Passage: §3.1, the combine side of the all-to-all). */
int moe_ep_wait(const moe_ep_peers* peers, int which, void* stream);

/* moe_combine_bwd under expert parallelism (Passage: §Architecture "Mixture of
 * Experts layer" and §3.1): dw [T, k] as there; each pick's dY
 * row goes to its owner's receive buffer (peers->rows[o]), then every owner's
 * arrival counter is raised.  Pad rows are zeroed by the owners
 * (moe_ep_zero_pads).  y [Rr, d] = this rank's routed rows returned by the
 * forward; topk_idx and offsets as for moe_ep_dispatch. */
int moe_ep_combine_bwd(const moe_dims* dims, const moe_ep_peers* peers, const void* dout,
                       const void* y, const int32_t* row_of, const float* topk_w,
                       const int32_t* topk_idx, const int32_t* offsets, float* dw, void* stream);

/* Passage: §3.1 (communication overlapped with computation) and §3.2.
 * grouped_gemm_fwd on an owner (dims_loc: E = E_l local experts, rows_cap =
 * recv_cap): the first GEMM starts with the shared experts' tiles and, before the
 * tiles of each local expert, waits (bounded) until every source's segment of that
 * expert has arrived; the second
 * GEMM writes each routed group's Y rows straight into the buffer of the rank
 * they came from (peers->rows[s], [rows_cap, d]: the source's routed rows, in its
 * permuted layout) instead of into y, then raises every source's counter.  The
 * shared experts' rows land in y at rows Rr_loc + s T as usual. */
int grouped_gemm_fwd_ep(const moe_dims* dims_loc, const void* ws, const moe_ep_peers* peers,
                        const void* x_recv, const void* x, const void* w1, const void* w2,
                        void* h, void* a1, void* y, void* stream);

/* Passage: §3.1 and §3.2, as grouped_gemm_fwd_ep.
 * grouped_gemm_bwd_dx on an owner: MOE_GEMM2 waits for every source's dY rows
 * (shared tiles first); MOE_GEMM1 writes each routed group's dX rows into the
 * buffer of the rank they came from (peers->rows[s]) and raises its counter. */
int grouped_gemm_bwd_dx_ep(const moe_dims* dims_loc, const void* ws, const moe_ep_peers* peers,
                           int which, const void* dy_recv, const void* dy_shared, const void* w,
                           const void* a1, void* out, void* stream);

/* Reads and clears the device status word of `ws` (synchronises `stream`).
 * Error reporting of this library: the pages have no counterpart.
 * *status_out receives MOE_OK or the first device error recorded. */
int moe_get_device_status(void* ws, int32_t* status_out, void* stream);

/* The CUDA error string behind the calling thread's most recent MOE_ERR_CUDA
 * ("no error" if there was none).  No counterpart on the pages. */
const char* moe_last_cuda_error(void);

/* Human-readable name of a moe_status value.  No counterpart on the pages. */
const char* moe_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
