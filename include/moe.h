/*
 * moe.h -- C ABI of the B200 (sm_100a) MoE-layer hot path:
 *          route -> balance -> dispatch -> expert FFN -> combine on one GPU.
 *
 * The R expert-parallel ranks are partitions of this GPU's HBM: rank u owns rows
 * [u*C, (u+1)*C) of every per-rank buffer, C = T*k/R ("a rank may mean one process, one
 * accelerator, or one partition", "MoE Load Balancing: Find Expert Hotspots", section
 * "Reject incomparable MoE load-balancing traces").
 *
 * Sources cited below (page title, section):
 *   [MoonEP]   "Moonshot AI drops MoonEP, claims 2.5x scaling boost for trillion-parameter
 *              models" (news article), paragraphs 2-4.
 *   [Primer]   "DeepEP-on-EFA Guidance, section 1: What is MoE", the four-phase
 *              expert-parallel pipeline (a) router, (b) dispatch, (c) expert FFN,
 *              (d) combine.
 *   [Hotspots] "MoE Load Balancing: Find Expert Hotspots".
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise, allocated and
 *     owned by the caller; the library never allocates, frees or synchronises.  All work
 *     is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default).
 *   - 16-bit tensors are passed as moe_bf16 / moe_f16 (raw bit patterns); layouts are
 *     row-major and contiguous.  Token rows and the up/gate projections W1, W3 are bf16;
 *     the down projection W2 and the activations h are fp16 (see moe_grouped_ffn).
 *   - Return value: a host status (MOE_OK, or an MOE_ERR_* code) decided from the
 *     scalar arguments and pointer nullness BEFORE anything is enqueued; on a non-zero
 *     status nothing was enqueued.  MOE_ERR_LAUNCH reports a failed launch.
 *   - Data-dependent errors are OR-ed into the caller's device word `*err` (int32) with
 *     the MOE_DERR_* bits.  moe_topk sets *err to 0 first (it begins a layer); a caller
 *     that skips moe_topk must zero *err itself.  Every other call reads *err on the
 *     device and does nothing when it is non-zero, so a bad trace stops the layer without
 *     a host sync; its outputs are then unspecified.  Nothing traps or asserts.
 *   - Size limits: 1 <= k <= min(E, 32), E <= 1024, E % R == 0, (T*k) % R == 0,
 *     d % 128 == 0, F % 128 == 0, R*(E/R + S) <= 4096, every element count < 2^31.
 *     T == 0 is allowed (every call is then a no-op apart from clearing outputs that
 *     are defined for it).
 */
#ifndef MOE_H_
#define MOE_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16;   /* bfloat16 bit pattern */
typedef uint16_t moe_f16;    /* IEEE binary16 bit pattern */
typedef void* moe_stream_t;  /* cudaStream_t */

/* host status codes */
enum {
  MOE_OK = 0,
  MOE_ERR_ARG = 1,     /* null pointer or negative size                              */
  MOE_ERR_SHAPE = 2,   /* a size limit above is violated                             */
  MOE_ERR_LAUNCH = 3,  /* a CUDA launch or attribute call failed                     */
  MOE_ERR_DEVICE = 4   /* no usable sm_100 device / driver entry point               */
};

/* device error-word bits */
enum {
  MOE_DERR_NONFINITE = 1,  /* a router logit is NaN or +-inf                         */
  MOE_DERR_ID_RANGE = 2,   /* an expert id outside [0, E)                            */
  MOE_DERR_DUPLICATE = 4,  /* a token names the same expert twice                    */
  MOE_DERR_SLOTS = 8,      /* the plan needs more than S replicas on some rank       */
  MOE_DERR_TIMEOUT = 16    /* a bounded wait inside a kernel gave up (FFN, copies)  */
};

/* Word offsets of the plan's fields inside the caller's int32 plan buffer. */
typedef struct moe_plan_layout {
  int64_t kept_rows;       /* [R]   rows of rank u held by experts kept whole at home      */
  int64_t room_prefix;     /* [R+1] exclusive prefix of the ranks' rooms (C - kept_rows)   */
  int64_t expert_home_off; /* [E]   local row offset of a kept expert at home, -1 streamed  */
  int64_t stream_off;      /* [E+1] exclusive prefix over e of (streamed ? count[e] : 0)    */
  int64_t replica_expert;  /* [R*S] expert held by pool slot u*S+s, -1 if empty            */
  int64_t replica_list;    /* [1+R*S] number of filled slots, then their ids ascending     */
  int64_t n_groups;        /* [R]   groups of rank u                                        */
  int64_t groups;          /* [R*(B+S)][4] {row_start (global row), rows, expert,
                                    weight_ref}; weight_ref = e (< E) reads the home
                                    tensors, E + u*S + s reads pool slot u*S+s; entries
                                    past n_groups[u] are all -1                             */
  int64_t words;           /* total int32 words of the plan buffer                          */
  int32_t max_groups_per_rank; /* B + S                                                     */
} moe_plan_layout;

/* Fills *out with the plan layout for (E, R, S).  Host only; returns a host status. */
int moe_plan_get_layout(int E, int R, int S, moe_plan_layout* out);

/* int32 words of the workspace moe_dispatch (and moe_dispatch_index,
 * moe_dispatch_capacity) needs for T tokens and E experts: a few words of status per
 * 256-token tile and two E-long count vectors per tile. */
int64_t moe_dispatch_workspace_words(int T, int E);

/* Static description of a host status code. */
const char* moe_status_string(int status);

/* ---------------------------------------------------------------------------------
 * (a) Router: top-k choice and gate weights.   [Primer] phase (a): the router scores
 * all experts per token, keeps the top-k and produces the routing table (token ->
 * experts plus combine weights).
 *   logits [T,E] fp32            router scores.
 *   idx    [T,k] int32  (out)    the k largest logits per token, descending; equal
 *                                logits are ordered by the lower expert id (+0 == -0).
 *   gate   [T,k] fp32   (out)    softmax over the k selected logits,
 *                                gate_j = exp(l_j - l_0) / sum_i exp(l_i - l_0).
 *   err    int32        (in/out) set to 0, then bit MOE_DERR_NONFINITE if any logit is
 *                                not finite (that token's outputs are unspecified).
 */
int moe_topk(const float* logits, int T, int E, int k,
             int32_t* idx, float* gate, int32_t* err, moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Router variant: bias-only balancing.   "MoE load balancing: 90/10 routing in
 * production" (interview page): DeepSeek-V3 balances with a per-expert bias kept outside
 * the gradient path, which moves the selection without distorting the gate.  The k
 * experts are chosen by the biased score s_e = logit_e + bias_e (one fp32 addition,
 * round-to-nearest), descending, equal scores by the lower expert id; the gates are the
 * softmax over the chosen experts' UNBIASED logits, in the chosen order.
 *   bias [E] fp32  per-expert selection bias (device).
 *   other arguments, outputs and err as moe_topk (a non-finite bias also sets
 *   MOE_DERR_NONFINITE).
 */
int moe_topk_biased(const float* logits, const float* bias, int T, int E, int k, int32_t* idx,
                    float* gate, int32_t* err, moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Demand histogram and imbalance.   [Hotspots] "Separate expert demand from rank
 * placement": count assignments per expert, then sum over an expert->rank mapping;
 * balancedness = mean/max.  [MoonEP] para. 2: maxvio is 0 when perfectly balanced,
 * here (max rank load - mean)/mean.  [Hotspots] "Work the 16-token hotspot fixture":
 * ids must be known experts and a token may not repeat one.
 *   idx            [T,k] int32        expert choices (e.g. from moe_topk).
 *   expert_to_rank [E] int32 or NULL  owning rank of each expert; NULL = e / (E/R).
 *                                     "If any expert is missing from a mapping, stop": an
 *                                     entry outside [0, R) sets MOE_DERR_ID_RANGE and that
 *                                     expert's demand is added to no rank.
 *   counts         [E] int32  (out)   assignments per expert (in-range ids only).
 *   loads          [R] int32  (out)   assignments per rank under the mapping.
 *   maxvio         [1] fp64   (out)   (R*max(loads) - T*k) / (T*k), one rounding;
 *                                     0 when T == 0.
 *   balancedness   [1] fp64   (out)   (T*k) / (R*max(loads)); 1 when T == 0.
 *   err            int32      (in/out) bits MOE_DERR_ID_RANGE, MOE_DERR_DUPLICATE; a
 *                                     no-op when already non-zero.  Every bit the trace
 *                                     deserves is set, counts/loads/maxvio/balancedness
 *                                     are still written, and none of them depends on the
 *                                     order in which the GPU runs its blocks.
 */
int moe_histogram_maxvio(const int32_t* idx, int T, int k, int E, int R,
                         const int32_t* expert_to_rank, int32_t* counts, int32_t* loads,
                         double* maxvio, double* balancedness, int32_t* err,
                         moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Fixed-capacity ledger.   [Hotspots] "Make expert capacity, overflow, and padding
 * explicit": per-expert capacity cap = ceil(A / E * cf), A = T*k assignments, with the
 * capacity factor given as the exact rational cf_num / cf_den (5/4 in the pages' example,
 * cap 5 for 32 assignments over 8 experts).  Per expert: processed = min(count, cap),
 * overflow = max(count - cap, 0), padding = max(cap - count, 0).  The ledger reports a
 * capacity mode; the layer path itself is dropless (no assignment is discarded).
 *   counts    [E] int32        expert demand (from moe_histogram_maxvio).
 *   processed, overflow, padding [E] int32 (out).
 *   totals    [4] int32 (out)  {cap, sum processed, sum overflow, sum padding}.
 *   err       no-op when non-zero.
 */
int moe_capacity_ledger(const int32_t* counts, int T, int k, int E, int cf_num, int cf_den,
                        int32_t* processed, int32_t* overflow, int32_t* padding,
                        int32_t* totals, const int32_t* err, moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Equal-load plan with redundant expert copies.   [MoonEP] para. 3-4: every rank
 * receives exactly the same number of tokens, by planning a few redundant expert copies
 * on the fly from the router output; copies live in S prefetch slots per rank drawn
 * from one process-global pool.  The article gives no algorithm; this one is
 * "keep small, stream the rest" (deterministic, scan-based):
 *   1. rank r owns experts [rB, (r+1)B), B = E/R; C = T*k/R;
 *   2. per rank, experts ordered by (count, id) ascending are kept whole while they fit
 *      in C; the first that does not fit and all after it are streamed;
 *   3. the streamed experts in id order form one stream; the ranks' leftover rooms,
 *      concatenated in rank order, cut it: each rank's piece fills its rows after its
 *      kept experts;
 *   4. each run of a foreign expert in a rank's piece is a replica taking the rank's
 *      next slot; more than S sets MOE_DERR_SLOTS.
 *   counts [E] int32   expert demand (from moe_histogram_maxvio).
 *   plan   int32[moe_plan_layout.words] (out)  the fields of moe_plan_layout.
 *   err    int32       (in/out) bit MOE_DERR_SLOTS; no-op when already non-zero.
 * One CTA; O(E*B + R*E) work.
 */
int moe_plan_balanced(const int32_t* counts, int T, int k, int E, int R, int S,
                      int32_t* plan, int32_t* err, moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Routing, histogram and plan fused: moe_topk (or moe_topk_biased when bias != NULL),
 * then moe_histogram_maxvio with the default home map (expert_to_rank = NULL), then
 * moe_plan_balanced, in one kernel launch (after a small one that zeroes err and the
 * workspace):
 * every block routes its tokens, counts the chosen ids in shared memory and adds its
 * counts to one of 16 partial histograms in the workspace (integer atomics); the last
 * block to finish sums them into counts and computes loads, maxvio, balancedness and the
 * plan.  Every
 * output equals the separate calls' bit for bit, including after a non-finite logit
 * (err = MOE_DERR_NONFINITE, counts and loads[0] zero, loads[1..R), maxvio,
 * balancedness and plan untouched) and after a slot overflow (MOE_DERR_SLOTS).
 *   logits [T,E] fp32; bias [E] fp32 or NULL; idx [T,k] int32, gate [T,k] fp32 (out);
 *   counts [E], loads [R] int32, maxvio, balancedness fp64 (out);
 *   plan int32[moe_plan_layout.words] (out); err int32 (out, reset to 0 first).
 *   workspace  int32[moe_route_plan_workspace_words(E)], caller-owned device scratch,
 *              any contents (zeroed by the call); one call at a time per workspace.
 * Shape rules and host statuses: those of the three calls.
 * moe_route_plan_workspace_words: words of that workspace, -1 for E outside [1, 1024].
 */
int64_t moe_route_plan_workspace_words(int E);
int moe_route_plan(const float* logits, const float* bias, int T, int E, int k, int R, int S,
                   int32_t* idx, float* gate, int32_t* counts, int32_t* loads, double* maxvio,
                   double* balancedness, int32_t* plan, int32_t* workspace, int32_t* err,
                   moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Prefetch of the replicas into the pool.   [MoonEP] para. 3: duplicated experts are
 * prefetched before computation from one process-global pool, not per layer; the
 * framework keeps one contiguous weight tensor per projection.
 *   W1, W3 [E,F,d] bf16, W2 [E,d,F] fp16     home expert weights.
 *   P1, P3 [R*S,F,d] bf16, P2 [R*S,d,F] fp16 (out) the pool; slot u*S+s receives a
 *          bitwise copy of expert replica_expert[u*S+s]; empty slots are not written.
 *          The pool is owned by the caller and may be shared by every layer.
 *          The copies run on the bulk-copy engine (32 KiB chunks staged in shared memory).
 *   err    no-op when non-zero; MOE_DERR_ID_RANGE if the plan lists a slot outside
 *          [0, R*S) or an expert outside [0, E) (that slot is skipped), MOE_DERR_TIMEOUT if
 *          a copy's bounded wait runs out.
 */
int moe_prefetch_replicas(const int32_t* plan, const moe_bf16* W1, const moe_bf16* W3,
                          const moe_f16* W2, int E, int R, int S, int d, int F,
                          moe_bf16* P1, moe_bf16* P3, moe_f16* P2, int32_t* err,
                          moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Zero-copy placement and dispatch.   [Primer] phase (b): every token is sent to its k
 * chosen experts (O(top-k) volume); [MoonEP] para. 3: tokens go straight to their final
 * row of a static-shape buffer.  Assignment (t,j) of expert e is the q-th assignment of
 * e in token order; a kept expert's q-th row is home(e)*C + expert_home_off[e] + q, a
 * streamed expert's is stream position p = stream_off[e] + q, on the rank u whose room
 * range holds p, row u*C + kept_rows[u] + p - room_prefix[u].
 *   x         [T,d] bf16      token rows.
 *   idx       [T,k] int32     expert choices (validated by moe_histogram_maxvio).
 *   workspace int32[moe_dispatch_workspace_words(T,E)]  scratch (caller-owned).
 *   recv      [R*C,d] bf16 (out)  recv[perm[t,j]] = x[t] bitwise.
 *   perm      [T,k] int32  (out)  row of each assignment.
 *   src       [R*C] int32  (out)  token of each row.
 *   err       no-op when non-zero.
 */
int moe_dispatch(const moe_bf16* x, const int32_t* idx, const int32_t* plan, int T, int k,
                 int E, int R, int S, int d, int32_t* workspace, moe_bf16* recv,
                 int32_t* perm, int32_t* src, int32_t* err, moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Grouped SwiGLU expert FFN.   [Primer] phase (c): each rank runs its local experts
 * over the rows it received as a batched grouped GEMM.  For every plan group (rows of
 * one rank holding one expert or replica):
 *   h = silu(X W1^T) * (X W3^T)   (bf16 x bf16, fp32 accumulate; silu(z) = z/(1+e^-z);
 *                                  stored as fp16, saturated to +-65504)
 *   y = h W2^T                    (fp16 x fp16, fp32 accumulate; bf16 out)
 * with the home tensors (weight_ref < E) or the pool slot (weight_ref >= E).  The down
 * projection runs in fp16 because a tensor-core MMA takes both operands in one type and
 * h rounded to bf16 (8 significant bits) leaves y's worst element near the 1e-2 parity
 * bound when F/d >= 2; fp16 holds 11 bits at the same rate.  bf16 weight values with
 * 2^-17 <= |w| <= 65504 convert to fp16 exactly.
 *   recv [R*C,d] bf16           rows from moe_dispatch.
 *   W1, W3 [E,F,d] bf16; W2 [E,d,F] fp16; P1, P3, P2 the pool (same types).
 *   h    [R*C,F] fp16 (out)     the SwiGLU activations (caller-owned scratch).
 *   y    [R*C,d] bf16 (out)     expert outputs.
 *   err  no-op when non-zero; MOE_DERR_TIMEOUT if a pipeline wait exceeded its bound.
 * Two persistent tcgen05/TMEM kernels fed by TMA.
 */
int moe_grouped_ffn(const moe_bf16* recv, const int32_t* plan, const moe_bf16* W1,
                    const moe_bf16* W3, const moe_f16* W2, const moe_bf16* P1,
                    const moe_bf16* P3, const moe_f16* P2, int T, int k, int E, int R,
                    int S, int d, int F, moe_f16* h, moe_bf16* y, int32_t* err,
                    moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Fused dispatch: the row copy folded into GEMM 1's operand load.   [MoonEP] para. 3
 * (zero-copy dispatch straight into the final static buffers) and [Primer], the second of
 * the three ideas it credits to DeepEP (routing layout and data movement fused into
 * dedicated GPU kernels): the rows a rank receives are read where they already are.
 *
 * moe_dispatch_index computes what moe_dispatch computes except recv: perm and src only
 * (same arguments minus x, d and recv; same errors).
 */
int moe_dispatch_index(const int32_t* idx, const int32_t* plan, int T, int k, int E, int R,
                       int S, int32_t* workspace, int32_t* perm, int32_t* src, int32_t* err,
                       moe_stream_t stream);
/*
 * moe_grouped_ffn_gather computes exactly what moe_grouped_ffn computes, bit for bit,
 * with GEMM 1's row r read as x[src[r]] instead of recv[r] (the same bf16 values), so no
 * [R*C,d] recv buffer is written or read.  The persistent GEMM-1 kernel's producer warp
 * gathers the rows with 16-byte copies into the swizzled operand tiles.
 *   x    [T,d] bf16             token rows (16-byte aligned).
 *   src  [R*C] int32            token of each row, from moe_dispatch_index (or
 *                               moe_dispatch).  An entry outside [0, T) sets
 *                               MOE_DERR_ID_RANGE (that row reads token 0 instead).
 *   other arguments, outputs and errors as moe_grouped_ffn.
 */
int moe_grouped_ffn_gather(const moe_bf16* x, const int32_t* src, const int32_t* plan,
                           const moe_bf16* W1, const moe_bf16* W3, const moe_f16* W2,
                           const moe_bf16* P1, const moe_bf16* P3, const moe_f16* P2, int T,
                           int k, int E, int R, int S, int d, int F, moe_f16* h, moe_bf16* y,
                           int32_t* err, moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Fused combine: the gate-weighted sum folded into GEMM 2's epilogue.   [Primer], the
 * third of the ideas it credits to DeepEP (the combine reduction fused into dedicated GPU
 * kernels), and phase (d): the expert outputs return to their token, summed with the gate
 * weights.  moe_grouped_ffn_combine computes moe_grouped_ffn followed by moe_combine
 * without writing y: GEMM 2's epilogue adds gate[t,j] * (h W2^T)_row, in fp32 straight from
 * the tensor-core accumulator, into out32[t] for the token t = src[row] and the choice j
 * with perm[t,j] == row (16-byte fp32 atomics), then out = bf16(out32).  The k
 * contributions of a token arrive in no fixed order, so out may differ from moe_combine's
 * j-ordered sum in the last bits (it also skips y's rounding to bf16); both are within the
 * combine's tolerance of the fp64 result.
 *   src [R*C], perm [T,k], gate [T,k] from moe_dispatch and the router; an src entry
 *   outside [0, T) sets MOE_DERR_ID_RANGE (that row is left out).
 *   out32 [T,d] fp32: caller-owned scratch, zeroed by the call.  out [T,d] bf16 (out).
 *   Other arguments, arithmetic and errors as moe_grouped_ffn (128-row tiles; the
 *   2-CTA tile mode does not apply).
 */
int moe_grouped_ffn_combine(const moe_bf16* recv, const int32_t* plan, const moe_bf16* W1,
                            const moe_bf16* W3, const moe_f16* W2, const moe_bf16* P1,
                            const moe_bf16* P3, const moe_f16* P2, const int32_t* src,
                            const int32_t* perm, const float* gate, int T, int k, int E, int R,
                            int S, int d, int F, moe_f16* h, float* out32, moe_bf16* out,
                            int32_t* err, moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Backward pass.   [MoonEP] para. 3: the duplicated experts' gradients are reduced back
 * home during the backward pass.  The pages give no formulas; these calls apply the
 * chain rule to the forward above, reading top-k selection as passing no gradient to the
 * experts it did not choose.  dout = dLoss/dout [T,d] bf16.  Same buffers, layouts and
 * error word as the forward; each call is a no-op when *err is non-zero.
 *
 * moe_combine_backward: dy[perm[t,j]] = gate[t,j] * dout[t] (bf16: its exponent range keeps
 *   the rows of small gates) and dgate[t,j] = <dout[t], y[perm[t,j]]> (fp32).
 *   dout [T,d] bf16; y [R*C,d] bf16 (forward output rows); dy [R*C,d] bf16 (out);
 *   dgate [T,k] fp32 (out).
 */
int moe_combine_backward(const moe_bf16* dout, const moe_bf16* y, const int32_t* perm,
                         const float* gate, int T, int k, int d, moe_bf16* dy, float* dgate,
                         const int32_t* err, moe_stream_t stream);
/*
 * moe_grouped_ffn_backward: for every plan group (rows of one rank, expert e; a replica
 * slot's rows use their expert's home weights, bitwise the same values):
 *   dH = dY W2,  dG = dH * u * silu'(g),  dU = dH * silu(g)   (g = X W1^T, u = X W3^T
 *   recomputed from recv), dX = dG W1 + dU W3;
 *   dW2[e] = sum over ALL groups of e (home and replica) of dY^T h, dW1[e] = sum dG^T X,
 *   dW3[e] = sum dU^T X -- replica gradients reduced home; experts without rows get 0.
 *   recv [R*C,d] bf16 (from moe_dispatch); dy [R*C,d] bf16 (moe_combine_backward);
 *   h [R*C,F] fp16: the forward's activations (from moe_grouped_ffn); not read (may be
 *   NULL): the SwiGLU-backward epilogue recomputes h = silu(g) u from the re-run gate/up
 *   GEMM and keeps it in bf16 for dW2.  W1, W3 [E,F,d] bf16; W2 [E,d,F] fp16.
 *   All GEMMs run in bf16 with fp32 accumulation: W2 is rounded to bf16 on the way into its
 *   transposed copy (exact for W2 values that are bf16 numbers).
 *   dx_rows [R*C,d] bf16 (out); dW1, dW3 [E,F,d] fp32 (out); dW2 [E,d,F] fp32 (out).
 *   workspace: caller-owned device scratch of moe_ffn_backward_workspace_bytes(...) bytes,
 *   256-byte aligned (W2 transposed in bf16, dH fp32, dG|dU and h bf16, the per-expert
 *   group lists).
 *   Returns MOE_ERR_ARG if workspace_bytes is too small.  Persistent tcgen05 kernels:
 *   dH, dG|dU (the gate/up GEMM re-run with a SwiGLU-backward epilogue), dX rows, and one
 *   weight-gradient GEMM per projection whose K loop runs over the rows of every group of
 *   the expert, 64 at a time, reading the row-major activations as MN-major operands.
 */
int64_t moe_ffn_backward_workspace_bytes(int T, int k, int E, int R, int S, int d, int F);
int moe_grouped_ffn_backward(const moe_bf16* recv, const moe_bf16* dy, const moe_f16* h,
                             const int32_t* plan, const moe_bf16* W1, const moe_bf16* W3,
                             const moe_f16* W2, int T, int k, int E, int R, int S, int d, int F,
                             moe_bf16* dx_rows, float* dW1, float* dW3, float* dW2,
                             void* workspace, int64_t workspace_bytes, int32_t* err,
                             moe_stream_t stream);
/*
 * moe_dispatch_backward: dx[t] = sum_j dx_rows[perm[t,j]] (fp32 accumulate, bf16 out).
 * moe_topk_backward: dlogits[t, idx[t,j]] = gate[t,j] (dgate[t,j] - sum_i gate[t,i]
 *   dgate[t,i]); every other entry of the row 0.  dlogits [T,E] fp32 (out).
 */
int moe_dispatch_backward(const moe_bf16* dx_rows, const int32_t* perm, int T, int k, int d,
                          moe_bf16* dx, const int32_t* err, moe_stream_t stream);
int moe_topk_backward(const float* gate, const float* dgate, const int32_t* idx, int T, int E,
                      int k, float* dlogits, const int32_t* err, moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Dispatch without a workspace argument.  The pages have no counterpart: this is a
 * convenience of this library for callers that cannot allocate device memory when they
 * dispatch -- an operator or plugin interface of another runtime that passes only its
 * input and output buffers, or a host program whose hot path must not call cudaMalloc
 * (which may synchronise the device).  It computes exactly what moe_dispatch computes,
 * with the same arguments minus `workspace`, and allocates nothing: the placement
 * counts live in a static device array of MOE_NOALLOC_SCRATCH_WORDS int32 words (2 MiB)
 * that every GPU loading the library holds until the process exits.
 *   - Returns MOE_ERR_SHAPE when moe_dispatch_workspace_words(T, E) exceeds
 *     MOE_NOALLOC_SCRATCH_WORDS (e.g. T = 65536 with E = 512 fits, with E = 1024 it does
 *     not; T = 32768 with E = 1024 fits).
 *   - The first call in each CUDA context of a device looks up the array's device
 *     address (cudaGetSymbolAddress, with that device current) and keeps it for that
 *     context; after a cudaDeviceReset the next call looks it up again.  Make the first
 *     call on a device before any stream capture.  MOE_ERR_DEVICE if the lookup fails.
 *   - All calls share the array and it keeps the last call's contents; each call clears
 *     the words it needs at zero itself.  Calls that overlap on the GPU (several streams or
 *     host threads on one device) race on it: serialise them.
 */
#define MOE_NOALLOC_SCRATCH_WORDS 524288
int moe_dispatch_noalloc(const moe_bf16* x, const int32_t* idx, const int32_t* plan, int T,
                         int k, int E, int R, int S, int d, moe_bf16* recv, int32_t* perm,
                         int32_t* src, int32_t* err, moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Fixed-capacity (dropping) mode.   [Hotspots] "Make expert capacity, overflow, and
 * padding explicit": each expert gets cap = ceil(A / E * cf) rows, the limit applied to
 * each expert independently; processed = min(demand, cap), overflow = max(demand - cap,
 * 0) (recorded before anything is excluded: moe_histogram_maxvio's counts and
 * moe_capacity_ledger), padding = max(cap - demand, 0) unused rows that still cost work.
 * Which assignments an expert keeps is not on the page: here its first cap assignments in
 * token order.  The layer path in this mode: moe_topk, moe_histogram_maxvio (raw demand),
 * moe_capacity_ledger, moe_dispatch_capacity, moe_grouped_ffn_capacity,
 * moe_combine_capacity.  (The default path above is dropless: zero drops, zero padding.)
 *
 * moe_capacity_rows: cap for T*k assignments over E experts at capacity factor
 *   cf_num / cf_den (an exact rational); -1 for a non-positive argument.  Host only.
 */
int64_t moe_capacity_rows(int T, int k, int E, int cf_num, int cf_den);
/*
 * moe_dispatch_capacity: expert e owns rows [e*cap, (e+1)*cap) of recv.  Assignment (t,j)
 * of expert e, the q-th of e in token order, goes to row e*cap + q when q < cap; otherwise
 * it overflows and is dropped (perm[t,j] = -1).  Rows e*cap + [min(counts[e], cap), cap)
 * are padding: zero rows in recv, src = -1.
 *   x [T,d] bf16; idx [T,k] int32; counts [E] int32 (expert demand of idx, from
 *   moe_histogram_maxvio); workspace int32[moe_dispatch_workspace_words(T, E)];
 *   recv [E*cap, d] bf16 (out); perm [T,k] int32 (out); src [E*cap] int32 (out).
 *   err  no-op when non-zero.
 */
int moe_dispatch_capacity(const moe_bf16* x, const int32_t* idx, const int32_t* counts, int T,
                          int k, int E, int cap, int d, int32_t* workspace, moe_bf16* recv,
                          int32_t* perm, int32_t* src, int32_t* err, moe_stream_t stream);
/*
 * moe_grouped_ffn_capacity: moe_grouped_ffn's SwiGLU expert over every row of every
 * expert's block (padding rows included: zeros in, zeros out), expert e's home weights on
 * rows [e*cap, (e+1)*cap).  recv [E*cap, d] bf16; W1, W3 [E,F,d] bf16; W2 [E,d,F] fp16;
 * h [E*cap, F] fp16 (out); y [E*cap, d] bf16 (out); arithmetic and errors as
 * moe_grouped_ffn.
 */
int moe_grouped_ffn_capacity(const moe_bf16* recv, const moe_bf16* W1, const moe_bf16* W3,
                             const moe_f16* W2, int E, int cap, int d, int F, moe_f16* h,
                             moe_bf16* y, int32_t* err, moe_stream_t stream);
/*
 * moe_combine_capacity: out[t] = sum over j with perm[t,j] >= 0 of gate[t,j] *
 * y[perm[t,j]] (fp32, j order; bf16 out): a dropped assignment adds nothing, a token with
 * every assignment dropped gets zeros.  Arguments as moe_combine.
 */
int moe_combine_capacity(const moe_bf16* y, const int32_t* perm, const float* gate, int T, int k,
                         int d, moe_bf16* out, const int32_t* err, moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Combine.   [Primer] phase (d): expert outputs return to their token and are summed
 * with the gate weights; the mirror (transpose) of dispatch.
 *   out[t] = sum_{j=0..k-1} gate[t,j] * y[perm[t,j]]   (fp32, j order; bf16 out)
 *   y [R*C,d] bf16, perm [T,k] int32, gate [T,k] fp32, out [T,d] bf16 (out).
 *   err  no-op when non-zero.
 *   perm must be the output of a moe_dispatch (or moe_dispatch_index) that left *err at
 *   0: its rows are not range-checked again here (the call has no R*C argument), and a
 *   perm from elsewhere must hold rows in [0, rows of y).
 */
int moe_combine(const moe_bf16* y, const int32_t* perm, const float* gate, int T, int k,
                int d, moe_bf16* out, const int32_t* err, moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Expert parallelism across GPUs: one process per GPU, rank `me` of W.   [MoonEP]
 * paragraphs 2-3: every rank receives exactly T*k/R rows under a plan computed on the fly
 * from the router output; [Primer] phases (b) dispatch and (d) combine are the two
 * all-to-all exchanges between the ranks.  Here the plan's R is W: rank u owns the home
 * experts [u*B, (u+1)*B), B = E/W, holds S pool slots, and every rank holds the same
 * number T of tokens.  The job's token order is rank-major (rank u's token t is job token
 * u*T + t), so the job computes the single-GPU layer of the concatenated batch with
 * R = W: the same plan, and rank u's receive buffer holds rows [u*C, (u+1)*C) of it,
 * C = T*k (the job's W*T*k rows over W ranks).
 *
 * One step on rank me:
 *   moe_topk (own logits) -> moe_ep_counts -> [all-gather of the (E+1)-word vectors] ->
 *   moe_ep_plan -> moe_ep_prefetch -> moe_ep_dispatch -> [barrier] -> moe_ep_grouped_ffn
 *   -> [barrier] -> moe_ep_combine.
 * The exchange and the barriers are the caller's (an NCCL all-gather and a one-word
 * all-reduce on the same stream order the ranks): every rank's dispatch must have
 * finished before any rank's FFN reads its receive buffer, every FFN before any combine
 * reads y, and every combine before the next step's FFN overwrites y (the next step's
 * all-gather orders that, and the dispatch of the next step after every FFN).
 *
 * Pointer tables: the arguments named *_ranks are HOST arrays of W device pointers, one
 * per rank in rank order, each that rank's buffer as addressed from THIS process (this
 * rank's own buffer at index me, a peer GPU's buffer mapped into this process -- e.g. by
 * moe_ipc_import -- elsewhere).  The library reads the tables when the call enqueues (they
 * are passed to the kernels by value; a captured graph keeps them).  Peer buffers are
 * written with plain 16-byte stores (dispatch) and read with plain 16-byte loads
 * (prefetch, combine) over NVLink; no call uses TMA multicast.
 *
 * Sizes: 1 <= W <= MOE_EP_MAX_RANKS, 0 <= me < W, E % W == 0, W*T*k < 2^31, and the
 * per-call limits of the single-GPU calls with R = W and T*k local rows.
 */
#define MOE_EP_MAX_RANKS 64

/*
 * moe_ep_counts: this rank's demand and error word, packed for the exchange.
 *   idx  [T,k] int32   this rank's top-k ids.
 *   err  int32 (in)    this rank's error word (set by moe_topk).
 *   send [E+1] int32 (out, device)  send[e] = assignments of this rank's tokens naming e
 *                      (ids in range only); send[E] = *err | MOE_DERR_ID_RANGE (an id
 *                      outside [0, E)) | MOE_DERR_DUPLICATE (a token repeating an id).
 *                      *err itself is not written: the bits reach every rank through
 *                      the exchanged vectors (moe_ep_plan).  With *err != 0 on entry,
 *                      send = {0, ..., 0, *err}.
 */
int moe_ep_counts(const int32_t* idx, int T, int k, int E, const int32_t* err, int32_t* send,
                  moe_stream_t stream);

/*
 * moe_ep_plan: the job's demand, this rank's base offsets and the plan (the same on every
 * rank, bit for bit, since every rank reads the same vectors).
 *   gathered [W][E+1] int32   every rank's send vector in rank order (the all-gather).
 *   T        tokens per rank.
 *   err      (in/out) |= the OR of every rank's send[E]; when that is non-zero nothing
 *            else is written (on every rank alike, so the ranks stop together).
 *   counts   [E] int32 (out)  the job's demand (sum over the ranks).
 *   q_base   [E] int32 (out)  assignments of expert e made by the ranks below me (the
 *                             position of this rank's first e-assignment in e's order).
 *   loads [W] int32, maxvio, balancedness (fp64, device) (out)  as moe_histogram_maxvio
 *            with R = W, the home map and A = W*T*k.
 *   plan     int32 buffer of moe_plan_get_layout(E, W, S) (out), as moe_plan_balanced on
 *            the job's demand with T_job = W*T; MOE_DERR_SLOTS as there.
 */
int moe_ep_plan(const int32_t* gathered, int W, int me, int T, int k, int E, int S,
                int32_t* counts, int32_t* q_base, int32_t* loads, double* maxvio,
                double* balancedness, int32_t* plan, int32_t* err, moe_stream_t stream);

/*
 * moe_ep_prefetch: this rank's pool slots receive their experts' weights from the home
 * ranks (a peer copy into local memory before any FFN reads them).
 *   W1_ranks, W3_ranks (moe_bf16, each [B,F,d]), W2_ranks (moe_f16, each [B,d,F]): HOST
 *            tables of every rank's home tensors (see "Pointer tables").
 *   P1, P3 [S,F,d] bf16, P2 [S,d,F] fp16 (out): this rank's slots; slot s receives
 *            expert e = replica_expert[me*S + s] (local expert e % B of rank e / B),
 *            bitwise; empty slots are untouched.  Bulk copies (no multicast) staged in
 *            this GPU's shared memory, as moe_prefetch_replicas.
 *   err  no-op when non-zero; MOE_DERR_ID_RANGE if a slot names an expert outside
 *        [0, W*B) (that slot is skipped), MOE_DERR_TIMEOUT if a copy's bounded wait runs out.
 */
int moe_ep_prefetch(const int32_t* plan, const moe_bf16* const* W1_ranks,
                    const moe_bf16* const* W3_ranks, const moe_f16* const* W2_ranks, int W,
                    int me, int E, int S, int d, int F, moe_bf16* P1, moe_bf16* P3, moe_f16* P2,
                    int32_t* err, moe_stream_t stream);

/*
 * moe_ep_dispatch: every assignment of this rank's tokens straight into its final row on
 * the rank that processes it.
 *   x [T,d] bf16, idx [T,k]: this rank's tokens and ids; q_base from moe_ep_plan.
 *   workspace  moe_dispatch_workspace_words(T, E) int32 words.
 *   recv_ranks HOST table of every rank's receive buffer [C,d] bf16, C = T*k.
 *   perm [T,k] int32 (out): the job-wide row of each assignment (rank perm / C, local
 *        row perm % C): the rows moe_dispatch assigns to these tokens in the
 *        concatenated batch.  Row perm receives x[t] bitwise.
 *   err  no-op when non-zero; MOE_DERR_ID_RANGE, MOE_DERR_TIMEOUT as moe_dispatch.
 */
int moe_ep_dispatch(const moe_bf16* x, const int32_t* idx, const int32_t* q_base,
                    const int32_t* plan, int W, int T, int k, int E, int S, int d,
                    int32_t* workspace, moe_bf16* const* recv_ranks, int32_t* perm,
                    int32_t* err, moe_stream_t stream);

/*
 * moe_ep_grouped_ffn: the grouped SwiGLU FFN over this rank's C rows and groups.
 *   recv [C,d] bf16: this rank's receive buffer; W1, W3 [B,F,d] bf16 and W2 [B,d,F] fp16:
 *   its home experts; P1, P3, P2: its pool (as moe_ep_prefetch).
 *   groups_ws [4*(B+S)] int32 (device scratch): the rank's group table re-based to local
 *   rows and local weights (row_start - me*C; expert e -> e - me*B; slot -> B + s).
 *   h [C,F] fp16, y [C,d] bf16 (out): as moe_grouped_ffn, row for row the rows
 *   [me*C, (me+1)*C) of the single-GPU layer's h and y.
 *   err  no-op when non-zero; MOE_DERR_TIMEOUT as moe_grouped_ffn, MOE_DERR_ID_RANGE if a
 *   group of this rank names weights that are not on it (never, for a plan of moe_ep_plan).
 */
int moe_ep_grouped_ffn(const moe_bf16* recv, const int32_t* plan, int W, int me,
                       const moe_bf16* W1, const moe_bf16* W3, const moe_f16* W2,
                       const moe_bf16* P1, const moe_bf16* P3, const moe_f16* P2, int T, int k,
                       int E, int S, int d, int F, int32_t* groups_ws, moe_f16* h, moe_bf16* y,
                       int32_t* err, moe_stream_t stream);

/*
 * moe_ep_combine: out[t] = sum_j gate[t,j] * y_{perm[t,j] / C}[perm[t,j] % C] (fp32, j
 * order; bf16 out), C = T*k: the same sums as moe_combine over the single-GPU layer.
 *   y_ranks  HOST table of every rank's y [C,d] bf16.
 *   perm, gate [T,k] of this rank (perm from moe_ep_dispatch with *err left at 0).
 *   out [T,d] bf16 (out).  err  no-op when non-zero.
 */
int moe_ep_combine(const moe_bf16* const* y_ranks, const int32_t* perm, const float* gate,
                   int W, int T, int k, int d, moe_bf16* out, const int32_t* err,
                   moe_stream_t stream);

/*
 * Backward of the expert-parallel layer.   [MoonEP] paragraph 3: the duplicated experts'
 * gradients are reduced back home during the backward pass -- here across GPUs.  One
 * backward step on rank me, after its forward:
 *   moe_ep_combine_backward -> [barrier] -> moe_ep_grouped_ffn_backward -> [barrier] ->
 *   moe_ep_reduce_home, moe_ep_dispatch_backward -> moe_topk_backward (local).
 * The results equal the single-GPU backward of the concatenated batch (moe_combine_backward,
 * moe_grouped_ffn_backward, moe_dispatch_backward with R = W): dx, dlogits and the rows bit
 * for bit; a home expert's weight gradient sums the same products, in a different order
 * (its own groups in one accumulator, then each copy's partial in fp32).
 *
 * moe_ep_combine_backward: for this rank's assignment (t, j) with row r = perm[t,j] on rank
 *   v = r / C (C = T*k): v's dy[r % C] = gate[t,j] * dout[t] (bf16, a peer store) and
 *   dgate[t,j] = <dout[t], y_v[r % C]> (fp32, peer loads).
 *   dout [T,d] bf16; y_ranks, dy_ranks: HOST tables of every rank's y and dy [C,d] bf16;
 *   perm, gate [T,k] from the forward; dgate [T,k] fp32 (out).  err  no-op when non-zero.
 */
int moe_ep_combine_backward(const moe_bf16* dout, const moe_bf16* const* y_ranks,
                            const int32_t* perm, const float* gate, int W, int T, int k, int d,
                            moe_bf16* const* dy_ranks, float* dgate, const int32_t* err,
                            moe_stream_t stream);
/*
 * moe_ep_grouped_ffn_backward: the grouped-FFN backward over this rank's C rows and its
 *   re-based groups (as moe_ep_grouped_ffn: home experts from W1, W3, W2 [B,...], replicas
 *   from its pool slots P1, P3, P2 [S,...]).
 *   recv, dy [C,d] bf16: this rank's rows and their gradients.
 *   dx_rows [C,d] bf16 (out).
 *   dP1, dP3 [B+S,F,d], dP2 [B+S,d,F] fp32 (out): the weight gradients of this rank's
 *   groups -- entry b < B its home expert me*B + b, entry B + s its pool slot s (the
 *   partial that moe_ep_reduce_home adds to the slot's home expert); entries without rows
 *   are 0.
 *   groups_ws [4*(B+S)] int32 scratch; workspace of moe_ep_ffn_backward_workspace_bytes
 *   bytes, 256-byte aligned.  Requires B + S <= 1024.  MOE_ERR_ARG if workspace_bytes is
 *   too small.  err  no-op when non-zero.
 * moe_ep_ffn_backward_workspace_bytes: that size, or -1 for an invalid shape.
 */
int64_t moe_ep_ffn_backward_workspace_bytes(int T, int k, int E, int W, int S, int d, int F);
int moe_ep_grouped_ffn_backward(const moe_bf16* recv, const moe_bf16* dy, const int32_t* plan,
                                int W, int me, const moe_bf16* W1, const moe_bf16* W3,
                                const moe_f16* W2, const moe_bf16* P1, const moe_bf16* P3,
                                const moe_f16* P2, int T, int k, int E, int S, int d, int F,
                                int32_t* groups_ws, moe_bf16* dx_rows, float* dP1, float* dP3,
                                float* dP2, void* workspace, int64_t workspace_bytes,
                                int32_t* err, moe_stream_t stream);
/*
 * moe_ep_reduce_home: in place on this rank's partials (dP*_ranks[me]): entry b, the
 *   gradient of home expert e = me*B + b, gets, for every pool slot (v, s) of the plan that
 *   held a copy of e and in (v, s) order, rank v's entry B + s added (peer loads, fp32);
 *   experts without copies are left as they are.  Afterwards entries 0..B-1 of this rank's
 *   dP1, dP3 [B+S,F,d] and dP2 [B+S,d,F] are its home experts' weight gradients.  No rank may
 *   run this before every rank's moe_ep_grouped_ffn_backward has finished, nor start its next
 *   backward before every rank's moe_ep_reduce_home has finished (a rank reads its peers'
 *   slot entries).
 *   dP1_ranks, dP3_ranks, dP2_ranks: HOST tables of every rank's dP1, dP3, dP2.
 *   err  no-op when non-zero.
 */
int moe_ep_reduce_home(const int32_t* plan, float* const* dP1_ranks, float* const* dP3_ranks,
                       float* const* dP2_ranks, int W, int me, int E, int S, int d, int F,
                       const int32_t* err, moe_stream_t stream);
/*
 * moe_ep_dispatch_backward: dx[t] = sum_j dx_rows_v[perm[t,j] % C], v = perm[t,j] / C
 *   (fp32 in j order, bf16 out; peer loads).  dx_rows_ranks: HOST table of every rank's
 *   dx_rows [C,d] bf16; dx [T,d] bf16 (out).  err  no-op when non-zero.
 */
int moe_ep_dispatch_backward(const moe_bf16* const* dx_rows_ranks, const int32_t* perm, int W,
                             int T, int k, int d, moe_bf16* dx, const int32_t* err,
                             moe_stream_t stream);

/*
 * Device-memory sharing between the processes of one node (CUDA IPC), for the pointer
 * tables above.  Host calls; nothing is enqueued.
 * moe_ipc_export: handle (host buffer of MOE_IPC_HANDLE_BYTES) names the allocation that
 *   holds the device pointer ptr; *offset = ptr - the allocation's base.  MOE_ERR_ARG for
 *   a null argument, MOE_ERR_DEVICE if the runtime refuses (not a device allocation, or
 *   one that cannot be shared).
 * moe_ipc_import: maps another process's exported allocation into this one (peer access
 *   enabled on first use); *ptr = base + offset, *base = the mapping to close later.  A
 *   process cannot import its own export (MOE_ERR_DEVICE): it uses its own pointer.
 * moe_ipc_close: unmaps a base returned by moe_ipc_import.
 */
#define MOE_IPC_HANDLE_BYTES 64
int moe_ipc_export(const void* ptr, void* handle, int64_t* offset);
int moe_ipc_import(const void* handle, int64_t offset, void** ptr, void** base);
int moe_ipc_close(void* base);

/* ---------------------------------------------------------------------------------
 * moe_w2_to_f16: the fp16 copy of a bf16 down projection that moe_prefetch_replicas,
 * moe_grouped_ffn and the other FFN calls take (GEMM 2 runs with h and W2 both fp16; one
 * tcgen05 MMA takes one operand type).  A caller holding bf16 weights ([MoonEP] para. 3:
 * one contiguous tensor per projection) converts W2 once per weight version, not per step.
 *   w2_bf16 [n] (any shape, e.g. [E,d,F]) bf16 -> w2_f16 [n] fp16 (out), round to nearest
 *   even: 0 and every bf16 value with 2^-17 <= |w| <= 65504 convert exactly (below 2^-14 as
 *   fp16 subnormals); smaller values round to the subnormal grid (spacing 2^-24), larger
 *   ones become +-inf.  n % 8 == 0, both 16-byte aligned.  No error word: a weight
 *   preparation step, not part of a layer's step.
 */
int moe_w2_to_f16(const moe_bf16* w2_bf16, int64_t n, moe_f16* w2_f16, moe_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Grouped-FFN tile mode (a B200 tiling choice; the pages fix no kernel design).
 *   0  one CTA per 128-row x N tile (tcgen05.mma.cta_group::1), the default.
 *   1  CTA pairs (2-CTA clusters) on 256-row x N tiles (tcgen05.mma.cta_group::2): each
 *      SM loads its 128 rows of A and half of B, a third fewer operand bytes per MAC at
 *      N = 256, at the price of padding each group's last tile to 256 rows.
 * Process-wide, read when moe_grouped_ffn enqueues its kernels (set it before capturing a
 * graph); moe_grouped_ffn_gather always uses mode 0.  Both modes compute the same sums in
 * the same K order: their h and y were bit-identical on every shape tested, and both stay
 * within the FFN tolerance of the oracle.
 * moe_set_ffn_tile_mode returns MOE_OK, or MOE_ERR_ARG (mode unchanged) for a mode other
 * than 0 or 1; moe_ffn_tile_mode returns the current mode.
 * moe_ffn_pair_clusters: 2-CTA clusters mode 1 launches per GEMM on the current device
 * (as many as fit at once), 0 before its first launch.
 */
int moe_set_ffn_tile_mode(int mode);
int moe_ffn_tile_mode(void);
int moe_ffn_pair_clusters(void);

/* ---------------------------------------------------------------------------------
 * Diagnostic (no counterpart in the pages): runs the grouped FFN's bounded mbarrier wait
 * on a barrier that nothing ever arrives at, with a limit of `limit_us` microseconds
 * (1 .. 10^7).  The wait gives up, ORs MOE_DERR_TIMEOUT into *err and the kernel returns;
 * the CUDA context stays usable.  Lets a caller check the timeout path without faulting or
 * hanging a GPU.
 */
int moe_selftest_bounded_wait(int32_t* err, int limit_us, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
