/*
 * moe_b200.h - C ABI of the token-choice Mixture-of-Experts forward pass on
 * NVIDIA B200 (sm_100a).
 *
 * The layer (page "Lab 18 - Mixture of experts", section 1):
 *     z = x W_r,  p = softmax(z),  y = sum over top-k(p) of g_i FFN_i(x)
 * plus the capacity limit of section 3, the balancing losses of section 2 and
 * shared experts that run on every token.  Each stage is one call; moe_forward
 * runs them all.
 *
 * Conventions for every call:
 *   - Pointers named x, W*, y, ... are DEVICE pointers unless marked "host".
 *     The caller allocates every buffer (including the workspace); the library
 *     never allocates, frees or synchronises.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is asynchronous to the host.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid call returns a status and launches nothing.  A failed launch
 *     returns MOE_ERR_CUDA.
 *   - Row-major layouts throughout.  "dtype" is the activation / expert-weight
 *     storage type chosen by moe_config.dtype: fp32, or bf16 (2-byte).  The
 *     router weights, biases, gates and losses are always fp32.
 *   - T = tokens, d = model dim, E = routed experts, k = experts per token,
 *     F = expert hidden dim (d_ff), S = shared experts, Fs = their hidden dim.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *moe_stream_t; /* same type as cudaStream_t */

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_NULL = 1,            /* a required pointer is NULL */
    MOE_ERR_SHAPE = 2,           /* T < 0, d < 1, k < 1, k > E, E > 256, k > 8, ... */
    MOE_ERR_CAPACITY_FACTOR = 3, /* capacity_factor < 1.0 or NaN ("Lab 01" traps) */
    MOE_ERR_ALIGN = 4,           /* a pointer or row pitch breaks the 16-byte rule */
    MOE_ERR_WORKSPACE = 5,       /* workspace smaller than the size query says */
    MOE_ERR_DTYPE = 6,           /* unknown dtype / activation / score code */
    MOE_ERR_CUDA = 7,            /* a CUDA launch or attribute call failed */
    MOE_ERR_DEVICE_TIMEOUT = 8   /* a kernel's bounded wait ran out (see moe_device_status) */
} moe_status;

enum { MOE_ACT_GELU = 0, MOE_ACT_SWIGLU = 1 };
enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 };
enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 };
enum { MOE_PRIORITY_TOKEN = 0, MOE_PRIORITY_RANK = 1, MOE_PRIORITY_SCORE = 2 };

/* Every expert's segment of the permuted row buffers starts on a multiple of
 * this many rows (the expert GEMM's M tile). */
#define MOE_ROW_ALIGN 128

/*
 * One layer's shape and options.
 *   act      MOE_ACT_GELU: two-matrix expert W2 gelu(W1 x), exact erf GELU;
 *            MOE_ACT_SWIGLU: three-matrix W2 (silu(W1 x) * (W3 x))
 *            ("Lab 18" section 1, expert description).
 *   score    MOE_SCORE_SOFTMAX, or MOE_SCORE_SIGMOID (DeepSeek-V3 note of
 *            "Lab 18" section 1; selection may add a per-expert bias).
 *   renorm   -1: renormalize the gates over the selected experts exactly when
 *            k > 1 (raw p for k = 1, "Lab 18" section 1 gate values); 0: raw;
 *            1: renormalized.
 *   dtype    MOE_DTYPE_F32 or MOE_DTYPE_BF16 for x, y and all expert weights.
 *   priority order in which assignments claim expert slots: token order, first
 *            come first served ("Lab 01", where to start step 4), rank-major
 *            (every first choice before any second, "Lab 18" section 3), or
 *            MOE_PRIORITY_SCORE, batch-prioritized: highest router score first
 *            (V-MoE, "Lab 18" section 3; see moe_capacity_scored).
 *   capacity_factor  C = ceil(capacity_factor * T * k / E) slots per expert
 *            ("Lab 18" section 3); +infinity = no limit.  Must be >= 1.0.
 * Limits: 1 <= k <= min(E, 8), E <= 256.  bf16 needs d, d_ff, d_ff_shared
 * multiples of 64.
 */
typedef struct moe_config {
    int32_t T, d, E, k, d_ff, n_shared, d_ff_shared;
    int32_t act, score, renorm, dtype, priority;
    double capacity_factor;
} moe_config;

/* Weights of one layer (device pointers, dtype unless noted).
 *   W_r [d, E] fp32 router ("Lab 18" section 1: z = x W_r; routers stay fp32,
 *       cs336 lecture 4, "Stability, fine-tuning, and upcycling").
 *   logit_bias [E] fp32, nullable: added to every token's logits.
 *   select_bias [E] fp32, nullable, sigmoid scores only: added to the scores
 *       used to pick the top k, never to the gates ("Lab 18" section 2,
 *       auxiliary-loss-free balancing).
 *   W1, W3 [E, F, d] (W3 only for SwiGLU), W2 [E, d, F]: hidden = W1 x, output
 *       = W2 hidden (row f of W1[e] holds hidden unit f's input weights).
 *   Ws1, Ws3 [S, Fs, d], Ws2 [S, d, Fs]: shared experts, NULL when S = 0. */
typedef struct moe_weights {
    const float *W_r;
    const float *logit_bias;
    const float *select_bias;
    const void *W1, *W3, *W2;
    const void *Ws1, *Ws3, *Ws2;
} moe_weights;

/* Outputs of moe_forward (device pointers).  y, aux and zloss are required;
 * every other field may be NULL, in which case the value lives only in the
 * workspace.
 *   y [T, d] dtype          the layer output; the residual x + y is the
 *                           caller's ("Lab 18", GPU scale-up listing)
 *   topk_idx [T, k] int32   experts of each token, best first
 *   gates [T, k] fp32
 *   keep [T, k] uint8       1 = the assignment got a slot
 *   dropped [T] uint8       1 = every assignment of the token was dropped
 *   counts [E] int32        assignments per expert before capacity
 *   n_dropped [1] int32     dropped assignments
 *   aux, zloss [1] fp32     unweighted L_aux and L_z ("Lab 18" section 2) */
typedef struct moe_outputs {
    void *y;
    int32_t *topk_idx;
    float *gates;
    uint8_t *keep;
    uint8_t *dropped;
    int32_t *counts;
    int32_t *n_dropped;
    float *aux;
    float *zloss;
} moe_outputs;

/* Human-readable text of a status code (static storage). */
const char *moe_status_string(moe_status s);

/* Validate a configuration (shape limits, codes, capacity factor). */
moe_status moe_validate(const moe_config *cfg);

/* C = ceil(capacity_factor * T * k / E), computed in double on the host in
 * exactly that order of operations, held at T when it exceeds T (an expert
 * receives at most T assignments, so that changes no decision); T when the
 * factor is +infinity ("Lab 18" section 3).  Writes *C (host). */
moe_status moe_capacity_value(const moe_config *cfg, int64_t *C);

/* Rows the caller must allocate for the permuted buffers x_perm and Y_perm:
 * min(T*k, E*C) kept assignments plus per-expert padding to MOE_ROW_ALIGN.
 * Returns -1 for an invalid configuration. */
int64_t moe_perm_rows(const moe_config *cfg);

/* Number of fp32 values moe_route writes to loss_partials. */
int64_t moe_loss_partials_count(const moe_config *cfg);

/* Scratch bytes the stage calls need (moe_route, moe_capacity,
 * moe_expert_ffn).  One workspace serves all of them, one call at a time. */
size_t moe_stage_workspace_size(const moe_config *cfg);

/* Workspace bytes moe_forward needs (includes the stage scratch).  0 for an
 * invalid configuration. */
size_t moe_workspace_size(const moe_config *cfg);

/*
 * moe_route - router, scores, top-k and gates ("Lab 18" section 1 and the
 * route() row of "What to implement"; router listing of "Mixture of Experts -
 * parameters without the FLOPs", section 2).
 *   x [T, d] dtype; W_r [d, E] fp32; logit_bias / select_bias as in moe_weights.
 *   topk_idx [T, k] int32 out: the k experts with the largest selection key,
 *     best first, equal keys to the lower index ("Lab 01" traps).  The key is
 *     the logit for softmax scores (the same order as p) and s + select_bias
 *     for sigmoid scores.
 *   gates [T, k] fp32 out: p or s of the selected experts, renormalized over
 *     them when cfg->renorm says so.
 *   loss_partials [moe_loss_partials_count] fp32 out: per token block, the sum
 *     of each expert's probability (sigmoid: s / sum s) and of lse^2, summed
 *     by moe_losses in a fixed order.
 *   logits_out [T, E] fp32, nullable: the router logits z.
 *   scores_out [T, E] fp32, nullable: p (softmax) or s (sigmoid).
 *   ws: scratch of at least moe_stage_workspace_size bytes, 256-byte aligned;
 *     its first word is the device status word (cleared by this call).
 * Logits are fp32: for bf16 x the tensor cores compute x W_hi + x W_mid +
 * x W_lo, where hi + mid + lo is an exact three-term bf16 split of each fp32
 * weight, so every product is exact and the sum accumulates in fp32; fp32 x
 * uses fp32 FMAs.  A wait that times out sets MOE_ERR_DEVICE_TIMEOUT in the
 * status word (see moe_device_status); the routing is then not valid.
 */
moe_status moe_route(const moe_config *cfg, const void *x, const float *W_r,
                     const float *logit_bias, const float *select_bias,
                     int32_t *topk_idx, float *gates, float *loss_partials,
                     float *logits_out, float *scores_out, void *ws, size_t ws_bytes,
                     moe_stream_t stream);

/*
 * moe_capacity - slot assignment under the capacity limit ("Lab 18" section 3;
 * "Lab 01", where to start step 4).  Bit-exact with a sequential walk over the
 * assignments in priority order that gives each one position = (number of
 * earlier assignments to the same expert) and keeps it while position < C.
 *   topk_idx [T, k] int32 in.
 *   counts [E] int32 out: assignments per expert before capacity.
 *   pos [T, k] int32 out: queue position of each assignment in its expert.
 *   keep [T, k] uint8 out: pos < C.
 *   kept [E] int32 out: min(counts, C).
 *   offsets [E + 1] int32 out: first row of each expert's segment in the
 *     permuted buffers; offsets[e + 1] - offsets[e] = kept[e] rounded up to
 *     MOE_ROW_ALIGN; offsets[E] = rows used.
 *   dropped [T] uint8 out: 1 when every slot of the token was dropped.
 *   n_dropped [1] int32 out: number of dropped assignments.
 *   ws: scratch of at least moe_stage_workspace_size bytes, 256-byte aligned.
 * Returns MOE_ERR_CAPACITY_FACTOR for capacity_factor < 1 ("Lab 01" traps),
 * MOE_ERR_DTYPE for MOE_PRIORITY_SCORE (that order needs the router scores:
 * moe_capacity_scored).
 */
moe_status moe_capacity(const moe_config *cfg, const int32_t *topk_idx,
                        int32_t *counts, int32_t *pos, uint8_t *keep,
                        int32_t *kept, int32_t *offsets, uint8_t *dropped,
                        int32_t *n_dropped, void *ws, size_t ws_bytes,
                        moe_stream_t stream);

/*
 * moe_capacity_sharded - moe_capacity for one shard of a batch split across
 * data-parallel ranks in token order (rank r holds the tokens after those of
 * ranks 0..r-1), keeping the capacity of the whole batch ("Lab 18" section 3:
 * C per expert per batch, first come first served in token order).
 *   capacity: C of the whole batch (moe_capacity_value of its config).
 *   shard_counts [n_shards][E] int32 in (device): every shard's assignments
 *     per expert (moe_capacity's counts, all-gathered in rank order); this
 *     shard is number `shard`.  The library sums the rows before it:
 *     count_base[e] = sum_{r < shard} shard_counts[r][e].
 *   cfg: this shard's shape; priority must be MOE_PRIORITY_TOKEN (else
 *     MOE_ERR_DTYPE: the other orders are not a prefix over shards).
 *   Outputs as for moe_capacity, for this shard: counts = its assignments per
 *   expert; pos = place in this shard's segment of the expert; keep = 1 while
 *   count_base[e] + pos < capacity; kept = min(counts, max(0, capacity -
 *   count_base)); offsets, dropped and n_dropped follow.  With one shard and
 *   capacity = moe_capacity_value(cfg) the results equal moe_capacity's.
 *   Returns MOE_ERR_SHAPE for capacity < 0 or shard outside [0, n_shards).
 */
moe_status moe_capacity_sharded(const moe_config *cfg, int64_t capacity,
                                const int32_t *shard_counts, int32_t n_shards,
                                int32_t shard, const int32_t *topk_idx,
                                int32_t *counts, int32_t *pos, uint8_t *keep,
                                int32_t *kept, int32_t *offsets, uint8_t *dropped,
                                int32_t *n_dropped, void *ws, size_t ws_bytes,
                                moe_stream_t stream);

/*
 * moe_capacity_scored - moe_capacity in batch-prioritized order ("Lab 18"
 * section 3: V-MoE ranks the assignments by router score).  The walk takes the
 * T*k assignments from the highest router score of the selected expert down;
 * equal scores go in token order, then slot order.  cfg->priority must be
 * MOE_PRIORITY_SCORE (else MOE_ERR_DTYPE).
 *   scores [T, E] fp32 in: the router scores, as moe_route writes them to
 *     scores_out (softmax p, or sigmoid s without the selection bias); the
 *     score of assignment (t, j) is scores[t, topk_idx[t, j]], compared as
 *     fp32 (-0 equals +0; NaN scores give an unspecified order).
 *   Every other argument as for moe_capacity; counts, kept, offsets and
 *   n_dropped do not depend on the order.
 *   ws: moe_stage_workspace_size bytes of a config with this priority (it
 *     holds 8 T k bytes of sort keys).
 */
moe_status moe_capacity_scored(const moe_config *cfg, const int32_t *topk_idx,
                               const float *scores, int32_t *counts, int32_t *pos,
                               uint8_t *keep, int32_t *kept, int32_t *offsets,
                               uint8_t *dropped, int32_t *n_dropped, void *ws,
                               size_t ws_bytes, moe_stream_t stream);

/*
 * moe_capacity_noalloc - moe_capacity with its scratch inside the library.
 * The pages have no counterpart: this entry point exists for callers that
 * cannot allocate device memory where they run the capacity step (memory
 * planned once at start-up that may not grow, or device memory owned by
 * another allocator that must not be bypassed).  The caller still allocates
 * and passes every input and output; the arguments mean what they mean for
 * moe_capacity, and the results are identical to it.
 *   - The scratch is a file-scope device array of 256 KiB (one table of
 *     65536 int32), held by every GPU that loads the library until the process
 *     exits.  Shapes that need more, ceil(T / 256) * k * E > 65536, return
 *     MOE_ERR_WORKSPACE and launch nothing.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make
 *     that first call before any stream capture.  The cached address is not
 *     refreshed: cudaDeviceReset after the first call on a device is not
 *     supported for this entry point.
 *   - No cudaMalloc, cudaFree or other allocating call is made.
 *   - All calls share the one array: calls whose work overlaps on the GPU
 *     (other streams, other threads) race and give wrong results.  Each call
 *     writes every scratch entry it reads, so nothing needs clearing between
 *     calls.
 */
moe_status moe_capacity_noalloc(const moe_config *cfg, const int32_t *topk_idx,
                                int32_t *counts, int32_t *pos, uint8_t *keep,
                                int32_t *kept, int32_t *offsets, uint8_t *dropped,
                                int32_t *n_dropped, moe_stream_t stream);

/*
 * moe_dispatch - permute token rows into expert-grouped order ("Lab 18" tips:
 * gather each expert's tokens and run the expert once on them).
 *   x [T, d] dtype in; topk_idx, pos, keep, offsets from moe_capacity.
 *   x_perm [moe_perm_rows, d] dtype out: row offsets[e] + pos[t, j] = x[t] for
 *     every kept (t, j).  Padding rows are left untouched.
 *   src_slot [moe_perm_rows] int32 out, nullable: entry offsets[e] + pos[t, j]
 *     = t k + j (the assignment the row holds) for every kept (t, j); padding
 *     entries are left untouched.  moe_expert_ffn_slots reads it.
 *   zero_rows [T, d] dtype out, nullable: the row of every token with all its
 *     slots dropped is set to zero (for a top-1 layer without shared experts
 *     whose combine is moe_expert_ffn_slots writing y directly); other rows
 *     are left untouched.
 */
moe_status moe_dispatch(const moe_config *cfg, const void *x,
                        const int32_t *topk_idx, const int32_t *pos,
                        const uint8_t *keep, const int32_t *offsets,
                        void *x_perm, int32_t *src_slot, void *zero_rows,
                        moe_stream_t stream);

/*
 * moe_dispatch_rows - the dispatch as a row table only, for the expert GEMM
 * that gathers its rows from x (moe_expert_ffn_gather, moe_expert_ffn_slots
 * without x_perm): src_slot[offsets[e] + pos[t, j]] = t k + j for every kept
 * (t, j) (the row is token t's); every other entry (segment padding) = -1.
 *   topk_idx, pos, keep, offsets from moe_capacity; src_slot [moe_perm_rows]
 *   int32 out (device).  Moves T k small entries instead of the rows.
 */
moe_status moe_dispatch_rows(const moe_config *cfg, const int32_t *topk_idx,
                             const int32_t *pos, const uint8_t *keep,
                             const int32_t *offsets, int32_t *src_slot,
                             moe_stream_t stream);

/*
 * moe_expert_ffn - the expert FFNs over the expert segments, and the shared
 * experts over all tokens ("Lab 18" section 1 expert definitions, tips: one
 * grouped matrix multiply over all experts).
 *   x_perm [moe_perm_rows, d] dtype in; offsets [E + 1] from moe_capacity.
 *   W1, W3, W2 routed weights; x [T, d] and Ws1, Ws3, Ws2 for the shared
 *     experts (all NULL when S = 0).
 *   Y_perm [moe_perm_rows, d] dtype out: FFN_e of each row of segment e.
 *   Y_shared [T, d] dtype out (NULL when S = 0): sum over s of FFN_s(x_t).
 *   ws: scratch (hidden activations), moe_stage_workspace_size bytes; its
 *     first word is the device status word (cleared by this call).
 * bf16 runs on the tensor cores (tcgen05, fp32 accumulation, hidden
 * activations rounded to bf16); fp32 runs on the CUDA cores in fp32.
 */
moe_status moe_expert_ffn(const moe_config *cfg, const void *x_perm,
                          const int32_t *offsets, const void *W1,
                          const void *W3, const void *W2, const void *x,
                          const void *Ws1, const void *Ws3, const void *Ws2,
                          void *Y_perm, void *Y_shared, void *ws,
                          size_t ws_bytes, moe_stream_t stream);

/*
 * moe_expert_ffn_gather - moe_expert_ffn with the dispatch fused in: row r of
 * segment e is token src_slot[r] / k of x, read by GEMM1 straight from x
 * (bf16: TMA row gathers into each tile; fp32: indexed loads), so x_perm is
 * never written.  Results are those of moe_dispatch + moe_expert_ffn on the
 * same rows.
 *   x [T, d] dtype in; src_slot [moe_perm_rows] from moe_dispatch_rows;
 *   every other argument as for moe_expert_ffn.
 */
moe_status moe_expert_ffn_gather(const moe_config *cfg, const void *x,
                                 const int32_t *src_slot, const int32_t *offsets,
                                 const void *W1, const void *W3, const void *W2,
                                 const void *Ws1, const void *Ws3, const void *Ws2,
                                 void *Y_perm, void *Y_shared, void *ws,
                                 size_t ws_bytes, moe_stream_t stream);

/*
 * moe_expert_ffn_slots - moe_expert_ffn with the combine's gate fused into
 * GEMM2's epilogue ("Lab 18" section 1, y = sum g_i FFN_i(x); section 3, a
 * dropped slot contributes nothing): every kept row r of segment e, holding
 * assignment a = src_slot[r] (token a / k, slot a % k), is written as
 *     Y_slot[a] = gates[a] * FFN_e(row)      (rounded once to dtype)
 * so the combine is left with a plain sum of a token's k contiguous rows
 * (moe_combine_slots), or with nothing for k = 1 and no shared expert: there
 * Y_slot may be y itself, and only the rows of tokens whose slot was dropped
 * are left to fill (they are not written).
 *   x_perm [moe_perm_rows, d]: the permuted rows (moe_dispatch), or NULL to
 *     gather them from x through src_slot (moe_dispatch_rows) as
 *     moe_expert_ffn_gather does.
 *   x [T, d]: the tokens (required when x_perm is NULL or S > 0).
 *   src_slot [moe_perm_rows] int32 (moe_dispatch or moe_dispatch_rows);
 *   kept [E] int32 (moe_capacity): rows past kept[e] in segment e are padding.
 *   gates [T, k] fp32 (moe_route).
 *   Y_slot [T k, d] dtype out: rows of dropped assignments are not written.
 *   Y_shared, ws and the weights as for moe_expert_ffn.
 */
moe_status moe_expert_ffn_slots(const moe_config *cfg, const void *x_perm, const void *x,
                                const int32_t *src_slot, const int32_t *offsets,
                                const int32_t *kept, const float *gates,
                                const void *W1, const void *W3, const void *W2,
                                const void *Ws1, const void *Ws3, const void *Ws2,
                                void *Y_slot, void *Y_shared, void *ws, size_t ws_bytes,
                                moe_stream_t stream);

/*
 * moe_combine_slots - the combine after moe_expert_ffn_slots ("Lab 18"
 * section 1 and section 3):
 *   y[t] = sum_{j = 0..k-1, keep[t, j]} Y_slot[t k + j] + Y_shared[t] (+ residual[t])
 * summed in fp32 in that order and stored as dtype; the k rows of a token are
 * contiguous.  A token with every slot dropped gets Y_shared[t] (or 0), plus
 * the residual when given.  Y_shared: required when S > 0; residual nullable.
 */
moe_status moe_combine_slots(const moe_config *cfg, const void *Y_slot, const void *Y_shared,
                             const uint8_t *keep, const void *residual, void *y,
                             moe_stream_t stream);

/*
 * moe_combine - gate-weighted sum plus shared experts ("Lab 18" section 1,
 * y = sum g_i FFN_i(x); section 3, a dropped slot contributes nothing):
 *   y[t] = sum_{j = 0..k-1, keep[t, j]} gates[t, j] * Y_perm[offsets[e] + pos[t, j]]
 *          + Y_shared[t] (+ residual[t])
 * summed in fp32 in that order and stored as dtype.  A token with every slot
 * dropped gets Y_shared[t] (or 0), plus the residual when given.
 *   Y_shared [T, d] dtype: required when S > 0, added whenever given.
 *   residual [T, d] dtype: nullable.
 */
moe_status moe_combine(const moe_config *cfg, const void *Y_perm,
                       const void *Y_shared, const float *gates,
                       const int32_t *topk_idx, const int32_t *pos,
                       const uint8_t *keep, const int32_t *offsets,
                       const void *residual, void *y, moe_stream_t stream);

/*
 * moe_losses - Switch load-balance loss and router z-loss ("Lab 18" section 2;
 * "Lab 01" step 3: f divides by the T k slots):
 *   aux = E * sum_i (counts_i / (T k)) * P_i,  P_i = (1/T) sum_t p_{t,i}
 *   zloss = (1/T) sum_t lse_t^2
 * from counts (moe_capacity) and loss_partials (moe_route), reduced in a fixed
 * order (deterministic).  aux, zloss: device fp32 scalars, unweighted.
 */
moe_status moe_losses(const moe_config *cfg, const int32_t *counts,
                      const float *loss_partials, float *aux, float *zloss,
                      moe_stream_t stream);

/*
 * moe_seq_balance_loss - sequence-wise balance loss: the Switch loss of
 * moe_losses with one sequence as the balancing unit (cs336 lecture 4 field
 * map, "Training a router you cannot differentiate": the balancing unit is
 * where the variants differ; DeepSeek-V3 keeps a small sequence-wise loss,
 * "Lab 18" section 2).  Tokens [b L, (b + 1) L) form sequence b:
 *   per_seq[b] = E * sum_i (count_i^b / (L k)) * P_i^b,
 *   count_i^b = assignments of sequence b to expert i (before capacity),
 *   P_i^b = (1/L) sum_{t in b} p_{t,i} (sigmoid: s_{t,i} / sum_j s_{t,j}),
 *   loss = (1/B) sum_b per_seq[b], B = T / L.
 *   seq_len L: a multiple of 32 that divides T (else MOE_ERR_SHAPE).
 *   topk_idx [T, k] and loss_partials (moe_route) in; per_seq [T / L] fp32
 *   and loss [1] fp32 out (device).  Fixed summation order (deterministic).
 */
moe_status moe_seq_balance_loss(const moe_config *cfg, int32_t seq_len,
                                const int32_t *topk_idx, const float *loss_partials,
                                float *per_seq, float *loss, moe_stream_t stream);

/*
 * moe_bias_update - one step of auxiliary-loss-free balancing ("Lab 18"
 * section 2, DeepSeek-V3; cs336 lecture 4, "Training a router you cannot
 * differentiate"): in place, select_bias[i] -= gamma when expert i is
 * overloaded (E counts[i] > T k), += gamma when underloaded (E counts[i] <
 * T k), unchanged at the balanced load; one fp32 addition each.
 *   counts [E] int32 in (moe_capacity: assignments before capacity);
 *   gamma: finite step (else MOE_ERR_SHAPE); select_bias [E] fp32 in/out,
 *   the bias moe_route adds to the sigmoid scores for selection only.
 */
moe_status moe_bias_update(const moe_config *cfg, const int32_t *counts, float gamma,
                           float *select_bias, moe_stream_t stream);

/*
 * moe_forward - the whole layer: route, capacity, dispatch, expert FFNs,
 * combine, losses ("Lab 18", MoE.forward row of "What to implement").
 *   x [T, d] dtype; weights; outputs as described at moe_outputs.
 *   ws: at least moe_workspace_size(cfg) bytes, 256-byte aligned.
 * The stages' kernels, no host synchronisation, safe to capture in a CUDA
 * graph; each kernel is launched so that it may start while the previous one
 * finishes (programmatic dependent launch) and waits for it on the device.
 * The losses are computed inside the capacity launch, with the same
 * fixed-order reduction as moe_losses (the same bits).  For k = 1 without
 * shared experts the combine is fused into the expert GEMM (as
 * moe_expert_ffn_slots writing y, the dispatch zeroing dropped tokens' rows),
 * so y is g FFN(x) rounded once instead of twice.  With
 * MOE_PRIORITY_SCORE the router also writes its scores [T, E] to the
 * workspace, the capacity stage is moe_capacity_scored and the losses are a
 * launch of their own.
 */
moe_status moe_forward(const moe_config *cfg, const moe_weights *w,
                       const void *x, const moe_outputs *out, void *ws,
                       size_t ws_bytes, moe_stream_t stream);

/*
 * moe_device_status - read the device status word that the bounded waits of
 * the tensor-core kernels (router, expert GEMMs) set when they give up
 * (MOE_OK or MOE_ERR_DEVICE_TIMEOUT).  moe_route and moe_expert_ffn clear it
 * when they start, moe_forward once for the whole layer.  ws is the workspace
 * passed to those calls; *status is host memory.  Synchronises `stream` (a cudaMemcpyAsync followed by a stream
 * synchronise) - the only call in this library that does.
 */
moe_status moe_device_status(const void *ws, int32_t *status,
                             moe_stream_t stream);

/* Clear the device status word (asynchronous, on `stream`). */
moe_status moe_clear_device_status(void *ws, moe_stream_t stream);

/*
 * moe_probe_wait_timeout - diagnostic of the failure path: launches one
 * thread that waits, with the bounded wait the expert GEMMs' roles use, on an
 * mbarrier that nothing arrives on.  After timeout_ns (at most 2 s, else
 * MOE_ERR_SHAPE) it gives up and writes MOE_ERR_DEVICE_TIMEOUT to the status
 * word at the start of ws; nothing else is touched and the CUDA context stays
 * usable.  Read the result with moe_device_status.
 */
moe_status moe_probe_wait_timeout(void *ws, uint64_t timeout_ns, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
