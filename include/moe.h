/*
 * moe.h — C ABI of the single-GPU Mixture-of-Experts FFN layer forward pass (sm_100a).
 *
 * The layer (DeepSpeed MoE and Model Compression, section "DeepSpeed-MoE：容量增长不等于
 * 每 token 计算增长", the MoE formula and the pipeline listing):
 *
 *     p(x) = softmax(W_r x)                     y = sum_{e in TopK(p(x), k)} p_e(x) E_e(x)
 *
 * i.e. score every expert for every token, keep each token's k best experts and their
 * probabilities as gates, pack the tokens expert by expert within a per-expert capacity, run
 * each expert's FFN on its packed rows, and sum each token's expert outputs weighted by its
 * gates.
 *
 * Entry points, in pipeline order:
 *     moe_router_topk   router logits, softmax, top-k, load-balance statistics
 *     moe_dispatch      capacity-limited first-come slots and the expert-major packed copy
 *     moe_expert_ffn    per-expert two-layer GeLU FFN on the packed rows (grouped GEMMs)
 *     moe_combine       gate-weighted sum of the kept expert rows plus the residual terms
 *     moe_layer_forward all of the above (plus the optional PR-MoE dense MLP branch)
 *
 * Conventions (every entry point):
 *   - Tensor pointers are caller-owned DEVICE memory, row-major, 16-byte aligned. The
 *     library never allocates or frees memory and never synchronises the device, except
 *     moe_get_device_error / moe_workspace_reset, which say so.
 *   - All work is enqueued asynchronously on `stream` (NULL = the legacy default stream).
 *   - Arguments are validated on the host before anything is enqueued; on failure the
 *     entry returns a status other than MOE_OK and enqueues nothing.
 *   - `ws` is caller-owned device scratch of at least the size the matching
 *     *_workspace_bytes query returns. Its first 256 bytes are the STATUS BLOCK: an int
 *     that kernels set (first error wins) when they detect bad device-side data or give
 *     up a bounded wait. Zero it once after allocation with moe_workspace_reset (or any
 *     memset) and read it with moe_get_device_error. Entry points never clear it.
 *   - Calls that share a workspace must not overlap on the GPU (same stream is enough).
 *   - bf16 tensors are stored as 16-bit words (the top half of an IEEE fp32 word).
 *   - Environment variable MOE_FAULT_INJECT=<entry point name> makes that entry point
 *     return MOE_ERR_CUDA without enqueueing anything (host-side fault injection for
 *     callers' error paths).
 *   - Performance switches, all on by default and all bit-identical in their results
 *     (set to 0 to turn one off, for A/B timing): MOE_PDL (programmatic dependent launch
 *     between the layer's kernels; read once per process), MOE_FUSED_ROUTER (softmax,
 *     top-k and the statistics in the tensor-core router's epilogue), MOE_COSCHEDULE (a
 *     PR-MoE layer's expert and dense GEMM layers share one launch), MOE_PAIR_MMA (expert
 *     GEMMs with 256-column tiles run as two-SM CTA pairs), MOE_W_EVICT_FIRST (the L2
 *     evict-first hint on expert weights read once per layer). All but MOE_PDL are read at
 *     every call.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 3
#define MOE_STATUS_BLOCK_BYTES 256
#define MOE_MAX_EXPERTS 1024
#define MOE_MAX_TOPK 8

struct CUstream_st;
typedef struct CUstream_st* moe_stream_t; /* the same handle as cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARGUMENT = 1,    /* NULL pointer, negative size, k > E, ... */
  MOE_ERR_UNSUPPORTED = 2,         /* valid but outside what the library implements */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below the *_workspace_bytes answer */
  MOE_ERR_CUDA = 4,                /* a CUDA runtime call failed (or fault injection) */
  MOE_ERR_DEVICE_FLAG = 5,         /* moe_get_device_error found a device-side error */
  MOE_ERR_MISALIGNED = 6           /* a tensor pointer is not 16-byte aligned */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Device-side error codes written to the status block (first error wins). */
typedef enum {
  MOE_DEVERR_NONE = 0,
  MOE_DEVERR_TIMEOUT = 1,      /* a bounded wait inside a kernel gave up (about 2 s) */
  MOE_DEVERR_BAD_EXPERT = 2,   /* an expert id outside [0, E) reached dispatch */
  MOE_DEVERR_BAD_OFFSETS = 3,  /* expert_offsets not non-decreasing or beyond rows_max */
  MOE_DEVERR_BAD_ROW = 4       /* combine met a (slot, offset) outside the packed rows */
} moe_device_error;

const char* moe_status_string(moe_status s);
int moe_abi_version(void);

/* ---------------------------------------------------------------- sizes
 * Expert capacity (Switch/DeepSpeed comparison article, section "Expert Capacity Overflow":
 * capacity = (tokens in the batch / experts) x capacity factor), with the k choices of
 * each token counted and rounded up: C = ceil(k * T / E * capacity_factor). The product is
 * formed in double in that order; one that lies within 8 units in the last place above an
 * integer counts as that integer, so a decimal factor gives the capacity the decimal number
 * means (T = 100, E = 10, k = 1, capacity_factor = 1.1 gives 11, although 1.1 is stored a
 * little above 1.1). capacity_factor must be finite and >= 0. */
moe_status moe_capacity(int64_t T, int E, int k, double capacity_factor, int64_t* C_out);

/* Rows of the expert-major packed buffers: min(T * k, E * C). Kept rows of expert e occupy
 * [expert_offsets[e], expert_offsets[e+1]) with no padding between experts. */
moe_status moe_packed_rows_max(int64_t T, int E, int k, int64_t C, int64_t* rows_out);

/* ---------------------------------------------------------------- router
 * logits[t,e] = sum_i x[t,i] * w_router[e,i] (+ router_bias[e])   (fp32 arithmetic)
 * p[t,:]      = softmax(logits[t,:]) over all E experts
 * expert_ids[t,0..k-1] = the k largest logits, descending; ties go to the lower index
 * gates[t,j]  = p[t, expert_ids[t,j]]  (not renormalised over the k choices)
 * lb_stats    = [f_0..f_{E-1}, Q_0..Q_{E-1}, aux]: f_i = share of tokens whose first choice is i,
 *               Q_i = mean over tokens of p[t,i], aux = aux_alpha * E * sum_i f_i * Q_i
 *               (MoE survey notes §1.1.4.1, Switch Transformer load-balance loss).
 * Cites: DeepSpeed MoE blog, MoE formula; comparison article, "Router computation" and
 * "Top-1 routing decision".
 *
 * x:          [T, d_model] in x_dtype.           w_router: [E, d_model] fp32 (row e = expert e).
 * router_bias:[E] fp32 or NULL.                   logits:   [T, E] fp32 output, or NULL.
 * expert_ids: [T, k] int32 output.                gates:    [T, k] fp32 output.
 * lb_stats:   [2E+1] fp32 output, or NULL.
 * Limits: 1 <= E <= 1024, 1 <= k <= min(E, 8), T >= 0 (T == 0 enqueues nothing), d_model >= 1;
 * bf16 x needs d_model % 8 == 0. */
moe_status moe_router_workspace_bytes(int64_t T, int E, int d_model, size_t* bytes);

/* The router weight prepared for the tensor-core logits kernel: W_r (fp32) split exactly into
 * three bf16 parts hi + mid + lo = W_r (each holds the next 8 significant bits), stored
 * [E, 3 * ceil64(d_model)]. The router entry points split W_r on every call; a caller that keeps
 * W_r fixed between calls (inference, or between optimizer steps) prepares it once per weight
 * version with moe_router_prepare and passes it as moe_layer_args.w_router_prepared, which
 * saves one launch per layer call. The prepared buffer is caller-owned device memory of
 * moe_router_prepare_bytes bytes; it must be prepared again whenever W_r changes (the library
 * cannot see a change). Prepared weights only serve bf16 x with d_model % 8 == 0 and T > 64
 * (the tensor-core path); elsewhere they are ignored and W_r is used directly. */
moe_status moe_router_prepare_bytes(int E, int d_model, size_t* bytes);
moe_status moe_router_prepare(const float* w_router, int E, int d_model, void* w_prepared,
                              size_t bytes, moe_stream_t stream);

moe_status moe_router_topk(const void* x, moe_dtype x_dtype, int64_t T, int d_model,
                           const float* w_router, const float* router_bias, int E, int k,
                           float* logits, int32_t* expert_ids, float* gates, float* lb_stats,
                           float aux_alpha, void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_router_topk with two routing variants (same workspace):
 * renormalize != 0: gates[t,j] = p[t,e_j] / sum_{j'} p[t,e_j'] (the k chosen probabilities
 *               renormalised to sum to 1: MoE survey notes §1.1.1.1, top-k after the softmax).
 * probs (NULL or [T, k] fp32 output): p[t, expert_ids[t,j]], the softmax probability of each
 *               choice before any renormalisation (equal to gates when renormalize == 0); the
 *               ranking key of moe_dispatch_priority.
 * router_losses (NULL or [3] fp32 output):
 *   [0] z-loss = (1/T) sum_t (log sum_e exp(logits[t,e]))^2 (comparison article, "Router
 *       Z-loss"; without the coefficient);
 *   [1] CoV^2 of Importance_i = sum of the gates routed to expert i (after renormalisation);
 *   [2] CoV^2 of Load_i = number of choices routed to expert i
 *   (MoE survey notes §1.1.4.1; CoV = standard deviation / mean with the population variance,
 *   0 when the mean is 0; without the coefficients). lb_stats still uses the softmax p. */
moe_status moe_router_topk_ex(const void* x, moe_dtype x_dtype, int64_t T, int d_model,
                              const float* w_router, const float* router_bias, int E, int k,
                              float* logits, int32_t* expert_ids, float* gates, float* lb_stats,
                              float aux_alpha, int renormalize, float* router_losses,
                              float* probs, void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------- dispatch
 * pack_by_expert with a capacity (DeepSpeed MoE blog, pipeline listing; DeepSpeed-MoE notes
 * §4.4: top-k + prefix-sum + scatter into a dense token-to-expert mapping table, then an
 * explicit re-order of rows by that table instead of a sparse einsum).
 * Pairs (t, j) are taken in token order (t ascending, then j); each gets the next position of
 * its expert: slot[t,j] = position if position < C, else -1 (overflow: the pair contributes
 * nothing and the token keeps only its residual).
 * expert_counts[e]   = demand of expert e (before the drop).
 * expert_offsets[e]  = sum_{e' < e} min(expert_counts[e'], C); expert_offsets[E] = kept rows.
 * row_token[r]       = token of packed row r for r < expert_offsets[E] (rows beyond: unspecified).
 * x_packed[offsets[e] + slot[t,j], :] = x[t, :] for every kept pair.
 * x, x_packed: [T, d_model] / [rows_max, d_model] in dtype; rows_max from moe_packed_rows_max.
 * Expert ids outside [0, E) set MOE_DEVERR_BAD_EXPERT and are treated as dropped. */
moe_status moe_dispatch_workspace_bytes(int64_t T, int E, int k, size_t* bytes);
moe_status moe_dispatch(const void* x, moe_dtype dtype, int64_t T, int d_model,
                        const int32_t* expert_ids, int E, int k, int64_t C, int32_t* slot,
                        int32_t* expert_counts, int32_t* expert_offsets, int32_t* row_token,
                        void* x_packed, int64_t rows_max, void* ws, size_t ws_bytes,
                        moe_stream_t stream);

/* moe_dispatch with overflow by priority (comparison article, "Expert Capacity Overflow": the
 * example ranks an expert's tokens by router probability and keeps the most probable): the
 * pairs of each expert are ranked by probs, largest first, ties to the lower pair index
 * p = t * k + j; slot[t,j] = rank if rank < C, else -1, and kept rows are packed in rank order.
 * probs: [T, k] fp32, the softmax probability of each choice BEFORE any renormalisation
 * (moe_router_topk's gates, or moe_router_topk_ex's probs output): renormalised top-1 gates are
 * all 1 and carry no preference. Finite values; the order is that of the fp32 numbers.
 * Counts, offsets, row_token and x_packed follow moe_dispatch. Same workspace as moe_dispatch.
 * Cost: O(n log^2 n) per expert of demand n (chunk ranks, then merge passes). */
moe_status moe_dispatch_priority(const void* x, moe_dtype dtype, int64_t T, int d_model,
                                 const int32_t* expert_ids, const float* probs, int E, int k,
                                 int64_t C, int32_t* slot, int32_t* expert_counts,
                                 int32_t* expert_offsets, int32_t* row_token, void* x_packed,
                                 int64_t rows_max, void* ws, size_t ws_bytes,
                                 moe_stream_t stream);

/* Allocation-free variant of moe_dispatch (no counterpart on the pages: it exists for callers).
 * Some callers cannot allocate device memory at all: a plug-in running inside a host application
 * that owns every device buffer and offers no allocation hook, or a latency-critical serving loop
 * that must never call cudaMalloc/cudaFree because they can block and synchronise the device.
 * Such a caller passes only its inputs and outputs; the dispatch scratch (per-pair ranks and
 * per-segment counts and bases: align256(4*T*k) + 2*align256(4*ceil(T*k/256)*E) bytes) comes
 * from one static device array of MOE_NOALLOC_SCRATCH_BYTES (4 MiB) that every GPU loading the
 * library holds until the process exits. Larger problems return MOE_ERR_WORKSPACE_TOO_SMALL
 * (use moe_dispatch with a workspace instead). Arguments, outputs and results are those of
 * moe_dispatch, except that no status block exists: ids outside [0, E) become dropped pairs
 * without a device error code. Each call looks up the array's device address on the current
 * device, except a call whose stream is being captured, which reuses the address an earlier call
 * on that device found: make the first call on each device before any stream capture begins
 * (after a device reset, too, the first call must come before a capture).
 * Nothing in the array needs to start at zero (every element read is written first in the same
 * call), but all calls share it: calls that overlap on the GPU race and must be serialised. */
#define MOE_NOALLOC_SCRATCH_BYTES (4u << 20)
moe_status moe_dispatch_noalloc(const void* x, moe_dtype dtype, int64_t T, int d_model,
                                const int32_t* expert_ids, int E, int k, int64_t C, int32_t* slot,
                                int32_t* expert_counts, int32_t* expert_offsets,
                                int32_t* row_token, void* x_packed, int64_t rows_max,
                                moe_stream_t stream);

/* ---------------------------------------------------------------- expert FFN
 * For every expert e and every packed row r in [expert_offsets[e], expert_offsets[e+1]):
 *     h[r,:] = GeLU(W1[e] x_packed[r,:] + b1[e])        GeLU(z) = 0.5 z (1 + erf(z / sqrt 2))
 *     y[r,:] = W2[e] h[r,:] + b2[e]
 * (an expert is a two-layer feed-forward network: MoE survey notes §1.1.2.1; DeepSpeed-MoE notes
 * §4.4/§5, "Sparse GEMM -> Dense GEMM": dense per-expert GEMMs on the packed rows).
 * w1: [E, d_ff, d_model], b1: [E, d_ff] or NULL, w2: [E, d_model, d_ff], b2: [E, d_model] or NULL,
 * all in dtype. h_packed: [rows_max, d_ff] in dtype (intermediate, bf16 rounds h);
 * y_packed: [rows_max, d_model] fp32. Rows outside every segment are not written.
 * With E = 1 and expert_offsets = {0, T} this is a dense MLP (the PR-MoE fixed MLP).
 * capacity_hint: an upper bound on the rows of any one expert (normally C); it only selects the
 * token tile width and never affects results. bf16 needs d_model % 8 == 0 and d_ff % 8 == 0.
 * bf16 runs on tcgen05 tensor cores (fp32 accumulate); fp32 runs on fp32 FMA (no TF32). */
moe_status moe_expert_ffn_workspace_bytes(size_t* bytes);
moe_status moe_expert_ffn(const void* x_packed, const int32_t* expert_offsets, int E,
                          int64_t rows_max, int d_model, int d_ff, moe_dtype dtype, const void* w1,
                          const void* b1, const void* w2, const void* b2, void* h_packed,
                          float* y_packed, int64_t capacity_hint, void* ws, size_t ws_bytes,
                          moe_stream_t stream);

/* One layer of the grouped expert GEMM (a single kernel launch):
 *     out[r, :] = act(W[e] x_packed[r, :] + bias[e])   for r in [expert_offsets[e], expert_offsets[e+1])
 * w: [E, N, K] in dtype, bias: [E, N] in dtype or NULL, x_packed: [rows_max, K] in dtype.
 * MOE_EPILOGUE_BIAS_GELU writes out [rows_max, N] in dtype (bf16 rounds GeLU(z));
 * MOE_EPILOGUE_BIAS writes out [rows_max, N] in fp32. moe_expert_ffn is this entry twice
 * (K=d_model, N=d_ff with GeLU; then K=d_ff, N=d_model). Same limits as moe_expert_ffn. */
typedef enum { MOE_EPILOGUE_BIAS_GELU = 0, MOE_EPILOGUE_BIAS = 1 } moe_epilogue;
moe_status moe_grouped_gemm(const void* x_packed, const int32_t* expert_offsets, int E,
                            int64_t rows_max, int K, int N, moe_dtype dtype, const void* w,
                            const void* bias, moe_epilogue epilogue, void* out,
                            int64_t capacity_hint, void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------- combine
 * out[t,:] = [residual[t,:]] + [dense[t,:]] + sum_{j : slot[t,j] >= 0} gates[t,j] *
 *            y_packed[expert_offsets[expert_ids[t,j]] + slot[t,j], :]
 * summed in fp32 in that order and rounded once to out_dtype (DeepSpeed MoE blog, the combine
 * step of the pipeline listing; comparison article, "Expert Capacity Overflow": a dropped token
 * passes through the residual only; PR-MoE "residual correction" example: fixed MLP output +
 * gate * expert).
 * residual: [T, d_model] in res_dtype or NULL. dense: [T, d_model] fp32 or NULL.
 * A (slot, offset) pointing outside [0, rows_max) sets MOE_DEVERR_BAD_ROW and is skipped. */
moe_status moe_combine_workspace_bytes(size_t* bytes);
moe_status moe_combine(const float* y_packed, const int32_t* expert_offsets,
                       const int32_t* expert_ids, const int32_t* slot, const float* gates,
                       int64_t T, int d_model, int E, int k, int64_t rows_max,
                       const void* residual, moe_dtype res_dtype, const float* dense, void* out,
                       moe_dtype out_dtype, void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------- whole layer */
typedef struct {
  int64_t T;
  int d_model, d_ff, E, k;
  double capacity_factor;
  moe_dtype dtype;      /* x, expert weights and biases, dense-branch weights */
  moe_dtype out_dtype;  /* output */
  const void* x;                         /* [T, d_model] */
  const float* w_router;                 /* [E, d_model] fp32 */
  const float* router_bias;              /* [E] fp32 or NULL */
  const void *w1, *b1, *w2, *b2;         /* experts; biases may be NULL */
  /* PR-MoE fixed dense MLP (DeepSpeed-MoE notes §3.1): all four NULL = no dense branch.
   * dense_w1 [d_ff, d_model], dense_b1 [d_ff], dense_w2 [d_model, d_ff], dense_b2 [d_model]. */
  const void *dense_w1, *dense_b1, *dense_w2, *dense_b2;
  int add_input_residual; /* 1: out += x */
  float aux_alpha;        /* alpha of the load-balance loss */
  int overflow_policy;    /* moe_overflow_policy */
  int renormalize_gates;  /* 1: gates renormalised over the k choices (moe_router_topk_ex) */
  /* w_router split by moe_router_prepare (NULL: split on every call inside the workspace) */
  const void* w_router_prepared;
} moe_layer_args;

/* Which pairs an expert keeps when its demand exceeds C: the first in token order (moe_dispatch),
 * or those of largest router probability (moe_dispatch_priority; the probability before any
 * renormalisation of the gates). */
typedef enum { MOE_OVERFLOW_FIRST_COME = 0, MOE_OVERFLOW_PRIORITY = 1 } moe_overflow_policy;

/* Optional device outputs of the intermediate results; any field may be NULL. */
typedef struct {
  float* logits;          /* [T, E] */
  int32_t* expert_ids;    /* [T, k] */
  float* gates;           /* [T, k] */
  int32_t* slot;          /* [T, k] */
  int32_t* expert_counts; /* [E] demand */
  int32_t* expert_offsets;/* [E+1] */
  float* lb_stats;        /* [2E+1] */
  float* router_losses;   /* [3]: z-loss, CoV^2 Importance, CoV^2 Load (moe_router_topk_ex) */
  float* topk_probs;      /* [T, k]: softmax probability of each choice before renormalisation */
} moe_layer_aux;

/* out = [x if add_input_residual] + [DenseMLP(x) if dense_*] + sum_j gate_j * Expert_{e_j}(x)
 * over the kept choices. Enqueues: router, dispatch, [dense MLP], expert FFN, combine.
 * T == 0 launches no kernel; it only zeroes aux expert_counts / expert_offsets when given. */
moe_status moe_layer_workspace_bytes(const moe_layer_args* args, size_t* bytes);
moe_status moe_layer_forward(const moe_layer_args* args, void* out, moe_layer_aux* aux, void* ws,
                             size_t ws_bytes, moe_stream_t stream);

/* moe_layer_forward that also records caller-created CUDA events (cudaEvent_t handles passed as
 * void*) on `stream` at stage boundaries: events[0] before the first kernel, then one after each
 * stage ("router", "dispatch", "expert_gemm1", "expert_gemm2" or "expert_gemm2_combine",
 * "dense_gemm1", "dense_gemm2_combine", "dense_ffn", "combine", as the layer's path has them).
 * *n_events receives the number recorded (at most max_events); `names` (may be NULL) receives the
 * comma-separated labels, starting with "start". Results are identical to moe_layer_forward. */
moe_status moe_layer_forward_profiled(const moe_layer_args* args, void* out, moe_layer_aux* aux,
                                      void* ws, size_t ws_bytes, moe_stream_t stream,
                                      void* const* events, int max_events, int* n_events,
                                      char* names, size_t names_len);

/* ---------------------------------------------------------------- token shards
 * The layer split over G GPUs by tokens, every weight replicated (data parallelism as the
 * DeepSpeed-MoE notes §4.2 use it: parameters copied, tokens divided). Shard r holds tokens [T_0 + ... + T_{r-1}, ... + T_r) of the batch of
 * T_global tokens, args->T = T_r. The capacity is the whole batch's, C = ceil(k T_global cf / E),
 * and the overflow rule is the single-GPU one: pairs in global token order, first come first
 * kept. One exchange step sits between the two halves:
 *   1. moe_layer_forward_shard_begin: router and top-k of the shard's tokens; writes the shard's
 *      demand per expert (demand [E] int32) and its integer router statistics
 *      (stat_partials [moe_router_partials_count(E)] int64: fixed-point sums of p, first-choice
 *      counts, gate sums, choice counts, (log Z)^2).
 *   2. the caller gathers every shard's demand into demand_all [G, E] (shard order) and sums
 *      the partials over shards into stat_totals (e.g. NCCL all-gather and all-reduce).
 *   3. moe_layer_forward_shard_end: the shard's global slot base per expert (sum of the earlier
 *      shards' demand), expert e keeps its first clamp(C - base_e, 0, demand_e) pairs; then
 *      dispatch, expert FFN and combine of the shard's tokens into out [T_r, d_model], and
 *      lb_stats / router_losses of the whole batch from stat_totals.
 * Results equal the single-GPU layer over the whole batch: ids, gates, slots and outputs of each
 * token bit for bit; lb_stats and router losses too when every shard but the last holds a
 * multiple of 64 tokens (the router's statistics blocks), else within fixed-point rounding.
 * Both calls take the same args, aux pointers and workspace (the workspace carries the shard's
 * routing from begin to end and must not be used in between). overflow_policy must be
 * MOE_OVERFLOW_FIRST_COME (MOE_ERR_UNSUPPORTED otherwise). begin's `out` is not used. */
moe_status moe_layer_shard_workspace_bytes(const moe_layer_args* args, int64_t T_global,
                                           size_t* bytes);
int64_t moe_router_partials_count(int E); /* 4 E + 1 */
moe_status moe_layer_forward_shard_begin(const moe_layer_args* args, int64_t T_global,
                                         moe_layer_aux* aux, int32_t* demand,
                                         int64_t* stat_partials, void* ws, size_t ws_bytes,
                                         moe_stream_t stream);
moe_status moe_layer_forward_shard_end(const moe_layer_args* args, int64_t T_global, int G,
                                       int rank, const int32_t* demand_all,
                                       const int64_t* stat_totals, void* out, moe_layer_aux* aux,
                                       void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------- training
 * The backward pass of the layer: gradients of the objective
 *     L = sum_{t,i} d_out[t,i] * out[t,i] + aux_weight * aux + z_weight * z_loss
 * (aux = lb_stats[2E], the load-balance loss; z_loss the router z-loss of moe_router_topk_ex),
 * by the chain rule through the forward pass. The routing decisions (top-k ids, slots, the
 * counts f_i) are held fixed; the gates carry the gradient to the router through the softmax
 * (and the renormalisation when enabled); a dropped choice contributes nothing (comparison
 * article, "Expert Capacity Overflow": no gradient for that expert).
 *
 * moe_layer_forward_train is moe_layer_forward that also keeps, in the workspace, what the
 * backward pass reads: logits, routing, the packed rows, h and GeLU'(z) of every expert row and
 * of the dense MLP, and the expert outputs y. moe_layer_backward then takes the same args and
 * workspace (unchanged in between) and the output gradient d_out [T, d_model] in args.dtype.
 * Results are identical to moe_layer_forward (the combine runs as its own kernel here).
 *
 * Gradients (fp32, overwritten; shapes those of the parameters): dw_router, db_router, dw1, db1,
 * dw2, db2 and the dense MLP's; dx [T, d_model] in args.dtype. A bias gradient pointer may be
 * NULL (not computed). T == 0 zeroes the parameter gradients. dgates [T, k] (dL/dgate) and dlogits [T, E] (dL/dlogits) are optional.
 * bf16 layers run the expert and dense GEMMs on tcgen05 (bf16 operands: dY, dZ rounded to bf16;
 * fp32 accumulation); the router's GEMMs and fp32 layers run on fp32 FMA. */
typedef struct {
  void* dx;                /* [T, d_model], args.dtype */
  float* dw_router;        /* [E, d_model] */
  float* db_router;        /* [E] or NULL */
  float* dw1;              /* [E, d_ff, d_model] */
  float* db1;              /* [E, d_ff] or NULL */
  float* dw2;              /* [E, d_model, d_ff] */
  float* db2;              /* [E, d_model] or NULL */
  float* dense_dw1;        /* [d_ff, d_model] (dense MLP only) */
  float* dense_db1;        /* [d_ff] or NULL */
  float* dense_dw2;        /* [d_model, d_ff] */
  float* dense_db2;        /* [d_model] or NULL */
  float* dgates;           /* [T, k] or NULL */
  float* dlogits;          /* [T, E] or NULL */
} moe_layer_grads;
moe_status moe_layer_train_workspace_bytes(const moe_layer_args* args, size_t* bytes);
moe_status moe_layer_forward_train(const moe_layer_args* args, void* out, moe_layer_aux* aux,
                                   void* ws, size_t ws_bytes, moe_stream_t stream);
moe_status moe_layer_backward(const moe_layer_args* args, const void* d_out, float aux_weight,
                              float z_weight, moe_layer_grads* grads, void* ws, size_t ws_bytes,
                              moe_stream_t stream);

/* ---------------------------------------------------------------- status block
 * moe_workspace_reset: zeroes the status block (asynchronous on stream).
 * moe_get_device_error: synchronises `stream`, copies the status word to *code_out and returns
 * MOE_ERR_DEVICE_FLAG if it is non-zero, MOE_OK otherwise. */
moe_status moe_workspace_reset(void* ws, size_t ws_bytes, moe_stream_t stream);
moe_status moe_get_device_error(const void* ws, int* code_out, moe_stream_t stream);

/* Number of kernel launches the last successful call of each entry point enqueued on this host
 * thread (for launch accounting in benchmarks). */
int moe_last_launch_count(void);

/* ---------------------------------------------------------------- failure-detection self-test
 * Checks, on the caller's GPU, that a kernel whose wait can never complete gives up instead of
 * hanging (no counterpart on the pages: it tests the library's own failure detection). Launches
 * the grouped expert GEMM once on a one-tile problem whose TMA role is told to issue no copy, so
 * the MMA role waits on a barrier that nobody arrives at. Every wait of that launch gives up after
 * wait_limit_ns (1000 <= wait_limit_ns <= 10^10), MOE_DEVERR_TIMEOUT is recorded in the status
 * block of ws, the roles stop, TMEM is freed and the kernel returns; nothing else in ws is read
 * or written, and the context stays usable. Read the result with moe_get_device_error.
 * ws: >= MOE_SELFTEST_WS_BYTES bytes, 256-byte aligned, status block zeroed by the caller. */
#define MOE_SELFTEST_WS_BYTES (256u + 32768u)
moe_status moe_selftest_bounded_wait(void* ws, size_t ws_bytes, uint64_t wait_limit_ns,
                                     moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
