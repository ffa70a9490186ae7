// Internal enqueue functions of the MoE-layer kernels (host side). Not part of the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Incremented once per kernel launch on the calling host thread (reset by every entry point).
void count_launch();
void reset_launch_count();

// Number of SMs of the current device (cached per device).
int num_sms();

// Whether launches carry the programmatic-dependent-launch attribute (MOE_PDL=0 disables it).
bool pdl_enabled();
// Whether bf16 PR-MoE layers co-schedule expert and dense GEMM layers (MOE_COSCHEDULE=0: no).
bool coschedule_enabled();
// Wide (256-token) expert GEMM tiles on CTA pairs (cta_group::2 MMAs); MOE_PAIR_MMA=0 keeps one
// CTA per tile. Read at every call.
bool pair_mma_enabled();

// Launches kern<<<grid, block, smem, stream>>>(args...) as a programmatic dependent launch and
// counts it.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
  count_launch();
  return e;
}

// ---------------------------------------------------------------- router
constexpr int kRouterTokensPerBlock = 64;
inline int64_t router_num_blocks(int64_t T) {
  return (T + kRouterTokensPerBlock - 1) / kRouterTokensPerBlock;
}
// Batches up to this many tokens use the GEMV router (one block per expert).
constexpr int64_t kRouterGemvMaxT = 64;
// K of each bf16 part of the split router weight, padded to the 64-element TMA block.
inline int router_split_dpad(int d) { return (d + 63) / 64 * 64; }
// The tensor-core router needs bf16 x whose rows are whole 16-byte units.
inline bool router_uses_tensor_cores(bool x_bf16, int d) { return x_bf16 && d % 8 == 0; }
// Load-balance statistics accumulators (zeroed by the router's first kernel each call).
struct RouterAccum {
  unsigned long long* q;    // [E] sums of p in 2^-32 fixed point
  unsigned* c;              // [E] counts of first choices
  unsigned long long* imp;  // [E] sums of the gates routed to each expert, 2^-24 fixed point
  unsigned* load;           // [E] counts of all choices routed to each expert
  unsigned long long* z;    // [1] sum over tokens of (log sum exp logits)^2, 2^-24 fixed point
  unsigned* ticket;         // blocks finished
};
struct RouterScratch {
  RouterAccum acc;
  uint16_t* w_split;      // [E, 3 * router_split_dpad(d)] bf16: hi | mid | lo parts of W_r
  float* logits_scratch;  // [T, E], used when the caller does not ask for the logits
};
// Optional: let the top-k kernel also rank each 64-token segment's (token, choice) pairs per
// expert for dispatch (segments of kRouterTokensPerBlock * k pairs).
struct RouterDispatchCount {
  int32_t* local_rank = nullptr;  // [T * k]
  int32_t* seg_counts = nullptr;  // [router_num_blocks(T), E]
};
// Integer statistics partials of one token shard: [q (E), c (E), imp (E), load (E), z (1)] as
// int64 (the accumulators' fixed-point values); sums over shards give the whole batch's.
inline int64_t router_partials_count(int E) { return 4 * (int64_t)E + 1; }
// logits may be nullptr (not returned).
// renormalize: gates of the k choices divided by their sum; probs (optional, [T, k]): the chosen
// experts' probabilities before that division (the priority ranking key). losses (optional): [z-loss,
// CoV^2 of Importance, CoV^2 of Load]. export_partials (optional): instead of finalising, the
// last block writes the integer partials there (lb_stats and losses must then be nullptr).
cudaError_t enqueue_router(const void* x, bool x_bf16, int64_t T, int d, const float* w_router,
                           const float* router_bias, int E, int k, float* logits, int32_t* ids,
                           float* gates, float* lb_stats, float aux_alpha,
                           const RouterScratch& scratch, int* status, cudaStream_t stream,
                           RouterDispatchCount dcount = RouterDispatchCount{},
                           bool renormalize = false, float* losses = nullptr,
                           int64_t* export_partials = nullptr, int64_t T_kernel_choice = -1,
                           float* probs = nullptr, const uint16_t* w_prepared = nullptr,
                           bool extra_stats = false);
// extra_stats: accumulate the z-loss, Importance and Load sums although losses == nullptr (a
// later kernel finalises them from the accumulators).
// w_prepared (optional): W_r already split (enqueue_router_prepare); the tensor-core path then
// skips the split, and the logits kernel zeroes the statistics accumulators instead.
// Splits W_r [E, d] into the three bf16 parts [E, 3 * router_split_dpad(d)].
cudaError_t enqueue_router_prepare(const float* w_router, int E, int d, uint16_t* out,
                                   cudaStream_t stream);
// T_kernel_choice (>= T): the batch size that selects the logits kernel (a token shard takes the
// whole batch's, so every token's logits come from the same arithmetic).
// f, Q, aux (lb_stats, optional) and the router losses (optional) from summed partials of T
// tokens, with the same arithmetic as the top-k kernel's own finalisation (one block).
cudaError_t enqueue_router_finalize(const int64_t* totals, int64_t T, int E, float aux_alpha,
                                    float* lb_stats, float* losses, cudaStream_t stream);
// logits = x W_r^T + b_r on tcgen05 from the exact split W_r = hi + mid + lo (bf16 each).
// zero_acc (optional): accumulators the kernel zeroes before its dependents start.
cudaError_t enqueue_router_logits_tc(const void* x, int64_t T, int d, const uint16_t* w_split,
                                     int dpad, const float* router_bias, int E, float* logits,
                                     int* status, cudaStream_t stream,
                                     const RouterAccum* zero_acc = nullptr);

// The tensor-core router with softmax, top-k, the statistics (and the dispatch ranks) fused into
// its epilogue (router_fused_supported: E <= 128). The statistics accumulators must be zero when it
// starts. logits may be nullptr (not written).
bool router_fused_supported(int E);
// Whether the router uses the fused kernel where it can (MOE_FUSED_ROUTER=0: the two kernels).
bool router_fusion_enabled();
cudaError_t enqueue_router_fused(const void* x, int64_t T, int d, const uint16_t* w_split,
                                 int dpad, const float* router_bias, int E, int k, float* logits,
                                 int32_t* ids, float* gates, float* probs, const RouterAccum& acc,
                                 float aux_alpha, float* lb_stats, RouterDispatchCount dc,
                                 bool renormalize, float* losses, int64_t* exported,
                                 bool extra_stats, int* status, cudaStream_t stream);

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current device, once per
// device (done_per_device: a zero-initialised [64] array owned by the launching function).
template <class Kern>
cudaError_t ensure_dynamic_smem(Kern kern, int bytes, int* done_per_device) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cached = dev >= 0 && dev < 64;
  if (cached && done_per_device[dev] >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && cached) done_per_device[dev] = bytes;
  return e;
}

// One layer of the experts and one layer of the PR-MoE dense MLP co-scheduled in one persistent
// launch (the expert tiles stream weights from HBM, the dense tiles keep the tensor pipe busy):
//   experts: out[r] = act(W[e] xp[r] + bias[e]) for the packed rows of every expert (offsets),
//   dense:   out_dense[t] = act(W_dense x_dense[t] + bias_dense) for t < T,
// both with K inputs and N outputs; gelu: bf16 GeLU outputs (layer 1), else fp32 (layer 2).
// co_gemm_supported: whether the expert token tile (from capacity_hint) allows it (<= 128 rows).
bool co_gemm_supported(int64_t capacity_hint);
cudaError_t enqueue_co_gemm_bf16(const void* xp, const int32_t* offsets, int E, int64_t rows_max,
                                 const void* w, const void* bias, void* out, int64_t capacity_hint,
                                 const void* x_dense, int64_t T, const void* w_dense,
                                 const void* bias_dense, void* out_dense, int K, int N, bool gelu,
                                 int* status, cudaStream_t stream);

// Failure-detection self-test: one grouped-GEMM launch whose TMA role issues no copy, so its MMA
// role waits on a barrier nobody arrives at; every wait gives up after wait_limit_ns, records
// MOE_DEVERR_TIMEOUT in *status and the kernel returns. scratch: >= 32 KB of device memory (the
// tensor maps' base; never read or written).
cudaError_t enqueue_selftest_bounded_wait(void* scratch, uint64_t wait_limit_ns, int* status,
                                         cudaStream_t stream);

// ---------------------------------------------------------------- dispatch
constexpr int kDispatchSeg = 256;  // (token, choice) pairs per counting segment (one warp)
inline int64_t dispatch_num_segments(int64_t pairs) {
  return (pairs + kDispatchSeg - 1) / kDispatchSeg;
}
// dropped_out (optional, top-1 layers whose combine is fused into layer 2): for every token whose
// only choice overflowed, writes out[t] = x[t] (dropped_add_x) or 0, in the output type.
struct DroppedRows {
  void* out = nullptr;
  bool out_bf16 = true;
  bool add_x = true;
};
// Overflow by priority (optional): each expert keeps its C pairs of largest router probability
// (ties -> lower pair index) and packs them in that order. keys [2 T k] (two ping-pong halves of
// 64-bit sort keys) and demand_offsets [E + 1] are scratch.
struct PriorityDispatch {
  const float* probs = nullptr;  // [T, k] probabilities before renormalisation; nullptr = first-come
  uint64_t* keys = nullptr;
  int32_t* demand_offsets = nullptr;
};
// Token shards (optional): this shard is `rank` of G consecutive token blocks; demand_all [G, E]
// holds every shard's demand. Expert e keeps the pairs whose global first-come position
// (sum of the earlier shards' demand + local position) is below C: cap_local[e] (scratch [E])
// = clamp(C - base_e, 0, demand_e) of them.
struct ShardBase {
  const int32_t* demand_all = nullptr;  // nullptr = one shard
  int G = 1;
  int rank = 0;
  int32_t* cap_local = nullptr;
};
// Optional: the router's load-balance statistics finalised by the dispatch scan kernel (the
// router then leaves them as integer accumulators): f, Q, aux into lb and the router losses into
// losses (either may be nullptr), from the accumulators of T tokens.
struct StatsFinalize {
  RouterAccum acc{};
  int64_t T = 0;
  float alpha = 0.0f;
  float* lb = nullptr;
  float* losses = nullptr;
};
cudaError_t enqueue_dispatch(const void* x, bool bf16, int64_t T, int d, const int32_t* ids, int E,
                             int k, int64_t C, int32_t* slot, int32_t* counts, int32_t* offsets,
                             int32_t* row_token, void* x_packed, int64_t rows_max,
                             int32_t* local_rank, int32_t* seg_counts, int32_t* seg_base,
                             int* status, cudaStream_t stream, DroppedRows dropped = DroppedRows{},
                             int counted_seg_len = 0, PriorityDispatch prio = PriorityDispatch{},
                             ShardBase shard = ShardBase{}, bool scan_only = false,
                             StatsFinalize fin = StatsFinalize{});
// counted_seg_len > 0: local_rank and seg_counts were already written (segments of that many
// pairs) by the router's top-k kernel; the counting kernel is skipped.

// ---------------------------------------------------------------- expert FFN
// One grouped GEMM layer: out = act(W[e] x + bias[e]) over every expert segment. offsets ==
// nullptr means one segment [0, rows_max) (E must be 1). gelu: GeLU epilogue with output in the
// input type; otherwise bias only with fp32 output.
// A bf16 tensor map over a row-major [rows, cols] matrix, boxes of box_cols x box_rows,
// 128-byte swizzle, out-of-range elements read as zero.
bool make_bf16_map_2d(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int box_cols,
                      int box_rows);
// Weight-gradient GEMM (tcgen05): for every expert e,
//     out[e][m][n] = sum over the rows r of segment e of a[r][m] * b[r][n]    (fp32, overwritten)
// a [rows_max, M] and b [rows_max, N] bf16, token-major; offsets == nullptr: one segment
// [0, rows_max) (E == 1). Experts without rows get zeros.
// splits > 1: split-K, out holds [splits][E][M][N] partial sums (add them in split order).
// b_period > 0 (a multiple of 64): row r of a pairs with row r % b_period of b, which has
// b_rows <= b_period rows (the rest read as zero); the router's weight gradient stacks three
// bf16 parts of dL/dlogits against x this way.
cudaError_t enqueue_wgrad_bf16(const void* a, const void* b, const int32_t* offsets, int E,
                               int64_t rows_max, int M, int N, float* out, int* status,
                               cudaStream_t stream, int splits = 1, int64_t b_period = 0,
                               int64_t b_rows = 0);
// Layer 1 for training: h = bf16(GeLU(W x + b)) and g = bf16(GeLU'(W x + b)), both [rows, N].
cudaError_t enqueue_grouped_gemm_bf16_train(const void* x, const int32_t* offsets, int E,
                                            int64_t rows_max, int K, int N, const void* w,
                                            const void* bias, void* h_out, void* g_out,
                                            int64_t capacity_hint, int* status,
                                            cudaStream_t stream);
// Backward data GEMM: out[r, n] = sum_k w_t[e][k][n] * dy[r, k] for the rows of expert e, with
// w_t the weight stored [E][K][N] (W1 [E][d_ff][d] gives dx = dz W1; W2 [E][d][d_ff] gives
// dh = dy W2). g_in (bf16 [rows, N]) given: out = bf16(result * g_in), else out fp32.
cudaError_t enqueue_grouped_gemm_dgrad_bf16(const void* dy, const int32_t* offsets, int E,
                                            int64_t rows_max, int K, int N, const void* w_t,
                                            const void* g_in, void* out, int64_t capacity_hint,
                                            int* status, cudaStream_t stream);
cudaError_t enqueue_grouped_gemm_bf16(const void* x, const int32_t* offsets, int E,
                                      int64_t rows_max, int K, int N, const void* w,
                                      const void* bias, bool gelu, void* out,
                                      int64_t capacity_hint, int* status, cudaStream_t stream);
// gelu_grad_out (optional, GeLU layer): also writes GeLU'(z) for the backward pass.
cudaError_t enqueue_grouped_gemm_f32(const float* x, const int32_t* offsets, int E,
                                     int64_t rows_max, int K, int N, const float* w,
                                     const float* bias, bool gelu, float* out, int* status,
                                     cudaStream_t stream, float* gelu_grad_out = nullptr);
// Layer 2 with the combine fused into its epilogue (bf16 layers):
//   dense == false: top-1 experts; row r of the packed buffer belongs to token row_token[r]:
//                   out[t] = [residual[t]] + gates[t] * (W2[e] h[r] + b2[e])
//   dense == true:  the PR-MoE dense MLP's layer 2 over all T tokens (offsets == nullptr, E == 1):
//                   out[t] = [residual[t]] + (W2d h[t] + b2d) + sum_{j kept} gates[t,j] * y[row_j]
struct FusedCombine {
  bool dense;
  const int32_t* row_token;
  const int32_t* slot;
  const int32_t* ids;
  const int32_t* offsets;   // expert offsets (dense mode)
  const float* gates;
  const float* y;           // expert outputs [rows_y, d] (dense mode)
  int64_t rows_y;
  const void* residual;     // bf16 x or nullptr
  void* out;
  bool out_bf16;
  int k, E_experts;
};
cudaError_t enqueue_gemm2_combine(const void* h, const int32_t* offsets, int E, int64_t rows_max,
                                  int K, int N, const void* w, const void* bias,
                                  const FusedCombine& fc, int64_t capacity_hint, int* status,
                                  cudaStream_t stream);
cudaError_t enqueue_expert_ffn_bf16(const void* x_packed, const int32_t* offsets, int E,
                                    int64_t rows_max, int d, int d_ff, const void* w1,
                                    const void* b1, const void* w2, const void* b2, void* h_packed,
                                    float* y_packed, int64_t capacity_hint, int* status,
                                    cudaStream_t stream);
cudaError_t enqueue_expert_ffn_f32(const float* x_packed, const int32_t* offsets, int E,
                                   int64_t rows_max, int d, int d_ff, const float* w1,
                                   const float* b1, const float* w2, const float* b2,
                                   float* h_packed, float* y_packed, int* status,
                                   cudaStream_t stream);
// Largest d_model / d_ff the fp32 FFN accepts (one activation row is staged in shared memory).
constexpr int kFfnF32MaxDim = 16384;

// ---------------------------------------------------------------- combine
cudaError_t enqueue_combine(const float* y_packed, const int32_t* offsets, const int32_t* ids,
                            const int32_t* slot, const float* gates, int64_t T, int d, int E,
                            int k, int64_t rows_max, const void* residual, bool res_bf16,
                            const float* dense, void* out, bool out_bf16, int* status,
                            cudaStream_t stream);

// ---------------------------------------------------------------- backward
cudaError_t enqueue_combine_backward(const void* dout, bool bf16, const float* y_packed,
                                     const int32_t* offsets, const int32_t* ids,
                                     const int32_t* slot, const float* gates, int64_t T, int d,
                                     int E, int k, int64_t rows_max, float* dgate, void* dy,
                                     int* status, cudaStream_t stream);
// first_counts: the forward's first-choice counts per expert (f_e * T).
cudaError_t enqueue_router_backward(const float* logits, const int32_t* ids, const float* dgate,
                                    const unsigned* first_counts, int64_t T, int E, int k,
                                    float alpha, float aux_weight, float z_weight,
                                    bool renormalize, float* dl, cudaStream_t stream);
// Row splits for a column sum over segments of at most longest_segment rows.
int colsum_splits(int64_t longest_segment);
// out[e][n] = sum of X[r][n] over segment e (offsets == nullptr: one segment of rows_max rows);
// S > 1 needs partial [E * S * N].
cudaError_t enqueue_colsum(const void* X, bool bf16, const int32_t* offsets, int E,
                           int64_t rows_max, int N, int S, float* partial, float* out,
                           cudaStream_t stream);
// out[g][n] = sum_s part[g][s][n] for n < N, rows of part N_stride apart (0: N).
cudaError_t enqueue_split_reduce(const float* part, int64_t groups, int S, int64_t N, float* out,
                                 cudaStream_t stream, int64_t N_stride = 0);
// bf16 parts of dL/dlogits and W_r for the router's backward GEMMs on tensor cores:
// dl3 [3 Tpad, Epad] (hi; mid; lo stacked by rows), dlx [T, Kx] ([hi | mid | hi | 0]),
// wx [Kx, d] ([W_hi; W_hi; W_mid; 0]); Tpad % 64 == 0, Epad % 8 == 0, Kx = roundup(3E, 8).
cudaError_t enqueue_router_bwd_split(const float* dl, int64_t T, int64_t Tpad, int E, int Epad,
                                     int Kx, uint16_t* dl3, uint16_t* dlx, const float* w_router,
                                     int d, uint16_t* wx, cudaStream_t stream);
cudaError_t enqueue_dx_gather(const void* dout, bool bf16, bool add_dout, const float* dense_dx,
                              const float* dxp, const int32_t* offsets, const int32_t* ids,
                              const int32_t* slot, int64_t T, int d, int E, int k,
                              int64_t rows_max, const float* dx_router, void* dx,
                              cudaStream_t stream);
// fp32 FMA GEMM C(m, n) = sum_k A(m, k) B(k, n) per expert e (blockIdx.z = e * splits + s):
// A(m, k) at a[e * a_e + m * a_m + k * a_k] (bf16 or fp32), B(k, n) at b[e * b_e + k * b_k +
// n * b_n], C at c (fp32) or c16 (bf16) [e * c_e + s * split_stride + m * c_m + n * c_n], times
// mul at the same index when given. ragged = 1: M is the rows of segment e and the m index of A
// and C is offset by the segment start; ragged = 2: the same for K and the k index of A and B.
struct SimtGemm {
  int64_t M = 0, N = 0, K = 0;
  int ragged = 0;
  const int32_t* offsets = nullptr;
  int E = 1;
  int64_t rows_max = 0;
  const void* a = nullptr;
  int a_bf16 = 0;
  int64_t a_e = 0, a_m = 0, a_k = 0;
  const void* b = nullptr;
  int b_bf16 = 0;
  int64_t b_e = 0, b_k = 0, b_n = 0;
  float* c = nullptr;
  uint16_t* c16 = nullptr;
  int64_t c_e = 0, c_m = 0, c_n = 0;
  const void* mul = nullptr;
  int mul_bf16 = 0;
  int splits = 1;
  int64_t split_stride = 0;
};
// m_extent: the largest M over the experts (grid rows).
cudaError_t enqueue_simt_gemm(const SimtGemm& p, int64_t m_extent, cudaStream_t stream);

}  // namespace moe
