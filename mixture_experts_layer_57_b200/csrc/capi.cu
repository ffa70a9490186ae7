// C ABI of the MoE-layer forward pass: argument validation, workspace layout, fault injection
// and launch accounting around the kernels' enqueue functions. See include/moe.h.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <utility>

#include "kernels.h"

namespace moe {

namespace {
thread_local int g_launches = 0;
}

void count_launch() { ++g_launches; }
void reset_launch_count() { g_launches = 0; }

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("MOE_PDL");
    return !(v != nullptr && v[0] == '0');
  }();
  return on;
}

// Whether the tensor-core router runs softmax, top-k and the statistics in its own epilogue
// (MOE_FUSED_ROUTER=0: a separate top-k kernel reads the logits back; both give the same bits).
// Read at every call.
bool router_fusion_enabled() {
  const char* v = std::getenv("MOE_FUSED_ROUTER");
  return !(v != nullptr && v[0] == '0');
}

// Whether bf16 PR-MoE layers co-schedule each expert GEMM layer with the dense MLP's layer in one
// launch (MOE_COSCHEDULE=0 runs them one after another, the dense layer 2 with the combine fused;
// both give the same bits). Read at every call.
bool coschedule_enabled() {
  const char* v = std::getenv("MOE_COSCHEDULE");
  return !(v != nullptr && v[0] == '0');
}

// Whether expert GEMMs with 256-column tiles run as two-SM CTA pairs that share each B tile
// (MOE_PAIR_MMA=0: one CTA per tile; both give the same bits). Read at every call.
bool pair_mma_enabled() {
  const char* v = std::getenv("MOE_PAIR_MMA");
  return !(v != nullptr && v[0] == '0');
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

}  // namespace moe

using namespace moe;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

bool fault_injected(const char* entry) {
  const char* v = std::getenv("MOE_FAULT_INJECT");
  return v != nullptr && std::strcmp(v, entry) == 0;
}

size_t esize(moe_dtype dt) { return dt == MOE_BF16 ? 2 : 4; }

bool valid_dtype(moe_dtype dt) { return dt == MOE_F32 || dt == MOE_BF16; }

// Bump allocator over the caller's workspace; the first kAlign bytes are the status block.
struct Carve {
  uint8_t* base;
  size_t off = kAlign;
  template <class T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += align_up(count * sizeof(T));
    return p;
  }
};

// ------------------------------------------------------------ workspace layouts

struct RouterWs {
  RouterScratch scr;
  float* logits;
};
RouterWs carve_router(Carve& c, int64_t T, int E, int d) {
  RouterWs w;
  w.scr.acc.q = c.take<unsigned long long>((size_t)E);
  w.scr.acc.c = c.take<unsigned>((size_t)E);
  w.scr.acc.imp = c.take<unsigned long long>((size_t)E);
  w.scr.acc.load = c.take<unsigned>((size_t)E);
  w.scr.acc.z = c.take<unsigned long long>(1);
  w.scr.acc.ticket = c.take<unsigned>(1);
  w.scr.w_split = c.take<uint16_t>((size_t)E * 3 * router_split_dpad(d));
  w.logits = c.take<float>((size_t)T * E);
  w.scr.logits_scratch = w.logits;
  return w;
}

struct DispatchWs {
  int32_t *local_rank, *seg_counts, *seg_base;
  uint64_t* prio_keys;       // overflow by priority: [2 T k] ping-pong sort keys
  int32_t* demand_offsets;   // overflow by priority: [E + 1]
};
DispatchWs carve_dispatch(Carve& c, int64_t T, int E, int k) {
  // segments of 256 pairs (counting kernel) or of one 64-token router block (layer forward)
  const int64_t nseg = dispatch_num_segments(T * k) > router_num_blocks(T)
                           ? dispatch_num_segments(T * k)
                           : router_num_blocks(T);
  DispatchWs w;
  w.local_rank = c.take<int32_t>((size_t)T * k);
  w.seg_counts = c.take<int32_t>((size_t)nseg * E);
  w.seg_base = c.take<int32_t>((size_t)nseg * E);
  w.prio_keys = c.take<uint64_t>((size_t)2 * T * k);
  w.demand_offsets = c.take<int32_t>((size_t)E + 1);
  return w;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// ------------------------------------------------------------ shared validation

moe_status check_router_shape(int64_t T, int d, int E, int k) {
  if (T < 0 || d < 1 || E < 1 || k < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (k > E) return MOE_ERR_INVALID_ARGUMENT;
  if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (T * (int64_t)k >= (int64_t)INT32_MAX || T * (int64_t)E >= ((int64_t)1 << 40))
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_ffn_shape(int E, int64_t rows_max, int d, int d_ff, moe_dtype dt) {
  if (E < 1 || rows_max < 0 || d < 1 || d_ff < 1 || !valid_dtype(dt)) return MOE_ERR_INVALID_ARGUMENT;
  if (E > MOE_MAX_EXPERTS || rows_max >= (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if ((int64_t)E * d >= (int64_t)INT32_MAX || (int64_t)E * d_ff >= (int64_t)INT32_MAX)
    return MOE_ERR_UNSUPPORTED;
  if (dt == MOE_BF16 && (d % 8 != 0 || d_ff % 8 != 0)) return MOE_ERR_UNSUPPORTED;
  if (dt == MOE_F32 && (d > kFfnF32MaxDim || d_ff > kFfnF32MaxDim)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARGUMENT: return "MOE_ERR_INVALID_ARGUMENT";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "MOE_ERR_WORKSPACE_TOO_SMALL";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_FLAG: return "MOE_ERR_DEVICE_FLAG";
    case MOE_ERR_MISALIGNED: return "MOE_ERR_MISALIGNED";
  }
  return "MOE_ERR_UNKNOWN";
}

int moe_abi_version(void) { return MOE_ABI_VERSION; }

int moe_last_launch_count(void) { return g_launches; }

moe_status moe_selftest_bounded_wait(void* ws, size_t ws_bytes, uint64_t wait_limit_ns,
                                     moe_stream_t stream) {
  if (!ws || wait_limit_ns < 1000 || wait_limit_ns > 10000000000ull) return MOE_ERR_INVALID_ARGUMENT;
  if (((uintptr_t)ws % kAlign) != 0) return MOE_ERR_MISALIGNED;
  if (ws_bytes < MOE_SELFTEST_WS_BYTES) return MOE_ERR_WORKSPACE_TOO_SMALL;
  g_launches = 0;
  return cuda_status(enqueue_selftest_bounded_wait((uint8_t*)ws + kAlign, wait_limit_ns, (int*)ws,
                                                   stream));
}

moe_status moe_capacity(int64_t T, int E, int k, double capacity_factor, int64_t* C_out) {
  if (!C_out || T < 0 || E < 1 || k < 1 || !std::isfinite(capacity_factor) || capacity_factor < 0)
    return MOE_ERR_INVALID_ARGUMENT;
  // k T / E first, then the factor; a product within 8 ulps above an integer is that integer
  // (the factor is a decimal number held in binary, e.g. 1.1 is stored slightly above 1.1)
  const double v = ((double)k * (double)T / (double)E) * capacity_factor;
  const double fl = std::floor(v);
  const double c = (v - fl <= 8.0 * (std::nextafter(v, INFINITY) - v)) ? fl : std::ceil(v);
  if (c > 9.0e18) return MOE_ERR_UNSUPPORTED;
  *C_out = (int64_t)c;
  return MOE_OK;
}

moe_status moe_packed_rows_max(int64_t T, int E, int k, int64_t C, int64_t* rows_out) {
  if (!rows_out || T < 0 || E < 1 || k < 1 || C < 0) return MOE_ERR_INVALID_ARGUMENT;
  const int64_t a = T * k;
  // min(T k, E C); when C >= T k the minimum is T k (E >= 1), which also avoids overflow
  *rows_out = C >= a ? a : ((int64_t)E * C < a ? (int64_t)E * C : a);
  return MOE_OK;
}

// ---------------------------------------------------------------- router

moe_status moe_router_workspace_bytes(int64_t T, int E, int d_model, size_t* bytes) {
  if (!bytes || T < 0 || E < 1 || d_model < 1) return MOE_ERR_INVALID_ARGUMENT;
  Carve c{nullptr};
  carve_router(c, T, E, d_model);
  *bytes = c.off;
  return MOE_OK;
}

namespace {
moe_status router_topk_impl(const char* entry, const void* x, moe_dtype x_dtype, int64_t T,
                            int d_model, const float* w_router, const float* router_bias, int E,
                            int k, float* logits, int32_t* expert_ids, float* gates,
                            float* lb_stats, float aux_alpha, int renormalize,
                            float* router_losses, float* probs, void* ws, size_t ws_bytes,
                            moe_stream_t stream) {
  if (!valid_dtype(x_dtype)) return MOE_ERR_INVALID_ARGUMENT;
  moe_status st = check_router_shape(T, d_model, E, k);
  if (st != MOE_OK) return st;
  if (T > 0 && (!x || !w_router || !expert_ids || !gates)) return MOE_ERR_INVALID_ARGUMENT;
  if (!ws) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(router_bias) || !aligned16(logits) ||
      !aligned16(expert_ids) || !aligned16(gates) || !aligned16(lb_stats) ||
      !aligned16(router_losses) || !aligned16(probs) || ((uintptr_t)ws % kAlign) != 0)
    return MOE_ERR_MISALIGNED;
  size_t need = 0;
  moe_router_workspace_bytes(T, E, d_model, &need);
  if (ws_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (fault_injected(entry)) return MOE_ERR_CUDA;
  g_launches = 0;
  if (T == 0) return MOE_OK;
  Carve c{(uint8_t*)ws};
  RouterWs w = carve_router(c, T, E, d_model);
  return cuda_status(enqueue_router(x, x_dtype == MOE_BF16, T, d_model, w_router, router_bias, E,
                                    k, logits, expert_ids, gates, lb_stats, aux_alpha, w.scr,
                                    (int*)ws, stream, RouterDispatchCount{}, renormalize != 0,
                                    router_losses, nullptr, -1, probs));
}
}  // namespace

moe_status moe_router_prepare_bytes(int E, int d_model, size_t* bytes) {
  if (!bytes || E < 1 || d_model < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  *bytes = (size_t)E * 3 * router_split_dpad(d_model) * sizeof(uint16_t);
  return MOE_OK;
}

moe_status moe_router_prepare(const float* w_router, int E, int d_model, void* w_prepared,
                              size_t bytes, moe_stream_t stream) {
  size_t need = 0;
  moe_status st = moe_router_prepare_bytes(E, d_model, &need);
  if (st != MOE_OK) return st;
  if (!w_router || !w_prepared) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(w_router) || !aligned16(w_prepared)) return MOE_ERR_MISALIGNED;
  if (bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (fault_injected("moe_router_prepare")) return MOE_ERR_CUDA;
  g_launches = 0;
  return cuda_status(enqueue_router_prepare(w_router, E, d_model, (uint16_t*)w_prepared, stream));
}

moe_status moe_router_topk(const void* x, moe_dtype x_dtype, int64_t T, int d_model,
                           const float* w_router, const float* router_bias, int E, int k,
                           float* logits, int32_t* expert_ids, float* gates, float* lb_stats,
                           float aux_alpha, void* ws, size_t ws_bytes, moe_stream_t stream) {
  return router_topk_impl("moe_router_topk", x, x_dtype, T, d_model, w_router, router_bias, E, k,
                          logits, expert_ids, gates, lb_stats, aux_alpha, 0, nullptr, nullptr, ws,
                          ws_bytes, stream);
}

moe_status moe_router_topk_ex(const void* x, moe_dtype x_dtype, int64_t T, int d_model,
                              const float* w_router, const float* router_bias, int E, int k,
                              float* logits, int32_t* expert_ids, float* gates, float* lb_stats,
                              float aux_alpha, int renormalize, float* router_losses,
                              float* probs, void* ws, size_t ws_bytes, moe_stream_t stream) {
  return router_topk_impl("moe_router_topk_ex", x, x_dtype, T, d_model, w_router, router_bias, E,
                          k, logits, expert_ids, gates, lb_stats, aux_alpha, renormalize,
                          router_losses, probs, ws, ws_bytes, stream);
}

// ---------------------------------------------------------------- dispatch

moe_status moe_dispatch_workspace_bytes(int64_t T, int E, int k, size_t* bytes) {
  if (!bytes || T < 0 || E < 1 || k < 1) return MOE_ERR_INVALID_ARGUMENT;
  Carve c{nullptr};
  carve_dispatch(c, T, E, k);
  *bytes = c.off;
  return MOE_OK;
}

namespace {
moe_status dispatch_impl(const char* entry, const void* x, moe_dtype dtype, int64_t T,
                         int d_model, const int32_t* expert_ids, const float* prio_probs, int E,
                         int k, int64_t C, int32_t* slot, int32_t* expert_counts,
                         int32_t* expert_offsets, int32_t* row_token, void* x_packed,
                         int64_t rows_max, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!valid_dtype(dtype) || C < 0) return MOE_ERR_INVALID_ARGUMENT;
  moe_status st = check_router_shape(T, d_model, E, k);
  if (st != MOE_OK) return st;
  int64_t need_rows = 0;
  moe_packed_rows_max(T, E, k, C, &need_rows);
  if (rows_max < need_rows) return MOE_ERR_INVALID_ARGUMENT;
  if (rows_max >= (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if (dtype == MOE_BF16 && d_model % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (!expert_counts || !expert_offsets || !ws) return MOE_ERR_INVALID_ARGUMENT;
  if (T > 0 && (!x || !expert_ids || !slot)) return MOE_ERR_INVALID_ARGUMENT;
  if (rows_max > 0 && (!row_token || !x_packed)) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(expert_ids) || !aligned16(slot) || !aligned16(expert_counts) ||
      !aligned16(expert_offsets) || !aligned16(row_token) || !aligned16(x_packed) ||
      !aligned16(prio_probs) || ((uintptr_t)ws % kAlign) != 0)
    return MOE_ERR_MISALIGNED;
  size_t need = 0;
  moe_dispatch_workspace_bytes(T, E, k, &need);
  if (ws_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (fault_injected(entry)) return MOE_ERR_CUDA;
  g_launches = 0;
  Carve c{(uint8_t*)ws};
  DispatchWs w = carve_dispatch(c, T, E, k);
  PriorityDispatch prio;
  prio.probs = prio_probs;
  prio.keys = w.prio_keys;
  prio.demand_offsets = w.demand_offsets;
  return cuda_status(enqueue_dispatch(x, dtype == MOE_BF16, T, d_model, expert_ids, E, k, C, slot,
                                      expert_counts, expert_offsets, row_token, x_packed, rows_max,
                                      w.local_rank, w.seg_counts, w.seg_base, (int*)ws, stream,
                                      DroppedRows{}, 0, prio));
}
}  // namespace

moe_status moe_dispatch(const void* x, moe_dtype dtype, int64_t T, int d_model,
                        const int32_t* expert_ids, int E, int k, int64_t C, int32_t* slot,
                        int32_t* expert_counts, int32_t* expert_offsets, int32_t* row_token,
                        void* x_packed, int64_t rows_max, void* ws, size_t ws_bytes,
                        moe_stream_t stream) {
  return dispatch_impl("moe_dispatch", x, dtype, T, d_model, expert_ids, nullptr, E, k, C, slot,
                       expert_counts, expert_offsets, row_token, x_packed, rows_max, ws, ws_bytes,
                       stream);
}

moe_status moe_dispatch_priority(const void* x, moe_dtype dtype, int64_t T, int d_model,
                                 const int32_t* expert_ids, const float* probs, int E, int k,
                                 int64_t C, int32_t* slot, int32_t* expert_counts,
                                 int32_t* expert_offsets, int32_t* row_token, void* x_packed,
                                 int64_t rows_max, void* ws, size_t ws_bytes,
                                 moe_stream_t stream) {
  if (T > 0 && !probs) return MOE_ERR_INVALID_ARGUMENT;
  return dispatch_impl("moe_dispatch_priority", x, dtype, T, d_model, expert_ids,
                       T > 0 ? probs : nullptr, E, k, C, slot, expert_counts, expert_offsets,
                       row_token, x_packed, rows_max, ws, ws_bytes, stream);
}

// ---------------------------------------------------------------- expert FFN

moe_status moe_expert_ffn_workspace_bytes(size_t* bytes) {
  if (!bytes) return MOE_ERR_INVALID_ARGUMENT;
  *bytes = kAlign;
  return MOE_OK;
}

moe_status moe_expert_ffn(const void* x_packed, const int32_t* expert_offsets, int E,
                          int64_t rows_max, int d_model, int d_ff, moe_dtype dtype, const void* w1,
                          const void* b1, const void* w2, const void* b2, void* h_packed,
                          float* y_packed, int64_t capacity_hint, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
  moe_status st = check_ffn_shape(E, rows_max, d_model, d_ff, dtype);
  if (st != MOE_OK) return st;
  if (capacity_hint < 0 || !expert_offsets || !w1 || !w2 || !ws) return MOE_ERR_INVALID_ARGUMENT;
  if (rows_max > 0 && (!x_packed || !h_packed || !y_packed)) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(x_packed) || !aligned16(expert_offsets) || !aligned16(w1) || !aligned16(b1) ||
      !aligned16(w2) || !aligned16(b2) || !aligned16(h_packed) || !aligned16(y_packed) ||
      ((uintptr_t)ws % kAlign) != 0)
    return MOE_ERR_MISALIGNED;
  if (ws_bytes < kAlign) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (fault_injected("moe_expert_ffn")) return MOE_ERR_CUDA;
  g_launches = 0;
  if (rows_max == 0) return MOE_OK;
  if (dtype == MOE_BF16)
    return cuda_status(enqueue_expert_ffn_bf16(x_packed, expert_offsets, E, rows_max, d_model, d_ff,
                                               w1, b1, w2, b2, h_packed, y_packed, capacity_hint,
                                               (int*)ws, stream));
  return cuda_status(enqueue_expert_ffn_f32((const float*)x_packed, expert_offsets, E, rows_max,
                                            d_model, d_ff, (const float*)w1, (const float*)b1,
                                            (const float*)w2, (const float*)b2, (float*)h_packed,
                                            y_packed, (int*)ws, stream));
}

moe_status moe_grouped_gemm(const void* x_packed, const int32_t* expert_offsets, int E,
                            int64_t rows_max, int K, int N, moe_dtype dtype, const void* w,
                            const void* bias, moe_epilogue epilogue, void* out,
                            int64_t capacity_hint, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_ffn_shape(E, rows_max, K, N, dtype);
  if (st != MOE_OK) return st;
  if (epilogue != MOE_EPILOGUE_BIAS_GELU && epilogue != MOE_EPILOGUE_BIAS)
    return MOE_ERR_INVALID_ARGUMENT;
  if (capacity_hint < 0 || !expert_offsets || !w || !ws) return MOE_ERR_INVALID_ARGUMENT;
  if (rows_max > 0 && (!x_packed || !out)) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(x_packed) || !aligned16(expert_offsets) || !aligned16(w) || !aligned16(bias) ||
      !aligned16(out) || ((uintptr_t)ws % kAlign) != 0)
    return MOE_ERR_MISALIGNED;
  if (ws_bytes < kAlign) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (fault_injected("moe_grouped_gemm")) return MOE_ERR_CUDA;
  g_launches = 0;
  const bool gelu = epilogue == MOE_EPILOGUE_BIAS_GELU;
  if (dtype == MOE_BF16)
    return cuda_status(enqueue_grouped_gemm_bf16(x_packed, expert_offsets, E, rows_max, K, N, w,
                                                 bias, gelu, out, capacity_hint, (int*)ws, stream));
  return cuda_status(enqueue_grouped_gemm_f32((const float*)x_packed, expert_offsets, E, rows_max,
                                              K, N, (const float*)w, (const float*)bias, gelu,
                                              (float*)out, (int*)ws, stream));
}

// ---------------------------------------------------------------- combine

moe_status moe_combine_workspace_bytes(size_t* bytes) {
  if (!bytes) return MOE_ERR_INVALID_ARGUMENT;
  *bytes = kAlign;
  return MOE_OK;
}

moe_status moe_combine(const float* y_packed, const int32_t* expert_offsets,
                       const int32_t* expert_ids, const int32_t* slot, const float* gates,
                       int64_t T, int d_model, int E, int k, int64_t rows_max,
                       const void* residual, moe_dtype res_dtype, const float* dense, void* out,
                       moe_dtype out_dtype, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!valid_dtype(res_dtype) || !valid_dtype(out_dtype) || rows_max < 0)
    return MOE_ERR_INVALID_ARGUMENT;
  moe_status st = check_router_shape(T, d_model, E, k);
  if (st != MOE_OK) return st;
  if (!ws || !expert_offsets) return MOE_ERR_INVALID_ARGUMENT;
  if (T > 0 && (!expert_ids || !slot || !gates || !out)) return MOE_ERR_INVALID_ARGUMENT;
  if (rows_max > 0 && !y_packed) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(y_packed) || !aligned16(expert_offsets) || !aligned16(expert_ids) ||
      !aligned16(slot) || !aligned16(gates) || !aligned16(residual) || !aligned16(dense) ||
      !aligned16(out) || ((uintptr_t)ws % kAlign) != 0)
    return MOE_ERR_MISALIGNED;
  if (ws_bytes < kAlign) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (fault_injected("moe_combine")) return MOE_ERR_CUDA;
  g_launches = 0;
  return cuda_status(enqueue_combine(y_packed, expert_offsets, expert_ids, slot, gates, T, d_model,
                                     E, k, rows_max, residual, res_dtype == MOE_BF16, dense, out,
                                     out_dtype == MOE_BF16, (int*)ws, stream));
}

// ---------------------------------------------------------------- whole layer

namespace {

struct LayerWs {
  RouterWs router;
  DispatchWs dispatch;
  float *gates, *probs, *lb_stats;
  int32_t *ids, *slot, *counts, *offsets, *row_token;
  void *x_packed, *h_packed;
  float* y_packed;
  void* h_dense;
  float* r_dense;
  int32_t* cap_local;
  int64_t C, rows_max;
};

// T_cap: the batch the capacity is computed from (T, or the whole batch of a token shard).
moe_status layer_layout(const moe_layer_args* a, uint8_t* base, LayerWs* w, size_t* bytes,
                        int64_t T_cap = -1) {
  if (!a) return MOE_ERR_INVALID_ARGUMENT;
  if (T_cap < 0) T_cap = a->T;
  if (T_cap < a->T) return MOE_ERR_INVALID_ARGUMENT;
  moe_status st = check_router_shape(a->T, a->d_model, a->E, a->k);
  if (st != MOE_OK) return st;
  if (!valid_dtype(a->dtype) || !valid_dtype(a->out_dtype)) return MOE_ERR_INVALID_ARGUMENT;
  if (a->overflow_policy != MOE_OVERFLOW_FIRST_COME && a->overflow_policy != MOE_OVERFLOW_PRIORITY)
    return MOE_ERR_INVALID_ARGUMENT;
  st = moe_capacity(T_cap, a->E, a->k, a->capacity_factor, &w->C);
  if (st != MOE_OK) return st;
  moe_packed_rows_max(a->T, a->E, a->k, w->C, &w->rows_max);
  st = check_ffn_shape(a->E, w->rows_max, a->d_model, a->d_ff, a->dtype);
  if (st != MOE_OK) return st;
  if (a->T >= (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  const int64_t T = a->T, R = w->rows_max;
  const int E = a->E, k = a->k, d = a->d_model, f = a->d_ff;
  const size_t es = esize(a->dtype);
  Carve c{base};
  w->router = carve_router(c, T, E, d);
  w->dispatch = carve_dispatch(c, T, E, k);
  w->gates = c.take<float>((size_t)T * k);
  w->probs = c.take<float>((size_t)T * k);
  w->lb_stats = c.take<float>((size_t)2 * E + 1);
  w->ids = c.take<int32_t>((size_t)T * k);
  w->slot = c.take<int32_t>((size_t)T * k);
  w->counts = c.take<int32_t>((size_t)E);
  w->offsets = c.take<int32_t>((size_t)E + 1);
  w->cap_local = c.take<int32_t>((size_t)E);
  w->row_token = c.take<int32_t>((size_t)R);
  w->x_packed = c.take<uint8_t>((size_t)R * d * es);
  w->h_packed = c.take<uint8_t>((size_t)R * f * es);
  w->y_packed = c.take<float>((size_t)R * d);
  const bool dense = a->dense_w1 != nullptr;
  w->h_dense = dense ? (void*)c.take<uint8_t>((size_t)T * f * es) : nullptr;
  // the dense MLP's fp32 output, read by the combine kernel (fp32 layers, and bf16 layers whose
  // dense layers are co-scheduled with the experts'; otherwise the combine is fused into the
  // dense layer 2 epilogue)
  w->r_dense = dense ? c.take<float>((size_t)T * d) : nullptr;
  *bytes = c.off;
  return MOE_OK;
}

}  // namespace

moe_status moe_layer_workspace_bytes(const moe_layer_args* args, size_t* bytes) {
  if (!bytes) return MOE_ERR_INVALID_ARGUMENT;
  LayerWs w;
  return layer_layout(args, nullptr, &w, bytes);
}

}  // extern "C"

namespace {

// Records caller-created CUDA events at stage boundaries (moe_layer_forward_profiled).
struct StageRecorder {
  void* const* events = nullptr;
  int max_events = 0;
  int n = 0;
  char* names = nullptr;
  size_t names_len = 0;
  size_t used = 0;
  cudaStream_t stream = nullptr;
  void mark(const char* name) {
    if (events == nullptr || n >= max_events) return;
    cudaEventRecord((cudaEvent_t)events[n], stream);
    ++n;
    if (names != nullptr && names_len > 0) {
      const size_t len = std::strlen(name);
      if (used + len + 2 <= names_len) {
        if (used > 0) names[used++] = ',';
        std::memcpy(names + used, name, len);
        used += len;
        names[used] = '\0';
      }
    }
  }
};

// A token shard's half of the layer (moe_layer_forward_shard_begin / _end), or the whole layer.
enum ShardMode { kWhole = 0, kShardBegin = 1, kShardEnd = 2 };
struct ShardCall {
  ShardMode mode = kWhole;
  int64_t T_global = -1;
  int32_t* demand_out = nullptr;    // begin
  int64_t* partials_out = nullptr;  // begin
  const int32_t* demand_all = nullptr;  // end
  const int64_t* totals = nullptr;      // end
  int G = 1, rank = 0;                  // end
};

moe_status layer_forward_impl(const moe_layer_args* a, void* out, moe_layer_aux* aux, void* ws,
                              size_t ws_bytes, moe_stream_t stream, StageRecorder& rec,
                              const ShardCall& sh = ShardCall{}) {
  LayerWs w;
  size_t need = 0;
  moe_status st = layer_layout(a, (uint8_t*)ws, &w, &need, sh.T_global);
  if (st != MOE_OK) return st;
  if (sh.mode != kWhole && a->overflow_policy != MOE_OVERFLOW_FIRST_COME)
    return MOE_ERR_UNSUPPORTED;  // a global priority order would need every shard's gates
  const bool dense = a->dense_w1 != nullptr;
  if (dense && !a->dense_w2) return MOE_ERR_INVALID_ARGUMENT;
  if (!ws) return MOE_ERR_INVALID_ARGUMENT;
  if (a->T > 0 && (!a->x || !a->w_router || !a->w1 || !a->w2 || (!out && sh.mode != kShardBegin)))
    return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(a->x) || !aligned16(a->w_router) || !aligned16(a->router_bias) ||
      !aligned16(a->w1) || !aligned16(a->b1) || !aligned16(a->w2) || !aligned16(a->b2) ||
      !aligned16(a->dense_w1) || !aligned16(a->dense_b1) || !aligned16(a->dense_w2) ||
      !aligned16(a->dense_b2) || !aligned16(out) || !aligned16(a->w_router_prepared) ||
      ((uintptr_t)ws % kAlign) != 0)
    return MOE_ERR_MISALIGNED;
  if (aux && (!aligned16(aux->logits) || !aligned16(aux->expert_ids) || !aligned16(aux->gates) ||
              !aligned16(aux->slot) || !aligned16(aux->expert_counts) ||
              !aligned16(aux->expert_offsets) || !aligned16(aux->lb_stats) ||
              !aligned16(aux->router_losses) || !aligned16(aux->topk_probs)))
    return MOE_ERR_MISALIGNED;
  if (ws_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  const char* entry = sh.mode == kShardBegin ? "moe_layer_forward_shard_begin"
                      : sh.mode == kShardEnd ? "moe_layer_forward_shard_end"
                                             : "moe_layer_forward";
  if (fault_injected(entry)) return MOE_ERR_CUDA;
  g_launches = 0;
  if (a->T == 0) {
    if (sh.mode == kShardBegin) {  // an empty shard demands nothing and adds nothing
      if (cudaMemsetAsync(sh.demand_out, 0, sizeof(int32_t) * a->E, stream) != cudaSuccess ||
          cudaMemsetAsync(sh.partials_out, 0, sizeof(int64_t) * router_partials_count(a->E),
                          stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    if (sh.mode == kShardEnd && aux &&
        enqueue_router_finalize(sh.totals, sh.T_global, a->E, a->aux_alpha, aux->lb_stats,
                                aux->router_losses, stream) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (sh.mode != kShardBegin && aux) {  // no demand and no packed rows
      if (aux->expert_counts &&
          cudaMemsetAsync(aux->expert_counts, 0, sizeof(int32_t) * a->E, stream) != cudaSuccess)
        return MOE_ERR_CUDA;
      if (aux->expert_offsets &&
          cudaMemsetAsync(aux->expert_offsets, 0, sizeof(int32_t) * (a->E + 1), stream) !=
              cudaSuccess)
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
  }

  float* logits = aux ? aux->logits : nullptr;  // the router keeps its own scratch if needed
  int32_t* ids = aux && aux->expert_ids ? aux->expert_ids : w.ids;
  float* gates = aux && aux->gates ? aux->gates : w.gates;
  int32_t* slot = aux && aux->slot ? aux->slot : w.slot;
  int32_t* counts = aux && aux->expert_counts ? aux->expert_counts : w.counts;
  int32_t* offsets = aux && aux->expert_offsets ? aux->expert_offsets : w.offsets;
  float* lb = aux ? aux->lb_stats : nullptr;
  float* losses = aux ? aux->router_losses : nullptr;
  // the priority ranking key: the probabilities before renormalisation (the gates themselves
  // when they are not renormalised)
  const bool prio_on = a->overflow_policy == MOE_OVERFLOW_PRIORITY;
  float* probs = aux && aux->topk_probs ? aux->topk_probs
                 : (prio_on && a->renormalize_gates) ? w.probs
                                                     : nullptr;
  const float* prio_key = a->renormalize_gates ? probs : gates;
  int* status = (int*)ws;
  const bool bf16 = a->dtype == MOE_BF16;
  const int64_t T = a->T;
  const int d = a->d_model, f = a->d_ff, E = a->E, k = a->k;

  rec.stream = stream;
  rec.mark("start");
  cudaError_t e = cudaSuccess;
  if (sh.mode != kShardEnd) {
    // the router's top-k kernel also ranks each 64-token segment's pairs for dispatch; a shard
    // exports its integer statistics instead of finalising them
    RouterDispatchCount dcount;
    dcount.local_rank = w.dispatch.local_rank;
    dcount.seg_counts = w.dispatch.seg_counts;
    const bool begin = sh.mode == kShardBegin;
    // the statistics are left as integer accumulators: the dispatch scan finalises them below,
    // off the router's critical path (a shard exports them instead)
    e = enqueue_router(a->x, bf16, T, d, a->w_router, a->router_bias, E, k, logits, ids, gates,
                       nullptr, a->aux_alpha, w.router.scr, status, stream, dcount,
                       a->renormalize_gates != 0, nullptr, begin ? sh.partials_out : nullptr,
                       sh.T_global, probs, (const uint16_t*)a->w_router_prepared,
                       losses != nullptr);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    rec.mark("router");
  }
  if (sh.mode == kShardBegin) {
    // the shard's demand per expert (what the other shards need for their global slot base)
    e = enqueue_dispatch(a->x, bf16, T, d, ids, E, k, w.C, slot, sh.demand_out, offsets,
                         w.row_token, w.x_packed, w.rows_max, w.dispatch.local_rank,
                         w.dispatch.seg_counts, w.dispatch.seg_base, status, stream,
                         DroppedRows{}, (int)kRouterTokensPerBlock * k, PriorityDispatch{},
                         ShardBase{}, true);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    rec.mark("demand");
    return MOE_OK;
  }
  ShardBase shard;
  if (sh.mode == kShardEnd) {
    e = enqueue_router_finalize(sh.totals, sh.T_global, E, a->aux_alpha, lb, losses, stream);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    shard.demand_all = sh.demand_all;
    shard.G = sh.G;
    shard.rank = sh.rank;
    shard.cap_local = w.cap_local;
  }

  // bf16 layers fuse the combine into a layer-2 epilogue: the PR-MoE dense MLP's (any k, experts
  // run first) or, without the dense branch, the top-1 experts' (dropped tokens are then written
  // by dispatch). Other layers use the gather combine kernel.
  const bool fuse_dense = bf16 && dense;
  const bool fuse_expert = bf16 && !dense && k == 1;
  const bool out_bf16 = a->out_dtype == MOE_BF16;
  const void* residual = a->add_input_residual ? a->x : nullptr;
  DroppedRows dropped;
  if (fuse_expert) {
    dropped.out = out;
    dropped.out_bf16 = out_bf16;
    dropped.add_x = a->add_input_residual != 0;
  }
  PriorityDispatch prio;
  if (prio_on) {
    prio.probs = prio_key;
    prio.keys = w.dispatch.prio_keys;
    prio.demand_offsets = w.dispatch.demand_offsets;
  }
  StatsFinalize fin;
  if (sh.mode == kWhole) {
    fin.acc = w.router.scr.acc;
    fin.T = T;
    fin.alpha = a->aux_alpha;
    fin.lb = lb;
    fin.losses = losses;
  }
  e = enqueue_dispatch(a->x, bf16, T, d, ids, E, k, w.C, slot, counts, offsets, w.row_token,
                       w.x_packed, w.rows_max, w.dispatch.local_rank, w.dispatch.seg_counts,
                       w.dispatch.seg_base, status, stream, dropped,
                       (int)kRouterTokensPerBlock * k, prio, shard, false, fin);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  rec.mark("dispatch");

  FusedCombine fc{};
  fc.row_token = w.row_token;
  fc.slot = slot;
  fc.ids = ids;
  fc.offsets = offsets;
  fc.gates = gates;
  fc.y = w.y_packed;
  fc.rows_y = w.rows_max;
  fc.residual = residual;
  fc.out = out;
  fc.out_bf16 = out_bf16;
  fc.k = k;
  fc.E_experts = E;

  // the tile width follows the whole batch, so a shard's rows get the whole batch's arithmetic
  const int64_t dense_hint = sh.T_global > T ? sh.T_global : T;
  if (fuse_dense && coschedule_enabled() && co_gemm_supported(w.C) && dense_hint >= 256) {
    // each expert layer co-scheduled with the dense MLP's layer (one launch per layer), then the
    // gather combine: out = [x] + dense + sum_j gate_j y_j, the fused epilogue's arithmetic
    e = enqueue_co_gemm_bf16(w.x_packed, offsets, E, w.rows_max, a->w1, a->b1, w.h_packed, w.C,
                             a->x, T, a->dense_w1, a->dense_b1, w.h_dense, d, f, true, status,
                             stream);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    rec.mark("experts_dense_gemm1");
    e = enqueue_co_gemm_bf16(w.h_packed, offsets, E, w.rows_max, a->w2, a->b2, w.y_packed, w.C,
                             w.h_dense, T, a->dense_w2, a->dense_b2, w.r_dense, f, d, false, status,
                             stream);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    rec.mark("experts_dense_gemm2");
    e = enqueue_combine(w.y_packed, offsets, ids, slot, gates, T, d, E, k, w.rows_max, residual,
                        bf16, w.r_dense, out, out_bf16, status, stream);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    rec.mark("combine");
    return MOE_OK;
  }
  if (fuse_dense) {
    if (w.rows_max > 0) {
      e = enqueue_grouped_gemm_bf16(w.x_packed, offsets, E, w.rows_max, d, f, a->w1, a->b1, true,
                                    w.h_packed, w.C, status, stream);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
      rec.mark("expert_gemm1");
      e = enqueue_grouped_gemm_bf16(w.h_packed, offsets, E, w.rows_max, f, d, a->w2, a->b2, false,
                                    w.y_packed, w.C, status, stream);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
      rec.mark("expert_gemm2");
    }
    e = enqueue_grouped_gemm_bf16(a->x, nullptr, 1, T, d, f, a->dense_w1, a->dense_b1, true,
                                  w.h_dense, dense_hint, status, stream);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    rec.mark("dense_gemm1");
    fc.dense = true;
    e = enqueue_gemm2_combine(w.h_dense, nullptr, 1, T, f, d, a->dense_w2, a->dense_b2, fc,
                              dense_hint, status, stream);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    rec.mark("dense_gemm2_combine");
    return MOE_OK;
  }
  if (fuse_expert) {
    if (w.rows_max > 0) {
      e = enqueue_grouped_gemm_bf16(w.x_packed, offsets, E, w.rows_max, d, f, a->w1, a->b1, true,
                                    w.h_packed, w.C, status, stream);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
      rec.mark("expert_gemm1");
      fc.dense = false;
      e = enqueue_gemm2_combine(w.h_packed, offsets, E, w.rows_max, f, d, a->w2, a->b2, fc, w.C,
                                status, stream);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
      rec.mark("expert_gemm2_combine");
    }
    return MOE_OK;
  }
  if (dense) {
    // fp32 PR-MoE: dense MLP on every token as one segment of all T rows of x
    e = enqueue_expert_ffn_f32((const float*)a->x, nullptr, 1, T, d, f, (const float*)a->dense_w1,
                               (const float*)a->dense_b1, (const float*)a->dense_w2,
                               (const float*)a->dense_b2, (float*)w.h_dense, w.r_dense, status,
                               stream);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    rec.mark("dense_ffn");
  }
  if (w.rows_max > 0) {
    if (bf16) {
      e = enqueue_grouped_gemm_bf16(w.x_packed, offsets, E, w.rows_max, d, f, a->w1, a->b1, true,
                                    w.h_packed, w.C, status, stream);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
      rec.mark("expert_gemm1");
      e = enqueue_grouped_gemm_bf16(w.h_packed, offsets, E, w.rows_max, f, d, a->w2, a->b2, false,
                                    w.y_packed, w.C, status, stream);
    } else {
      e = enqueue_grouped_gemm_f32((const float*)w.x_packed, offsets, E, w.rows_max, d, f,
                                   (const float*)a->w1, (const float*)a->b1, true,
                                   (float*)w.h_packed, status, stream);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
      rec.mark("expert_gemm1");
      e = enqueue_grouped_gemm_f32((const float*)w.h_packed, offsets, E, w.rows_max, f, d,
                                   (const float*)a->w2, (const float*)a->b2, false, w.y_packed,
                                   status, stream);
    }
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    rec.mark("expert_gemm2");
  }
  e = enqueue_combine(w.y_packed, offsets, ids, slot, gates, T, d, E, k, w.rows_max, residual, bf16,
                      dense ? w.r_dense : nullptr, out, out_bf16, status, stream);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  rec.mark("combine");
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_layer_forward(const moe_layer_args* a, void* out, moe_layer_aux* aux, void* ws,
                             size_t ws_bytes, moe_stream_t stream) {
  StageRecorder rec;
  return layer_forward_impl(a, out, aux, ws, ws_bytes, stream, rec);
}

moe_status moe_layer_forward_profiled(const moe_layer_args* a, void* out, moe_layer_aux* aux,
                                      void* ws, size_t ws_bytes, moe_stream_t stream,
                                      void* const* events, int max_events, int* n_events,
                                      char* names, size_t names_len) {
  if (!events || max_events < 1 || !n_events) return MOE_ERR_INVALID_ARGUMENT;
  for (int i = 0; i < max_events; ++i)
    if (!events[i]) return MOE_ERR_INVALID_ARGUMENT;
  StageRecorder rec;
  rec.events = events;
  rec.max_events = max_events;
  rec.names = names;
  rec.names_len = names_len;
  if (names && names_len > 0) names[0] = '\0';
  const moe_status st = layer_forward_impl(a, out, aux, ws, ws_bytes, stream, rec);
  *n_events = rec.n;
  return st;
}

moe_status moe_layer_shard_workspace_bytes(const moe_layer_args* args, int64_t T_global,
                                           size_t* bytes) {
  if (!bytes || !args || T_global < args->T) return MOE_ERR_INVALID_ARGUMENT;
  LayerWs w;
  return layer_layout(args, nullptr, &w, bytes, T_global);
}

int64_t moe_router_partials_count(int E) { return E < 1 ? 0 : router_partials_count(E); }

moe_status moe_layer_forward_shard_begin(const moe_layer_args* args, int64_t T_global,
                                         moe_layer_aux* aux, int32_t* demand,
                                         int64_t* stat_partials, void* ws, size_t ws_bytes,
                                         moe_stream_t stream) {
  if (!args || T_global < args->T || !demand || !stat_partials) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(demand) || !aligned16(stat_partials)) return MOE_ERR_MISALIGNED;
  ShardCall sh;
  sh.mode = kShardBegin;
  sh.T_global = T_global;
  sh.demand_out = demand;
  sh.partials_out = stat_partials;
  StageRecorder rec;
  return layer_forward_impl(args, nullptr, aux, ws, ws_bytes, stream, rec, sh);
}

moe_status moe_layer_forward_shard_end(const moe_layer_args* args, int64_t T_global, int G,
                                       int rank, const int32_t* demand_all,
                                       const int64_t* stat_totals, void* out, moe_layer_aux* aux,
                                       void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!args || T_global < args->T || G < 1 || rank < 0 || rank >= G || !demand_all ||
      !stat_totals)
    return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(demand_all) || !aligned16(stat_totals)) return MOE_ERR_MISALIGNED;
  ShardCall sh;
  sh.mode = kShardEnd;
  sh.T_global = T_global;
  sh.demand_all = demand_all;
  sh.totals = stat_totals;
  sh.G = G;
  sh.rank = rank;
  StageRecorder rec;
  return layer_forward_impl(args, out, aux, ws, ws_bytes, stream, rec, sh);
}

// ---------------------------------------------------------------- status block

// ---------------------------------------------------------------- training

}  // extern "C"

namespace {

// Training workspace: the forward layout, then what the backward pass needs beyond it.
struct TrainWs {
  LayerWs L;
  void* g_packed;      // [R, d_ff] GeLU'(z) of the experts' layer 1 (dtype)
  void* g_dense;       // [T, d_ff] the dense MLP's (dtype)
  float* r_dense;      // [T, d] dense MLP output (fp32)
  float* dgate;        // [T, k]
  float* dl;           // [T, E]
  void* dy;            // [R, d] (dtype)
  void* dz;            // [R, d_ff] (dtype)
  float* dxp;          // [R, d]
  float* dx_router;    // [T, d]
  void* dzd;           // [T, d_ff] (dtype)
  float* dxd;          // [T, d]
  float* part_colsum;
  float* part_router;
  int S_e, S_d, S_rb, splits_r;
  // bf16 layers: the router's backward GEMMs on tensor cores
  int64_t Tpad;
  int Epad, Kx, S_rt;
  uint16_t *dl3, *dlx, *wx;
};

int router_wgrad_splits(int64_t T) {
  const int64_t s = (T + 1023) / 1024;
  return (int)(s < 1 ? 1 : (s > 64 ? 64 : s));
}

moe_status train_layout(const moe_layer_args* a, uint8_t* base, TrainWs* w, size_t* bytes) {
  size_t fwd = 0;
  moe_status st = layer_layout(a, base, &w->L, &fwd);
  if (st != MOE_OK) return st;
  const int64_t T = a->T, R = w->L.rows_max;
  const int E = a->E, k = a->k, d = a->d_model, f = a->d_ff;
  const size_t es = esize(a->dtype);
  const bool dense = a->dense_w1 != nullptr;
  Carve c{base};
  c.off = fwd;
  w->g_packed = c.take<uint8_t>((size_t)R * f * es);
  w->g_dense = dense ? (void*)c.take<uint8_t>((size_t)T * f * es) : nullptr;
  w->r_dense = dense ? (w->L.r_dense ? w->L.r_dense : c.take<float>((size_t)T * d)) : nullptr;
  w->dgate = c.take<float>((size_t)T * k);
  w->dl = c.take<float>((size_t)T * E);
  w->dy = c.take<uint8_t>((size_t)R * d * es);
  w->dz = c.take<uint8_t>((size_t)R * f * es);
  w->dxp = c.take<float>((size_t)R * d);
  w->dx_router = c.take<float>((size_t)T * d);
  w->dzd = dense ? (void*)c.take<uint8_t>((size_t)T * f * es) : nullptr;
  w->dxd = dense ? c.take<float>((size_t)T * d) : nullptr;
  const int64_t seg = w->L.C < T ? w->L.C : T;
  w->S_e = colsum_splits(seg);
  w->S_d = colsum_splits(T);
  w->S_rb = (int)std::min<int64_t>(256, std::max<int64_t>(1, (T + 127) / 128));
  const int64_t wide = d > f ? d : f;
  int64_t pc = (int64_t)E * w->S_e * wide;
  if ((int64_t)w->S_d * wide > pc) pc = (int64_t)w->S_d * wide;
  if ((int64_t)w->S_rb * E > pc) pc = (int64_t)w->S_rb * E;
  w->part_colsum = c.take<float>((size_t)pc);
  w->splits_r = router_wgrad_splits(T);
  w->Tpad = (T + 63) / 64 * 64;
  w->Epad = (E + 7) / 8 * 8;
  w->Kx = (3 * E + 7) / 8 * 8;
  {
    // split-K of dW_r = dl^T x over the three stacked parts: about one tile per SM
    const int bn = d <= 64 ? 64 : (d <= 128 ? 128 : 256);
    const int64_t tiles = (int64_t)((w->Epad + 127) / 128) * ((d + bn - 1) / bn);
    const int64_t n_kb = 3 * w->Tpad / 64;
    int64_t s = (148 + tiles - 1) / tiles;
    if (s > 64) s = 64;
    if (s > n_kb) s = n_kb;
    w->S_rt = (int)(s < 1 ? 1 : s);
  }
  const bool bf16 = a->dtype == MOE_BF16;
  int64_t pr = (int64_t)w->splits_r * E * d;
  if (bf16 && (int64_t)w->S_rt * w->Epad * d > pr) pr = (int64_t)w->S_rt * w->Epad * d;
  w->part_router = c.take<float>((size_t)pr);
  w->dl3 = bf16 ? c.take<uint16_t>((size_t)3 * w->Tpad * w->Epad) : nullptr;
  w->dlx = bf16 ? c.take<uint16_t>((size_t)T * w->Kx) : nullptr;
  w->wx = bf16 ? c.take<uint16_t>((size_t)w->Kx * d) : nullptr;
  *bytes = c.off;
  return MOE_OK;
}

moe_status copy_out(void* dst, const void* src, size_t n, cudaStream_t stream) {
  if (dst == nullptr || n == 0) return MOE_OK;
  return cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToDevice, stream) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status check_layer_pointers(const moe_layer_args* a, const void* out, const void* ws) {
  const bool dense = a->dense_w1 != nullptr;
  if (dense && !a->dense_w2) return MOE_ERR_INVALID_ARGUMENT;
  if (!ws) return MOE_ERR_INVALID_ARGUMENT;
  if (a->T > 0 && (!a->x || !a->w_router || !a->w1 || !a->w2 || !out))
    return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(a->x) || !aligned16(a->w_router) || !aligned16(a->router_bias) ||
      !aligned16(a->w1) || !aligned16(a->b1) || !aligned16(a->w2) || !aligned16(a->b2) ||
      !aligned16(a->dense_w1) || !aligned16(a->dense_b1) || !aligned16(a->dense_w2) ||
      !aligned16(a->dense_b2) || !aligned16(out) || !aligned16(a->w_router_prepared) ||
      ((uintptr_t)ws % kAlign) != 0)
    return MOE_ERR_MISALIGNED;
  return MOE_OK;
}

moe_status forward_train_impl(const moe_layer_args* a, void* out, moe_layer_aux* aux, void* ws,
                              size_t ws_bytes, cudaStream_t stream) {
  TrainWs w;
  size_t need = 0;
  moe_status st = train_layout(a, (uint8_t*)ws, &w, &need);
  if (st != MOE_OK) return st;
  st = check_layer_pointers(a, out, ws);
  if (st != MOE_OK) return st;
  if (aux && (!aligned16(aux->logits) || !aligned16(aux->expert_ids) || !aligned16(aux->gates) ||
              !aligned16(aux->slot) || !aligned16(aux->expert_counts) ||
              !aligned16(aux->expert_offsets) || !aligned16(aux->lb_stats) ||
              !aligned16(aux->router_losses) || !aligned16(aux->topk_probs)))
    return MOE_ERR_MISALIGNED;
  if (ws_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (fault_injected("moe_layer_forward_train")) return MOE_ERR_CUDA;
  g_launches = 0;
  if (a->T == 0) return MOE_OK;
  const LayerWs& L = w.L;
  int* status = (int*)ws;
  const bool bf16 = a->dtype == MOE_BF16;
  const bool dense = a->dense_w1 != nullptr;
  const int64_t T = a->T;
  const int d = a->d_model, f = a->d_ff, E = a->E, k = a->k;
  // routing state stays in the workspace for the backward pass; aux receives copies
  RouterDispatchCount dcount;
  dcount.local_rank = L.dispatch.local_rank;
  dcount.seg_counts = L.dispatch.seg_counts;
  cudaError_t e = enqueue_router(a->x, bf16, T, d, a->w_router, a->router_bias, E, k,
                                 L.router.logits, L.ids, L.gates, L.lb_stats, a->aux_alpha,
                                 L.router.scr, status, stream, dcount, a->renormalize_gates != 0,
                                 aux ? aux->router_losses : nullptr, nullptr, -1, L.probs,
                                 (const uint16_t*)a->w_router_prepared);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  PriorityDispatch prio;
  if (a->overflow_policy == MOE_OVERFLOW_PRIORITY) {
    prio.probs = L.probs;  // before renormalisation
    prio.keys = L.dispatch.prio_keys;
    prio.demand_offsets = L.dispatch.demand_offsets;
  }
  e = enqueue_dispatch(a->x, bf16, T, d, L.ids, E, k, L.C, L.slot, L.counts, L.offsets,
                       L.row_token, L.x_packed, L.rows_max, L.dispatch.local_rank,
                       L.dispatch.seg_counts, L.dispatch.seg_base, status, stream, DroppedRows{},
                       (int)kRouterTokensPerBlock * k, prio);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (bf16) {
    if (L.rows_max > 0) {
      e = enqueue_grouped_gemm_bf16_train(L.x_packed, L.offsets, E, L.rows_max, d, f, a->w1, a->b1,
                                          L.h_packed, w.g_packed, L.C, status, stream);
      if (e == cudaSuccess)
        e = enqueue_grouped_gemm_bf16(L.h_packed, L.offsets, E, L.rows_max, f, d, a->w2, a->b2,
                                      false, L.y_packed, L.C, status, stream);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (dense) {
      e = enqueue_grouped_gemm_bf16_train(a->x, nullptr, 1, T, d, f, a->dense_w1, a->dense_b1,
                                          L.h_dense, w.g_dense, T, status, stream);
      if (e == cudaSuccess)
        e = enqueue_grouped_gemm_bf16(L.h_dense, nullptr, 1, T, f, d, a->dense_w2, a->dense_b2,
                                      false, w.r_dense, T, status, stream);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
  } else {
    if (L.rows_max > 0) {
      e = enqueue_grouped_gemm_f32((const float*)L.x_packed, L.offsets, E, L.rows_max, d, f,
                                   (const float*)a->w1, (const float*)a->b1, true,
                                   (float*)L.h_packed, status, stream, (float*)w.g_packed);
      if (e == cudaSuccess)
        e = enqueue_grouped_gemm_f32((const float*)L.h_packed, L.offsets, E, L.rows_max, f, d,
                                     (const float*)a->w2, (const float*)a->b2, false, L.y_packed,
                                     status, stream);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (dense) {
      e = enqueue_grouped_gemm_f32((const float*)a->x, nullptr, 1, T, d, f,
                                   (const float*)a->dense_w1, (const float*)a->dense_b1, true,
                                   (float*)L.h_dense, status, stream, (float*)w.g_dense);
      if (e == cudaSuccess)
        e = enqueue_grouped_gemm_f32((const float*)L.h_dense, nullptr, 1, T, f, d,
                                     (const float*)a->dense_w2, (const float*)a->dense_b2, false,
                                     w.r_dense, status, stream);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
  }
  e = enqueue_combine(L.y_packed, L.offsets, L.ids, L.slot, L.gates, T, d, E, k, L.rows_max,
                      a->add_input_residual ? a->x : nullptr, bf16, dense ? w.r_dense : nullptr,
                      out, a->out_dtype == MOE_BF16, status, stream);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (aux) {
    if ((st = copy_out(aux->logits, L.router.logits, sizeof(float) * T * E, stream)) != MOE_OK ||
        (st = copy_out(aux->expert_ids, L.ids, sizeof(int32_t) * T * k, stream)) != MOE_OK ||
        (st = copy_out(aux->gates, L.gates, sizeof(float) * T * k, stream)) != MOE_OK ||
        (st = copy_out(aux->slot, L.slot, sizeof(int32_t) * T * k, stream)) != MOE_OK ||
        (st = copy_out(aux->expert_counts, L.counts, sizeof(int32_t) * E, stream)) != MOE_OK ||
        (st = copy_out(aux->expert_offsets, L.offsets, sizeof(int32_t) * (E + 1), stream)) !=
            MOE_OK ||
        (st = copy_out(aux->lb_stats, L.lb_stats, sizeof(float) * (2 * E + 1), stream)) != MOE_OK ||
        (st = copy_out(aux->topk_probs, L.probs, sizeof(float) * T * k, stream)) != MOE_OK)
      return st;
  }
  return MOE_OK;
}

moe_status backward_impl(const moe_layer_args* a, const void* dout, float aux_weight,
                         float z_weight, moe_layer_grads* g, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
  if (!g) return MOE_ERR_INVALID_ARGUMENT;
  TrainWs w;
  size_t need = 0;
  moe_status st = train_layout(a, (uint8_t*)ws, &w, &need);
  if (st != MOE_OK) return st;
  st = check_layer_pointers(a, dout, ws);
  if (st != MOE_OK) return st;
  const bool dense = a->dense_w1 != nullptr;
  if (a->T > 0 && (!g->dx || !g->dw_router || !g->dw1 || !g->dw2)) return MOE_ERR_INVALID_ARGUMENT;
  if (a->T > 0 && dense && (!g->dense_dw1 || !g->dense_dw2)) return MOE_ERR_INVALID_ARGUMENT;
  if (!std::isfinite(aux_weight) || !std::isfinite(z_weight)) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(g->dx) || !aligned16(g->dw_router) || !aligned16(g->db_router) ||
      !aligned16(g->dw1) || !aligned16(g->db1) || !aligned16(g->dw2) || !aligned16(g->db2) ||
      !aligned16(g->dense_dw1) || !aligned16(g->dense_db1) || !aligned16(g->dense_dw2) ||
      !aligned16(g->dense_db2) || !aligned16(g->dgates) || !aligned16(g->dlogits))
    return MOE_ERR_MISALIGNED;
  if (ws_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (fault_injected("moe_layer_backward")) return MOE_ERR_CUDA;
  g_launches = 0;
  const int64_t T = a->T;
  const int d = a->d_model, f = a->d_ff, E = a->E, k = a->k;
  const LayerWs& L = w.L;
  if (T == 0) {
    // no tokens: every parameter gradient is zero (dx has no rows)
    const size_t ef = (size_t)E * f, ed = (size_t)E * d, fd = (size_t)f * d;
    const std::pair<float*, size_t> zero[] = {
        {g->dw_router, ed}, {g->db_router, (size_t)E}, {g->dw1, ef * d}, {g->db1, ef},
        {g->dw2, ed * f},   {g->db2, ed},              {g->dense_dw1, fd}, {g->dense_db1, (size_t)f},
        {g->dense_dw2, fd}, {g->dense_db2, (size_t)d}};
    for (const auto& z : zero)
      if (z.first != nullptr && z.second > 0 &&
          cudaMemsetAsync(z.first, 0, sizeof(float) * z.second, stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
  }
  int* status = (int*)ws;
  const bool bf16 = a->dtype == MOE_BF16;
  const int64_t R = L.rows_max;
  cudaError_t e;
  auto fail = [&](cudaError_t err) { return err != cudaSuccess; };

  // ---- combine: dgate, dY
  e = enqueue_combine_backward(dout, bf16, L.y_packed, L.offsets, L.ids, L.slot, L.gates, T, d, E,
                               k, R, w.dgate, w.dy, status, stream);
  if (fail(e)) return MOE_ERR_CUDA;
  if (g->dgates && copy_out(g->dgates, w.dgate, sizeof(float) * T * k, stream) != MOE_OK)
    return MOE_ERR_CUDA;
  // ---- router: dl, then dW_r = dl^T x, db_r = column sums of dl, dx_r = dl W_r
  e = enqueue_router_backward(L.router.logits, L.ids, w.dgate, L.router.scr.acc.c, T, E, k,
                              a->aux_alpha, aux_weight, z_weight, a->renormalize_gates != 0, w.dl,
                              stream);
  if (fail(e)) return MOE_ERR_CUDA;
  if (g->dlogits && copy_out(g->dlogits, w.dl, sizeof(float) * T * E, stream) != MOE_OK)
    return MOE_ERR_CUDA;
  if (g->db_router &&
      fail(enqueue_colsum(w.dl, false, nullptr, 1, T, E, w.S_rb, w.part_colsum, g->db_router, stream)))
    return MOE_ERR_CUDA;
  if (bf16) {
    // tensor cores on bf16 parts: dW_r = sum of the three stacked parts^T x (split-K),
    // dx_r = [dl_hi | dl_mid | dl_hi] [W_hi; W_hi; W_mid]
    e = enqueue_router_bwd_split(w.dl, T, w.Tpad, E, w.Epad, w.Kx, w.dl3, w.dlx, a->w_router, d,
                                 w.wx, stream);
    if (!fail(e))
      e = enqueue_wgrad_bf16(w.dl3, a->x, nullptr, 1, 3 * w.Tpad, w.Epad, d, w.part_router, status,
                             stream, w.S_rt, w.Tpad, T);
    if (!fail(e))
      e = enqueue_split_reduce(w.part_router, 1, w.S_rt, (int64_t)E * d, g->dw_router, stream,
                               (int64_t)w.Epad * d);
    if (!fail(e))
      e = enqueue_grouped_gemm_dgrad_bf16(w.dlx, nullptr, 1, T, w.Kx, d, w.wx, nullptr,
                                          w.dx_router, T, status, stream);
    if (fail(e)) return MOE_ERR_CUDA;
  } else {
    SimtGemm p;
    p.M = E; p.N = d; p.K = T;
    p.a = w.dl; p.a_m = 1; p.a_k = E;
    p.b = a->x; p.b_k = d; p.b_n = 1;
    p.c = w.part_router; p.c_m = d; p.c_n = 1;
    p.splits = w.splits_r; p.split_stride = (int64_t)E * d;
    e = enqueue_simt_gemm(p, E, stream);
    if (fail(e) || fail(enqueue_split_reduce(w.part_router, 1, w.splits_r, (int64_t)E * d,
                                             g->dw_router, stream)))
      return MOE_ERR_CUDA;
    SimtGemm q;
    q.M = T; q.N = d; q.K = E;
    q.a = w.dl; q.a_m = E; q.a_k = 1;
    q.b = a->w_router; q.b_k = d; q.b_n = 1;
    q.c = w.dx_router; q.c_m = d; q.c_n = 1;
    if (fail(enqueue_simt_gemm(q, T, stream))) return MOE_ERR_CUDA;
  }
  // ---- experts
  const int64_t m_ext = L.C < T ? L.C : T;  // rows of one expert at most
  if (R > 0) {
    if (bf16) {
      e = enqueue_grouped_gemm_dgrad_bf16(w.dy, L.offsets, E, R, d, f, a->w2, w.g_packed, w.dz,
                                          L.C, status, stream);
      if (!fail(e))
        e = enqueue_grouped_gemm_dgrad_bf16(w.dz, L.offsets, E, R, f, d, a->w1, nullptr, w.dxp,
                                            L.C, status, stream);
      if (!fail(e)) e = enqueue_wgrad_bf16(w.dy, L.h_packed, L.offsets, E, R, d, f, g->dw2, status, stream);
      if (!fail(e)) e = enqueue_wgrad_bf16(w.dz, L.x_packed, L.offsets, E, R, f, d, g->dw1, status, stream);
      if (fail(e)) return MOE_ERR_CUDA;
    } else {
      SimtGemm p;  // dZ = (dY W2[e]) * GeLU'(z)
      p.M = 0; p.N = f; p.K = d; p.ragged = 1; p.offsets = L.offsets; p.E = E; p.rows_max = R;
      p.a = w.dy; p.a_m = d; p.a_k = 1;
      p.b = a->w2; p.b_e = (int64_t)d * f; p.b_k = f; p.b_n = 1;
      p.c = (float*)w.dz; p.c_m = f; p.c_n = 1;
      p.mul = w.g_packed;
      if (fail(enqueue_simt_gemm(p, m_ext, stream))) return MOE_ERR_CUDA;
      SimtGemm q;  // dX_packed = dZ W1[e]
      q.N = d; q.K = f; q.ragged = 1; q.offsets = L.offsets; q.E = E; q.rows_max = R;
      q.a = w.dz; q.a_m = f; q.a_k = 1;
      q.b = a->w1; q.b_e = (int64_t)f * d; q.b_k = d; q.b_n = 1;
      q.c = w.dxp; q.c_m = d; q.c_n = 1;
      if (fail(enqueue_simt_gemm(q, m_ext, stream))) return MOE_ERR_CUDA;
      SimtGemm r;  // dW2[e] = dY^T h
      r.M = d; r.N = f; r.ragged = 2; r.offsets = L.offsets; r.E = E; r.rows_max = R;
      r.a = w.dy; r.a_m = 1; r.a_k = d;
      r.b = L.h_packed; r.b_k = f; r.b_n = 1;
      r.c = g->dw2; r.c_e = (int64_t)d * f; r.c_m = f; r.c_n = 1;
      if (fail(enqueue_simt_gemm(r, d, stream))) return MOE_ERR_CUDA;
      SimtGemm u;  // dW1[e] = dZ^T x
      u.M = f; u.N = d; u.ragged = 2; u.offsets = L.offsets; u.E = E; u.rows_max = R;
      u.a = w.dz; u.a_m = 1; u.a_k = f;
      u.b = L.x_packed; u.b_k = d; u.b_n = 1;
      u.c = g->dw1; u.c_e = (int64_t)f * d; u.c_m = d; u.c_n = 1;
      if (fail(enqueue_simt_gemm(u, f, stream))) return MOE_ERR_CUDA;
    }
  } else {
    if (cudaMemsetAsync(g->dw1, 0, sizeof(float) * E * f * d, stream) != cudaSuccess ||
        cudaMemsetAsync(g->dw2, 0, sizeof(float) * E * d * f, stream) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (g->db2 && fail(enqueue_colsum(w.dy, bf16, L.offsets, E, R, d, w.S_e, w.part_colsum, g->db2, stream)))
    return MOE_ERR_CUDA;
  if (g->db1 && fail(enqueue_colsum(w.dz, bf16, L.offsets, E, R, f, w.S_e, w.part_colsum, g->db1, stream)))
    return MOE_ERR_CUDA;
  // ---- dense MLP (one segment of all T rows; its output gradient is dout itself)
  if (dense) {
    if (bf16) {
      e = enqueue_grouped_gemm_dgrad_bf16(dout, nullptr, 1, T, d, f, a->dense_w2, w.g_dense, w.dzd,
                                          T, status, stream);
      if (!fail(e))
        e = enqueue_grouped_gemm_dgrad_bf16(w.dzd, nullptr, 1, T, f, d, a->dense_w1, nullptr, w.dxd,
                                            T, status, stream);
      if (!fail(e)) e = enqueue_wgrad_bf16(dout, L.h_dense, nullptr, 1, T, d, f, g->dense_dw2, status, stream);
      if (!fail(e)) e = enqueue_wgrad_bf16(w.dzd, a->x, nullptr, 1, T, f, d, g->dense_dw1, status, stream);
      if (fail(e)) return MOE_ERR_CUDA;
    } else {
      SimtGemm p;
      p.N = f; p.K = d; p.ragged = 1; p.E = 1; p.rows_max = T;
      p.a = dout; p.a_m = d; p.a_k = 1;
      p.b = a->dense_w2; p.b_k = f; p.b_n = 1;
      p.c = (float*)w.dzd; p.c_m = f; p.c_n = 1;
      p.mul = w.g_dense;
      if (fail(enqueue_simt_gemm(p, T, stream))) return MOE_ERR_CUDA;
      SimtGemm q;
      q.N = d; q.K = f; q.ragged = 1; q.E = 1; q.rows_max = T;
      q.a = w.dzd; q.a_m = f; q.a_k = 1;
      q.b = a->dense_w1; q.b_k = d; q.b_n = 1;
      q.c = w.dxd; q.c_m = d; q.c_n = 1;
      if (fail(enqueue_simt_gemm(q, T, stream))) return MOE_ERR_CUDA;
      SimtGemm r;
      r.M = d; r.N = f; r.ragged = 2; r.E = 1; r.rows_max = T;
      r.a = dout; r.a_m = 1; r.a_k = d;
      r.b = L.h_dense; r.b_k = f; r.b_n = 1;
      r.c = g->dense_dw2; r.c_m = f; r.c_n = 1;
      r.splits = 1;
      if (fail(enqueue_simt_gemm(r, d, stream))) return MOE_ERR_CUDA;
      SimtGemm u;
      u.M = f; u.N = d; u.ragged = 2; u.E = 1; u.rows_max = T;
      u.a = w.dzd; u.a_m = 1; u.a_k = f;
      u.b = a->x; u.b_k = d; u.b_n = 1;
      u.c = g->dense_dw1; u.c_m = d; u.c_n = 1;
      if (fail(enqueue_simt_gemm(u, f, stream))) return MOE_ERR_CUDA;
    }
    if (g->dense_db2 &&
        fail(enqueue_colsum(dout, bf16, nullptr, 1, T, d, w.S_d, w.part_colsum, g->dense_db2, stream)))
      return MOE_ERR_CUDA;
    if (g->dense_db1 &&
        fail(enqueue_colsum(w.dzd, bf16, nullptr, 1, T, f, w.S_d, w.part_colsum, g->dense_db1, stream)))
      return MOE_ERR_CUDA;
  }
  // ---- dx = [dout] + [dense dx] + packed expert dx rows + router dx
  e = enqueue_dx_gather(dout, bf16, a->add_input_residual != 0, dense ? w.dxd : nullptr, w.dxp,
                        L.offsets, L.ids, L.slot, T, d, E, k, R, w.dx_router, g->dx, stream);
  return fail(e) ? MOE_ERR_CUDA : MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_layer_train_workspace_bytes(const moe_layer_args* args, size_t* bytes) {
  if (!bytes) return MOE_ERR_INVALID_ARGUMENT;
  TrainWs w;
  return train_layout(args, nullptr, &w, bytes);
}

moe_status moe_layer_forward_train(const moe_layer_args* args, void* out, moe_layer_aux* aux,
                                   void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!args) return MOE_ERR_INVALID_ARGUMENT;
  return forward_train_impl(args, out, aux, ws, ws_bytes, stream);
}

moe_status moe_layer_backward(const moe_layer_args* args, const void* d_out, float aux_weight,
                              float z_weight, moe_layer_grads* grads, void* ws, size_t ws_bytes,
                              moe_stream_t stream) {
  if (!args) return MOE_ERR_INVALID_ARGUMENT;
  return backward_impl(args, d_out, aux_weight, z_weight, grads, ws, ws_bytes, stream);
}

moe_status moe_workspace_reset(void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!ws || ws_bytes < kAlign) return MOE_ERR_INVALID_ARGUMENT;
  return cuda_status(cudaMemsetAsync(ws, 0, kAlign, stream));
}

moe_status moe_get_device_error(const void* ws, int* code_out, moe_stream_t stream) {
  if (!ws || !code_out) return MOE_ERR_INVALID_ARGUMENT;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  int code = 0;
  if (cudaMemcpy(&code, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  *code_out = code;
  return code ? MOE_ERR_DEVICE_FLAG : MOE_OK;
}

}  // extern "C"
