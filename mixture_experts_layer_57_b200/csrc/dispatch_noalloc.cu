// moe_dispatch_noalloc: the dispatch step for callers that cannot hand the library a workspace.
//
// Some callers have no way to allocate device memory of their own: a plug-in that runs inside a
// host application which owns every device buffer and exposes no allocation hook, or a
// latency-critical serving loop that must never call cudaMalloc/cudaFree (both can block and
// synchronise the whole device). They still own their inputs and outputs, but not scratch.
// This entry point runs the same three dispatch kernels as moe_dispatch; the scratch they need
// (per-pair rank inside its segment, per-segment expert counts and bases) lives in the
// file-scope array below, which every GPU that loads the library holds until the process exits.
//
// Host code cannot use the array's name as a device address (on the host it names a stand-in
// object), so each call looks the address up with cudaGetSymbolAddress on the current device and
// keeps it per device. A call made while its stream is being captured into a CUDA graph reuses the
// kept address instead (the first call on a device must therefore come before any capture); every
// other call looks it up again, so a device reset, which unloads the module and with it the
// array, cannot leave a stale address behind.
//
// The kernels write every scratch element they later read (counts and bases for all segments and
// experts, a rank for every pair), so nothing has to start at zero and the contents left by the
// previous call do no harm. All calls share the one array: calls that overlap on the GPU (two
// streams, or two host threads, at the same time) race on it and must be serialised by the
// caller. No status word is written: expert ids outside [0, E) are treated as dropped pairs
// (slot -1), as moe_dispatch treats them, without a device error code.
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "kernels.h"

static __device__ __align__(256) unsigned char g_dispatch_scratch[MOE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_dispatch_scratch on the current device: looked up again unless `stream` is
// capturing (then the address kept from an earlier call on this device is used).
cudaError_t scratch_address(cudaStream_t stream, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  bool capturing = true;
  if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess) capturing = cs != cudaStreamCaptureStatusNone;
  else (void)cudaGetLastError();  // the query failed: keep the kept address, clear the error
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!capturing || g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dispatch_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" moe_status moe_dispatch_noalloc(const void* x, moe_dtype dtype, int64_t T, int d_model,
                                           const int32_t* expert_ids, int E, int k, int64_t C,
                                           int32_t* slot, int32_t* expert_counts,
                                           int32_t* expert_offsets, int32_t* row_token,
                                           void* x_packed, int64_t rows_max, moe_stream_t stream) {
  // the same argument rules as moe_dispatch
  if ((dtype != MOE_F32 && dtype != MOE_BF16) || C < 0) return MOE_ERR_INVALID_ARGUMENT;
  if (T < 0 || d_model < 1 || E < 1 || k < 1 || k > E) return MOE_ERR_INVALID_ARGUMENT;
  if (E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK) return MOE_ERR_UNSUPPORTED;
  if (T * (int64_t)k >= (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  const int64_t pairs = T * k;
  const int64_t need_rows = C >= pairs ? pairs : ((int64_t)E * C < pairs ? (int64_t)E * C : pairs);
  if (rows_max < need_rows) return MOE_ERR_INVALID_ARGUMENT;
  if (rows_max >= (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  if (dtype == MOE_BF16 && d_model % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (!expert_counts || !expert_offsets) return MOE_ERR_INVALID_ARGUMENT;
  if (T > 0 && (!x || !expert_ids || !slot)) return MOE_ERR_INVALID_ARGUMENT;
  if (rows_max > 0 && (!row_token || !x_packed)) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(expert_ids) || !aligned16(slot) || !aligned16(expert_counts) ||
      !aligned16(expert_offsets) || !aligned16(row_token) || !aligned16(x_packed))
    return MOE_ERR_MISALIGNED;
  // scratch layout inside the static array: ranks [pairs], segment counts and bases [nseg, E]
  const int64_t nseg = moe::dispatch_num_segments(pairs);
  const size_t rank_bytes = align_up((size_t)pairs * sizeof(int32_t));
  const size_t seg_bytes = align_up((size_t)nseg * E * sizeof(int32_t));
  if (rank_bytes + 2 * seg_bytes > (size_t)MOE_NOALLOC_SCRATCH_BYTES)
    return MOE_ERR_WORKSPACE_TOO_SMALL;
  const char* inj = std::getenv("MOE_FAULT_INJECT");
  if (inj && std::strcmp(inj, "moe_dispatch_noalloc") == 0) return MOE_ERR_CUDA;
  void* base = nullptr;
  if (scratch_address(stream, &base) != cudaSuccess) return MOE_ERR_CUDA;
  moe::reset_launch_count();
  unsigned char* b = static_cast<unsigned char*>(base);
  int32_t* local_rank = reinterpret_cast<int32_t*>(b);
  int32_t* seg_counts = reinterpret_cast<int32_t*>(b + rank_bytes);
  int32_t* seg_base = reinterpret_cast<int32_t*>(b + rank_bytes + seg_bytes);
  const cudaError_t e = moe::enqueue_dispatch(
      x, dtype == MOE_BF16, T, d_model, expert_ids, E, k, C, slot, expert_counts, expert_offsets,
      row_token, x_packed, rows_max, local_rank, seg_counts, seg_base, /*status=*/nullptr, stream);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
