// Expert FFN for fp32 tensors on fp32 FMA units (no TF32): one block per (packed row, 128
// output features); the row is staged in shared memory and each thread accumulates one output
// feature over K in index order. Used for fp32 layers, whose tolerance (1e-5) TF32 or bf16
// tensor-core inputs cannot meet; bf16 layers use the tcgen05 grouped GEMM.
//     h[r, :] = GeLU(W1[e] x[r, :] + b1[e]),   y[r, :] = W2[e] h[r, :] + b2[e]
// (MoE survey notes §1.1.2.1: an expert is a two-layer feed-forward network.)
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kFeat = 128;

template <bool GELU>
__global__ void __launch_bounds__(kFeat)
    ffn_f32_kernel(const float* __restrict__ X, const int32_t* __restrict__ offsets, int E,
                   int n_out, int K, int64_t rows_max, const float* __restrict__ W,
                   const float* __restrict__ bias, float* __restrict__ out, int* status,
                   float* __restrict__ gout) {
  extern __shared__ float xs[];
  pdl_wait();
  // offsets == nullptr: one segment covering all rows_max rows (dense MLP, E == 1)
  const int64_t start = offsets ? offsets[0] : 0, total = offsets ? offsets[E] : rows_max;
  if (start < 0 || total < start || total > rows_max) {
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
      set_device_error(status, MOE_DEVERR_BAD_OFFSETS);
    return;
  }
  const int f = blockIdx.y * kFeat + threadIdx.x;
  for (int64_t r = start + blockIdx.x; r < total; r += gridDim.x) {
    // expert owning row r: largest e with offsets[e] <= r
    int lo = 0, hi = E;
    while (offsets && hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (offsets[mid] <= r) lo = mid;
      else hi = mid;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < K; i += kFeat) xs[i] = X[r * K + i];
    __syncthreads();
    if (f < n_out) {
      const float* w = W + ((int64_t)lo * n_out + f) * K;
      float acc = 0.0f;
      for (int i = 0; i < K; ++i) acc = fmaf(xs[i], w[i], acc);
      float v = acc + (bias ? bias[(int64_t)lo * n_out + f] : 0.0f);
      if (GELU) {
        if (gout != nullptr) gout[r * n_out + f] = gelu_erf_grad(v);  // saved for the backward
        v = gelu_erf(v);
      }
      out[r * n_out + f] = v;
    }
  }
  pdl_trigger();
}

}  // namespace

cudaError_t enqueue_grouped_gemm_f32(const float* x, const int32_t* offsets, int E,
                                     int64_t rows_max, int K, int N, const float* w,
                                     const float* bias, bool gelu, float* out, int* status,
                                     cudaStream_t stream, float* gelu_grad_out) {
  if (rows_max == 0) return cudaSuccess;
  const unsigned gx = (unsigned)(rows_max < 65536 ? rows_max : 65536);
  const size_t smem = (size_t)K * sizeof(float);
  if (smem > 48 * 1024) {  // above the default limit: raise it once per device
    static int attr_done[2][64] = {{0}};
    cudaError_t e = ensure_dynamic_smem(gelu ? ffn_f32_kernel<true> : ffn_f32_kernel<false>,
                                        (int)smem, attr_done[gelu ? 1 : 0]);
    if (e != cudaSuccess) return e;
  }
  const dim3 grid(gx, (N + kFeat - 1) / kFeat);
  return launch_kernel(gelu ? ffn_f32_kernel<true> : ffn_f32_kernel<false>, grid, dim3(kFeat), smem,
                       stream, x, offsets, E, N, K, rows_max, w, bias, out, status,
                       gelu ? gelu_grad_out : nullptr);
}

cudaError_t enqueue_expert_ffn_f32(const float* x_packed, const int32_t* offsets, int E,
                                   int64_t rows_max, int d, int d_ff, const float* w1,
                                   const float* b1, const float* w2, const float* b2,
                                   float* h_packed, float* y_packed, int* status,
                                   cudaStream_t stream) {
  cudaError_t e = enqueue_grouped_gemm_f32(x_packed, offsets, E, rows_max, d, d_ff, w1, b1, true,
                                           h_packed, status, stream);
  if (e != cudaSuccess) return e;
  return enqueue_grouped_gemm_f32(h_packed, offsets, E, rows_max, d_ff, d, w2, b2, false, y_packed,
                                  status, stream);
}

}  // namespace moe
