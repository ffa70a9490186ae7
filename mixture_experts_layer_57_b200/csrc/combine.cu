// Combine: gate-weighted sum of each token's kept expert rows plus the residual terms.
//     out[t] = [residual[t]] + [dense[t]] + sum_{j : slot[t,j] >= 0} gate[t,j] * y[row(t,j)]
//     row(t,j) = offsets[expert_ids[t,j]] + slot[t,j]
// in fp32, in that order, rounded once to the output type.
// DeepSpeed MoE blog, the combine step of its pipeline listing, gates p_e(x); comparison article,
// "Expert Capacity Overflow" (a dropped token passes through the residual only) and the PR-MoE
// "residual correction" example (fixed MLP output + gate * expert output).
//
// One warp per token (gather form: each output row is written once, no atomics); VEC floats per
// lane per step (VEC = 4 when d % 4 == 0: 16-byte loads of y).
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

template <int VEC, bool RES_BF16, bool OUT_BF16>
__global__ void __launch_bounds__(256, 4)
    combine_kernel(const float* __restrict__ y, const int32_t* __restrict__ offsets,
                   const int32_t* __restrict__ ids, const int32_t* __restrict__ slot,
                   const float* __restrict__ gates, int64_t T, int d, int E, int k,
                   int64_t rows_max, const void* __restrict__ residual,
                   const float* __restrict__ dense, void* __restrict__ out, int* status) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  // the kept choices in order, held in registers (fully unrolled over the largest k): row -1 and
  // gate 0 for a choice that is dropped or out of range
  int64_t row[MOE_MAX_TOPK];
  float g[MOE_MAX_TOPK];
#pragma unroll
  for (int j = 0; j < MOE_MAX_TOPK; ++j) {
    row[j] = -1;
    g[j] = 0.0f;
    if (j >= k) continue;
    const int s = slot[t * k + j];
    if (s < 0) continue;
    const int e = ids[t * k + j];
    int64_t r = -1;
    if (e >= 0 && e < E) r = (int64_t)offsets[e] + s;
    if (r < 0 || r >= rows_max) {
      if (lane == 0) set_device_error(status, MOE_DEVERR_BAD_ROW);
      continue;
    }
    row[j] = r;
    g[j] = gates[t * k + j];
  }
  // (VEC == 4: the loop is unrolled so that each lane has several rows' loads in flight; with at
  // most 64 registers four blocks fit an SM. Launch durations: gpt1.3b-prmoe128 67.5 -> 54 us,
  // top2-e8-zipf 104 -> 74 us against unroll 4 at three blocks per SM)
#pragma unroll 8
  for (int c = lane * VEC; c < d; c += 32 * VEC) {
    float acc[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = 0.0f;
    if (residual) {
      if constexpr (VEC == 4 && RES_BF16) {
        const uint2 rb = *reinterpret_cast<const uint2*>(
            reinterpret_cast<const uint16_t*>(residual) + t * d + c);
        acc[0] = __uint_as_float(rb.x << 16);
        acc[1] = __uint_as_float(rb.x & 0xffff0000u);
        acc[2] = __uint_as_float(rb.y << 16);
        acc[3] = __uint_as_float(rb.y & 0xffff0000u);
      } else {
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[v] = load_elem<RES_BF16>(residual, t * d + c + v);
      }
    }
    if (dense) {
      if constexpr (VEC == 4) {
        const float4 q = *reinterpret_cast<const float4*>(dense + t * d + c);
        acc[0] += q.x;
        acc[1] += q.y;
        acc[2] += q.z;
        acc[3] += q.w;
      } else {
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[v] += dense[t * d + c + v];
      }
    }
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOPK; ++j) {
      if (row[j] < 0) continue;
      const float* src = y + row[j] * d + c;
      float yv[VEC];
      if constexpr (VEC == 4) {
        const float4 q = *reinterpret_cast<const float4*>(src);
        yv[0] = q.x; yv[1] = q.y; yv[2] = q.z; yv[3] = q.w;
      } else {
#pragma unroll
        for (int v = 0; v < VEC; ++v) yv[v] = src[v];
      }
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[v] = fmaf(g[j], yv[v], acc[v]);
    }
    if constexpr (OUT_BF16 && VEC == 4) {
      // one 8-byte store of the 4 rounded values (d % 4 == 0, so t * d + c is a multiple of 4)
      uint2 o;
      o.x = (uint32_t)f32_to_bf16_rn(acc[0]) | ((uint32_t)f32_to_bf16_rn(acc[1]) << 16);
      o.y = (uint32_t)f32_to_bf16_rn(acc[2]) | ((uint32_t)f32_to_bf16_rn(acc[3]) << 16);
      *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(out) + t * d + c) = o;
    } else if constexpr (OUT_BF16) {
      uint16_t* o = reinterpret_cast<uint16_t*>(out) + t * d + c;
#pragma unroll
      for (int v = 0; v < VEC; ++v) o[v] = f32_to_bf16_rn(acc[v]);
    } else if constexpr (VEC == 4) {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + t * d + c) =
          make_float4(acc[0], acc[1], acc[2], acc[3]);
    } else {
      float* o = reinterpret_cast<float*>(out) + t * d + c;
#pragma unroll
      for (int v = 0; v < VEC; ++v) o[v] = acc[v];
    }
  }
  pdl_trigger();
}

template <int VEC>
cudaError_t launch(const float* y, const int32_t* offsets, const int32_t* ids, const int32_t* slot,
                   const float* gates, int64_t T, int d, int E, int k, int64_t rows_max,
                   const void* residual, bool res_bf16, const float* dense, void* out,
                   bool out_bf16, int* status, cudaStream_t stream) {
  const unsigned blocks = (unsigned)((T * 32 + 255) / 256);
#define MOE_COMBINE_LAUNCH(RB, OB)                                                              \
  launch_kernel(combine_kernel<VEC, RB, OB>, dim3(blocks), dim3(256), 0, stream, y, offsets, ids, \
                slot, gates, T, d, E, k, rows_max, residual, dense, out, status)
  cudaError_t e;
  if (res_bf16 && out_bf16) e = MOE_COMBINE_LAUNCH(true, true);
  else if (res_bf16) e = MOE_COMBINE_LAUNCH(true, false);
  else if (out_bf16) e = MOE_COMBINE_LAUNCH(false, true);
  else e = MOE_COMBINE_LAUNCH(false, false);
#undef MOE_COMBINE_LAUNCH
  return e;
}

}  // namespace

cudaError_t enqueue_combine(const float* y_packed, const int32_t* offsets, const int32_t* ids,
                            const int32_t* slot, const float* gates, int64_t T, int d, int E,
                            int k, int64_t rows_max, const void* residual, bool res_bf16,
                            const float* dense, void* out, bool out_bf16, int* status,
                            cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  if (d % 4 == 0)
    return launch<4>(y_packed, offsets, ids, slot, gates, T, d, E, k, rows_max, residual, res_bf16,
                     dense, out, out_bf16, status, stream);
  return launch<1>(y_packed, offsets, ids, slot, gates, T, d, E, k, rows_max, residual, res_bf16,
                   dense, out, out_bf16, status, stream);
}

}  // namespace moe
