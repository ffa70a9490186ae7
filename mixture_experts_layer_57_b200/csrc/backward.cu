// Backward pass of the MoE layer, the parts that are not expert GEMMs on tensor cores:
//
//   combine_backward_kernel   one warp per token: dL/dgate_j = <dout[t], y[row_j]> for each kept
//                             choice and dY[row_j] = gate_j * dout[t] (the experts' output
//                             gradient, packed like y)
//   router_backward_kernel    one warp per token: gates -> p (renormalisation), the load-balance
//                             term alpha E f_e / T on every p_e, softmax backward and the z-loss
//                             term 2 log Z p_e / T: dL/dlogits [T, E]
//   colsum_kernel             bias gradients: column sums over each segment's rows, split over
//                             row chunks with a fixed-order second pass when a segment is long
//   dx_gather_kernel          one warp per token: dx = [dout] + [dense MLP dx] + the kept
//                             choices' packed dx rows + the router's dx, in that order
//   simt_gemm_kernel          fp32 FMA GEMM with arbitrary strides and one ragged dimension
//                             (expert segments), optional split-K: the router's dW_r = dl^T x and
//                             dx_r = dl W_r, and every GEMM of fp32 layers
//   split_reduce_kernel       fixed-order sum of split-K partials
//
// Chain rule through the forward pass of the comparison article's Switch layer and the DeepSpeed
// MoE formula (gate-weighted experts), the survey notes' load-balance loss and the article's
// router z-loss. Every sum has a fixed order, so results are deterministic.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

template <bool BF16>
__device__ __forceinline__ float ld_any(const void* p, int64_t i) {
  if constexpr (BF16) return bf16_to_f32(reinterpret_cast<const uint16_t*>(p)[i]);
  else return reinterpret_cast<const float*>(p)[i];
}
template <bool BF16>
__device__ __forceinline__ void st_any(void* p, int64_t i, float v) {
  if constexpr (BF16) reinterpret_cast<uint16_t*>(p)[i] = f32_to_bf16_rn(v);
  else reinterpret_cast<float*>(p)[i] = v;
}

template <bool BF16>
__global__ void __launch_bounds__(256)
    combine_backward_kernel(const void* __restrict__ dout, const float* __restrict__ y,
                            const int32_t* __restrict__ offsets, const int32_t* __restrict__ ids,
                            const int32_t* __restrict__ slot, const float* __restrict__ gates,
                            int64_t T, int d, int E, int k, int64_t rows_max,
                            float* __restrict__ dgate, void* __restrict__ dy, int* status) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int s = slot[t * k + j];
      const int e = ids[t * k + j];
      int64_t r = -1;
      if (s >= 0 && e >= 0 && e < E) r = (int64_t)offsets[e] + s;
      if (s >= 0 && (r < 0 || r >= rows_max)) {
        if (lane == 0) set_device_error(status, MOE_DEVERR_BAD_ROW);
        r = -1;
      }
      float acc = 0.0f;
      if (r >= 0) {
        const float g = gates[t * k + j];
        for (int c = lane; c < d; c += 32) {
          const float go = ld_any<BF16>(dout, t * d + c);
          acc = fmaf(go, y[r * d + c], acc);
          st_any<BF16>(dy, r * d + c, g * go);
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0 && dgate != nullptr) dgate[t * k + j] = acc;
    }
  }
  pdl_trigger();
}

// EPL experts per lane (expert e in lane e % 32, slot e / 32), as in the forward top-k kernel,
// whose arithmetic for p (max, exp, sum, divide) this repeats so that p is the forward's.
template <int EPL>
__global__ void __launch_bounds__(256)
    router_backward_kernel(const float* __restrict__ logits, const int32_t* __restrict__ ids,
                           const float* __restrict__ dgate, const unsigned* __restrict__ first,
                           int64_t T, int E, int k, float alpha, float aux_weight, float z_weight,
                           int renorm, float* __restrict__ dl) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t < T) {
    float l[EPL];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      l[i] = e < E ? logits[t * E + e] : -INFINITY;
      m = fmaxf(m, l[i]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float ex[EPL];
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      ex[i] = (lane + 32 * i) < E ? expf(l[i] - m) : 0.0f;
      s += ex[i];
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    float p[EPL], dp[EPL];
    // load-balance loss alpha * E * sum_e f_e Q_e with f_e = first_e / T, Q_e = mean_t p_te
    const float aux_c = aux_weight * alpha * (float)E / ((float)T * (float)T);
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      p[i] = ex[i] / s;
      dp[i] = e < E ? aux_c * (float)first[e] : 0.0f;
    }
    // gates: g_j = p_{e_j}, or p_{e_j} / S with S the sum of the chosen p
    float S = 0.0f, gdg = 0.0f;
    if (renorm) {
      for (int j = 0; j < k; ++j) {
        const int e = ids[t * k + j];
        float pe = 0.0f;
#pragma unroll
        for (int i = 0; i < EPL; ++i)
          if (i == (e >> 5)) pe = p[i];
        S += __shfl_sync(0xffffffffu, pe, e & 31);
      }
      for (int j = 0; j < k; ++j) {
        const int e = ids[t * k + j];
        float pe = 0.0f;
#pragma unroll
        for (int i = 0; i < EPL; ++i)
          if (i == (e >> 5)) pe = p[i];
        pe = __shfl_sync(0xffffffffu, pe, e & 31);
        gdg += dgate[t * k + j] * (pe / S);
      }
    }
    for (int j = 0; j < k; ++j) {
      const int e = ids[t * k + j];
      const float g = dgate[t * k + j];
      const float add = renorm ? (g - gdg) / S : g;
      if (lane == (e & 31)) {
#pragma unroll
        for (int i = 0; i < EPL; ++i)
          if (i == (e >> 5)) dp[i] += add;
      }
    }
    float pdp = 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) pdp = fmaf(p[i], dp[i], pdp);
#pragma unroll
    for (int o = 16; o; o >>= 1) pdp += __shfl_xor_sync(0xffffffffu, pdp, o);
    const float zc = z_weight != 0.0f ? z_weight * 2.0f * (m + logf(s)) / (float)T : 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) dl[t * E + e] = p[i] * (dp[i] - pdp) + zc * p[i];
    }
  }
  pdl_trigger();
}

// out[(e * S + s) * N + n] = sum of X[r][n] over rows r of split s of segment e.
template <bool BF16>
__global__ void __launch_bounds__(256)
    colsum_kernel(const void* __restrict__ X, const int32_t* __restrict__ offsets, int64_t rows_max,
                  int N, int S, float* __restrict__ out) {
  pdl_wait();
  const int n = blockIdx.x * 256 + threadIdx.x;
  const int e = blockIdx.y, sidx = blockIdx.z;
  int64_t a = offsets ? offsets[e] : 0, b = offsets ? offsets[e + 1] : rows_max;
  if (a < 0 || b < a || b > rows_max) a = b = 0;
  const int64_t len = b - a, chunk = (len + S - 1) / S;
  const int64_t r0 = a + sidx * chunk, r1 = min(b, r0 + chunk);
  if (n < N) {
    float acc = 0.0f;
    for (int64_t r = r0; r < r1; ++r) acc += ld_any<BF16>(X, r * N + n);
    out[((int64_t)e * S + sidx) * N + n] = acc;
  }
  pdl_trigger();
}

// out[g * N + n] = sum_{s < S} part[(g * S + s) * N_stride + n], s ascending (N <= N_stride).
__global__ void __launch_bounds__(256)
    split_reduce_kernel(const float* __restrict__ part, int64_t groups, int S, int64_t N,
                        int64_t N_stride, float* __restrict__ out) {
  pdl_wait();
  const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (i < groups * N) {
    const int64_t g = i / N, n = i - g * N;
    float acc = 0.0f;
    for (int s = 0; s < S; ++s) acc += part[(g * S + s) * N_stride + n];
    out[i] = acc;
  }
  pdl_trigger();
}

// Exact three-way bf16 split v = hi + mid + lo (each part the next 8 significant bits).
__device__ __forceinline__ void split3(float v, uint16_t* hi, uint16_t* mid, uint16_t* lo) {
  *hi = f32_to_bf16_rn(v);
  const float r1 = v - bf16_to_f32(*hi);
  *mid = f32_to_bf16_rn(r1);
  *lo = f32_to_bf16_rn(r1 - bf16_to_f32(*mid));
}

// The router's backward GEMMs on tensor cores from bf16 parts of fp32 operands:
//   dl3 [3 Tpad, Epad]: rows p * Tpad + t hold part p (hi, mid, lo) of dl[t, :]; padding zero
//     (dW_r = sum_p part_p^T x: x is bf16, so the three products are exact and the sum is fp32-
//     accurate);
//   dlx [T, Kx]: columns [dl_hi | dl_mid | dl_hi | 0], wx [Kx, d]: rows [W_hi; W_hi; W_mid; 0]
//     (dx_r = dl W_r as W_hi dl_hi + W_hi dl_mid + W_mid dl_hi: 16 significant bits of each
//     operand, for a dx that is returned in bf16).
__global__ void __launch_bounds__(256)
    router_bwd_split_kernel(const float* __restrict__ dl, int64_t T, int64_t Tpad, int E,
                            int Epad, int Kx, uint16_t* __restrict__ dl3,
                            uint16_t* __restrict__ dlx) {
  pdl_wait();
  const int64_t n = Tpad * Epad;
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (int64_t)gridDim.x * 256) {
    const int64_t t = i / Epad;
    const int e = (int)(i - t * Epad);
    const float v = (t < T && e < E) ? dl[t * E + e] : 0.0f;
    uint16_t hi, mid, lo;
    split3(v, &hi, &mid, &lo);
    dl3[t * Epad + e] = hi;
    dl3[(Tpad + t) * Epad + e] = mid;
    dl3[(2 * Tpad + t) * Epad + e] = lo;
    if (t < T) {
      if (e < E) {
        dlx[t * Kx + e] = hi;
        dlx[t * Kx + E + e] = mid;
        dlx[t * Kx + 2 * E + e] = hi;
      }
      for (int c = 3 * E + e; c < Kx; c += Epad) dlx[t * Kx + c] = 0;  // padding columns
    }
  }
  pdl_trigger();
}

__global__ void __launch_bounds__(256)
    router_w_split_kernel(const float* __restrict__ w, int E, int d, int Kx,
                          uint16_t* __restrict__ wx) {
  pdl_wait();
  const int64_t n = (int64_t)Kx * d;
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (int64_t)gridDim.x * 256) {
    const int r = (int)(i / d), c = (int)(i - (int64_t)r * d);
    const int part = r / E, e = r - part * E;
    uint16_t v = 0;
    if (part < 3) {
      uint16_t hi, mid, lo;
      split3(w[(int64_t)e * d + c], &hi, &mid, &lo);
      v = part == 2 ? mid : hi;
    }
    wx[i] = v;
  }
  pdl_trigger();
}

template <bool BF16, int VEC>
__global__ void __launch_bounds__(256)
    dx_gather_kernel(const void* __restrict__ dout, int add_dout, const float* __restrict__ dense_dx,
                     const float* __restrict__ dxp, const int32_t* __restrict__ offsets,
                     const int32_t* __restrict__ ids, const int32_t* __restrict__ slot, int64_t T,
                     int d, int E, int k, int64_t rows_max, const float* __restrict__ dx_router,
                     void* __restrict__ dx) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (t < T) {
    int64_t rows[MOE_MAX_TOPK];
    int nk = 0;
    for (int j = 0; j < k; ++j) {
      const int s = slot[t * k + j];
      const int e = ids[t * k + j];
      if (s < 0 || e < 0 || e >= E) continue;
      const int64_t r = (int64_t)offsets[e] + s;
      if (r < rows_max) rows[nk++] = r;
    }
    for (int c = lane * VEC; c < d; c += 32 * VEC) {
      float acc[VEC];
#pragma unroll
      for (int v = 0; v < VEC; ++v) acc[v] = 0.0f;
      auto add4 = [&](const float* src) {
        if constexpr (VEC == 4) {
          const float4 q = *reinterpret_cast<const float4*>(src);
          acc[0] += q.x; acc[1] += q.y; acc[2] += q.z; acc[3] += q.w;
        } else {
#pragma unroll
          for (int v = 0; v < VEC; ++v) acc[v] += src[v];
        }
      };
      if (add_dout) {
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[v] = ld_any<BF16>(dout, t * d + c + v);
      }
      if (dense_dx) add4(dense_dx + t * d + c);
      for (int j = 0; j < nk; ++j) add4(dxp + rows[j] * d + c);
      if (dx_router) add4(dx_router + t * d + c);
#pragma unroll
      for (int v = 0; v < VEC; ++v) st_any<BF16>(dx, t * d + c + v, acc[v]);
    }
  }
  pdl_trigger();
}

constexpr int kSBM = 64, kSBN = 64, kSBK = 16;

template <bool ABF, bool BBF>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const SimtGemm p) {
  __shared__ float As[kSBK][kSBM + 4];
  __shared__ float Bs[kSBK][kSBN + 4];
  pdl_wait();
  const int e = blockIdx.z / p.splits, sidx = blockIdx.z - e * p.splits;
  int64_t r0 = 0, len = 0;
  if (p.ragged) {
    int64_t a = p.offsets ? p.offsets[e] : 0, b = p.offsets ? p.offsets[e + 1] : p.rows_max;
    if (a < 0 || b < a || b > p.rows_max) a = b = 0;
    r0 = a;
    len = b - a;
  }
  const int64_t M = p.ragged == 1 ? len : p.M;
  const int64_t Kfull = p.ragged == 2 ? len : p.K;
  const int64_t kchunk = (Kfull + p.splits - 1) / p.splits;
  const int64_t k0 = sidx * kchunk, k1 = min(Kfull, k0 + kchunk);
  const int64_t m0 = (int64_t)blockIdx.y * kSBM, n0 = (int64_t)blockIdx.x * kSBN;
  if (m0 < M) {
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int64_t am = p.ragged == 1 ? r0 : 0, ak = p.ragged == 2 ? r0 : 0;
    const int64_t bk = p.ragged == 2 ? r0 : 0, cm = p.ragged == 1 ? r0 : 0;
    const int64_t ea = (int64_t)e * p.a_e, eb = (int64_t)e * p.b_e;
    float acc[4][4] = {};
    for (int64_t kt = k0; kt < k1; kt += kSBK) {
      __syncthreads();
      for (int i = tid; i < kSBM * kSBK; i += 256) {
        const int mm = i % kSBM, kk = i / kSBM;
        const int64_t gm = m0 + mm, gk = kt + kk;
        As[kk][mm] = (gm < M && gk < k1) ? ld_any<ABF>(p.a, ea + (am + gm) * p.a_m + (ak + gk) * p.a_k)
                                         : 0.0f;
      }
      for (int i = tid; i < kSBN * kSBK; i += 256) {
        const int nn = i % kSBN, kk = i / kSBN;
        const int64_t gn = n0 + nn, gk = kt + kk;
        Bs[kk][nn] = (gn < p.N && gk < k1) ? ld_any<BBF>(p.b, eb + (bk + gk) * p.b_k + gn * p.b_n)
                                           : 0.0f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kSBK; ++kk) {
        float av[4], bv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
    }
    const int64_t ec = (int64_t)e * p.c_e + (int64_t)sidx * p.split_stride;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t gm = m0 + ty * 4 + i;
      if (gm >= M) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t gn = n0 + tx * 4 + j;
        if (gn >= p.N) continue;
        const int64_t ci = ec + (cm + gm) * p.c_m + gn * p.c_n;
        float v = acc[i][j];
        if (p.mul) v *= p.mul_bf16 ? bf16_to_f32(reinterpret_cast<const uint16_t*>(p.mul)[ci])
                                   : reinterpret_cast<const float*>(p.mul)[ci];
        if (p.c16) p.c16[ci] = f32_to_bf16_rn(v);
        else p.c[ci] = v;
      }
    }
  }
  pdl_trigger();
}

}  // namespace

cudaError_t enqueue_combine_backward(const void* dout, bool bf16, const float* y_packed,
                                     const int32_t* offsets, const int32_t* ids,
                                     const int32_t* slot, const float* gates, int64_t T, int d,
                                     int E, int k, int64_t rows_max, float* dgate, void* dy,
                                     int* status, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const dim3 grid((unsigned)((T * 32 + 255) / 256));
  return bf16 ? launch_kernel(combine_backward_kernel<true>, grid, dim3(256), 0, stream, dout,
                              y_packed, offsets, ids, slot, gates, T, d, E, k, rows_max, dgate, dy,
                              status)
              : launch_kernel(combine_backward_kernel<false>, grid, dim3(256), 0, stream, dout,
                              y_packed, offsets, ids, slot, gates, T, d, E, k, rows_max, dgate, dy,
                              status);
}

cudaError_t enqueue_router_backward(const float* logits, const int32_t* ids, const float* dgate,
                                    const unsigned* first_counts, int64_t T, int E, int k,
                                    float alpha, float aux_weight, float z_weight,
                                    bool renormalize, float* dl, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const dim3 grid((unsigned)((T * 32 + 255) / 256));
  const int rn = renormalize ? 1 : 0;
  auto go = [&](auto kern) {
    return launch_kernel(kern, grid, dim3(256), 0, stream, logits, ids, dgate, first_counts, T, E,
                         k, alpha, aux_weight, z_weight, rn, dl);
  };
  if (E <= 32) return go(router_backward_kernel<1>);
  if (E <= 64) return go(router_backward_kernel<2>);
  if (E <= 128) return go(router_backward_kernel<4>);
  if (E <= 256) return go(router_backward_kernel<8>);
  if (E <= 512) return go(router_backward_kernel<16>);
  return go(router_backward_kernel<32>);
}

int colsum_splits(int64_t longest_segment) {
  const int64_t s = (longest_segment + 511) / 512;
  return (int)(s < 1 ? 1 : (s > 64 ? 64 : s));
}

cudaError_t enqueue_colsum(const void* X, bool bf16, const int32_t* offsets, int E,
                           int64_t rows_max, int N, int S, float* partial, float* out,
                           cudaStream_t stream) {
  if (E <= 0 || N <= 0) return cudaSuccess;
  const dim3 grid((unsigned)((N + 255) / 256), (unsigned)E, (unsigned)S);
  float* dst = S == 1 ? out : partial;
  cudaError_t e = bf16 ? launch_kernel(colsum_kernel<true>, grid, dim3(256), 0, stream, X, offsets,
                                       rows_max, N, S, dst)
                       : launch_kernel(colsum_kernel<false>, grid, dim3(256), 0, stream, X,
                                       offsets, rows_max, N, S, dst);
  if (e != cudaSuccess || S == 1) return e;
  return enqueue_split_reduce(partial, E, S, N, out, stream);
}

cudaError_t enqueue_split_reduce(const float* part, int64_t groups, int S, int64_t N, float* out,
                                 cudaStream_t stream, int64_t N_stride) {
  const int64_t n = groups * N;
  if (n == 0) return cudaSuccess;
  return launch_kernel(split_reduce_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0,
                       stream, part, groups, S, N, N_stride > 0 ? N_stride : N, out);
}

cudaError_t enqueue_router_bwd_split(const float* dl, int64_t T, int64_t Tpad, int E, int Epad,
                                     int Kx, uint16_t* dl3, uint16_t* dlx, const float* w_router,
                                     int d, uint16_t* wx, cudaStream_t stream) {
  const int64_t n = Tpad * Epad;
  const unsigned blocks = (unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  cudaError_t e = launch_kernel(router_bwd_split_kernel, dim3(blocks), dim3(256), 0, stream, dl,
                                T, Tpad, E, Epad, Kx, dl3, dlx);
  if (e != cudaSuccess) return e;
  const int64_t nw = (int64_t)Kx * d;
  const unsigned bw = (unsigned)((nw + 255) / 256 < 4096 ? (nw + 255) / 256 : 4096);
  return launch_kernel(router_w_split_kernel, dim3(bw), dim3(256), 0, stream, w_router, E, d, Kx,
                       wx);
}

cudaError_t enqueue_dx_gather(const void* dout, bool bf16, bool add_dout, const float* dense_dx,
                              const float* dxp, const int32_t* offsets, const int32_t* ids,
                              const int32_t* slot, int64_t T, int d, int E, int k,
                              int64_t rows_max, const float* dx_router, void* dx,
                              cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const dim3 grid((unsigned)((T * 32 + 255) / 256));
  const int ad = add_dout ? 1 : 0;
  auto go = [&](auto kern) {
    return launch_kernel(kern, grid, dim3(256), 0, stream, dout, ad, dense_dx, dxp, offsets, ids,
                         slot, T, d, E, k, rows_max, dx_router, dx);
  };
  if (d % 4 == 0) return bf16 ? go(dx_gather_kernel<true, 4>) : go(dx_gather_kernel<false, 4>);
  return bf16 ? go(dx_gather_kernel<true, 1>) : go(dx_gather_kernel<false, 1>);
}

cudaError_t enqueue_simt_gemm(const SimtGemm& p, int64_t m_extent, cudaStream_t stream) {
  if (p.N <= 0 || m_extent <= 0) return cudaSuccess;
  const dim3 grid((unsigned)((p.N + kSBN - 1) / kSBN), (unsigned)((m_extent + kSBM - 1) / kSBM),
                  (unsigned)(p.E * p.splits));
  auto go = [&](auto kern) { return launch_kernel(kern, grid, dim3(256), 0, stream, p); };
  if (p.a_bf16 && p.b_bf16) return go(simt_gemm_kernel<true, true>);
  if (p.a_bf16) return go(simt_gemm_kernel<true, false>);
  if (p.b_bf16) return go(simt_gemm_kernel<false, true>);
  return go(simt_gemm_kernel<false, false>);
}

}  // namespace moe
