// Router: logits = x W_r^T (+ b_r) in fp32, softmax over all E experts, top-k, and the Switch
// load-balance statistics (f_i, Q_i, aux).
//
// DeepSpeed MoE blog, MoE formula p(x) = softmax(W_r x) and the top-k step of its pipeline
// listing (expert ids and gates per token); comparison article, "Router computation"
// (logits = x W_r, p = softmax(logits)) and "Top-1 routing decision"; MoE survey notes
// §1.1.4.1 (f_i = share of tokens whose first choice is i, Q_i = mean p_i,
// loss = alpha * N * sum_i f_i Q_i).
//
// Kernels, in launch order:
//   router_prep_kernel    zeroes the statistics accumulators; for bf16 x also splits W_r (fp32)
//                         into three bf16 parts hi + mid + lo that sum to W_r exactly (each takes
//                         the next 8 significant bits), for the tensor-core logits
//   logits                router_logits_tc_kernel (router_fused.cu, tcgen05: x * W_r =
//                         x*hi + x*mid + x*lo from exact products, fp32 accumulation) for bf16 x,
//                         or router_logits_kernel below (fp32 FMA) for fp32 x
//   router_topk_tile_kernel (E <= 128) 128 tokens per block, two threads per token, the code
//                         the tensor-core router runs in its epilogue (router_topk.cuh);
//   router_topk_kernel    (E > 128) one warp per token. Both: max, sum of exp,
//                         p = exp(l - max) / sum,
//                         k rounds of argmax on the logits (ties -> lower index), gates
//                         (optionally renormalised over the k choices: survey notes §1.1.1.1);
//                         per-block sums of p (fixed order), first-choice counts, gate sums
//                         (Importance), choice counts (Load) and (log Z)^2 (comparison article,
//                         "Router Z-loss") are added to global accumulators as integers (fixed
//                         point), so the totals do not depend on the order of the blocks; the last
//                         block to finish turns them into f, Q, aux, z-loss and the CoV^2 of
//                         Importance and Load (survey notes §1.1.4.1)
#include "common.cuh"
#include "kernels.h"
#include "router_topk.cuh"

namespace moe {
namespace {

// fp32-FMA logits for fp32 x: 64 tokens x 64 experts per block, K in index order.
constexpr int kLBM = 64, kLBN = 64, kLBK = 32;

template <bool XBF16>
__global__ void __launch_bounds__(256) router_logits_kernel(const void* __restrict__ x,
                                                            const float* __restrict__ w,
                                                            const float* __restrict__ bias,
                                                            int64_t T, int d, int E,
                                                            float* __restrict__ logits) {
  __shared__ float xs[kLBK][kLBM + 4];
  __shared__ float ws[kLBK][kLBN + 4];
  pdl_wait();
  const int tx = threadIdx.x & 15;   // expert lane
  const int ty = threadIdx.x >> 4;   // token lane
  const int64_t t0 = (int64_t)blockIdx.x * kLBM;
  const int e0 = blockIdx.y * kLBN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < d; k0 += kLBK) {
    // stage x[t0 .. t0+64, k0 .. k0+32] and w[e0 .. e0+64, k0 .. k0+32] (transposed in smem)
    for (int i = threadIdx.x; i < kLBM * kLBK; i += 256) {
      const int r = i / kLBK, c = i % kLBK;
      const int64_t t = t0 + r;
      const int kk = k0 + c;
      xs[c][r] = (t < T && kk < d) ? load_elem<XBF16>(x, t * d + kk) : 0.0f;
      const int e = e0 + r;
      ws[c][r] = (e < E && kk < d) ? w[(int64_t)e * d + kk] : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < kLBK; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[c][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = ws[c][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t t = t0 + ty + 16 * i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx + 16 * j;
      if (e < E) logits[t * E + e] = acc[i][j] + (bias ? bias[e] : 0.0f);
    }
  }
  pdl_trigger();
}

// Decode-sized batches (T <= kRouterGemvMaxT): one block per expert, a warp per token (four at a
// time), lanes over K with 16-byte loads, fp32 FMA, fixed-order warp reduction; block 0 also
// zeroes the statistics accumulators (this kernel then replaces the prep kernel).
template <bool XBF16>
__global__ void __launch_bounds__(256) router_gemv_kernel(const void* __restrict__ x,
                                                          const float* __restrict__ w,
                                                          const float* __restrict__ bias,
                                                          int64_t T, int d, int E,
                                                          float* __restrict__ logits,
                                                          RouterAccum acc) {
  pdl_wait();
  const int e = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (e == 0) {
    for (int i = threadIdx.x; i < E; i += blockDim.x) {
      acc.q[i] = 0ull;
      acc.c[i] = 0u;
      acc.imp[i] = 0ull;
      acc.load[i] = 0u;
    }
    if (threadIdx.x == 0) {
      *acc.z = 0ull;
      *acc.ticket = 0u;
    }
  }
  const float* wr = w + (int64_t)e * d;
  if constexpr (XBF16) {
    if ((d & 7) == 0) {
      // Each lane owns elements lane*8 + 256 j (j = 0, 1, ...) of the weight row; a warp takes
      // tokens warp, warp + 8, ... four at a time. Per chunk of four j, the lane's weights and the
      // four tokens' x values are all requested before the first FMA (24 independent 16/32-byte
      // loads in flight instead of one round trip per j). Every sum adds its products in the
      // same order as one token at a time would (j ascending, 8 elements each), then the same
      // warp reduction.
      const uint16_t* xb = reinterpret_cast<const uint16_t*>(x);
      for (int64_t t0 = warp; t0 < T; t0 += 32) {
        float s[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int j0 = 0; j0 < d; j0 += 1024) {
          float4 wv[8];
          uint4 xv[4][4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int i = j0 + 256 * q + lane * 8;
            const bool in = i < d;
            wv[2 * q] = in ? *reinterpret_cast<const float4*>(wr + i) : make_float4(0, 0, 0, 0);
            wv[2 * q + 1] = in ? *reinterpret_cast<const float4*>(wr + i + 4) : make_float4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int64_t t = t0 + 8 * u;
              xv[u][q] = (in && t < T) ? *reinterpret_cast<const uint4*>(xb + t * d + i)
                                       : make_uint4(0, 0, 0, 0);
            }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (j0 + 256 * q + lane * 8 >= d) continue;
              const uint4 xq = xv[u][q];
              const float4 w0 = wv[2 * q], w1 = wv[2 * q + 1];
              float a = s[u];
              a = fmaf(__uint_as_float(xq.x << 16), w0.x, a);
              a = fmaf(__uint_as_float(xq.x & 0xffff0000u), w0.y, a);
              a = fmaf(__uint_as_float(xq.y << 16), w0.z, a);
              a = fmaf(__uint_as_float(xq.y & 0xffff0000u), w0.w, a);
              a = fmaf(__uint_as_float(xq.z << 16), w1.x, a);
              a = fmaf(__uint_as_float(xq.z & 0xffff0000u), w1.y, a);
              a = fmaf(__uint_as_float(xq.w << 16), w1.z, a);
              a = fmaf(__uint_as_float(xq.w & 0xffff0000u), w1.w, a);
              s[u] = a;
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float v = s[u];
#pragma unroll
          for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          const int64_t t = t0 + 8 * u;
          if (lane == 0 && t < T) logits[t * E + e] = v + (bias ? bias[e] : 0.0f);
        }
      }
      pdl_trigger();
      return;
    }
  }
  for (int64_t t = warp; t < T; t += 8) {
    float s = 0.0f;
    if constexpr (XBF16) {
      const uint16_t* xr = reinterpret_cast<const uint16_t*>(x) + t * d;
      if ((d & 7) == 0) {
        for (int i = lane * 8; i < d; i += 256) {
          const uint4 xv = *reinterpret_cast<const uint4*>(xr + i);
          const float4 w0 = *reinterpret_cast<const float4*>(wr + i);
          const float4 w1 = *reinterpret_cast<const float4*>(wr + i + 4);
          s = fmaf(__uint_as_float(xv.x << 16), w0.x, s);
          s = fmaf(__uint_as_float(xv.x & 0xffff0000u), w0.y, s);
          s = fmaf(__uint_as_float(xv.y << 16), w0.z, s);
          s = fmaf(__uint_as_float(xv.y & 0xffff0000u), w0.w, s);
          s = fmaf(__uint_as_float(xv.z << 16), w1.x, s);
          s = fmaf(__uint_as_float(xv.z & 0xffff0000u), w1.y, s);
          s = fmaf(__uint_as_float(xv.w << 16), w1.z, s);
          s = fmaf(__uint_as_float(xv.w & 0xffff0000u), w1.w, s);
        }
      } else {
        for (int i = lane; i < d; i += 32) s = fmaf(bf16_to_f32(xr[i]), wr[i], s);
      }
    } else {
      const float* xr = reinterpret_cast<const float*>(x) + t * d;
      if ((d & 3) == 0) {
        for (int i = lane * 4; i < d; i += 128) {
          const float4 xv = *reinterpret_cast<const float4*>(xr + i);
          const float4 wv = *reinterpret_cast<const float4*>(wr + i);
          s = fmaf(xv.x, wv.x, s);
          s = fmaf(xv.y, wv.y, s);
          s = fmaf(xv.z, wv.z, s);
          s = fmaf(xv.w, wv.w, s);
        }
      } else {
        for (int i = lane; i < d; i += 32) s = fmaf(xr[i], wr[i], s);
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) logits[t * E + e] = s + (bias ? bias[e] : 0.0f);
  }
  pdl_trigger();
}

__global__ void __launch_bounds__(256) router_prep_kernel(const float* __restrict__ w, int E,
                                                          int d, int dpad, uint16_t* __restrict__ out,
                                                          RouterAccum acc) {
  pdl_wait();
  if (blockIdx.x == 0 && acc.q != nullptr) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      acc.q[e] = 0ull;
      acc.c[e] = 0u;
      acc.imp[e] = 0ull;
      acc.load[e] = 0u;
    }
    if (threadIdx.x == 0) {
      *acc.z = 0ull;
      *acc.ticket = 0u;
    }
  }
  if (out == nullptr) {
    pdl_trigger();
    return;
  }
  const int64_t n = (int64_t)E * dpad;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int e = (int)(idx / dpad), i = (int)(idx % dpad);
    const float v = i < d ? w[(int64_t)e * d + i] : 0.0f;
    const uint16_t hi = f32_to_bf16_rn(v);
    const float r1 = v - bf16_to_f32(hi);     // exact: hi is v rounded to 8 significant bits
    const uint16_t mid = f32_to_bf16_rn(r1);
    const float r2 = r1 - bf16_to_f32(mid);   // exact, at most 8 significant bits left
    const uint16_t lo = f32_to_bf16_rn(r2);   // == r2
    uint16_t* row = out + (int64_t)e * 3 * dpad;
    row[i] = hi;
    row[dpad + i] = mid;
    row[2 * dpad + i] = lo;
  }
  pdl_trigger();
}

__global__ void __launch_bounds__(256)
    router_finalize_kernel(const int64_t* __restrict__ tot, int64_t T, int E, float alpha,
                           float* __restrict__ lb, float* __restrict__ losses) {
  __shared__ float prod[MOE_MAX_EXPERTS];
  pdl_wait();
  router_finalize_block(
      E, T, alpha, [&](int e) { return (unsigned long long)tot[e]; },
      [&](int e) { return (unsigned long long)tot[E + e]; },
      [&](int e) { return (unsigned long long)tot[2 * E + e]; },
      [&](int e) { return (unsigned long long)tot[3 * E + e]; }, (unsigned long long)tot[4 * E],
      lb, losses, prod, threadIdx.x, blockDim.x, BlockSync{});
  pdl_trigger();
}

template <int EPL, bool COUNT, bool EXTRA>
__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ logits,
                                                          const TopkOut ko) {
  __shared__ TopkShared<MOE_MAX_EXPERTS, COUNT, EXTRA> sh;
  pdl_wait();
  const int64_t tb = (int64_t)blockIdx.x * kRouterTokensPerBlock;
  const int E = ko.E;
  topk_block<EPL, COUNT, EXTRA>(
      ko, (int64_t)blockIdx.x, [&](int r, int e) { return logits[(tb + r) * E + e]; },
      BlockSync{}, (int)threadIdx.x, sh);
  pdl_trigger();
  topk_block_last(ko, gridDim.x, BlockSync{}, (int)threadIdx.x, sh);
}

// E <= 128: one 128-token tile per block, its logits staged in shared memory in the layout of
// the tensor-core router's epilogue, then the tile top-k that epilogue runs.
template <int NE, bool COUNT, bool EXTRA>
__global__ void __launch_bounds__(256) router_topk_tile_kernel(const float* __restrict__ logits,
                                                               const TopkOut ko) {
  extern __shared__ __align__(16) uint8_t tile_smem[];
  float* L = reinterpret_cast<float*>(tile_smem);
  auto& sh = *reinterpret_cast<TileShared<COUNT, EXTRA>*>(tile_smem + tile_logits_bytes<NE>());
  pdl_wait();
  const int64_t tile = blockIdx.x;
  const int64_t t0 = tile * kTileTokens;
  const int E = ko.E;
  const int n = (int)min((int64_t)kTileTokens, ko.T - t0) * E;
  for (int i = threadIdx.x; i < n; i += 256) {
    const int r = i / E, e = i - r * E;
    L[lpos<NE>(r, e)] = logits[t0 * E + i];
  }
  __syncthreads();
  topk_tile<NE, COUNT, EXTRA>(ko, tile, L, BlockSync{}, (int)threadIdx.x, sh);
  pdl_trigger();
  const unsigned n_blocks = (unsigned)((ko.T + kRouterTokensPerBlock - 1) / kRouterTokensPerBlock);
  topk_tile_last(ko, tile, n_blocks, BlockSync{}, (int)threadIdx.x, sh);
}

template <int NE, bool COUNT, bool EXTRA>
cudaError_t launch_topk_tile(const float* logits, const TopkOut& ko, cudaStream_t stream) {
  auto kern = router_topk_tile_kernel<NE, COUNT, EXTRA>;
  constexpr int smem = tile_logits_bytes<NE>() + (int)sizeof(TileShared<COUNT, EXTRA>);
  static int attr_done[64] = {0};  // per device
  cudaError_t e = ensure_dynamic_smem(kern, smem, attr_done);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((ko.T + kTileTokens - 1) / kTileTokens));
  return launch_kernel(kern, grid, dim3(256), smem, stream, logits, ko);
}

template <int NE>
cudaError_t launch_topk_tile_ne(const float* logits, const TopkOut& ko, bool count, bool extra,
                                cudaStream_t stream) {
  if (count)
    return extra ? launch_topk_tile<NE, true, true>(logits, ko, stream)
                 : launch_topk_tile<NE, true, false>(logits, ko, stream);
  return extra ? launch_topk_tile<NE, false, true>(logits, ko, stream)
               : launch_topk_tile<NE, false, false>(logits, ko, stream);
}

template <int EPL>
cudaError_t launch_topk(const float* logits, int64_t T, int E, int k, int32_t* ids, float* gates,
                        const RouterAccum& acc, float alpha, float* lb, RouterDispatchCount dc,
                        int renorm, float* losses, int64_t* exported, float* probs,
                        bool extra_stats, cudaStream_t stream) {
  const dim3 grid((unsigned)router_num_blocks(T));
  const bool extra = losses != nullptr || exported != nullptr || extra_stats;
  const TopkOut ko{T, E, k,     ids,    gates,    probs,   acc,
                   alpha, lb, dc, renorm, losses, exported, extra_stats ? 1 : 0};
  if constexpr (EPL * 32 <= kTileExperts) {
    (void)grid;
    const bool count = dc.local_rank != nullptr;
    if (E <= 16) return launch_topk_tile_ne<16>(logits, ko, count, extra, stream);
    if (E <= 32) return launch_topk_tile_ne<32>(logits, ko, count, extra, stream);
    if (E <= 64) return launch_topk_tile_ne<64>(logits, ko, count, extra, stream);
    return launch_topk_tile_ne<128>(logits, ko, count, extra, stream);
  } else {
    auto go = [&](auto kern) {
      return launch_kernel(kern, grid, dim3(256), 0, stream, (const float*)logits, ko);
    };
    if (dc.local_rank != nullptr)
      return extra ? go(router_topk_kernel<EPL, true, true>)
                   : go(router_topk_kernel<EPL, true, false>);
    return extra ? go(router_topk_kernel<EPL, false, true>)
                 : go(router_topk_kernel<EPL, false, false>);
  }
}

}  // namespace

cudaError_t enqueue_router(const void* x, bool x_bf16, int64_t T, int d, const float* w_router,
                           const float* router_bias, int E, int k, float* logits, int32_t* ids,
                           float* gates, float* lb_stats, float aux_alpha,
                           const RouterScratch& scr, int* status, cudaStream_t stream,
                           RouterDispatchCount dc, bool renormalize, float* losses,
                           int64_t* exported, int64_t T_kernel_choice, float* probs,
                           const uint16_t* w_prepared, bool extra_stats) {
  if (T == 0) return cudaSuccess;
  float* const logits_out = logits;  // the caller's (may be nullptr)
  if (!logits) logits = scr.logits_scratch;
  const bool gemv = (T_kernel_choice > T ? T_kernel_choice : T) <= kRouterGemvMaxT;
  const bool tc = !gemv && router_uses_tensor_cores(x_bf16, d);
  const bool prepared = tc && w_prepared != nullptr;
  const bool fused = tc && router_fused_supported(E) && router_fusion_enabled();
  const int dpad = router_split_dpad(d);
  const int64_t n = tc ? (int64_t)E * dpad : 0;
  const unsigned blocks = (unsigned)(n == 0 ? 1 : ((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096));
  cudaError_t err = cudaSuccess;
  if (gemv) {
    err = launch_kernel(x_bf16 ? router_gemv_kernel<true> : router_gemv_kernel<false>, dim3(E),
                        dim3(256), 0, stream, x, w_router, router_bias, T, d, E, logits, scr.acc);
  } else if (!prepared) {
    err = launch_kernel(router_prep_kernel, dim3(blocks), dim3(256), 0, stream, w_router, E, d, dpad,
                        tc ? scr.w_split : nullptr, scr.acc);
  }
  if (err != cudaSuccess) return err;
  if (fused) {
    if (prepared) {
      // no split kernel ran to zero the statistics accumulators (contiguous in the workspace)
      const size_t n = (size_t)((const char*)(scr.acc.ticket + 1) - (const char*)scr.acc.q);
      err = cudaMemsetAsync(scr.acc.q, 0, n, stream);
      if (err != cudaSuccess) return err;
    }
    return enqueue_router_fused(x, T, d, prepared ? w_prepared : scr.w_split, dpad, router_bias, E,
                                k, logits_out, ids, gates, probs, scr.acc, aux_alpha, lb_stats, dc,
                                renormalize, losses, exported, extra_stats, status, stream);
  }
  if (tc) {
    cudaError_t e = enqueue_router_logits_tc(x, T, d, prepared ? w_prepared : scr.w_split, dpad,
                                             router_bias, E, logits, status, stream,
                                             prepared ? &scr.acc : nullptr);
    if (e != cudaSuccess) return e;
  } else if (!gemv) {
    dim3 grid((unsigned)((T + kLBM - 1) / kLBM), (E + kLBN - 1) / kLBN);
    err = launch_kernel(x_bf16 ? router_logits_kernel<true> : router_logits_kernel<false>, grid,
                        dim3(256), 0, stream, x, w_router, router_bias, T, d, E, logits);
    if (err != cudaSuccess) return err;
  }
  const RouterAccum& a = scr.acc;
  const int rn = renormalize ? 1 : 0;
  if (E <= 128)  // the tile top-k (launch_topk's E <= 128 branch)
    return launch_topk<4>(logits, T, E, k, ids, gates, a, aux_alpha, lb_stats, dc, rn,
                          losses, exported, probs, extra_stats, stream);
  if (E <= 256)
    return launch_topk<8>(logits, T, E, k, ids, gates, a, aux_alpha, lb_stats, dc, rn,
                          losses, exported, probs, extra_stats, stream);
  if (E <= 512)
    return launch_topk<16>(logits, T, E, k, ids, gates, a, aux_alpha, lb_stats, dc, rn,
                           losses, exported, probs, extra_stats, stream);
  return launch_topk<32>(logits, T, E, k, ids, gates, a, aux_alpha, lb_stats, dc, rn,
                         losses, exported, probs, extra_stats, stream);
}

cudaError_t enqueue_router_prepare(const float* w_router, int E, int d, uint16_t* out,
                                   cudaStream_t stream) {
  const int dpad = router_split_dpad(d);
  const int64_t n = (int64_t)E * dpad;
  const unsigned blocks = (unsigned)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  // no statistics here: an accumulator set whose pointers are all null is skipped by block 0
  return launch_kernel(router_prep_kernel, dim3(blocks), dim3(256), 0, stream, w_router, E, d,
                       dpad, out, RouterAccum{});
}

cudaError_t enqueue_router_finalize(const int64_t* totals, int64_t T, int E, float aux_alpha,
                                    float* lb_stats, float* losses, cudaStream_t stream) {
  if (lb_stats == nullptr && losses == nullptr) return cudaSuccess;
  return launch_kernel(router_finalize_kernel, dim3(1), dim3(256), 0, stream, totals, T, E,
                       aux_alpha, lb_stats, losses);
}

}  // namespace moe
