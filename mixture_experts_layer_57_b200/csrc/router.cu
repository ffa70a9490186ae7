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
//   router_topk_kernel    one warp per token: max, sum of exp, p = exp(l - max) / sum,
//                         k rounds of warp argmax on the logits (ties -> lower index), gates
//                         (optionally renormalised over the k choices: survey notes §1.1.1.1);
//                         per-block sums of p (fixed order), first-choice counts, gate sums
//                         (Importance), choice counts (Load) and (log Z)^2 (comparison article,
//                         "Router Z-loss") are added to global accumulators as integers (fixed
//                         point), so the totals do not depend on the order of the blocks; the last
//                         block to finish turns them into f, Q, aux, z-loss and the CoV^2 of
//                         Importance and Load (survey notes §1.1.4.1)
#include "common.cuh"
#include "kernels.h"

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

// Decode-sized batches (T <= kRouterGemvMaxT): one block per expert, warp per token, lanes over
// K with 16-byte loads, fp32 FMA, fixed-order warp reduction; block 0 also zeroes the statistics
// accumulators (this kernel then replaces the prep kernel).
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

constexpr double kQScale = 4294967296.0;  // 2^32: fixed-point scale of the p sums
constexpr double kZScale = 16777216.0;    // 2^24: fixed-point scale of the (log Z)^2 sums
constexpr double kIScale = 16777216.0;    // 2^24: fixed-point scale of the gate sums

// f, Q, aux and the router losses from the integer totals of T tokens; called by every thread
// of one 256-thread block (prod: E floats of shared memory). Totals are read through accessors so
// that the top-k kernel's last block and the shard finalisation run the same arithmetic.
template <class Q, class Cn, class I, class L>
__device__ void router_finalize_block(int E, int64_t T, float alpha, Q q_at, Cn c_at, I imp_at,
                                      L load_at, unsigned long long zsum, float* lb, float* losses,
                                      float* prod) {
  if (lb != nullptr) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      const float Qe = (float)((double)q_at(e) / kQScale / (double)T);
      const float f = (float)c_at(e) / (float)T;
      lb[e] = f;
      lb[E + e] = Qe;
      prod[e] = f * Qe;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float s = 0.0f;
      for (int e = 0; e < E; ++e) s += prod[e];
      lb[2 * E] = alpha * (float)E * s;
    }
  }
  if (losses != nullptr && threadIdx.x == 0) {
    // z-loss = mean over tokens of (log Z)^2; CoV^2 = population variance / mean^2 over experts
    losses[0] = (float)((double)zsum / kZScale / (double)T);
    double mi = 0.0, ml = 0.0;
    for (int e = 0; e < E; ++e) {
      mi += (double)imp_at(e) / kIScale;
      ml += (double)load_at(e);
    }
    mi /= E;
    ml /= E;
    double vi = 0.0, vl = 0.0;
    for (int e = 0; e < E; ++e) {
      const double a = (double)imp_at(e) / kIScale - mi;
      const double b = (double)load_at(e) - ml;
      vi += a * a;
      vl += b * b;
    }
    vi /= E;
    vl /= E;
    losses[1] = mi > 0.0 ? (float)(vi / (mi * mi)) : 0.0f;
    losses[2] = ml > 0.0 ? (float)(vl / (ml * ml)) : 0.0f;
  }
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
      lb, losses, prod);
  pdl_trigger();
}

// EPL = experts per lane (E <= 32 * EPL); expert e lives in lane e % 32, slot e / 32.
// COUNT: also rank this block's (token, choice) pairs per expert in pair order for dispatch.
template <int EPL, bool COUNT, bool EXTRA>
__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ logits,
                                                          int64_t T, int E, int k,
                                                          int32_t* __restrict__ ids,
                                                          float* __restrict__ gates,
                                                          RouterAccum acc, float alpha,
                                                          float* __restrict__ lb,
                                                          RouterDispatchCount dc, int renorm,
                                                          float* __restrict__ losses,
                                                          int64_t* __restrict__ exported,
                                                          float* __restrict__ probs) {
  __shared__ float qs[8][MOE_MAX_EXPERTS];
  // per expert: first-choice count << 16 | choice count (each at most kRouterTokensPerBlock)
  __shared__ unsigned cs[MOE_MAX_EXPERTS];
  // gate sums, 2^-24 fixed point (< 2^31 per block); only with the extra statistics
  __shared__ unsigned imp_s[EXTRA ? MOE_MAX_EXPERTS : 1];
  __shared__ float zs[8];
  __shared__ float prod[MOE_MAX_EXPERTS];
  __shared__ int is_last;
  __shared__ int blk_ids[COUNT ? kRouterTokensPerBlock * MOE_MAX_TOPK : 1];
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < E; e += 256) {
    cs[e] = 0u;
    if constexpr (EXTRA) imp_s[e] = 0u;
  }
  __syncthreads();
  float zw = 0.0f;  // this warp's sum of (log Z)^2 over its tokens, in token order
  float q[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) q[i] = 0.0f;
  const int64_t tb = (int64_t)blockIdx.x * kRouterTokensPerBlock;
  for (int r = warp; r < kRouterTokensPerBlock; r += 8) {
    const int64_t t = tb + r;
    if (t >= T) break;
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
    if constexpr (EXTRA) {
      const float lz = m + logf(s);  // log sum_e exp(l_e)
      zw += lz * lz;
    }
    float p[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      p[i] = ex[i] / s;
      q[i] += p[i];
    }
    // first choice: the lowest expert index holding the maximum logit (ballot per slot)
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = EPL - 1; i >= 0; --i) {
      const unsigned b = __ballot_sync(0xffffffffu, (lane + 32 * i) < E && l[i] == m);
      if (b) bi = 32 * i + __ffs(b) - 1;
    }
    // per-block integer counts (order-independent): first choices, and with the extra
    // statistics every choice and its gate
    auto count_choice = [&](int e, int j, float g) {
      if constexpr (EXTRA) {
        atomicAdd(&cs[e], j == 0 ? 0x10001u : 1u);
        atomicAdd(&imp_s[e], __float2uint_rn(g * (float)kIScale));
      } else if (j == 0) {
        atomicAdd(&cs[e], 0x10000u);
      }
    };
    uint32_t taken = 0;
    float gv[MOE_MAX_TOPK];
    int gi[MOE_MAX_TOPK];
    float gsum = 0.0f;
    for (int j = 0; j < k; ++j) {
      if (j > 0) {
        // later choices: (value desc, index asc) warp argmax over the experts not yet taken
        float bv = -INFINITY;
        bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const int e = lane + 32 * i;
          if (e < E && !(taken >> i & 1u) && (l[i] > bv || bi == 0x7fffffff)) {
            bv = l[i];
            bi = e;
          }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
          if (ov > bv || (ov == bv && oi < bi)) {
            bv = ov;
            bi = oi;
          }
        }
      }
      const int owner = bi & 31, slot_i = bi >> 5;
      float pv = 0.0f;
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (i == slot_i) pv = p[i];
      pv = __shfl_sync(0xffffffffu, pv, owner);
      if (lane == owner) taken |= 1u << slot_i;
      if (lane == 0) {
        ids[t * k + j] = bi;
        if (probs != nullptr) probs[t * k + j] = pv;  // before any renormalisation
        if (!renorm) {
          gates[t * k + j] = pv;
          count_choice(bi, j, pv);
        }
        if constexpr (COUNT) blk_ids[r * k + j] = bi;
      }
      if (renorm) {
#pragma unroll
        for (int jj = 0; jj < MOE_MAX_TOPK; ++jj)
          if (jj == j) {
            gv[jj] = pv;
            gi[jj] = bi;
          }
        gsum += pv;
      }
    }
    if (renorm && lane == 0) {
#pragma unroll
      for (int j = 0; j < MOE_MAX_TOPK; ++j) {
        if (j >= k) break;
        const float g = gv[j] / gsum;
        gates[t * k + j] = g;
        count_choice(gi[j], j, g);
      }
    }
  }
  if (lane == 0) zs[warp] = zw;
  if constexpr (COUNT) {
    // rank the block's pairs per expert in pair order (warp 0), write ranks and segment counts
    __syncthreads();
    int* run = reinterpret_cast<int*>(prod);  // reused as running counts until the finalize
    for (int e = threadIdx.x; e < E; e += 256) run[e] = 0;
    __syncthreads();
    const int64_t ntok = min((int64_t)kRouterTokensPerBlock, T - tb);
    const int npairs = (int)ntok * k;
    if (warp == 0) {
      const unsigned lt = (1u << lane) - 1u;
      for (int c = 0; c < npairs; c += 32) {
        const int pl = c + lane;
        const int e = pl < npairs ? blk_ids[pl] : -1;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(same & lt);
        const int base = e >= 0 ? run[e] : 0;
        __syncwarp();
        if (e >= 0 && rank == 0) run[e] = base + __popc(same);
        __syncwarp();
        if (pl < npairs) dc.local_rank[tb * k + pl] = base + rank;
      }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += 256) dc.seg_counts[(int64_t)blockIdx.x * E + e] = run[e];
    __syncthreads();
  }
  // block sums of p in a fixed order (warps ascending), then integer accumulation
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) qs[warp][e] = q[i];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += 256) {
    float sum = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) sum += qs[w][e];
    const unsigned long long fx = (unsigned long long)llrint((double)sum * kQScale);
    if (fx) atomicAdd(&acc.q[e], fx);
    if (cs[e] >> 16) atomicAdd(&acc.c[e], cs[e] >> 16);
    if constexpr (EXTRA) {
      if (cs[e] & 0xffffu) atomicAdd(&acc.load[e], cs[e] & 0xffffu);
      if (imp_s[e]) atomicAdd(&acc.imp[e], (unsigned long long)imp_s[e]);
    }
  }
  if (EXTRA && threadIdx.x == 0) {
    float zb = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) zb += zs[w];
    atomicAdd(acc.z, (unsigned long long)llrint((double)zb * kZScale));
  }
  pdl_trigger();
  if (lb == nullptr && losses == nullptr && exported == nullptr) return;
  // the last block to finish turns the totals into f, Q, aux (and the losses), or exports them
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(acc.ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (exported != nullptr) {
    for (int e = threadIdx.x; e < E; e += 256) {
      exported[e] = (int64_t)atomicAdd(&acc.q[e], 0ull);
      exported[E + e] = (int64_t)atomicAdd(&acc.c[e], 0u);
      exported[2 * E + e] = (int64_t)atomicAdd(&acc.imp[e], 0ull);
      exported[3 * E + e] = (int64_t)atomicAdd(&acc.load[e], 0u);
    }
    if (threadIdx.x == 0) exported[4 * E] = (int64_t)atomicAdd(acc.z, 0ull);
    return;
  }
  router_finalize_block(
      E, T, alpha, [&](int e) { return atomicAdd(&acc.q[e], 0ull); },
      [&](int e) { return (unsigned long long)atomicAdd(&acc.c[e], 0u); },
      [&](int e) { return atomicAdd(&acc.imp[e], 0ull); },
      [&](int e) { return (unsigned long long)atomicAdd(&acc.load[e], 0u); },
      atomicAdd(acc.z, 0ull), lb, losses, prod);
}

template <int EPL>
cudaError_t launch_topk(const float* logits, int64_t T, int E, int k, int32_t* ids, float* gates,
                        const RouterAccum& acc, float alpha, float* lb, RouterDispatchCount dc,
                        int renorm, float* losses, int64_t* exported, float* probs,
                        cudaStream_t stream) {
  const dim3 grid((unsigned)router_num_blocks(T));
  const bool extra = losses != nullptr || exported != nullptr;
  auto go = [&](auto kern) {
    return launch_kernel(kern, grid, dim3(256), 0, stream, (const float*)logits, T, E, k, ids,
                         gates, acc, alpha, lb, dc, renorm, losses, exported, probs);
  };
  if (dc.local_rank != nullptr)
    return extra ? go(router_topk_kernel<EPL, true, true>)
                 : go(router_topk_kernel<EPL, true, false>);
  return extra ? go(router_topk_kernel<EPL, false, true>)
               : go(router_topk_kernel<EPL, false, false>);
}

}  // namespace

cudaError_t enqueue_router(const void* x, bool x_bf16, int64_t T, int d, const float* w_router,
                           const float* router_bias, int E, int k, float* logits, int32_t* ids,
                           float* gates, float* lb_stats, float aux_alpha,
                           const RouterScratch& scr, int* status, cudaStream_t stream,
                           RouterDispatchCount dc, bool renormalize, float* losses,
                           int64_t* exported, int64_t T_kernel_choice, float* probs,
                           const uint16_t* w_prepared) {
  if (T == 0) return cudaSuccess;
  if (!logits) logits = scr.logits_scratch;
  const bool gemv = (T_kernel_choice > T ? T_kernel_choice : T) <= kRouterGemvMaxT;
  const bool tc = !gemv && router_uses_tensor_cores(x_bf16, d);
  const bool prepared = tc && w_prepared != nullptr;
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
  if (E <= 32)
    return launch_topk<1>(logits, T, E, k, ids, gates, a, aux_alpha, lb_stats, dc, rn,
                          losses, exported, probs, stream);
  if (E <= 64)
    return launch_topk<2>(logits, T, E, k, ids, gates, a, aux_alpha, lb_stats, dc, rn,
                          losses, exported, probs, stream);
  if (E <= 128)
    return launch_topk<4>(logits, T, E, k, ids, gates, a, aux_alpha, lb_stats, dc, rn,
                          losses, exported, probs, stream);
  if (E <= 256)
    return launch_topk<8>(logits, T, E, k, ids, gates, a, aux_alpha, lb_stats, dc, rn,
                          losses, exported, probs, stream);
  if (E <= 512)
    return launch_topk<16>(logits, T, E, k, ids, gates, a, aux_alpha, lb_stats, dc, rn,
                           losses, exported, probs, stream);
  return launch_topk<32>(logits, T, E, k, ids, gates, a, aux_alpha, lb_stats, dc, rn,
                         losses, exported, probs, stream);
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
