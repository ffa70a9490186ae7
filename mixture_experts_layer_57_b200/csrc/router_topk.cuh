// Softmax, top-k and load-balance statistics of the router, one 64-token block at a time, as
// device code shared by the standalone top-k kernel (router.cu) and the tensor-core router kernel
// whose epilogue runs it on logits held in shared memory (router_fused.cu). Both therefore give
// the same bits.
//
// DeepSpeed MoE blog, MoE formula p(x) = softmax(W_r x) and the top-k step of its pipeline
// listing; comparison article, "Top-1 routing decision" and "Router Z-loss"; MoE survey notes
// §1.1.1.1 (renormalised top-k gates) and §1.1.4.1 (f_i, Q_i, alpha * N * sum_i f_i Q_i,
// Importance and Load).
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr double kQScale = 4294967296.0;  // 2^32: fixed-point scale of the p sums
constexpr double kZScale = 16777216.0;    // 2^24: fixed-point scale of the (log Z)^2 sums
constexpr double kIScale = 16777216.0;    // 2^24: fixed-point scale of the gate sums

// Barrier of a whole thread block, or of a named subset of its warps.
struct BlockSync {
  __device__ __forceinline__ void operator()() const { __syncthreads(); }
};
struct NamedSync {
  int id, nthreads;
  __device__ __forceinline__ void operator()() const {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
  }
};

// f, Q, aux and the router losses from the integer totals of T tokens; called by all `nthr`
// threads of a group synchronised by `sync` (tid = 0..nthr-1; prod: E floats of shared memory).
// Totals are read through accessors so that the top-k's last block and the shard finalisation run
// the same arithmetic.
template <class Q, class Cn, class I, class L, class Sync>
__device__ void router_finalize_block(int E, int64_t T, float alpha, Q q_at, Cn c_at, I imp_at,
                                      L load_at, unsigned long long zsum, float* lb, float* losses,
                                      float* prod, int tid, int nthr, Sync sync) {
  if (lb != nullptr) {
    for (int e = tid; e < E; e += nthr) {
      const float Qe = (float)((double)q_at(e) / kQScale / (double)T);
      const float f = (float)c_at(e) / (float)T;
      lb[e] = f;
      lb[E + e] = Qe;
      prod[e] = f * Qe;
    }
    sync();
    if (tid == 0) {
      float s = 0.0f;
      for (int e = 0; e < E; ++e) s += prod[e];
      lb[2 * E] = alpha * (float)E * s;
    }
  }
  if (losses != nullptr && tid == 0) {
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

// Shared memory of one 64-token statistics block of the top-k (E_MAX experts at most).
template <int E_MAX, bool COUNT, bool EXTRA>
struct TopkShared {
  float qs[8][E_MAX];
  // per expert: first-choice count << 16 | choice count (each at most kRouterTokensPerBlock)
  unsigned cs[E_MAX];
  // gate sums, 2^-24 fixed point (< 2^31 per block); only with the extra statistics
  unsigned imp_s[EXTRA ? E_MAX : 1];
  float zs[8];
  float prod[E_MAX];
  int is_last;
  int blk_ids[COUNT ? kRouterTokensPerBlock * MOE_MAX_TOPK : 1];
};

// What the top-k writes and accumulates.
struct TopkOut {
  int64_t T;
  int E, k;
  int32_t* ids;
  float* gates;
  float* probs;  // optional: the chosen probabilities before renormalisation
  RouterAccum acc;
  float alpha;
  float* lb;
  RouterDispatchCount dc;
  int renorm;
  float* losses;
  int64_t* exported;
  // accumulate the z-loss, Importance and Load sums although this launch writes no losses (the
  // dispatch scan finalises them)
  int extra_stats;
};

// Softmax, top-k and the statistics of the 64-token block `blk` (tokens [64 blk, 64 blk + 64)),
// by 256 threads (tid 0..255, 8 warps) synchronised by `sync`; logit_at(r, e) gives the fp32
// logit of expert e for the block's token r. One warp per token: max, sum of exp,
// p = exp(l - max) / sum, k rounds of warp argmax on the logits (ties -> lower index), gates
// (optionally renormalised over the k choices: survey notes §1.1.1.1); per-block sums of p (fixed
// order: warps ascending, each warp's tokens ascending), first-choice counts, gate sums
// (Importance), choice counts (Load) and (log Z)^2 (comparison article, "Router Z-loss") are added
// to the global accumulators as integers (fixed point), so the totals do not depend on the order
// of the blocks. EPL = experts per lane (E <= 32 * EPL); expert e lives in lane e % 32, slot e / 32.
// COUNT: also rank the block's (token, choice) pairs per expert in pair order for dispatch.
template <int EPL, bool COUNT, bool EXTRA, int E_MAX, class Logit, class Sync>
__device__ __forceinline__ void topk_block(const TopkOut& ko, int64_t blk, Logit logit_at,
                                           Sync sync, int tid,
                                           TopkShared<E_MAX, COUNT, EXTRA>& sh) {
  const int64_t T = ko.T;
  const int E = ko.E, k = ko.k;
  int32_t* __restrict__ ids = ko.ids;
  float* __restrict__ gates = ko.gates;
  float* __restrict__ probs = ko.probs;
  const RouterAccum& acc = ko.acc;
  const RouterDispatchCount& dc = ko.dc;
  const int renorm = ko.renorm;
  auto& qs = sh.qs;
  auto& cs = sh.cs;
  auto& imp_s = sh.imp_s;
  auto& zs = sh.zs;
  auto& prod = sh.prod;
  auto& blk_ids = sh.blk_ids;
  const int warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < E; e += 256) {
    cs[e] = 0u;
    if constexpr (EXTRA) imp_s[e] = 0u;
  }
  sync();
  float zw = 0.0f;  // this warp's sum of (log Z)^2 over its tokens, in token order
  float q[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) q[i] = 0.0f;
  const int64_t tb = blk * kRouterTokensPerBlock;
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
  // A warp takes its tokens r = warp, warp + 8, ... TPI at a time (r, r + 8, ...): their softmaxes
  // are computed with the shuffle reductions interleaved (independent dependency chains), and each
  // token's p is added to this warp's sums in token order, as one at a time would. Two tokens for
  // up to 128 experts; one beyond (the registers would not hold two).
  constexpr int TPI = EPL <= 4 ? 2 : 1;
  for (int r0 = warp; r0 < kRouterTokensPerBlock; r0 += 8 * TPI) {
    int rr[TPI];
    bool ok[TPI];
    float l[TPI][EPL], m[TPI], s[TPI], p[TPI][EPL];
#pragma unroll
    for (int u = 0; u < TPI; ++u) {
      rr[u] = r0 + 8 * u;
      ok[u] = rr[u] < kRouterTokensPerBlock && tb + rr[u] < T;
      m[u] = -INFINITY;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        l[u][i] = (ok[u] && e < E) ? logit_at(rr[u], e) : -INFINITY;
        m[u] = fmaxf(m[u], l[u][i]);
      }
    }
    if (!ok[0]) break;
#pragma unroll
    for (int o = 16; o; o >>= 1)
#pragma unroll
      for (int u = 0; u < TPI; ++u) m[u] = fmaxf(m[u], __shfl_xor_sync(0xffffffffu, m[u], o));
    float ex[TPI][EPL];
#pragma unroll
    for (int u = 0; u < TPI; ++u) {
      s[u] = 0.0f;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        ex[u][i] = (ok[u] && (lane + 32 * i) < E) ? expf(l[u][i] - m[u]) : 0.0f;
        s[u] += ex[u][i];
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
#pragma unroll
      for (int u = 0; u < TPI; ++u) s[u] += __shfl_xor_sync(0xffffffffu, s[u], o);
#pragma unroll
    for (int u = 0; u < TPI; ++u) {
      if (!ok[u]) continue;
      if constexpr (EXTRA) {
        const float lz = m[u] + logf(s[u]);  // log sum_e exp(l_e)
        zw += lz * lz;
      }
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        p[u][i] = ex[u][i] / s[u];
        q[i] += p[u][i];
      }
    }
#pragma unroll
    for (int u = 0; u < TPI; ++u) {
      if (!ok[u]) break;
      const int r = rr[u];
      const int64_t t = tb + r;
      // first choice: the lowest expert index holding the maximum logit (ballot per slot)
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = EPL - 1; i >= 0; --i) {
        const unsigned b = __ballot_sync(0xffffffffu, (lane + 32 * i) < E && l[u][i] == m[u]);
        if (b) bi = 32 * i + __ffs(b) - 1;
      }
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
            if (e < E && !(taken >> i & 1u) && (l[u][i] > bv || bi == 0x7fffffff)) {
              bv = l[u][i];
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
          if (i == slot_i) pv = p[u][i];
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
  }
  if (lane == 0) zs[warp] = zw;
  if constexpr (COUNT) {
    // rank the block's pairs per expert in pair order (warp 0), write ranks and segment counts
    sync();
    int* run = reinterpret_cast<int*>(prod);  // reused as running counts until the finalize
    for (int e = tid; e < E; e += 256) run[e] = 0;
    sync();
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
    sync();
    for (int e = tid; e < E; e += 256) dc.seg_counts[blk * E + e] = run[e];
    sync();
  }
  // block sums of p in a fixed order (warps ascending), then integer accumulation
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) qs[warp][e] = q[i];
  }
  sync();
  for (int e = tid; e < E; e += 256) {
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
  if (EXTRA && tid == 0) {
    float zb = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) zb += zs[w];
    atomicAdd(acc.z, (unsigned long long)llrint((double)zb * kZScale));
  }
}

// After topk_block: the last of the n_blocks statistics blocks to finish turns the totals into
// f, Q, aux (and the losses), or exports them (token shards).
template <int E_MAX, bool COUNT, bool EXTRA, class Sync>
__device__ __forceinline__ void topk_block_last(const TopkOut& ko, unsigned n_blocks, Sync sync,
                                                int tid, TopkShared<E_MAX, COUNT, EXTRA>& sh) {
  if (ko.lb == nullptr && ko.losses == nullptr && ko.exported == nullptr) return;
  const int64_t T = ko.T;
  const int E = ko.E;
  const RouterAccum& acc = ko.acc;
  const float alpha = ko.alpha;
  float* lb = ko.lb;
  float* losses = ko.losses;
  int64_t* exported = ko.exported;
  int& is_last = sh.is_last;
  auto& prod = sh.prod;
    // the last block to finish turns the totals into f, Q, aux (and the losses), or exports them
  __threadfence();
  sync();
  if (tid == 0) is_last = atomicAdd(acc.ticket, 1u) == n_blocks - 1;
  sync();
  if (!is_last) return;
  __threadfence();
  if (exported != nullptr) {
    for (int e = tid; e < E; e += 256) {
      exported[e] = (int64_t)atomicAdd(&acc.q[e], 0ull);
      exported[E + e] = (int64_t)atomicAdd(&acc.c[e], 0u);
      exported[2 * E + e] = (int64_t)atomicAdd(&acc.imp[e], 0ull);
      exported[3 * E + e] = (int64_t)atomicAdd(&acc.load[e], 0u);
    }
    if (tid == 0) exported[4 * E] = (int64_t)atomicAdd(acc.z, 0ull);
    return;
  }
  router_finalize_block(
      E, T, alpha, [&](int e) { return atomicAdd(&acc.q[e], 0ull); },
      [&](int e) { return (unsigned long long)atomicAdd(&acc.c[e], 0u); },
      [&](int e) { return atomicAdd(&acc.imp[e], 0ull); },
      [&](int e) { return (unsigned long long)atomicAdd(&acc.load[e], 0u); },
      atomicAdd(acc.z, 0ull), lb, losses, prod, tid, 256, sync);
}

}  // namespace
}  // namespace moe
