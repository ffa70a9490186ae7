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

// The last of the n_blocks statistics blocks to finish turns the totals into f, Q, aux (and the
// losses), or exports them (token shards). The calling group has just completed `nb` blocks; it
// finds out whether they were the last through a ticket counter.
template <class Sync>
__device__ __forceinline__ void topk_finish(const TopkOut& ko, unsigned nb, unsigned n_blocks,
                                            Sync sync, int tid, int& is_last, float* prod) {
  if (ko.lb == nullptr && ko.losses == nullptr && ko.exported == nullptr) return;
  const int64_t T = ko.T;
  const int E = ko.E;
  const RouterAccum& acc = ko.acc;
  int64_t* exported = ko.exported;
  __threadfence();
  sync();
  if (tid == 0) is_last = atomicAdd(acc.ticket, nb) + nb == n_blocks;
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
      E, T, ko.alpha, [&](int e) { return atomicAdd(&acc.q[e], 0ull); },
      [&](int e) { return (unsigned long long)atomicAdd(&acc.c[e], 0u); },
      [&](int e) { return atomicAdd(&acc.imp[e], 0ull); },
      [&](int e) { return (unsigned long long)atomicAdd(&acc.load[e], 0u); },
      atomicAdd(acc.z, 0ull), ko.lb, ko.losses, prod, tid, 256, sync);
}

// After topk_block (one statistics block).
template <int E_MAX, bool COUNT, bool EXTRA, class Sync>
__device__ __forceinline__ void topk_block_last(const TopkOut& ko, unsigned n_blocks, Sync sync,
                                                int tid, TopkShared<E_MAX, COUNT, EXTRA>& sh) {
  topk_finish(ko, 1u, n_blocks, sync, tid, sh.is_last, sh.prod);
}

// ------------------------------------------------------------------------------------------------
// Up to 128 experts: the tile variant. A tile is 128 tokens (two statistics blocks) whose logits
// sit in shared memory as fp32 rows of NE columns (NE = E rounded up to a power of two >= 16) with
// a row stride of NE + 4 floats: rows stay 16-byte aligned, and a warp moving 16 bytes per lane
// along 32 consecutive rows, or along one row, touches every bank equally often (no conflicts).
// Token r of the tile belongs to lane r % 32 of warps r / 32 (experts [0, NE/2)) and r / 32 + 4
// (experts [NE/2, NE)); each thread loads its half of the row into registers with 16-byte loads,
// works on it in expert order with independent partial results, and the two halves meet through
// shared memory. All 128 tokens of a tile are thus in flight at once.

constexpr int kTileTokens = 2 * kRouterTokensPerBlock;
constexpr int kTileExperts = 128;

template <int NE>
__device__ __forceinline__ int lpos(int row, int col) {
  return row * (NE + 4) + col;
}
// Bytes of a tile's logits in shared memory.
template <int NE>
constexpr int tile_logits_bytes() {
  return kTileTokens * (NE + 4) * 4;
}

// Shared memory of one tile's top-k besides the logits.
template <bool COUNT, bool EXTRA>
struct TileShared {
  float part_v[2][kTileTokens];  // per half of a row: max, then the best candidate's logit
  int part_i[2][kTileTokens];    // per half: the best candidate's expert
  float part_s[2][kTileTokens];  // per half: the sum of exp(l - max)
  float rs[kTileTokens];         // per token: 1 / sum of exp(l - max)
  float qpart[2][4][kTileExperts];  // per block, row quarter and expert: partial sums of p
  // per block and expert: first-choice count << 16 | choice count
  unsigned cs[2][kTileExperts];
  // gate sums per block and expert, 2^-24 fixed point (extra statistics only)
  unsigned imp_s[EXTRA ? 2 : 1][kTileExperts];
  float z2[EXTRA ? kTileTokens : 1];  // (log Z)^2 per token
  int choice[kTileTokens][MOE_MAX_TOPK];  // per token: the chosen experts in choice order
  int run[COUNT ? 2 : 1][kTileExperts];
  int blk_ids[COUNT ? 2 : 1][COUNT ? kRouterTokensPerBlock * MOE_MAX_TOPK : 1];
  float prod[kTileExperts];
  int is_last;
};

// (value desc, index asc): is (v, i) ahead of (bv, bi)?
__device__ __forceinline__ bool topk_ahead(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

// Softmax, top-k and the statistics of tile `tile` (tokens [128 tile, 128 tile + 128), statistics
// blocks 2 tile and 2 tile + 1) by 256 threads synchronised by `sync`. L holds the tile's fp32
// logits (rows = tokens, lpos<NE> layout); the exponentials below overwrite them. Per token: the
// largest logit m and k rounds of (logit desc, index asc) argmax over the experts not yet taken
// (the first round is the max pass itself); then x_e = exp(l_e - m), s = the sum of x_e (each
// thread adds its half in expert order as four interleaved partial sums, then s = s_lo + s_hi),
// p_e = x_e * (1 / s), gates = the chosen p (optionally renormalised over the k choices in choice
// order: survey notes §1.1.1.1). Per block: the sums of p per expert (token order within
// quarters of 16 tokens, then the quarters in order), the first-choice counts, and with the extra statistics the gate sums (Importance), the choice
// counts (Load) and the sum of (log Z)^2 in token order (comparison article, "Router Z-loss");
// all are added to the global accumulators as integers (fixed point), so the totals do not
// depend on the order of the tiles. COUNT: also rank each block's (token, choice) pairs per
// expert in pair order for dispatch.
template <int NE, bool COUNT, bool EXTRA, class Sync>
__device__ __forceinline__ void topk_tile(const TopkOut& ko, int64_t tile, float* L, Sync sync,
                                          int tid, TileShared<COUNT, EXTRA>& sh) {
  static_assert(NE >= 16 && NE <= kTileExperts && (NE & (NE - 1)) == 0, "expert tile");
  constexpr int NPT = NE / 2;  // experts per thread
  static_assert(NPT <= 64 && NPT % 4 == 0, "taken mask, 16-byte loads");
  const int64_t T = ko.T;
  const int E = ko.E, k = ko.k;
  const int renorm = ko.renorm;
  const RouterAccum& acc = ko.acc;
  const RouterDispatchCount& dc = ko.dc;
  const int64_t t0 = tile * kTileTokens;
  const int ntok = (int)min((int64_t)kTileTokens, T - t0);
  for (int i = tid; i < 2 * kTileExperts; i += 256) {
    (&sh.cs[0][0])[i] = 0u;
    if constexpr (EXTRA) (&sh.imp_s[0][0])[i] = 0u;
    if constexpr (COUNT) (&sh.run[0][0])[i] = 0;
  }
  const int warp = tid >> 5, lane = tid & 31;
  const int h = warp >> 2;                // half of the row
  const int r = (warp & 3) * 32 + lane;   // token row in the tile
  const int b = r / kRouterTokensPerBlock;
  const bool ok = r < ntok;
  const int e0 = h * NPT;
  const int ne = ok ? max(0, min(NPT, E - e0)) : 0;  // experts of this half
  float4* rowv = reinterpret_cast<float4*>(L + lpos<NE>(r, e0));
  float v[NPT];  // this half's logits, then -inf past the last expert
#pragma unroll
  for (int q = 0; q < NPT / 4; ++q) {
    const float4 f = rowv[q];
    v[4 * q] = f.x;
    v[4 * q + 1] = f.y;
    v[4 * q + 2] = f.z;
    v[4 * q + 3] = f.w;
  }
#pragma unroll
  for (int i = 0; i < NPT; ++i)
    if (i >= ne) v[i] = -INFINITY;
  // the best (logit desc, index asc) among this half's experts not yet taken: four chains in
  // expert order (a later equal logit never wins within a chain), merged
  unsigned long long taken = 0ull;  // bit i: expert e0 + i already chosen
  auto best_of_half = [&](float& bv, int& bi) {
    float cv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    int ci[4] = {0x7fffffff, 0x7fffffff, 0x7fffffff, 0x7fffffff};
#pragma unroll
    for (int i = 0; i < NPT; ++i) {
      if (!((taken >> i) & 1ull) && v[i] > cv[i & 3]) {
        cv[i & 3] = v[i];
        ci[i & 3] = e0 + i;
      }
    }
    bv = cv[0];
    bi = ci[0];
#pragma unroll
    for (int c = 1; c < 4; ++c)
      if (topk_ahead(cv[c], ci[c], bv, bi)) {
        bv = cv[c];
        bi = ci[c];
      }
  };
  // one round: both halves offer their best; the winner is the same for both threads
  auto choose = [&](int j, float& wv) {
    float bv;
    int bi;
    best_of_half(bv, bi);
    sync();  // the previous round's reads of part_v / part_i are done
    sh.part_v[h][r] = bv;
    sh.part_i[h][r] = bi;
    sync();
    const float ov = sh.part_v[h ^ 1][r];
    const int oi = sh.part_i[h ^ 1][r];
    const bool mine = !topk_ahead(ov, oi, bv, bi);
    const int wi = mine ? bi : oi;
    wv = mine ? bv : ov;
    if (mine && bi >= e0 && bi < e0 + ne) taken |= 1ull << (bi - e0);
    if (h == 0) sh.choice[r][j] = wi;
  };
  float m;  // the largest logit: the first round's winner
  choose(0, m);
  for (int j = 1; j < k; ++j) {
    float wv;
    choose(j, wv);
  }
  // x_e = exp(l_e - m) in place of the logits, and their sum (past the last expert v = -inf, so
  // x = 0 there without a branch; rows past the tile's tokens are never read back)
  float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int q = 0; q < NPT / 4; ++q) {
    float x[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      x[c] = expf(v[4 * q + c] - m);
      a[c] += x[c];
    }
    rowv[q] = make_float4(x[0], x[1], x[2], x[3]);
  }
  sh.part_s[h][r] = (a[0] + a[1]) + (a[2] + a[3]);
  sync();  // the halves' sums and exponentials are in shared memory
  const int64_t t = t0 + r;
  if (ok && h == 0) {
    const float s = sh.part_s[0][r] + sh.part_s[1][r];
    const float rs = 1.0f / s;
    sh.rs[r] = rs;
    if constexpr (EXTRA) {
      const float lz = m + logf(s);  // log sum_e exp(l_e)
      sh.z2[r] = lz * lz;
    }
    const float* xr = L + lpos<NE>(r, 0);
    // per-block integer counts (order-independent): first choices, and with the extra
    // statistics every choice and its gate
    auto count_choice = [&](int e, int j, float g) {
      if (e < 0 || e >= E) return;
      if constexpr (EXTRA) {
        atomicAdd(&sh.cs[b][e], j == 0 ? 0x10001u : 1u);
        atomicAdd(&sh.imp_s[b][e], __float2uint_rn(g * (float)kIScale));
      } else if (j == 0) {
        atomicAdd(&sh.cs[b][e], 0x10000u);
      }
    };
    auto p_of = [&](int e) { return (e >= 0 && e < E) ? xr[e] * rs : 0.0f; };
    float gsum = 0.0f;
    for (int j = 0; j < k; ++j) {
      const int e = sh.choice[r][j];
      const float pv = p_of(e);
      ko.ids[t * k + j] = e;
      if (ko.probs != nullptr) ko.probs[t * k + j] = pv;  // before any renormalisation
      if (!renorm) {
        ko.gates[t * k + j] = pv;
        count_choice(e, j, pv);
      }
      if constexpr (COUNT)
        sh.blk_ids[b][(r - b * kRouterTokensPerBlock) * k + j] = (e >= 0 && e < E) ? e : -1;
      gsum += pv;
    }
    if (renorm) {
      for (int j = 0; j < k; ++j) {
        const int e = sh.choice[r][j];
        const float g = p_of(e) / gsum;
        ko.gates[t * k + j] = g;
        count_choice(e, j, g);
      }
    }
  }
  sync();
  // tokens of each block present in this tile
  const int nb0 = min(ntok, kRouterTokensPerBlock);
  const int nb1 = max(0, ntok - kRouterTokensPerBlock);
  if constexpr (COUNT) {
    // rank each block's pairs per expert in pair order (warp 0: block 0, warp 4: block 1)
    if ((warp & 3) == 0) {
      const int bb = warp >> 2;
      const int npairs = (bb == 0 ? nb0 : nb1) * k;
      const int64_t pair0 = (t0 + bb * kRouterTokensPerBlock) * k;
      const unsigned lt = (1u << lane) - 1u;
      for (int c = 0; c < npairs; c += 32) {
        const int pl = c + lane;
        const int e = pl < npairs ? sh.blk_ids[bb][pl] : -1;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(same & lt);
        const int base = e >= 0 ? sh.run[bb][e] : 0;
        __syncwarp();
        if (e >= 0 && rank == 0) sh.run[bb][e] = base + __popc(same);
        __syncwarp();
        if (pl < npairs) dc.local_rank[pair0 + pl] = e >= 0 ? base + rank : -1;
      }
    }
  }
  // per block and expert: the sum of p over the block's tokens. Thread (block, quarter, quad)
  // adds rows [16 quarter, 16 quarter + 16) of its block in token order for experts
  // [4 quad, 4 quad + 4); the quarters' sums are then added in quarter order.
  {
    const int bb = tid >> 7, quarter = (tid >> 5) & 3, quad = tid & 31;
    const int n = bb == 0 ? nb0 : nb1;
    const int row0 = bb * kRouterTokensPerBlock + quarter * 16;
    const int nr = min(16, max(0, n - quarter * 16));
    if (4 * quad < NE) {
      float q[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      for (int u = 0; u < nr; ++u) {
        const float4 f = *reinterpret_cast<const float4*>(L + lpos<NE>(row0 + u, 4 * quad));
        const float rs = sh.rs[row0 + u];
        q[0] += f.x * rs;
        q[1] += f.y * rs;
        q[2] += f.z * rs;
        q[3] += f.w * rs;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) sh.qpart[bb][quarter][4 * quad + c] = q[c];
    }
  }
  sync();
  {
    const int bb = tid >> 7, e = tid & (kTileExperts - 1);
    const int n = bb == 0 ? nb0 : nb1;
    if (n > 0 && e < E) {
      const float sum = ((sh.qpart[bb][0][e] + sh.qpart[bb][1][e]) + sh.qpart[bb][2][e]) +
                        sh.qpart[bb][3][e];
      const unsigned long long fx = (unsigned long long)llrint((double)sum * kQScale);
      if (fx) atomicAdd(&acc.q[e], fx);
      const unsigned cs = sh.cs[bb][e];
      if (cs >> 16) atomicAdd(&acc.c[e], cs >> 16);
      if constexpr (EXTRA) {
        if (cs & 0xffffu) atomicAdd(&acc.load[e], cs & 0xffffu);
        if (sh.imp_s[bb][e]) atomicAdd(&acc.imp[e], (unsigned long long)sh.imp_s[bb][e]);
      }
    }
    if (EXTRA && n > 0 && e == 0) {
      float zb = 0.0f;
      for (int u = 0; u < n; ++u) zb += sh.z2[bb * kRouterTokensPerBlock + u];
      atomicAdd(acc.z, (unsigned long long)llrint((double)zb * kZScale));
    }
  }
  if constexpr (COUNT) {
    const int64_t blk0 = tile * 2;
    for (int i = tid; i < 2 * E; i += 256) {
      const int bb = i / E, e = i - bb * E;
      if ((bb == 0 ? nb0 : nb1) > 0) dc.seg_counts[(blk0 + bb) * E + e] = sh.run[bb][e];
    }
  }
}

// After topk_tile: the tile completed one or two statistics blocks.
template <bool COUNT, bool EXTRA, class Sync>
__device__ __forceinline__ void topk_tile_last(const TopkOut& ko, int64_t tile, unsigned n_blocks,
                                               Sync sync, int tid, TileShared<COUNT, EXTRA>& sh) {
  const int64_t t0 = tile * kTileTokens;
  const unsigned nb = ko.T - t0 > kRouterTokensPerBlock ? 2u : 1u;
  topk_finish(ko, nb, n_blocks, sync, tid, sh.is_last, sh.prod);
}

}  // namespace
}  // namespace moe
