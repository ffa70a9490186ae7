// Dispatch: capacity-limited first-come slots and the expert-major packed copy of x.
//
// DeepSpeed-MoE notes §4.4: the gating kernel fuses top-k, a parallel prefix sum (cumsum) and a
// scatter into a dense token-to-expert mapping table, and the layout transformation re-orders
// rows explicitly by that table instead of multiplying by a sparse dispatch mask; comparison
// article, "Expert Capacity Overflow": capacity = tokens / experts * capacity_factor, tokens
// beyond it skip the expert and keep only the residual.
//
// Pairs p = t * k + j are ranked per expert in pair order (token order), with no atomics, so
// the result is unique and deterministic:
//   dispatch_count_kernel   one warp per segment of 256 consecutive pairs: in-warp ranks from
//                           __match_any_sync, running per-expert counts in shared memory;
//                           writes each pair's rank inside its segment and the segment totals
//                           (inside the layer forward the router's top-k kernel does this for its
//                           own 64-token segments and this kernel is skipped)
//   dispatch_scan_kernel    one block: per expert, exclusive prefix over segments (segment
//                           bases, runs of segments in parallel) and the demand;
//                           kept = min(demand, C); exclusive scan over experts -> offsets
//   dispatch_scatter_kernel one warp per pair: position = segment base + rank, slot = position
//                           or -1 beyond C, row_token, and 16-byte vector copies of the row
//
// Overflow by priority (comparison article, "Expert Capacity Overflow": the example ranks an
// expert's tokens by router probability and keeps the most probable): the scan also writes the
// demand offsets (exclusive prefix of the demands), then each expert's pairs are sorted by the
// 64-bit key (probability descending, pair index ascending; the probability is the softmax value
// before any renormalisation of the gates):
//   dispatch_prio_keys_kernel   one thread per pair: its key at its first-come place in its
//                               expert's list (every expert's pairs in token order)
//   dispatch_prio_chunk_kernel  one block per (expert, 1024 list entries): sorts the chunk in
//                               shared memory (rank = number of smaller keys)
//   dispatch_prio_merge_kernel  log2(T / 1024) passes, one thread per entry: runs of L merge
//                               pairwise, each entry placed by a binary search in its partner run
// the last launch writes slot = sorted position, or -1 from C on, and the scatter takes those
// slots instead of the first-come positions. Work is O(n log^2 n) for an expert of demand n.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "router_topk.cuh"

namespace moe {
namespace {

constexpr int kCountWarps = 8;

__global__ void __launch_bounds__(kCountWarps * 32)
    dispatch_count_kernel(const int32_t* __restrict__ ids, int64_t pairs, int64_t nseg, int E,
                          int32_t* __restrict__ local_rank, int32_t* __restrict__ seg_counts,
                          int* status) {
  extern __shared__ int cnt_all[];  // [kCountWarps][E]
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* cnt = cnt_all + warp * E;
  const int64_t seg = (int64_t)blockIdx.x * kCountWarps + warp;
  if (seg >= nseg) return;
  for (int e = lane; e < E; e += 32) cnt[e] = 0;
  __syncwarp();
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int c = 0; c < kDispatchSeg / 32; ++c) {
    const int64_t p = seg * kDispatchSeg + c * 32 + lane;
    int e = -1;
    if (p < pairs) {
      e = ids[p];
      if (e < 0 || e >= E) {
        set_device_error(status, MOE_DEVERR_BAD_EXPERT);
        e = -1;
      }
    }
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(same & lt_mask);
    const int base = e >= 0 ? cnt[e] : 0;
    __syncwarp();
    if (e >= 0 && rank == 0) cnt[e] = base + __popc(same);
    __syncwarp();
    if (p < pairs) local_rank[p] = e >= 0 ? base + rank : -1;
  }
  for (int e = lane; e < E; e += 32) seg_counts[seg * E + e] = cnt[e];
  pdl_trigger();
}

// Thread (g, e) owns a contiguous run of segments of expert e (G = 1024 / E runs per expert): it
// sums them, takes the sum of the earlier runs from shared memory as its base, then writes the
// exclusive prefix of its run (the segment bases). The last run's end is the demand.
// Exclusive prefix over experts of v (one element per thread of a 1024-thread block); thread
// E - 1 also writes the total to out[E].
__device__ void block_exclusive_scan_experts(int v, int E, int* warp_sums, int32_t* out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int ws = warp_sums[lane];
    int wincl = ws;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, wincl, o);
      if (lane >= o) wincl += u;
    }
    warp_sums[lane] = wincl - ws;  // exclusive prefix of warp totals
  }
  __syncthreads();
  const int excl = incl - v + warp_sums[warp];
  if (tid < E) out[tid] = excl;
  if (tid == E - 1) out[E] = excl + v;
}

__global__ void __launch_bounds__(1024)
    dispatch_scan_kernel(const int32_t* __restrict__ seg_counts, int64_t nseg, int E, int64_t C,
                         int32_t* __restrict__ seg_base, int32_t* __restrict__ counts,
                         int32_t* __restrict__ offsets, int32_t* __restrict__ demand_offsets,
                         ShardBase shard, StatsFinalize fin) {
  __shared__ int run_sum[1024];
  __shared__ float prod[MOE_MAX_EXPERTS];
  __shared__ int kept[MOE_MAX_EXPERTS];
  __shared__ int warp_sums[32];
  pdl_wait();
  const int tid = threadIdx.x;
  int G = 1024 / E;
  if ((int64_t)G > nseg) G = nseg > 0 ? (int)nseg : 1;
  const int64_t chunk = (nseg + G - 1) / G;
  const bool active = tid < G * E;
  const int e = active ? tid % E : 0, g = active ? tid / E : 0;
  const int64_t s0 = (int64_t)g * chunk, s1 = min(nseg, s0 + chunk);
  // runs of up to kBatch segments are held in registers: one sweep of independent loads
  constexpr int kBatch = 32;
  int vals[kBatch];
  const bool in_regs = chunk <= kBatch;
  int sum = 0;
  if (active) {
    if (in_regs) {
#pragma unroll
      for (int b = 0; b < kBatch; ++b) vals[b] = (s0 + b < s1) ? seg_counts[(s0 + b) * E + e] : 0;
#pragma unroll
      for (int b = 0; b < kBatch; ++b) sum += vals[b];
    } else {
#pragma unroll 8
      for (int64_t s = s0; s < s1; ++s) sum += seg_counts[s * E + e];
    }
    run_sum[tid] = sum;
  }
  __syncthreads();
  if (active) {
    int run = 0;
    for (int gg = 0; gg < g; ++gg) run += run_sum[gg * E + e];
    if (in_regs) {
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        if (s0 + b < s1) seg_base[(s0 + b) * E + e] = run;
        run += vals[b];
      }
    } else {
#pragma unroll 8
      for (int64_t s = s0; s < s1; ++s) {
        const int v = seg_counts[s * E + e];
        seg_base[s * E + e] = run;
        run += v;
      }
    }
    if (g == G - 1) {
      counts[e] = run;
      int64_t cap = C;
      if (shard.demand_all != nullptr) {
        // global first-come: the earlier shards' pairs of expert e come first
        int64_t base = 0;
        for (int r = 0; r < shard.rank; ++r) base += shard.demand_all[(int64_t)r * E + e];
        cap = C - base;
        if (cap < 0) cap = 0;
        if (cap > run) cap = run;
        shard.cap_local[e] = (int32_t)cap;
      }
      kept[e] = (int)min((int64_t)run, cap);
    }
  }
  __syncthreads();
  // exclusive scans over experts (E <= 1024), one element per thread
  block_exclusive_scan_experts(tid < E ? kept[tid] : 0, E, warp_sums, offsets);
  if (demand_offsets != nullptr) {
    __syncthreads();  // warp_sums is reused; counts (global) were written before the first sync
    block_exclusive_scan_experts(tid < E ? counts[tid] : 0, E, warp_sums, demand_offsets);
  }
  pdl_trigger();
  if (fin.lb != nullptr || fin.losses != nullptr) {
    // the router's statistics from its integer accumulators (complete: the router kernel ended)
    const RouterAccum& a = fin.acc;
    router_finalize_block(
        E, fin.T, fin.alpha, [&](int e) { return a.q[e]; },
        [&](int e) { return (unsigned long long)a.c[e]; }, [&](int e) { return a.imp[e]; },
        [&](int e) { return (unsigned long long)a.load[e]; }, *a.z, fin.lb, fin.losses, prod, tid,
        1024, BlockSync{});
  }
}

// Sort key of a pair for the priority order: ascending keys = probability descending, then pair
// index ascending. The fp32 probability is mapped to an unsigned integer of the same order
// (negative zero folded onto zero, so equal probabilities tie), inverted, and followed by the pair.
__device__ __forceinline__ uint64_t priority_key(float prob, int64_t pair) {
  uint32_t u = __float_as_uint(prob == 0.0f ? 0.0f : prob);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // float order -> unsigned order
  return ((uint64_t)(~u) << 32) | (uint64_t)(uint32_t)pair;
}

// One thread per pair: the pair's key at its first-come place in its expert's list
// (keys[demand_offset[e] + position]), i.e. every expert's pairs in token order.
__global__ void __launch_bounds__(256)
    dispatch_prio_keys_kernel(const int32_t* __restrict__ ids, const float* __restrict__ probs,
                              int64_t pairs, int E, const int32_t* __restrict__ local_rank,
                              const int32_t* __restrict__ seg_base, int seg_len,
                              const int32_t* __restrict__ demand_offsets,
                              uint64_t* __restrict__ keys) {
  pdl_wait();
  const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p < pairs) {
    const int e = ids[p];
    const int r = local_rank[p];
    if (e >= 0 && e < E && r >= 0)
      keys[demand_offsets[e] + seg_base[(p / seg_len) * E + e] + r] = priority_key(probs[p], p);
  }
  pdl_trigger();
}

constexpr int kPrioChunk = 1024;  // list entries ranked together in shared memory

// Block (c, e): entries [1024 c, 1024 c + 1024) of expert e's list are sorted in shared memory
// (each key's rank is the number of smaller keys in the chunk; keys are unique). The expert's
// demand is at most T (a token chooses an expert once), so gridDim.x = ceil(T / 1024) covers
// every list. final: no merge pass follows, so the rank is the slot (-1 from C on).
__global__ void __launch_bounds__(kPrioChunk)
    dispatch_prio_chunk_kernel(const uint64_t* __restrict__ in, uint64_t* __restrict__ out,
                               const int32_t* __restrict__ demand_offsets, int64_t C, int final,
                               int32_t* __restrict__ slot) {
  __shared__ uint64_t tile[kPrioChunk];
  pdl_wait();
  const int e = blockIdx.y;
  const int start = demand_offsets[e];
  const int n = demand_offsets[e + 1] - start;
  const int c0 = blockIdx.x * kPrioChunk;
  if (c0 < n) {  // block-uniform
    const int m = min(kPrioChunk, n - c0);
    const int i = threadIdx.x;
    uint64_t key = 0;
    if (i < m) {
      key = in[start + c0 + i];
      tile[i] = key;
    }
    __syncthreads();
    if (i < m) {
      int rank = 0;
      for (int u = 0; u < m; ++u) rank += tile[u] < key ? 1 : 0;
      const int pos = c0 + rank;
      out[start + pos] = key;
      if (final) slot[(uint32_t)key] = pos < C ? pos : -1;
    }
  }
  pdl_trigger();
}

// One merge pass: every expert's list is a sequence of sorted runs of L entries; runs 2q and
// 2q + 1 merge into one. Entry i of run r finds how many entries of the partner run r ^ 1 are
// smaller (binary search; keys are unique) and moves to its place in the merged run.
// final: the last pass, which also writes slot = position (-1 from C on).
__global__ void __launch_bounds__(256)
    dispatch_prio_merge_kernel(const uint64_t* __restrict__ in, uint64_t* __restrict__ out,
                               const int32_t* __restrict__ ids,
                               const int32_t* __restrict__ demand_offsets, int E, int L,
                               int64_t C, int final, int32_t* __restrict__ slot) {
  pdl_wait();
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j < demand_offsets[E]) {
    const uint64_t key = in[j];
    const int64_t pair = (uint32_t)key;
    const int e = ids[pair];
    const int start = demand_offsets[e];
    const int n = demand_offsets[e + 1] - start;
    const int i = (int)(j - start);
    const int r = i / L;
    const int partner = r ^ 1;
    const int64_t ps = (int64_t)partner * L;
    int pos = i;
    if (ps < n) {
      const int plen = (int)min((int64_t)L, n - ps);
      const uint64_t* run = in + start + ps;
      int lo = 0, hi = plen;  // first partner entry not smaller than key
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (run[mid] < key) lo = mid + 1;
        else hi = mid;
      }
      pos = min(r, partner) * L + (i - r * L) + lo;
    }
    out[start + pos] = key;
    if (final) slot[pair] = pos < C ? pos : -1;
  }
  pdl_trigger();
}

constexpr int kScatterPairsPerWarp = 1;  // measured: more pairs per warp is slower

// One warp per kScatterPairsPerWarp consecutive pairs: the first lanes resolve the pairs' slots and
// packed rows, then the warp copies the kept rows, each lane issuing its loads before its stores
// (16-byte vectors when the row allows).
template <int VEC_BYTES>
__global__ void __launch_bounds__(256)
    dispatch_scatter_kernel(const uint8_t* __restrict__ x, int64_t row_bytes, int64_t pairs, int k,
                            int E, int64_t C, const int32_t* __restrict__ ids,
                            const int32_t* __restrict__ local_rank,
                            const int32_t* __restrict__ seg_base,
                            const int32_t* __restrict__ offsets, int32_t* __restrict__ slot,
                            int32_t* __restrict__ row_token, uint8_t* __restrict__ x_packed,
                            int64_t rows_max, DroppedRows dropped, int d, int seg_len,
                            int prio, const int32_t* __restrict__ cap_local) {
  constexpr int P = kScatterPairsPerWarp;
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t p0 = (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5) * P;
  if (p0 >= pairs) return;
  int my_s = -1;
  int64_t my_row = -1;
  if (lane < P && p0 + lane < pairs) {
    const int64_t p = p0 + lane;
    const int e = ids[p];
    const int r = local_rank[p];
    if (e >= 0 && e < E && r >= 0) {
      if (prio) {
        my_s = slot[p];  // the priority rank kernel's slot
      } else {
        const int pos = seg_base[(p / seg_len) * E + e] + r;
        if (pos < (cap_local != nullptr ? (int64_t)cap_local[e] : C)) my_s = pos;
      }
    }
    slot[p] = my_s;
    if (my_s >= 0) {
      my_row = (int64_t)offsets[e] + my_s;
      if (my_row < rows_max) row_token[my_row] = (int32_t)(p / k);
      else my_row = -1;  // cannot happen with rows_max >= min(T k, E C)
    }
  }
  int64_t rows[P], toks[P];
  int ss[P];
#pragma unroll
  for (int q = 0; q < P; ++q) {
    ss[q] = __shfl_sync(0xffffffffu, my_s, q);
    rows[q] = __shfl_sync(0xffffffffu, my_row, q);
    toks[q] = (p0 + q) / k;
    if (p0 + q >= pairs) ss[q] = -2;  // no such pair
  }
  if (dropped.out != nullptr) {
    // top-1 with the combine fused into layer 2: a dropped token's output is its residual alone
#pragma unroll
    for (int q = 0; q < P; ++q) {
      if (ss[q] != -1) continue;
      const int64_t t = toks[q];
      for (int64_t i = lane; i < d; i += 32) {
        float v = 0.0f;
        if (dropped.add_x)
          v = row_bytes == (int64_t)d * 2 ? bf16_to_f32(reinterpret_cast<const uint16_t*>(x)[t * d + i])
                                          : reinterpret_cast<const float*>(x)[t * d + i];
        if (dropped.out_bf16) reinterpret_cast<uint16_t*>(dropped.out)[t * d + i] = f32_to_bf16_rn(v);
        else reinterpret_cast<float*>(dropped.out)[t * d + i] = v;
      }
    }
  }
  using V = typename std::conditional<VEC_BYTES == 16, uint4,
            typename std::conditional<VEC_BYTES == 8, uint2, uint32_t>::type>::type;
  const int64_t n = row_bytes / VEC_BYTES;
  for (int64_t i0 = lane; i0 < n; i0 += 4 * 32) {
    V v[P][4];
#pragma unroll
    for (int q = 0; q < P; ++q) {
      if (rows[q] < 0) continue;
      const V* src = reinterpret_cast<const V*>(x + toks[q] * row_bytes);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (i0 + 32 * u < n) v[q][u] = src[i0 + 32 * u];
    }
#pragma unroll
    for (int q = 0; q < P; ++q) {
      if (rows[q] < 0) continue;
      V* dst = reinterpret_cast<V*>(x_packed + rows[q] * row_bytes);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (i0 + 32 * u < n) dst[i0 + 32 * u] = v[q][u];
    }
  }
  pdl_trigger();
}

}  // namespace

cudaError_t enqueue_dispatch(const void* x, bool bf16, int64_t T, int d, const int32_t* ids, int E,
                             int k, int64_t C, int32_t* slot, int32_t* counts, int32_t* offsets,
                             int32_t* row_token, void* x_packed, int64_t rows_max,
                             int32_t* local_rank, int32_t* seg_counts, int32_t* seg_base,
                             int* status, cudaStream_t stream, DroppedRows dropped,
                             int counted_seg_len, PriorityDispatch prio, ShardBase shard,
                             bool scan_only, StatsFinalize fin) {
  const int64_t pairs = T * k;
  const int seg_len = counted_seg_len > 0 ? counted_seg_len : kDispatchSeg;
  const int64_t nseg = (pairs + seg_len - 1) / seg_len;
  if (pairs > 0 && counted_seg_len <= 0) {
    const unsigned blocks = (unsigned)((nseg + kCountWarps - 1) / kCountWarps);
    cudaError_t e = launch_kernel(dispatch_count_kernel, dim3(blocks), dim3(kCountWarps * 32),
                                  kCountWarps * E * sizeof(int), stream, ids, pairs, nseg, E,
                                  local_rank, seg_counts, status);
    if (e != cudaSuccess) return e;
  }
  {
    cudaError_t e = launch_kernel(dispatch_scan_kernel, dim3(1), dim3(1024), 0, stream,
                                  (const int32_t*)seg_counts, nseg, E, C, seg_base, counts, offsets,
                                  prio.probs != nullptr ? prio.demand_offsets : nullptr, shard, fin);
    if (e != cudaSuccess) return e;
  }
  if (scan_only) return cudaGetLastError();
  const int use_prio = prio.probs != nullptr && pairs > 0 ? 1 : 0;
  if (use_prio) {
    // keys in first-come order per expert, sorted chunks of 1024, then merge passes until a run
    // covers the largest possible list (T entries)
    uint64_t* buf[2] = {prio.keys, prio.keys + pairs};
    cudaError_t e = launch_kernel(dispatch_prio_keys_kernel, dim3((unsigned)((pairs + 255) / 256)),
                                  dim3(256), 0, stream, ids, prio.probs, pairs, E,
                                  (const int32_t*)local_rank, (const int32_t*)seg_base, seg_len,
                                  (const int32_t*)prio.demand_offsets, buf[0]);
    if (e != cudaSuccess) return e;
    int passes = 0;
    for (int64_t L = kPrioChunk; L < T; L *= 2) ++passes;
    const dim3 grid((unsigned)((T + kPrioChunk - 1) / kPrioChunk), (unsigned)E);
    e = launch_kernel(dispatch_prio_chunk_kernel, grid, dim3(kPrioChunk), 0, stream,
                      (const uint64_t*)buf[0], buf[1], (const int32_t*)prio.demand_offsets, C,
                      passes == 0 ? 1 : 0, slot);
    if (e != cudaSuccess) return e;
    int cur = 1;
    int64_t L = kPrioChunk;
    for (int q = 0; q < passes; ++q, L *= 2) {
      e = launch_kernel(dispatch_prio_merge_kernel, dim3((unsigned)((pairs + 255) / 256)),
                        dim3(256), 0, stream, (const uint64_t*)buf[cur], buf[cur ^ 1], ids,
                        (const int32_t*)prio.demand_offsets, E, (int)L, C,
                        q == passes - 1 ? 1 : 0, slot);
      if (e != cudaSuccess) return e;
      cur ^= 1;
    }
  }
  if (pairs > 0) {
    const int64_t row_bytes = (int64_t)d * (bf16 ? 2 : 4);
    const int64_t warps = (pairs + kScatterPairsPerWarp - 1) / kScatterPairsPerWarp;
    const unsigned blocks = (unsigned)((warps * 32 + 255) / 256);
    const uint8_t* xs = (const uint8_t*)x;
    uint8_t* xp = (uint8_t*)x_packed;
    auto launch = [&](auto kern) {
      return launch_kernel(kern, dim3(blocks), dim3(256), 0, stream, xs, row_bytes, pairs, k, E, C,
                           ids, (const int32_t*)local_rank, (const int32_t*)seg_base,
                           (const int32_t*)offsets, slot, row_token, xp, rows_max, dropped, d,
                           seg_len, use_prio, (const int32_t*)shard.cap_local);
    };
    cudaError_t e = row_bytes % 16 == 0  ? launch(dispatch_scatter_kernel<16>)
                    : row_bytes % 8 == 0 ? launch(dispatch_scatter_kernel<8>)
                                         : launch(dispatch_scatter_kernel<4>);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace moe
