// Router logits on sm_100a tensor cores, token-major: logits[t, e] = x[t, :] . W_r[e, :] + b_r[e].
//
// DeepSpeed MoE blog, MoE formula p(x) = softmax(W_r x); comparison article, "Router computation"
// (logits = x W_r).
//
// Arithmetic: x is bf16 and W_r (fp32) arrives split exactly into bf16 parts hi + mid + lo (each
// holds the next 8 significant bits; router.cu), so x * W_r = x*hi + x*mid + x*lo is formed from
// exact products and accumulated in fp32 by tcgen05.mma; b_r is added in fp32.
//
// Tile = 128 tokens x NE experts (one 128-expert slice of E, NE = the slice rounded up to a
// power of two >= 16): the x tile is the MMA's A operand (M = 128, TMEM lane = token) and the three
// weight parts are three B operands over the same A tile, so each x tile is read once per slice.
// Roles per CTA (persistent over tiles, two TMEM accumulators):
//     warp 0      TMA: x [128 x 64] and the three W parts [NE x 64] per stage, 128-byte swizzle
//     warp 1      TMEM allocation; one thread issues 3 x 4 MMAs per stage
//     warps 2..5  tcgen05.ld of 16-expert chunks, + bias, staged in shared memory and stored as
//                 64-byte runs of a token's logits row (two tokens per warp store)
// Bounded waits as in the grouped GEMM (MOE_DEVERR_TIMEOUT, drain, free TMEM).
#include "common.cuh"
#include "kernels.h"
#include "router_topk.cuh"

namespace moe {
namespace {

constexpr int kTM = 128;       // tokens per tile
constexpr int kBK = 64;        // K per stage
constexpr int kSlice = 128;    // experts per tile (at most)
constexpr int kThreads = 192;  // 6 warps

template <int NE>
struct RCfg {
  static constexpr int kABytes = kTM * kBK * 2;           // 16 KB
  static constexpr int kBPartBytes = NE * kBK * 2;        // per weight part
  static constexpr int kStageBytes = kABytes + 3 * kBPartBytes;
  static constexpr int kStagesFit = (200 * 1024) / kStageBytes;  // 3 stages at NE = 128
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kTmemCols = (2 * NE) < 32 ? 32 : (2 * NE);
  static constexpr int kBarBytes = 8 * 32;
  static constexpr int kStageTile = 32 * 16 * 4;          // per epilogue warp: 32 tokens x 16 fp32
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 4 * kStageTile + kBarBytes + 16;
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kStages >= 2, "pipeline depth");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

struct RParams {
  int64_t T;
  int E, dpad, n_slices;
  const float* bias;  // [E] fp32 or nullptr
  float* logits;      // [T, E]
  int* status;
  RouterAccum acc;    // zeroed by block 0 when zero_acc (no split kernel ran before this one)
  int zero_acc;
};

__device__ __forceinline__ void mbar_wait_drain_r(uint32_t bar, uint32_t parity, int* status) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      set_device_error(status, MOE_DEVERR_TIMEOUT);
      return;
    }
  }
}

template <int NE>
__global__ void __launch_bounds__(kThreads, 1)
    router_logits_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                            const __grid_constant__ CUtensorMap tmW, const RParams p) {
  using C = RCfg<NE>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_addr - raw_addr);
  uint8_t* stage_tiles = base + C::kStages * C::kStageBytes;
  uint8_t* aux = stage_tiles + 4 * C::kStageTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(aux);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(aux + C::kBarBytes);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(aux + C::kBarBytes + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = C::kStages;
  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[S + s]); };
  auto tfull_bar = [&](int a) { return smem_u32(&bars[2 * S + a]); };
  auto tempty_bar = [&](int a) { return smem_u32(&bars[2 * S + 2 + a]); };
  const uint32_t drain_bar = smem_u32(&bars[2 * S + 4]);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 128);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  pdl_wait();  // global memory and TMEM only after the preceding kernels have completed
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (p.zero_acc && blockIdx.x == 0) {
    for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
      p.acc.q[e] = 0ull;
      p.acc.c[e] = 0u;
      p.acc.imp[e] = 0ull;
      p.acc.load[e] = 0u;
    }
    if (threadIdx.x == 0) {
      *p.acc.z = 0ull;
      *p.acc.ticket = 0u;
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int ntiles = (int)((p.T + kTM - 1) / kTM) * p.n_slices;
  const int n_kb = p.dpad / kBK;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      // the weight parts into L2 first, a share per CTA (see the fused kernel)
      for (int b = blockIdx.x; b < 3 * n_kb * p.n_slices; b += gridDim.x) {
        const int sl = b / (3 * n_kb), rem = b % (3 * n_kb);
        tma_prefetch_l2_2d(&tmW, (rem / n_kb) * p.dpad + (rem % n_kb) * kBK, sl * kSlice);
      }
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const int tok_tile = t / p.n_slices, slice = t % p.n_slices;
        if (slice == 0)  // the tile's x rows into L2 at once (see the fused kernel)
          for (int kb = 0; kb < n_kb; ++kb) tma_prefetch_l2_2d(&tmX, kb * kBK, tok_tile * kTM);
        for (int kb = 0; kb < n_kb; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const uint32_t sa = base_addr + stage * C::kStageBytes;
          mbar_arrive_expect_tx(full_bar(stage), C::kStageBytes);
          tma_load_2d(sa, &tmX, kb * kBK, tok_tile * kTM, full_bar(stage));
#pragma unroll
          for (int part = 0; part < 3; ++part)
            tma_load_2d(sa + C::kABytes + part * C::kBPartBytes, &tmW, part * p.dpad + kb * kBK,
                        slice * kSlice, full_bar(stage));
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      for (int i = max(0, issued - S); i < issued; ++i)
        mbar_wait_drain_r(full_bar(i % S), (uint32_t)((i / S) & 1), p.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      constexpr uint32_t idesc = idesc_bf16_f32(kTM, NE);
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        if (!mbar_wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * NE);
        for (int kb = 0; kb < n_kb; ++kb) {
          if (!mbar_wait_bounded(full_bar(stage), phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base_addr + stage * C::kStageBytes;
          const uint64_t adesc = smem_desc_sw128(sa);
#pragma unroll
          for (int part = 0; part < 3; ++part) {
            const uint64_t bdesc = smem_desc_sw128(sa + C::kABytes + part * C::kBPartBytes);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              tc_mma_bf16(d_tmem, adesc + (uint64_t)(2 * kk), bdesc + (uint64_t)(2 * kk), idesc,
                          (kb | part | kk) != 0 ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      tc_commit(drain_bar);
      mbar_wait_drain_r(drain_bar, 0, p.status);
    }
  } else {
    // ---------------------------------------------------------- epilogue: logits rows
    const int quarter = warp & 3;  // TMEM lanes (tokens) [32*quarter, 32*quarter + 32)
    float* st = reinterpret_cast<float*>(stage_tiles + (warp - 2) * C::kStageTile);  // [32][16]
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      const int tok_tile = t / p.n_slices, slice = t % p.n_slices;
      if (!mbar_wait_bounded_warp(tfull_bar(acc), acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      const int64_t tok0 = (int64_t)tok_tile * kTM + quarter * 32;  // this warp's first token
      const int e_base = slice * kSlice;
      const int ne = min(NE, p.E - e_base);
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * NE);
      for (int c0 = 0; c0 < ne; c0 += 16) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(taddr + (uint32_t)c0, r);
        tmem_ld_wait();
        // row = this lane's token, 16 experts; columns rotated by the row to spread banks
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int e = e_base + c0 + c;
          const float b = (p.bias && e < p.E) ? p.bias[e] : 0.0f;
          st[lane * 16 + ((c + lane) & 15)] = __uint_as_float(r[c]) + b;
        }
        __syncwarp();
        const int nc = min(16, ne - c0);
        const int j = lane & 15;  // expert within the chunk
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
          const int row = 2 * i + (lane >> 4);  // two tokens per store instruction
          const int64_t tok = tok0 + row;
          if (j < nc && tok < p.T)
            p.logits[tok * p.E + e_base + c0 + j] = st[row * 16 + ((j + row) & 15)];
        }
        __syncwarp();
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  pdl_trigger();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// The router with softmax, top-k and the statistics fused into the tensor-core kernel's epilogue
// (E <= 128, one expert slice): after a tile's MMAs, the 8 epilogue warps copy the 128 x NE fp32
// logits (+ bias) from TMEM into shared memory, reusing pipeline stage 0 (the tile's MMAs have
// read it; the TMA role loads the next tile into stage 0 only after the epilogue is done with it),
// with the column index XOR-ed by the token (row) index so that both the column-wise copy and the
// reads of the top-k are free of bank conflicts. They then run the tile top-k (router_topk.cuh:
// two threads per token, all 128 tokens at once) that the standalone top-k kernel also runs for
// E <= 128, so ids, gates, statistics and dispatch ranks are those of the two-kernel path bit for
// bit, and the logits reach global memory only when the caller asks for them.
constexpr int kFusedThreads = 320;  // TMA, MMA, 8 epilogue warps

// The tile's logits (128 rows of NE + 1 floats) take stage 0 and, where they are longer, a gap of
// whole KB between stage 0 and stage 1 (stages stay 1024-byte aligned for the 128-byte swizzle).
template <int NE>
constexpr int fused_stage_gap() {
  constexpr int over = tile_logits_bytes<NE>() - RCfg<NE>::kStageBytes;
  return over <= 0 ? 0 : (over + 1023) / 1024 * 1024;
}

// Epilogue helpers of the fused kernels. One warp copies its 32 TMEM lanes (tokens `row`) of the
// accumulator at taddr, 16-expert chunks half, half + 2, ..., plus the bias, into the tile's
// logits rows in shared memory (16-byte stores).
template <int NE>
__device__ __forceinline__ void router_acc_to_smem(uint32_t taddr, int row, int half,
                                                   const RParams& p, float* L) {
  for (int c0 = half * 16; c0 < NE; c0 += 32) {
    uint32_t r[16];
    tmem_ld_32x32b_x16(taddr + (uint32_t)c0, r);
    tmem_ld_wait();
    float4* dst = reinterpret_cast<float4*>(L + lpos<NE>(row, c0));
#pragma unroll
    for (int c = 0; c < 16; c += 4) {
      float f[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = c0 + c + u;
        f[u] = __uint_as_float(r[c + u]) + ((p.bias && e < p.E) ? p.bias[e] : 0.0f);
      }
      dst[c / 4] = make_float4(f[0], f[1], f[2], f[3]);
    }
  }
}
// The tile's logits output (when asked for) and its top-k, by the 256 epilogue threads.
template <int NE, bool COUNT, bool EXTRA>
__device__ __forceinline__ void router_tile_outputs(const RParams& p, const TopkOut& ko,
                                                    int64_t tile, float* L, NamedSync sync,
                                                    int tid, TileShared<COUNT, EXTRA>& sh,
                                                    unsigned n_blocks) {
  const int64_t t0 = tile * kTM;
  if (p.logits != nullptr) {
    // whole rows: thread i writes experts i, i + 256, ... of the tile, row-major
    const int ne = p.E;
    for (int i = tid; i < kTM * ne; i += 256) {
      const int rr = i / ne, e = i - rr * ne;
      if (t0 + rr < p.T) p.logits[(t0 + rr) * ne + e] = L[lpos<NE>(rr, e)];
    }
  }
  topk_tile<NE, COUNT, EXTRA>(ko, tile, L, sync, tid, sh);
  topk_tile_last(ko, tile, n_blocks, sync, tid, sh);
}

template <int NE, bool COUNT, bool EXTRA>
__global__ void __launch_bounds__(kFusedThreads, 1)
    router_fused_kernel(const __grid_constant__ CUtensorMap tmX,
                        const __grid_constant__ CUtensorMap tmW, const RParams p,
                        const TopkOut ko) {
  using C = RCfg<NE>;
  constexpr int kGap = fused_stage_gap<NE>();
  static_assert(tile_logits_bytes<NE>() <= C::kStageBytes + kGap, "the logits tile must fit");
  static_assert(kTM == kTileTokens, "one top-k tile per MMA tile");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_addr - raw_addr);
  float* L = reinterpret_cast<float*>(base);  // stage 0 (and the gap after it): the tile's logits
  using Sh = TileShared<COUNT, EXTRA>;
  Sh& sh = *reinterpret_cast<Sh*>(base + C::kStages * C::kStageBytes + kGap);
  uint8_t* aux = base + C::kStages * C::kStageBytes + kGap + ((sizeof(Sh) + 15) / 16) * 16;
  auto stage_addr = [&](int s) {
    return base_addr + (uint32_t)(s * C::kStageBytes + (s > 0 ? kGap : 0));
  };
  uint64_t* bars = reinterpret_cast<uint64_t*>(aux);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(aux + C::kBarBytes);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(aux + C::kBarBytes + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = C::kStages;
  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[S + s]); };
  auto tfull_bar = [&](int a) { return smem_u32(&bars[2 * S + a]); };
  auto tempty_bar = [&](int a) { return smem_u32(&bars[2 * S + 2 + a]); };
  const uint32_t drain_bar = smem_u32(&bars[2 * S + 4]);
  const uint32_t lfree_bar = smem_u32(&bars[2 * S + 5]);  // the epilogue is done with stage 0

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 8 * 32);
    }
    mbar_init(drain_bar, 1);
    mbar_init(lfree_bar, 8 * 32);
    *abort_flag = 0;
    fence_barrier_init();
  }
  pdl_wait();
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int ntiles = (int)((p.T + kTM - 1) / kTM);
  const int n_kb = p.dpad / kBK;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0, issued = 0, n_local = 0;
      uint32_t phase = 0;
      bool ok = true;
      // every CTA runs the K blocks in the same order at about the same time, so each weight box
      // would be requested by all of them before its first copy reached L2: the CTAs first pull
      // the split weight (3 * dpad / 64 boxes) into L2 between them, a share each
      for (int b = blockIdx.x; b < 3 * n_kb; b += gridDim.x)
        tma_prefetch_l2_2d(&tmW, (b / n_kb) * p.dpad + (b % n_kb) * kBK, 0);
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++n_local) {
        bool waited = n_local == 0;  // this CTA's first tile: stage 0 holds no logits yet
        for (int kb = 0; kb < n_kb; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          if (stage == 0 && !waited) {
            // the previous tile's epilogue reads its logits from stage 0
            if (!mbar_wait_bounded(lfree_bar, (uint32_t)((n_local - 1) & 1), abort_flag, p.status)) {
              ok = false;
              break;
            }
            waited = true;
          }
          const uint32_t sa = stage_addr(stage);
          mbar_arrive_expect_tx(full_bar(stage), C::kStageBytes);
          tma_load_2d(sa, &tmX, kb * kBK, t * kTM, full_bar(stage));
#pragma unroll
          for (int part = 0; part < 3; ++part)
            tma_load_2d(sa + C::kABytes + part * C::kBPartBytes, &tmW, part * p.dpad + kb * kBK, 0,
                        full_bar(stage));
          // once the ring is full, the rest of the tile's x rows (read from HBM once) are asked
          // into L2 at once: the ring alone keeps too few bytes in flight to hide DRAM latency
          // (the weight parts are L2 hits); asking first would delay the ring's first loads
          if (kb == min(S, n_kb) - 1)
            for (int kq = kb + 1; kq < n_kb; ++kq) tma_prefetch_l2_2d(&tmX, kq * kBK, t * kTM);
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      for (int i = max(0, issued - S); i < issued; ++i)
        mbar_wait_drain_r(full_bar(i % S), (uint32_t)((i / S) & 1), p.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      constexpr uint32_t idesc = idesc_bf16_f32(kTM, NE);
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        if (!mbar_wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * NE);
        for (int kb = 0; kb < n_kb; ++kb) {
          if (!mbar_wait_bounded(full_bar(stage), phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = stage_addr(stage);
          const uint64_t adesc = smem_desc_sw128(sa);
#pragma unroll
          for (int part = 0; part < 3; ++part) {
            const uint64_t bdesc = smem_desc_sw128(sa + C::kABytes + part * C::kBPartBytes);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              tc_mma_bf16(d_tmem, adesc + (uint64_t)(2 * kk), bdesc + (uint64_t)(2 * kk), idesc,
                          (kb | part | kk) != 0 ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      tc_commit(drain_bar);
      mbar_wait_drain_r(drain_bar, 0, p.status);
    }
  } else {
    // ---------------------------------------------------------- epilogue: top-k of the tile
    const int tid = threadIdx.x - 64;  // 0..255
    const int ew = warp - 2;
    const int quarter = warp & 3;      // TMEM lanes (tokens) [32*quarter, 32*quarter + 32)
    const int half = ew >> 2;          // 16-expert chunks half, half + 2, ...
    const NamedSync sync{1, 256};
    const unsigned n_blocks = (unsigned)((p.T + kRouterTokensPerBlock - 1) / kRouterTokensPerBlock);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      // the 8 warps meet at named barriers below: they leave together if any wait gave up
      const bool ok = mbar_wait_bounded_warp(tfull_bar(acc), acc_phase, abort_flag, p.status);
      if (named_barrier_any(1, 256, !ok)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * NE);
      router_acc_to_smem<NE>(taddr, quarter * 32 + lane, half, p, L);
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));  // the accumulator is free for the tile after next
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
      sync();
      router_tile_outputs<NE, COUNT, EXTRA>(p, ko, t, L, sync, tid, sh, n_blocks);
      mbar_arrive(lfree_bar);  // stage 0 may take the next tile's data
    }
  }

  tc_fence_before();
  __syncthreads();
  pdl_trigger();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}



using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_map(CUtensorMap* m, const void* ptr, int64_t rows, int K, int box_rows) {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  cuuint32_t estride[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NE>
cudaError_t launch_tc(const CUtensorMap& tmX, const CUtensorMap& tmW, const RParams& p,
                      int ntiles, cudaStream_t stream) {
  auto kern = router_logits_tc_kernel<NE>;
  static int attr_done[64] = {0};  // per device
  cudaError_t e = ensure_dynamic_smem(kern, RCfg<NE>::kSmemBytes, attr_done);
  if (e != cudaSuccess) return e;
  const int grid = ntiles < num_sms() ? ntiles : num_sms();
  return launch_kernel(kern, dim3(grid), dim3(kThreads), RCfg<NE>::kSmemBytes, stream, tmX, tmW, p);
}

template <int NE, bool COUNT, bool EXTRA>
cudaError_t launch_fused(const CUtensorMap& tmX, const CUtensorMap& tmW, const RParams& p,
                         const TopkOut& ko, int ntiles, cudaStream_t stream) {
  auto kern = router_fused_kernel<NE, COUNT, EXTRA>;
  constexpr int smem = 1024 + RCfg<NE>::kStages * RCfg<NE>::kStageBytes + fused_stage_gap<NE>() +
                       (int)((sizeof(TileShared<COUNT, EXTRA>) + 15) / 16 * 16) +
                       RCfg<NE>::kBarBytes + 16;
  static_assert(smem <= 227 * 1024, "shared memory budget");
  static_assert(2 * RCfg<NE>::kStages + 6 <= RCfg<NE>::kBarBytes / 8, "barrier area too small");
  static int attr_done[64] = {0};  // per device
  cudaError_t e = ensure_dynamic_smem(kern, smem, attr_done);
  if (e != cudaSuccess) return e;
  const int grid = ntiles < num_sms() ? ntiles : num_sms();
  return launch_kernel(kern, dim3(grid), dim3(kFusedThreads), smem, stream, tmX, tmW, p, ko);
}

template <int NE>
cudaError_t launch_fused_ne(const CUtensorMap& tmX, const CUtensorMap& tmW, const RParams& p,
                            const TopkOut& ko, int ntiles, cudaStream_t stream) {
  const bool count = ko.dc.local_rank != nullptr;
  const bool extra = ko.losses != nullptr || ko.exported != nullptr || ko.extra_stats != 0;
  if (count)
    return extra ? launch_fused<NE, true, true>(tmX, tmW, p, ko, ntiles, stream)
                 : launch_fused<NE, true, false>(tmX, tmW, p, ko, ntiles, stream);
  return extra ? launch_fused<NE, false, true>(tmX, tmW, p, ko, ntiles, stream)
               : launch_fused<NE, false, false>(tmX, tmW, p, ko, ntiles, stream);
}

}  // namespace

bool router_fused_supported(int E) { return E <= kSlice; }

cudaError_t enqueue_router_fused(const void* x, int64_t T, int d, const uint16_t* w_split,
                                 int dpad, const float* router_bias, int E, int k, float* logits,
                                 int32_t* ids, float* gates, float* probs, const RouterAccum& acc,
                                 float aux_alpha, float* lb_stats, RouterDispatchCount dc,
                                 bool renormalize, float* losses, int64_t* exported,
                                 bool extra_stats, int* status, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  if (E > kSlice) return cudaErrorInvalidValue;
  int NE = 16;
  while (NE < E) NE <<= 1;
  CUtensorMap tmX, tmW;
  if (!make_map(&tmX, x, T, d, kTM) || !make_map(&tmW, w_split, E, 3 * dpad, NE))
    return cudaErrorInvalidValue;
  const RParams p{T, E, dpad, 1, router_bias, logits, status, RouterAccum{}, 0};
  const TopkOut ko{T,  E,  k,  ids, gates, probs, acc, aux_alpha, lb_stats, dc, renormalize ? 1 : 0,
                   losses, exported, extra_stats ? 1 : 0};
  const int ntiles = (int)((T + kTM - 1) / kTM);
  switch (NE) {
    case 16: return launch_fused_ne<16>(tmX, tmW, p, ko, ntiles, stream);
    case 32: return launch_fused_ne<32>(tmX, tmW, p, ko, ntiles, stream);
    case 64: return launch_fused_ne<64>(tmX, tmW, p, ko, ntiles, stream);
    default: return launch_fused_ne<128>(tmX, tmW, p, ko, ntiles, stream);
  }
}

cudaError_t enqueue_router_logits_tc(const void* x, int64_t T, int d, const uint16_t* w_split,
                                     int dpad, const float* router_bias, int E, float* logits,
                                     int* status, cudaStream_t stream, const RouterAccum* zero_acc) {
  if (T == 0) return cudaSuccess;
  const int slice = E < kSlice ? E : kSlice;
  int NE = 16;
  while (NE < slice) NE <<= 1;  // instantiated N tiles: 16, 32, 64, 128
  const int n_slices = (E + kSlice - 1) / kSlice;
  CUtensorMap tmX, tmW;
  if (!make_map(&tmX, x, T, d, kTM) || !make_map(&tmW, w_split, E, 3 * dpad, NE))
    return cudaErrorInvalidValue;
  const RParams p{T, E, dpad, n_slices, router_bias, logits, status,
                  zero_acc ? *zero_acc : RouterAccum{}, zero_acc ? 1 : 0};
  const int ntiles = (int)((T + kTM - 1) / kTM) * n_slices;
  switch (NE) {
    case 16: return launch_tc<16>(tmX, tmW, p, ntiles, stream);
    case 32: return launch_tc<32>(tmX, tmW, p, ntiles, stream);
    case 64: return launch_tc<64>(tmX, tmW, p, ntiles, stream);
    default: return launch_tc<128>(tmX, tmW, p, ntiles, stream);
  }
}

}  // namespace moe
