// Grouped expert GEMM on sm_100a tensor cores (tcgen05 + TMEM + TMA), with the bias(+GeLU)
// epilogue fused.
//
// Computes, for every expert e and every packed row r of its segment
// [offsets[e], offsets[e+1]):
//     out[r, f] = act( sum_k W[e*N + f, k] * X[r, k] + bias[e, f] ),   f < N
// which is one layer of the expert FFN ("Sparse GEMM -> Dense GEMM": dense per-expert GEMMs on
// the rows the layout transform packed together, DeepSpeed-MoE notes §4.4 / §5).
//
// Orientation: the weights are the MMA's A operand (M = 128 output features per tile) and the
// packed token rows are the B operand (N = BN tokens per tile, 16..256). The accumulator tile
// is therefore [features x tokens] in TMEM (lane = feature, column = token). A tile of an
// expert with few rows (decode: one row) issues an MMA with N = 16 instead of padding tokens
// to M = 128, so ragged and tiny experts cost no extra tensor work; the weight tiles stream
// from HBM once per token tile.
//
// Schedule: persistent CTAs (one per SM) walk tiles t = blockIdx.x, blockIdx.x + gridDim.x, ...
// of a list ordered (expert, feature tile, token tile), built in shared memory from the device
// offsets, so no host synchronisation is needed for the ragged sizes. A tile may hold FT = 2
// feature tiles of 128 that multiply the same token tile (two accumulators per buffer), so each
// token tile is read from L2 half as often; the host picks FT = 2 when the layer has more than
// one feature tile and the halved tile count still fills the persistent grid's waves.
// A_MN (backward pass): the weights arrive stored [E][K][N] and are read MN-major (two 64-feature
// boxes per feature tile, MN-major shared-memory descriptors), for dH = dY W2 and dX = dZ W1.
// Roles per CTA:
//     warp 0      TMA producer: FT 128x64 weight tiles and a BNx64 token tile per stage,
//                 128-byte swizzle, STAGES-deep mbarrier ring
//     warp 1      allocates TMEM, one thread issues tcgen05.mma (K = 16 per instruction) into
//                 one of two accumulators, commits stage release and accumulator-full barriers
//     warps 2..9  epilogue, two warps per TMEM lane quarter taking alternate 16-column chunks:
//                 tcgen05.ld of the accumulator, + bias, GeLU (erf form) and bf16 rounding for
//                 the first layer or fp32 for the second, transposed through a per-warp shared
//                 staging tile into 16-byte stores of whole token rows, masked to the valid
//                 rows/features; then release the accumulator
// Every wait is bounded (about 2 s): on expiry the kernel records MOE_DEVERR_TIMEOUT in the
// status word, the other roles stop, in-flight TMA copies and MMAs are drained, TMEM is freed.
#include <algorithm>
#include <cstdlib>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

#ifndef MOE_GG_MAX_STAGES
#define MOE_GG_MAX_STAGES 12
#endif

constexpr int kBM = 128;         // output features per tile (MMA M)
constexpr int kBK = 64;          // K per stage: one 128-byte swizzle row of bf16
constexpr int kUmmaK = 16;       // K per tcgen05.mma (kind::f16)
constexpr int kThreads = 320;    // 10 warps: TMA, MMA, 8 epilogue
constexpr int kEpiWarps = 8;
constexpr int kStageTileBytes = 16 * 32 * 4;  // per epilogue warp: 16 tokens x 32 features, fp32

// Epilogue kinds.
constexpr int kEpiGeluBf16 = 0;  // out = bf16(GeLU(acc + bias)), bias bf16   (expert layer 1)
constexpr int kEpiF32 = 1;       // out = acc + bias (fp32), bias bf16          (expert layer 2)
// Layer 2 with the combine fused (see CombineArgs): y = acc + bias stays in registers and the
// epilogue writes the layer output row of the token instead of y.
constexpr int kEpiCombineExpert = 2;  // top-1: out[token(r)] = [x] + gate * y[r]
constexpr int kEpiCombineDense = 3;   // PR-MoE dense MLP, row = token t:
                                      // out[t] = [x] + y_dense[t] + sum_j gate_j * y_expert[row_j]
// Training.
constexpr int kEpiGeluGradBf16 = 4;   // out = bf16(acc * g[r, f]), g = GeLU'(z) saved by the
                                      // forward (backward through layer 2 into layer 1's input)
constexpr int kEpiGeluBf16Train = 5;  // layer 1 forward that also saves g = bf16(GeLU'(z))

// FT: 128-feature tiles per CTA tile. With FT = 2 both feature tiles multiply the same token
// tile, so each token tile is read from L2 half as often (two accumulators per buffer).
template <int BN, int FT = 1>
struct Cfg {
  static constexpr int kABytes = FT * kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStagesFit = (200 * 1024) / kStageBytes;
  static constexpr int kStages = kStagesFit > MOE_GG_MAX_STAGES ? MOE_GG_MAX_STAGES : kStagesFit;
  static constexpr int kNumAcc = 2;  // the epilogue of tile i overlaps the MMAs of tile i + 1
  static constexpr int kTmemCols = (kNumAcc * FT * BN) < 32 ? 32 : (kNumAcc * FT * BN);
  static_assert(kNumAcc * FT * BN <= 512, "two buffers of FT accumulators must fit TMEM");
  // barriers: full[S], empty[S], tmem_full[2], tmem_empty[2], drain  (8 bytes each, <= 64 of them)
  static constexpr int kBarBytes = 8 * 64;
  static constexpr int kAuxBytes = kBarBytes + 16 + 2 * 4 * (MOE_MAX_EXPERTS + 1);
  static constexpr int kSmemBytes =
      1024 + kStages * kStageBytes + kEpiWarps * kStageTileBytes + kAuxBytes;
  static_assert(kStageBytes % 1024 == 0, "stage tiles must stay 1024-byte aligned");
  static_assert(2 * kStages + 5 <= 64, "barrier area too small");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// Operands of the fused combine epilogues. The arithmetic is the combine kernel's, in its order:
// acc = [x] + [y_dense]; acc = fma(gate_j, y_j, acc) for the kept choices j ascending; one rounding.
struct CombineArgs {
  const int32_t* row_token;  // [rows] token of each packed row (expert mode)
  const int32_t* slot;       // [T, k] (dense mode)
  const int32_t* ids;        // [T, k] (dense mode)
  const int32_t* offsets;    // [E_experts + 1] (dense mode)
  const float* gates;        // [T, k]
  const float* y;            // [rows_y, n_out] fp32 expert outputs (dense mode)
  const uint16_t* residual;  // [T, n_out] bf16 x, or nullptr
  void* out;                 // [T, n_out] bf16 or fp32
  int out_bf16, k, E_experts;
  int64_t rows_y;            // rows of y (bounds check)
};

struct Params {
  const int32_t* offsets;  // [E+1], or nullptr: one segment [0, rows_max) (E == 1)
  int E;
  int n_out;               // output features per expert
  int K;                   // reduction length of the weight operand
  int64_t rows_max;
  const void* bias;        // [E, n_out] bf16, or nullptr
  void* out;               // [rows_max, n_out]: bf16 (GeLU layer) or fp32
  int* status;
  CombineArgs cmb;         // used by the combine epilogues only
  const uint16_t* g_in;    // [rows_max, n_out] bf16 GeLU'(z) (kEpiGeluGradBf16)
  uint16_t* g_out;         // [rows_max, n_out] bf16 GeLU'(z) (kEpiGeluBf16Train)
  // Failure-detection self-test only (moe_selftest_bounded_wait): the TMA role issues no copy, so
  // the MMA role's first wait can never complete, and every bounded wait gives up after
  // wait_limit_ns. Normal launches: selftest_no_copies = 0, wait_limit_ns = kWaitLimitNs.
  int selftest_no_copies = 0;
  uint64_t wait_limit_ns = kWaitLimitNs;
  // The weights are read once (one token tile per expert): their TMA loads carry an L2
  // evict-first policy, so the stream does not push reused operands out of L2.
  int w_read_once = 0;
};

struct Tile {
  int e, f0, row0, n_valid;
};

template <int BN, int FT>
__device__ __forceinline__ Tile decode_tile(int t, const int* prefix, const int* seg, int E,
                                            int n_ftiles) {
  int lo = 0, hi = E;  // prefix[lo] <= t < prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= t) lo = mid;
    else hi = mid;
  }
  const int rows = seg[lo + 1] - seg[lo];
  const int ntt = (rows + BN - 1) / BN;
  const int local = t - prefix[lo];
  const int ft = local / ntt;
  const int jt = local - ft * ntt;
  Tile tl;
  tl.e = lo;
  tl.f0 = ft * kBM * FT;
  tl.row0 = seg[lo] + jt * BN;
  tl.n_valid = min(BN, rows - jt * BN);
  return tl;
}

// Tile order of a one-segment problem (the dense MLP: rows = tokens): groups of token tiles;
// inside a group, every token tile of the group for feature tile 0, then for feature tile 1, and
// so on. The tiles in flight at one time then share a few weight tiles and a few token tiles (a
// working set that stays in L2), where a feature-tile-major order would sweep all the tokens once
// per feature tile. A group holds about 24 MB of token rows (16 tiles at K = 2048, 6 at K = 8192)
// and at most 16 tiles.
__host__ __device__ __forceinline__ int dense_group_tiles(int BN, int K) {
  const int64_t per_tile = (int64_t)BN * K * 2;
  const int64_t g = (int64_t)(24 << 20) / (per_tile > 0 ? per_tile : 1);
  return g < 1 ? 1 : (g > 16 ? 16 : (int)g);
}
template <int BN, int FT>
__device__ __forceinline__ Tile decode_dense_tile(int u, int64_t rows, int n_ftiles, int K) {
  const int group = dense_group_tiles(BN, K);
  const int n_tt = (int)((rows + BN - 1) / BN);
  const int per_group = n_ftiles * group;
  const int g = u / per_group;
  const int in = u - g * per_group;
  const int gt = min(group, n_tt - g * group);
  const int ft = in / gt;
  const int jt = g * group + (in - ft * gt);
  Tile tl;
  tl.e = 0;
  tl.f0 = ft * kBM * FT;
  tl.row0 = jt * BN;
  tl.n_valid = (int)min((int64_t)BN, rows - (int64_t)jt * BN);
  return tl;
}

// Wait bounded by time only (used to drain in-flight copies/MMAs while unwinding).
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity, int* status) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      set_device_error(status, MOE_DEVERR_TIMEOUT);
      return;
    }
  }
}

// The mbarriers of one CTA: S stage-full, S stage-empty, 2 accumulator-full, 2 accumulator-empty
// and one drain barrier, 8 bytes each from `base`.
struct Bars {
  uint32_t base;
  int S;
  __device__ __forceinline__ uint32_t full(int s) const { return base + 8u * s; }
  __device__ __forceinline__ uint32_t empty(int s) const { return base + 8u * (S + s); }
  __device__ __forceinline__ uint32_t tfull(int a) const { return base + 8u * (2 * S + a); }
  __device__ __forceinline__ uint32_t tempty(int a) const { return base + 8u * (2 * S + 2 + a); }
  __device__ __forceinline__ uint32_t drain() const { return base + 8u * (2 * S + 4); }
};

// Position in the stage ring (shared by the TMA and MMA roles' loops).
struct Ring {
  int stage = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void next(int S) {
    if (++stage == S) {
      stage = 0;
      phase ^= 1u;
    }
  }
};

// TMA role, one tile: per 64-wide K block, FT weight boxes of 128 rows (A) and one token box of BN
// rows (B) into the next stage (A at the stage start, B at +a_bytes). Returns false if a wait
// gave up.
template <int BN, int FT, bool A_MN>
__device__ __forceinline__ bool produce_tile(const Tile& tl, const CUtensorMap* tmW,
                                             const CUtensorMap* tmX, const Params& p, int n_kb,
                                             uint32_t base_addr, uint32_t stage_stride,
                                             uint32_t a_bytes, const Bars& B, Ring& ring,
                                             int& issued, volatile int* abort_flag,
                                             int x_rows = BN) {
  // x_rows: the token box height of tmX (at least the tile's MMA N; rows past it are not read)
  const uint32_t kTx = FT * kBM * kBK * 2 + (uint32_t)x_rows * kBK * 2;
  const int w_row = tl.e * p.n_out + tl.f0;
  const uint64_t w_policy = p.w_read_once ? l2_policy_evict_first() : 0ull;
  for (int kb = 0; kb < n_kb; ++kb) {
    if (!mbar_wait_bounded(B.empty(ring.stage), ring.phase ^ 1u, abort_flag, p.status,
                           p.wait_limit_ns))
      return false;
    const uint32_t sa = base_addr + ring.stage * stage_stride;
    mbar_arrive_expect_tx(B.full(ring.stage), kTx);
#pragma unroll
    for (int i = 0; i < FT; ++i) {
      const uint32_t sai = sa + i * (kBM * kBK * 2);
      if constexpr (A_MN) {
        const int k_row = tl.e * p.K + kb * kBK;
        tma_load_2d(sai, tmW, tl.f0 + i * kBM, k_row, B.full(ring.stage));
        tma_load_2d(sai + kBM * kBK, tmW, tl.f0 + i * kBM + 64, k_row, B.full(ring.stage));
      } else {
        // rows past this expert's n_out (odd tile count) belong to the next expert or are out
        // of range; the epilogue masks those features
        if (p.w_read_once)
          tma_load_2d_hint(sai, tmW, kb * kBK, w_row + i * kBM, B.full(ring.stage), w_policy);
        else
          tma_load_2d(sai, tmW, kb * kBK, w_row + i * kBM, B.full(ring.stage));
      }
    }
    tma_load_2d(sa + a_bytes, tmX, kb * kBK, tl.row0, B.full(ring.stage));
    ++issued;
    ring.next(B.S);
  }
  return true;
}

// MMA role, one tile: K blocks of FT MMAs (M = 128 features, N = the tile's tokens rounded up to
// 16, K = 16 each) into FT accumulators of BN columns at d_tmem. Returns false if a wait gave up.
template <int BN, int FT, bool A_MN>
__device__ __forceinline__ bool mma_tile(const Tile& tl, uint32_t d_tmem, const Params& p,
                                         int n_kb, uint32_t base_addr, uint32_t stage_stride,
                                         uint32_t a_bytes, const Bars& B, Ring& ring,
                                         volatile int* abort_flag) {
  const int n_mma = max(16, (tl.n_valid + 15) & ~15);
  const uint32_t idesc = idesc_bf16_f32_major(kBM, n_mma, A_MN, false);
  for (int kb = 0; kb < n_kb; ++kb) {
    if (!mbar_wait_bounded(B.full(ring.stage), ring.phase, abort_flag, p.status, p.wait_limit_ns))
      return false;
    tc_fence_after();
    const uint32_t sa = base_addr + ring.stage * stage_stride;
    const uint64_t bdesc = smem_desc_sw128(sa + a_bytes);
    // K step: +32 bytes inside a K-major 128-byte row (+2 in the 16-byte address field),
    // or two 8-row groups of an MN-major tile
    constexpr uint64_t a_step = A_MN ? (kMnKStepBytes >> 4) : 2;
#pragma unroll
    for (int i = 0; i < FT; ++i) {
      const uint32_t sai = sa + i * (kBM * kBK * 2);
      const uint64_t adesc = A_MN ? smem_desc_sw128_mn(sai) : smem_desc_sw128(sai);
#pragma unroll
      for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
        tc_mma_bf16(d_tmem + (uint32_t)(i * BN), adesc + a_step * (uint64_t)kk,
                    bdesc + (uint64_t)(2 * kk), idesc, (kb | kk) != 0 ? 1u : 0u);
      }
    }
    tc_commit(B.empty(ring.stage));
    ring.next(B.S);
  }
  return true;
}

// Epilogue role (one of warps 2..9), one tile: reads the FT accumulators at acc_tmem (this warp's
// TMEM lane quarter, alternate 16-column chunks by `half`) and writes the tile's outputs.
template <int BN, int FT, int EPI>
__device__ __forceinline__ void epilogue_tile(const Tile& tl, const Params& p, uint32_t acc_tmem,
                                              int quarter, int half, int lane, uint8_t* st) {
#pragma unroll 1
  for (int fi = 0; fi < FT; ++fi) {
    const int fw = tl.f0 + fi * kBM + quarter * 32;  // first feature of this warp
    const int f = fw + lane;
    const bool f_ok = f < p.n_out;
    const float bv = (p.bias != nullptr && f_ok)
                         ? bf16_to_f32(reinterpret_cast<const uint16_t*>(p.bias)[(int64_t)tl.e * p.n_out + f])
                         : 0.0f;
    const uint32_t taddr = acc_tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(fi * BN);
    for (int c0 = half * 16; c0 < tl.n_valid; c0 += 32) {
      uint32_t r[16];
      tmem_ld_32x32b_x16(taddr + (uint32_t)c0, r);
      tmem_ld_wait();
      const int nc = min(16, tl.n_valid - c0);
      if constexpr (EPI == kEpiGeluGradBf16) {
        // dZ = dH * GeLU'(z): stage dH [16 tokens][32 features] fp32, then each lane takes 8
        // features of one token: 16-byte loads of GeLU'(z) and 16-byte stores of dZ
        float* s32 = reinterpret_cast<float*>(st);
#pragma unroll
        for (int c = 0; c < 16; ++c) s32[c * 32 + lane] = __uint_as_float(r[c]);
        __syncwarp();
#pragma unroll
        for (int id = lane; id < 64; id += 32) {
          const int row = id >> 2, q = id & 3;
          const int ff = fw + 8 * q;
          if (row < nc && ff < p.n_out) {
            const int64_t o = (int64_t)(tl.row0 + c0 + row) * p.n_out + ff;
            const uint4 gv = *reinterpret_cast<const uint4*>(p.g_in + o);
            const float4 h0 = *reinterpret_cast<const float4*>(s32 + row * 32 + 8 * q);
            const float4 h1 = *reinterpret_cast<const float4*>(s32 + row * 32 + 8 * q + 4);
            uint4 ov;
            ov.x = (uint32_t)f32_to_bf16_rn(h0.x * __uint_as_float(gv.x << 16)) |
                   ((uint32_t)f32_to_bf16_rn(h0.y * __uint_as_float(gv.x & 0xffff0000u)) << 16);
            ov.y = (uint32_t)f32_to_bf16_rn(h0.z * __uint_as_float(gv.y << 16)) |
                   ((uint32_t)f32_to_bf16_rn(h0.w * __uint_as_float(gv.y & 0xffff0000u)) << 16);
            ov.z = (uint32_t)f32_to_bf16_rn(h1.x * __uint_as_float(gv.z << 16)) |
                   ((uint32_t)f32_to_bf16_rn(h1.y * __uint_as_float(gv.z & 0xffff0000u)) << 16);
            ov.w = (uint32_t)f32_to_bf16_rn(h1.z * __uint_as_float(gv.w << 16)) |
                   ((uint32_t)f32_to_bf16_rn(h1.w * __uint_as_float(gv.w & 0xffff0000u)) << 16);
            *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) + o) = ov;
          }
        }
        __syncwarp();
      } else if constexpr (EPI == kEpiGeluBf16 || EPI == kEpiGeluBf16Train) {
        // stage [16 tokens][32 features] bf16, then 16-byte stores of 8 features of one token
        // (the training variant stages GeLU'(z) the same way, after GeLU(z))
        uint16_t* s16 = reinterpret_cast<uint16_t*>(st);
#pragma unroll
        for (int c = 0; c < 16; ++c) s16[c * 32 + lane] = f32_to_bf16_rn(gelu_erf(__uint_as_float(r[c]) + bv));
        __syncwarp();
        if constexpr (EPI == kEpiGeluBf16Train) {
          uint16_t* g16 = s16 + 16 * 32;
#pragma unroll
          for (int c = 0; c < 16; ++c)
            g16[c * 32 + lane] = f32_to_bf16_rn(gelu_erf_grad(__uint_as_float(r[c]) + bv));
          __syncwarp();
#pragma unroll
          for (int id = lane; id < 64; id += 32) {
            const int row = id >> 2, q = id & 3;
            const int ff = fw + 8 * q;
            if (row < nc && ff < p.n_out)
              *reinterpret_cast<uint4*>(p.g_out + (int64_t)(tl.row0 + c0 + row) * p.n_out + ff) =
                  *reinterpret_cast<const uint4*>(st + 1024 + row * 64 + q * 16);
          }
        }
#pragma unroll
        for (int id = lane; id < 64; id += 32) {
          const int row = id >> 2, q = id & 3;
          const int ff = fw + 8 * q;
          if (row < nc && ff < p.n_out)
            *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) +
                                      (int64_t)(tl.row0 + c0 + row) * p.n_out + ff) =
                *reinterpret_cast<const uint4*>(st + row * 64 + q * 16);
        }
        __syncwarp();
      } else if constexpr (EPI == kEpiF32) {
        // stage [16 tokens][32 features] fp32, then 16-byte stores of 4 features of one token
        float* s32 = reinterpret_cast<float*>(st);
#pragma unroll
        for (int c = 0; c < 16; ++c) s32[c * 32 + lane] = __uint_as_float(r[c]) + bv;
        __syncwarp();
#pragma unroll
        for (int id = lane; id < 128; id += 32) {
          const int row = id >> 3, q = id & 7;
          const int ff = fw + 4 * q;
          if (row < nc && ff < p.n_out)
            *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) +
                                       (int64_t)(tl.row0 + c0 + row) * p.n_out + ff) =
                *reinterpret_cast<const float4*>(st + row * 128 + q * 16);
        }
        __syncwarp();
      } else {
        // fused combine: y (or the dense MLP output) = acc + bias staged as fp32 [16][32]; each
        // lane then finishes 4 features of one token row of the layer output
        const CombineArgs& cb = p.cmb;
        float* s32 = reinterpret_cast<float*>(st);
#pragma unroll
        for (int c = 0; c < 16; ++c) s32[c * 32 + lane] = __uint_as_float(r[c]) + bv;
        __syncwarp();
#pragma unroll
        for (int id = lane; id < 128; id += 32) {
          const int row = id >> 3, q = id & 7;
          const int ff = fw + 4 * q;
          if (row < nc && ff < p.n_out) {
            const int64_t pr = (int64_t)(tl.row0 + c0 + row);  // packed row (dense: token)
            const float4 v = *reinterpret_cast<const float4*>(st + row * 128 + q * 16);
            int64_t t;
            float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            if constexpr (EPI == kEpiCombineExpert) {
              t = cb.row_token[pr];
            } else {
              t = pr;
            }
            if (cb.residual) {
              const uint2 rb = *reinterpret_cast<const uint2*>(cb.residual + t * p.n_out + ff);
              a[0] = __uint_as_float(rb.x << 16);
              a[1] = __uint_as_float(rb.x & 0xffff0000u);
              a[2] = __uint_as_float(rb.y << 16);
              a[3] = __uint_as_float(rb.y & 0xffff0000u);
            }
            if constexpr (EPI == kEpiCombineExpert) {
              const float g = cb.gates[t];
              a[0] = fmaf(g, v.x, a[0]);
              a[1] = fmaf(g, v.y, a[1]);
              a[2] = fmaf(g, v.z, a[2]);
              a[3] = fmaf(g, v.w, a[3]);
            } else {
              a[0] += v.x;
              a[1] += v.y;
              a[2] += v.z;
              a[3] += v.w;
              for (int j = 0; j < cb.k; ++j) {
                const int sl = cb.slot[t * cb.k + j];
                if (sl < 0) continue;
                const int e = cb.ids[t * cb.k + j];
                if (e < 0 || e >= cb.E_experts) continue;
                const int64_t yr = (int64_t)cb.offsets[e] + sl;
                if (yr >= cb.rows_y) {
                  set_device_error(p.status, MOE_DEVERR_BAD_ROW);
                  continue;
                }
                const float g = cb.gates[t * cb.k + j];
                const float4 y = *reinterpret_cast<const float4*>(cb.y + yr * p.n_out + ff);
                a[0] = fmaf(g, y.x, a[0]);
                a[1] = fmaf(g, y.y, a[1]);
                a[2] = fmaf(g, y.z, a[2]);
                a[3] = fmaf(g, y.w, a[3]);
              }
            }
            if (cb.out_bf16) {
              uint2 o;
              o.x = (uint32_t)f32_to_bf16_rn(a[0]) | ((uint32_t)f32_to_bf16_rn(a[1]) << 16);
              o.y = (uint32_t)f32_to_bf16_rn(a[2]) | ((uint32_t)f32_to_bf16_rn(a[3]) << 16);
              *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(cb.out) + t * p.n_out + ff) = o;
            } else {
              *reinterpret_cast<float4*>(reinterpret_cast<float*>(cb.out) + t * p.n_out + ff) =
                  make_float4(a[0], a[1], a[2], a[3]);
            }
          }
        }
        __syncwarp();
      }
    }
  }
}

// Builds the tile list of a grouped problem in shared memory (one warp): seg[e] = first packed
// row of expert e, prefix[e] = first tile of expert e, prefix[E] = the tile count (0 and a device
// error if the offsets are not non-decreasing within [0, rows_max]).
template <int BN>
__device__ __forceinline__ void build_tile_list(const Params& p, int n_ftiles, int* prefix,
                                                int* seg, int lane) {
  const int E = p.E;
  const int chunk = (E + 31) / 32;
  const int e0 = min(E, lane * chunk), e1 = min(E, e0 + chunk);
  bool bad = false;
  int local = 0;
  // offsets == nullptr: one segment covering all rows_max rows (dense MLP, E == 1)
  auto off = [&](int e) -> int {
    return p.offsets ? p.offsets[e] : (e == 0 ? 0 : (int)p.rows_max);
  };
  for (int e = e0; e < e1; ++e) {
    const int a = off(e), b = off(e + 1);
    seg[e] = a;
    if (a < 0 || b < a || (int64_t)b > p.rows_max) bad = true;
    else local += n_ftiles * ((b - a + BN - 1) / BN);
  }
  if (lane == 0) seg[E] = off(E);
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  int run = incl - local;
  for (int e = e0; e < e1; ++e) {
    prefix[e] = run;
    const int a = seg[e], b = off(e + 1);
    if (!(a < 0 || b < a || (int64_t)b > p.rows_max)) run += n_ftiles * ((b - a + BN - 1) / BN);
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  bad = __any_sync(0xffffffffu, bad);
  __syncwarp();
  if (lane == 0) {
    prefix[E] = bad ? 0 : total;
    if (bad && blockIdx.x == 0) set_device_error(p.status, MOE_DEVERR_BAD_OFFSETS);
  }
}

// A_MN: the weight operand is stored [E][K][n_out] (the transpose of the forward layout, as the
// backward pass reads W1 and W2) and loaded MN-major: two 64-feature x 64-K boxes per stage.
template <int BN, int EPI, bool A_MN = false, int FT = 1>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmW,
                        const __grid_constant__ CUtensorMap tmX, const Params p) {
  using C = Cfg<BN, FT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_addr - raw_addr);

  uint8_t* stage_tiles = base + C::kStages * C::kStageBytes;
  uint8_t* aux = stage_tiles + kEpiWarps * kStageTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(aux);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(aux + C::kBarBytes);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(aux + C::kBarBytes + 4);
  int* prefix = reinterpret_cast<int*>(aux + C::kBarBytes + 16);
  int* seg = prefix + (MOE_MAX_EXPERTS + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = C::kStages;
  const Bars B{smem_u32(bars), S};

  // ------------------------------------------------------------ prologue
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(B.full(s), 1);
      mbar_init(B.empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(B.tfull(a), 1);
      mbar_init(B.tempty(a), kEpiWarps * 32);
    }
    mbar_init(B.drain(), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // everything above touches shared memory only; wait for the preceding kernels before any global
  // access or TMEM allocation
  pdl_wait();
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  const int n_ftiles = (p.n_out + kBM * FT - 1) / (kBM * FT);
  if (warp == 2) build_tile_list<BN>(p, n_ftiles, prefix, seg, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total_tiles = prefix[p.E];
  const int n_kb = (p.K + kBK - 1) / kBK;
  const bool one_seg = p.offsets == nullptr;
  auto tile_at = [&](int t) {
    return one_seg ? decode_dense_tile<BN, FT>(t, p.rows_max, n_ftiles, p.K)
                   : decode_tile<BN, FT>(t, prefix, seg, p.E, n_ftiles);
  };

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      Ring ring;
      int issued = 0;
      for (int t = blockIdx.x; t < total_tiles && !p.selftest_no_copies; t += gridDim.x) {
        if (!produce_tile<BN, FT, A_MN>(tile_at(t), &tmW, &tmX, p, n_kb, base_addr, C::kStageBytes,
                                        C::kABytes, B, ring, issued, abort_flag))
          break;
      }
      // drain: the last min(issued, S) loads may still be landing
      for (int i = max(0, issued - S); i < issued; ++i)
        mbar_wait_drain(B.full(i % S), (uint32_t)((i / S) & 1), p.status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      Ring ring;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
        if (!mbar_wait_bounded(B.tempty(acc), acc_phase ^ 1u, abort_flag, p.status,
                               p.wait_limit_ns))
          break;
        tc_fence_after();
        if (!mma_tile<BN, FT, A_MN>(tile_at(t), tmem_base + (uint32_t)(acc * FT * BN), p, n_kb,
                                    base_addr, C::kStageBytes, C::kABytes, B, ring, abort_flag))
          break;
        tc_commit(B.tfull(acc));
        if (++acc == C::kNumAcc) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // drain every MMA this thread issued before TMEM is released
      tc_commit(B.drain());
      mbar_wait_drain(B.drain(), 0, p.status);
    }
  } else {
    // ---------------------------------------------------------- epilogue (warps 2..9)
    const int ew = warp - 2;         // 0..7
    const int quarter = warp & 3;    // TMEM lanes this warp may access: [32*quarter, 32*quarter+32)
    const int half = ew >> 2;        // this warp takes 16-column chunks half, half+2, half+4, ...
    uint8_t* st = stage_tiles + ew * kStageTileBytes;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      if (!mbar_wait_bounded_warp(B.tfull(acc), acc_phase, abort_flag, p.status,
                                  p.wait_limit_ns))
        break;
      tc_fence_after();
      epilogue_tile<BN, FT, EPI>(tile_at(t), p, tmem_base + (uint32_t)(acc * FT * BN), quarter,
                                 half, lane, st);
      tc_fence_before();
      mbar_arrive(B.tempty(acc));
      if (++acc == C::kNumAcc) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  pdl_trigger();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Two GEMM problems of one layer co-scheduled in one persistent launch: problem 0 is the grouped
// expert layer (BN0 tokens per tile, two 128-feature tiles per CTA tile), problem 1 the PR-MoE
// dense MLP layer (one segment of all tokens, 256 tokens x 128 features per tile), with the same
// epilogue kind. The expert layers stream their weights from HBM with the tensor pipe mostly idle,
// the dense layers keep it busy with little HBM traffic: interleaving their tiles on every SM lets
// the two overlap instead of taking turns. The combined tile sequence takes problem-0 tile number
// floor(t n0 / N) when floor((t + 1) n0 / N) > floor(t n0 / N), else problem-1 tile
// t - floor(t n0 / N) (N = n0 + n1), so any window of consecutive tiles holds both in proportion;
// CTA b takes tiles b, b + gridDim.x, ... as in the single-problem kernel. Stages are 48 KB (the
// larger of the two problems' stage sizes) and each accumulator is 256 TMEM columns.
constexpr int kCoBN1 = 256;
constexpr int kCoStageBytes = 48 * 1024;
constexpr int kCoStages = (200 * 1024) / kCoStageBytes;
constexpr int kCoAccCols = 256;
constexpr int kCoSmemBytes = 1024 + kCoStages * kCoStageBytes + kEpiWarps * kStageTileBytes +
                             Cfg<kCoBN1, 1>::kAuxBytes;
static_assert(Cfg<kCoBN1, 1>::kStageBytes == kCoStageBytes, "dense stage size");
static_assert(Cfg<128, 2>::kStageBytes <= kCoStageBytes, "expert stage size");
static_assert(2 * kCoStages + 5 <= 64, "barrier area too small");
static_assert(kCoSmemBytes <= 227 * 1024, "shared memory budget");

template <int BN0, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    co_gemm_kernel(const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmX0,
                   const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmX1,
                   const __grid_constant__ CUtensorMap tmX0_32,
                   const __grid_constant__ CUtensorMap tmX0_64, const Params p0, const Params p1) {
  static_assert(2 * BN0 <= kCoAccCols, "two expert accumulators per buffer");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_addr - raw_addr);

  uint8_t* stage_tiles = base + kCoStages * kCoStageBytes;
  uint8_t* aux = stage_tiles + kEpiWarps * kStageTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(aux);
  constexpr int kBarBytes = Cfg<kCoBN1, 1>::kBarBytes;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(aux + kBarBytes);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(aux + kBarBytes + 4);
  int* prefix = reinterpret_cast<int*>(aux + kBarBytes + 16);
  int* seg = prefix + (MOE_MAX_EXPERTS + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = kCoStages;
  const Bars B{smem_u32(bars), S};

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(B.full(s), 1);
      mbar_init(B.empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(B.tfull(a), 1);
      mbar_init(B.tempty(a), kEpiWarps * 32);
    }
    mbar_init(B.drain(), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  pdl_wait();
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmW0);
    tma_prefetch_desc(&tmX0);
    tma_prefetch_desc(&tmW1);
    tma_prefetch_desc(&tmX1);
    if (BN0 > 32) tma_prefetch_desc(&tmX0_32);
    if (BN0 > 64) tma_prefetch_desc(&tmX0_64);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 2 * kCoAccCols);
    tmem_relinquish();
  }
  const int nft0 = (p0.n_out + 2 * kBM - 1) / (2 * kBM);
  const int nft1 = (p1.n_out + kBM - 1) / kBM;
  if (warp == 2) build_tile_list<BN0>(p0, nft0, prefix, seg, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int n0 = prefix[p0.E];
  const int n1 = nft1 * (int)((p1.rows_max + kCoBN1 - 1) / kCoBN1);
  const int total = n0 + n1;
  const int nkb0 = (p0.K + kBK - 1) / kBK;
  const int nkb1 = (p1.K + kBK - 1) / kBK;
  // problem and tile of combined tile t
  auto which = [&](int t, int& local) -> int {
    const int c = (int)(((int64_t)t * n0) / total);
    const int c1 = (int)(((int64_t)(t + 1) * n0) / total);
    if (c1 > c) {
      local = c;
      return 0;
    }
    local = t - c;
    return 1;
  };
  constexpr uint32_t kA0 = 2 * kBM * kBK * 2;  // two weight boxes
  constexpr uint32_t kA1 = kBM * kBK * 2;      // one weight box

  if (warp == 0) {
    if (lane == 0) {
      Ring ring;
      int issued = 0;
      for (int t = blockIdx.x; t < total; t += gridDim.x) {
        int u;
        bool ok;
        if (which(t, u) == 0) {
          // an expert tile loads only the token rows its MMAs read (the tile's rows rounded up to
          // 16, then to a box of 32, 64 or BN0 rows): the stage fill that short segments leave
          // for the weight stream, which is what bounds these tiles
          const Tile tl = decode_tile<BN0, 2>(u, prefix, seg, p0.E, nft0);
          const int n_mma = max(16, (tl.n_valid + 15) & ~15);
          const bool r32 = BN0 > 32 && n_mma <= 32, r64 = !r32 && BN0 > 64 && n_mma <= 64;
          ok = produce_tile<BN0, 2, false>(tl, &tmW0, r32 ? &tmX0_32 : (r64 ? &tmX0_64 : &tmX0), p0,
                                           nkb0, base_addr, kCoStageBytes, kA0, B, ring, issued,
                                           abort_flag, r32 ? 32 : (r64 ? 64 : BN0));
        } else {
          ok = produce_tile<kCoBN1, 1, false>(
                                  decode_dense_tile<kCoBN1, 1>(u, p1.rows_max, nft1, p1.K), &tmW1, &tmX1,
                                  p1, nkb1, base_addr, kCoStageBytes, kA1, B, ring, issued,
                                  abort_flag);
        }
        if (!ok) break;
      }
      for (int i = max(0, issued - S); i < issued; ++i)
        mbar_wait_drain(B.full(i % S), (uint32_t)((i / S) & 1), p0.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      Ring ring;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int t = blockIdx.x; t < total; t += gridDim.x) {
        if (!mbar_wait_bounded(B.tempty(acc), acc_phase ^ 1u, abort_flag, p0.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kCoAccCols);
        int u;
        const bool ok = which(t, u) == 0
                            ? mma_tile<BN0, 2, false>(decode_tile<BN0, 2>(u, prefix, seg, p0.E, nft0),
                                                      d_tmem, p0, nkb0, base_addr, kCoStageBytes,
                                                      kA0, B, ring, abort_flag)
                            : mma_tile<kCoBN1, 1, false>(
                                  decode_dense_tile<kCoBN1, 1>(u, p1.rows_max, nft1, p1.K), d_tmem, p1,
                                  nkb1, base_addr, kCoStageBytes, kA1, B, ring, abort_flag);
        if (!ok) break;
        tc_commit(B.tfull(acc));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      tc_commit(B.drain());
      mbar_wait_drain(B.drain(), 0, p0.status);
    }
  } else {
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int half = ew >> 2;
    uint8_t* st = stage_tiles + ew * kStageTileBytes;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      if (!mbar_wait_bounded_warp(B.tfull(acc), acc_phase, abort_flag, p0.status)) break;
      tc_fence_after();
      const uint32_t acc_tmem = tmem_base + (uint32_t)(acc * kCoAccCols);
      int u;
      if (which(t, u) == 0)
        epilogue_tile<BN0, 2, EPI>(decode_tile<BN0, 2>(u, prefix, seg, p0.E, nft0), p0, acc_tmem,
                                   quarter, half, lane, st);
      else
        epilogue_tile<kCoBN1, 1, EPI>(decode_dense_tile<kCoBN1, 1>(u, p1.rows_max, nft1, p1.K), p1,
                                      acc_tmem, quarter, half, lane, st);
      tc_fence_before();
      mbar_arrive(B.tempty(acc));
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
    tmem_dealloc(tmem_base, 2 * kCoAccCols);
  }
}


// Tiles on CTA pairs (cta_group::2). A cluster of two CTAs takes each tile together with MMAs of
// M = 256: each CTA holds 128 of the 256 output features of an MMA (its A half) and half of the
// tile's tokens (its B half), so each SM loads half of the token operand instead of all of it:
// for a tile of 256 features x 256 tokens a CTA loads 32 KB per K step (one 128-row weight box
// and 128 token rows), against 48 KB for the same tensor work per SM with one CTA per tile. This
// pays where the tensor pipe is the bound (wide expert tiles of a compute-bound layer, the PR-MoE
// dense MLP); where the expert weights stream from HBM the two SMs in lockstep wait for the
// slower copy of every stage, and one CTA per tile is faster (measured). Problem 0 is the expert
// GEMM (tiles of NB0 x 256 features x BN0 tokens: NB0 MMAs of M = 256 per K step, NB0 weight
// boxes and BN0 / 2 token rows per CTA and stage), problem 1 an optional dense GEMM (256 x 256
// tiles), interleaved as in co_gemm_kernel. Protocol per stage: both CTAs' producers wait their
// own empty barrier and load their halves; the loads count on the leader's full barrier, whose
// expected bytes the leader's producer sets for both; the leader's MMA warp waits it, issues the
// MMAs (K = 16 each) and commits to the empty barrier of both CTAs. Per tile: the leader commits
// to both CTAs' accumulator-full barriers; both CTAs' epilogues read their 128 TMEM lanes and
// arrive on the leader's accumulator-empty barrier (2 x 256 arrivals). Waits stay bounded; both
// CTAs meet at a cluster barrier after set-up and before freeing TMEM and exiting.
constexpr int kPairBN1 = 256;  // dense tile tokens (128 per CTA)
constexpr int kPairAccCols = 256;
template <int BN0, int NB0, int STAGE_BYTES, int STAGES>
struct PairCfg {
  static constexpr int kSmemBytes =
      1024 + STAGES * STAGE_BYTES + kEpiWarps * kStageTileBytes + Cfg<128, 1>::kAuxBytes;
  static_assert(kBM * kBK * 2 + (kPairBN1 / 2) * kBK * 2 <= STAGE_BYTES, "dense pair stage");
  static_assert(NB0 * kBM * kBK * 2 + (BN0 / 2) * kBK * 2 <= STAGE_BYTES, "expert pair stage");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(NB0 * BN0 <= kPairAccCols, "expert accumulators per buffer");
  static_assert(2 * STAGES + 5 <= 64, "barrier area too small");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

template <int EPI, int BN0, int NB0, int STAGE_BYTES, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    co_pair_kernel(const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmX0,
                   const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmX1,
                   const Params p0, const Params p1) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_addr - raw_addr);
  uint8_t* stage_tiles = base + STAGES * STAGE_BYTES;
  uint8_t* aux = stage_tiles + kEpiWarps * kStageTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(aux);
  constexpr int kBarBytes = Cfg<128, 1>::kBarBytes;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(aux + kBarBytes);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(aux + kBarBytes + 4);
  int* prefix = reinterpret_cast<int*>(aux + kBarBytes + 16);
  int* seg = prefix + (MOE_MAX_EXPERTS + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = STAGES;
  const Bars B{smem_u32(bars), S};
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = (int)(blockIdx.x >> 1), n_pairs = (int)(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(B.full(s), 1);
      mbar_init(B.empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(B.tfull(a), 1);
      mbar_init(B.tempty(a), 2 * kEpiWarps * 32);
    }
    mbar_init(B.drain(), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  pdl_wait();
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmW0);
    tma_prefetch_desc(&tmX0);
    tma_prefetch_desc(&tmW1);
    tma_prefetch_desc(&tmX1);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), 2 * kPairAccCols);
    tmem_relinquish_pair();
  }
  const int nft0 = (p0.n_out + NB0 * 2 * kBM - 1) / (NB0 * 2 * kBM);  // expert tiles
  const int nft1 = (p1.n_out + 2 * kBM - 1) / (2 * kBM);  // dense tiles of 256 features
  if (warp == 2) build_tile_list<BN0>(p0, nft0, prefix, seg, lane);
  tc_fence_before();
  __syncwarp();
  cluster_sync();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int n0 = prefix[p0.E];
  const int n1 = nft1 * (int)((p1.rows_max + kPairBN1 - 1) / kPairBN1);
  const int total = n0 + n1;
  const int nkb0 = (p0.K + kBK - 1) / kBK;
  const int nkb1 = (p1.K + kBK - 1) / kBK;
  // problem 0's tile u: (expert, feature tile, token tile) order, or for one segment (the dense
  // MLP run alone) the grouped order of decode_dense_tile
  auto tile0 = [&](int u) -> Tile {
    return p0.offsets != nullptr ? decode_tile<BN0, 2 * NB0>(u, prefix, seg, p0.E, nft0)
                                 : decode_dense_tile<BN0, 2 * NB0>(u, p0.rows_max, nft0, p0.K);
  };
  auto which = [&](int t, int& local) -> int {
    const int c = (int)(((int64_t)t * n0) / total);
    const int c1 = (int)(((int64_t)(t + 1) * n0) / total);
    if (c1 > c) {
      local = c;
      return 0;
    }
    local = t - c;
    return 1;
  };
  constexpr uint32_t kBox = kBM * kBK * 2;  // one 128-row weight box
  // stage layout per CTA: weight boxes at 0 (and kBox), this CTA's token rows after them

  if (warp == 0) {
    if (lane == 0) {
      Ring ring;
      int issued = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += n_pairs) {
        int u;
        const int prob = which(t, u);
        const Tile tl = prob == 0 ? tile0(u)
                                  : decode_dense_tile<kPairBN1, 2>(u, p1.rows_max, nft1, p1.K);
        const Params& p = prob == 0 ? p0 : p1;
        const CUtensorMap* tmW = prob == 0 ? &tmW0 : &tmW1;
        const CUtensorMap* tmX = prob == 0 ? &tmX0 : &tmX1;
        const int n_box = prob == 0 ? NB0 : 1;  // weight boxes per CTA and stage
        const int half_rows = (prob == 0 ? BN0 : kPairBN1) / 2;
        const uint32_t x_off = (uint32_t)n_box * kBox;
        const uint32_t tx = 2u * (x_off + (uint32_t)half_rows * kBK * 2);
        // MMA i of the tile covers features [f0 + 256 i, f0 + 256 i + 256); this CTA holds its
        // rows 128 rank ..
        const int w_row = tl.e * p.n_out + tl.f0 + (int)rank * kBM;
        const int x_row = tl.row0 + (int)rank * half_rows;
        const int nkb = prob == 0 ? nkb0 : nkb1;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(B.empty(ring.stage), ring.phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const uint32_t sa = base_addr + ring.stage * STAGE_BYTES;
          const uint32_t full_leader = cluster_addr(B.full(ring.stage), 0);
          if (leader) mbar_arrive_expect_tx(B.full(ring.stage), tx);
          for (int i = 0; i < n_box; ++i)
            tma_load_2d_pair(sa + i * kBox, tmW, kb * kBK, w_row + i * 2 * kBM, full_leader);
          tma_load_2d_pair(sa + x_off, tmX, kb * kBK, x_row, full_leader);
          ++issued;
          ring.next(S);
        }
      }
      // the leader's full barriers count both CTAs' copies: it waits for the last ones; the
      // other CTA stays resident until then (cluster barrier below)
      if (leader)
        for (int i = max(0, issued - S); i < issued; ++i)
          mbar_wait_drain(B.full(i % S), (uint32_t)((i / S) & 1), p0.status);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      Ring ring;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += n_pairs) {
        if (!mbar_wait_bounded(B.tempty(acc), acc_phase ^ 1u, abort_flag, p0.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kPairAccCols);
        int u;
        const int prob = which(t, u);
        const int nkb = prob == 0 ? nkb0 : nkb1;
        const int n_box = prob == 0 ? NB0 : 1;
        const int n_tok = prob == 0 ? BN0 : kPairBN1;
        const uint32_t idesc = idesc_bf16_f32(2 * kBM, n_tok);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(B.full(ring.stage), ring.phase, abort_flag, p0.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base_addr + ring.stage * STAGE_BYTES;
          const uint64_t bdesc = smem_desc_sw128(sa + (uint32_t)n_box * kBox);
          for (int i = 0; i < n_box; ++i) {
            const uint64_t adesc = smem_desc_sw128(sa + i * kBox);
#pragma unroll
            for (int kk = 0; kk < kBK / kUmmaK; ++kk)
              tc_mma_bf16_pair(d_tmem + (uint32_t)(i * n_tok), adesc + (uint64_t)(2 * kk),
                               bdesc + (uint64_t)(2 * kk), idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit_pair_both(B.empty(ring.stage), cluster_addr(B.empty(ring.stage), 1));
          ring.next(S);
        }
        if (!ok) break;
        tc_commit_pair_both(B.tfull(acc), cluster_addr(B.tfull(acc), 1));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      tc_commit_pair_local(B.drain());
      mbar_wait_drain(B.drain(), 0, p0.status);
    }
  } else {
    const int ew = warp - 2;
    const int quarter = warp & 3;
    const int half = ew >> 2;
    uint8_t* st = stage_tiles + ew * kStageTileBytes;
    const uint32_t tempty0 = cluster_addr(B.tempty(0), 0), tempty1 = cluster_addr(B.tempty(1), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < total; t += n_pairs) {
      if (!mbar_wait_bounded_warp(B.tfull(acc), acc_phase, abort_flag, p0.status)) break;
      tc_fence_after();
      const uint32_t acc_tmem = tmem_base + (uint32_t)(acc * kPairAccCols);
      int u;
      if (which(t, u) == 0) {
        const Tile t4 = tile0(u);
#pragma unroll 1
        for (int i = 0; i < NB0; ++i) {
          Tile tl = t4;
          tl.f0 += i * 2 * kBM + (int)rank * kBM;
          epilogue_tile<BN0, 1, EPI>(tl, p0, acc_tmem + (uint32_t)(i * BN0), quarter,
                                          half, lane, st);
        }
      } else {
        Tile tl = decode_dense_tile<kPairBN1, 2>(u, p1.rows_max, nft1, p1.K);
        tl.f0 += (int)rank * kBM;
        epilogue_tile<kPairBN1, 1, EPI>(tl, p1, acc_tmem, quarter, half, lane, st);
      }
      tc_fence_before();
      mbar_arrive_cluster(acc == 0 ? tempty0 : tempty1);  // the leader's barrier
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync();  // no copy, commit or arrive targets either CTA after this
  pdl_trigger();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 2 * kPairAccCols);
  }
}

// ---------------------------------------------------------------- host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// K-major bf16 matrix [rows, K] (row stride K elements) read in boxes of box_rows x 64.
bool make_kmajor_map(CUtensorMap* m, const void* ptr, int64_t rows, int K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  cuuint32_t estride[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// MN-major bf16 matrix [rows, cols] (row stride cols elements) read in boxes of 64 x 64.
bool make_mn_map(CUtensorMap* m, const void* ptr, int64_t rows, int cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estride[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int EPI, bool A_MN = false, int FT = 1>
cudaError_t launch_one(const CUtensorMap& tmW, const CUtensorMap& tmX, const Params& p,
                       cudaStream_t stream) {
  auto kern = grouped_gemm_kernel<BN, EPI, A_MN, FT>;
  constexpr int smem = Cfg<BN, FT>::kSmemBytes;
  static int attr_done[64] = {0};  // per instantiation and device
  cudaError_t e = ensure_dynamic_smem(kern, smem, attr_done);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, dim3(num_sms()), dim3(kThreads), smem, stream, tmW, tmX, p);
}

template <int BN0, int EPI>
cudaError_t launch_co(const CUtensorMap& tmW0, const CUtensorMap& tmX0, const CUtensorMap& tmW1,
                      const CUtensorMap& tmX1, const CUtensorMap& tmX0_32,
                      const CUtensorMap& tmX0_64, const Params& p0, const Params& p1,
                      cudaStream_t stream) {
  auto kern = co_gemm_kernel<BN0, EPI>;
  static int attr_done[64] = {0};  // per instantiation and device
  cudaError_t e = ensure_dynamic_smem(kern, kCoSmemBytes, attr_done);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, dim3(num_sms()), dim3(kThreads), kCoSmemBytes, stream, tmW0, tmX0,
                       tmW1, tmX1, tmX0_32, tmX0_64, p0, p1);
}

// Launch as clusters of two CTAs (co_pair_kernel), with programmatic dependent launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_pair(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                        cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
  count_launch();
  return e;
}

template <int EPI, int BN0, int NB0, int STAGE_BYTES, int STAGES>
cudaError_t launch_co_pair(const CUtensorMap& tmW0, const CUtensorMap& tmX0,
                           const CUtensorMap& tmW1, const CUtensorMap& tmX1, const Params& p0,
                           const Params& p1, cudaStream_t stream) {
  auto kern = co_pair_kernel<EPI, BN0, NB0, STAGE_BYTES, STAGES>;
  constexpr int smem = PairCfg<BN0, NB0, STAGE_BYTES, STAGES>::kSmemBytes;
  static int attr_done[64] = {0};  // per instantiation and device
  cudaError_t e = ensure_dynamic_smem(kern, smem, attr_done);
  if (e != cudaSuccess) return e;
  const int grid = num_sms() & ~1;
  return launch_pair(kern, dim3(grid), dim3(kThreads), smem, stream, tmW0, tmX0, tmW1, tmX1, p0,
                     p1);
}

}  // namespace

bool make_bf16_map_2d(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int box_cols,
                      int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estride[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Co-scheduled layers with one token tile per expert: each expert weight row is read once per
// layer, and the evict-first hint keeps that stream from pushing the dense MLP's reused operands
// out of L2. Measured (launch durations, gpt1.3b-prmoe128): layer 1 907 -> 868 us, layer 2
// 842 -> 856 us, expert-only layers 1-2% slower; so it is given to the first co-scheduled layer
// only. MOE_W_EVICT_FIRST=0 turns it off; read at every call.
static int weights_read_once(int64_t capacity_hint, int BN) {
  const char* v = std::getenv("MOE_W_EVICT_FIRST");
  if (v != nullptr && v[0] == '0') return 0;
  return capacity_hint <= BN ? 1 : 0;
}

static int pick_token_tile(int64_t capacity_hint) {
  if (capacity_hint <= 16) return 16;
  if (capacity_hint <= 32) return 32;
  if (capacity_hint <= 64) return 64;
  if (capacity_hint <= 128) return 128;
  return 256;
}

#ifndef MOE_GG_FT
#define MOE_GG_FT 2
#endif

// Fraction of the last wave's CTA slots that hold a tile (tiles over persistent CTAs).
static double wave_efficiency(int64_t tiles) {
  const int64_t s = num_sms();
  if (tiles <= 0) return 1.0;
  return (double)tiles / (double)(((tiles + s - 1) / s) * s);
}

// Two feature tiles per CTA tile (each token tile read from L2 half as often) when the layer has
// more than one feature tile, TMEM holds them, and halving the tile count does not leave the
// last wave of the persistent grid emptier (estimated from E and the capacity hint).
template <int EPI, bool A_MN = false>
cudaError_t launch_bn(int BN, const CUtensorMap& tmW, const CUtensorMap& tmX, const Params& p,
                      cudaStream_t stream, int64_t capacity_hint) {
  bool two = MOE_GG_FT == 2 && p.n_out > kBM && BN <= 128;
  if (two) {
    const int64_t rows = std::min<int64_t>(std::max<int64_t>(capacity_hint, 1), p.rows_max);
    const int64_t tok_tiles = (int64_t)p.E * ((rows + BN - 1) / BN);
    const int64_t t1 = tok_tiles * ((p.n_out + kBM - 1) / kBM);
    const int64_t t2 = tok_tiles * ((p.n_out + 2 * kBM - 1) / (2 * kBM));
    two = wave_efficiency(t2) >= wave_efficiency(t1) - 0.02;
  }
  switch (BN) {
    case 16: return two ? launch_one<16, EPI, A_MN, 2>(tmW, tmX, p, stream)
                        : launch_one<16, EPI, A_MN, 1>(tmW, tmX, p, stream);
    case 32: return two ? launch_one<32, EPI, A_MN, 2>(tmW, tmX, p, stream)
                        : launch_one<32, EPI, A_MN, 1>(tmW, tmX, p, stream);
    case 64: return two ? launch_one<64, EPI, A_MN, 2>(tmW, tmX, p, stream)
                        : launch_one<64, EPI, A_MN, 1>(tmW, tmX, p, stream);
    case 128: return two ? launch_one<128, EPI, A_MN, 2>(tmW, tmX, p, stream)
                         : launch_one<128, EPI, A_MN, 1>(tmW, tmX, p, stream);
    default: return launch_one<256, EPI, A_MN, 1>(tmW, tmX, p, stream);
  }
}

cudaError_t enqueue_grouped_gemm_bf16(const void* x, const int32_t* offsets, int E,
                                      int64_t rows_max, int K, int N, const void* w,
                                      const void* bias, bool gelu, void* out,
                                      int64_t capacity_hint, int* status, cudaStream_t stream) {
  if (rows_max == 0) return cudaSuccess;
  const int BN = pick_token_tile(capacity_hint);
  CUtensorMap tmW, tmX;
  if (!make_kmajor_map(&tmW, w, (int64_t)E * N, K, kBM) || !make_kmajor_map(&tmX, x, rows_max, K, BN))
    return cudaErrorInvalidValue;
  Params p{offsets, E, N, K, rows_max, bias, out, status, CombineArgs{}, nullptr, nullptr};
  if (BN == 256 && pair_mma_enabled() && num_sms() >= 2) {
    // wide (compute-bound) expert tiles on CTA pairs: 256 features x 256 tokens, 128 token rows
    // per CTA; no second problem (its maps point at this one's operands and it has no tiles)
    CUtensorMap tmXh;
    if (!make_kmajor_map(&tmXh, x, rows_max, K, 128)) return cudaErrorInvalidValue;
    Params none{nullptr, 1, N, K, 0, nullptr, nullptr, status, CombineArgs{}, nullptr, nullptr};
    return gelu ? launch_co_pair<kEpiGeluBf16, 256, 1, 32 * 1024, 6>(tmW, tmXh, tmW, tmXh, p, none,
                                                                     stream)
                : launch_co_pair<kEpiF32, 256, 1, 32 * 1024, 6>(tmW, tmXh, tmW, tmXh, p, none,
                                                                stream);
  }
  return gelu ? launch_bn<kEpiGeluBf16>(BN, tmW, tmX, p, stream, capacity_hint)
              : launch_bn<kEpiF32>(BN, tmW, tmX, p, stream, capacity_hint);
}

cudaError_t enqueue_grouped_gemm_bf16_train(const void* x, const int32_t* offsets, int E,
                                            int64_t rows_max, int K, int N, const void* w,
                                            const void* bias, void* h_out, void* g_out,
                                            int64_t capacity_hint, int* status,
                                            cudaStream_t stream) {
  if (rows_max == 0) return cudaSuccess;
  const int BN = pick_token_tile(capacity_hint);
  CUtensorMap tmW, tmX;
  if (!make_kmajor_map(&tmW, w, (int64_t)E * N, K, kBM) || !make_kmajor_map(&tmX, x, rows_max, K, BN))
    return cudaErrorInvalidValue;
  Params p{offsets, E, N, K, rows_max, bias, h_out, status, CombineArgs{}, nullptr,
           (uint16_t*)g_out};
  return launch_bn<kEpiGeluBf16Train>(BN, tmW, tmX, p, stream, capacity_hint);
}

cudaError_t enqueue_grouped_gemm_dgrad_bf16(const void* dy, const int32_t* offsets, int E,
                                            int64_t rows_max, int K, int N, const void* w_t,
                                            const void* g_in, void* out, int64_t capacity_hint,
                                            int* status, cudaStream_t stream) {
  if (rows_max == 0) return cudaSuccess;
  const int BN = pick_token_tile(capacity_hint);
  CUtensorMap tmW, tmX;
  if (!make_mn_map(&tmW, w_t, (int64_t)E * K, N) || !make_kmajor_map(&tmX, dy, rows_max, K, BN))
    return cudaErrorInvalidValue;
  Params p{offsets, E, N, K, rows_max, nullptr, out, status, CombineArgs{},
           (const uint16_t*)g_in, nullptr};
  return g_in != nullptr ? launch_bn<kEpiGeluGradBf16, true>(BN, tmW, tmX, p, stream, capacity_hint)
                         : launch_bn<kEpiF32, true>(BN, tmW, tmX, p, stream, capacity_hint);
}

cudaError_t enqueue_gemm2_combine(const void* h, const int32_t* offsets, int E, int64_t rows_max,
                                  int K, int N, const void* w, const void* bias,
                                  const FusedCombine& fc, int64_t capacity_hint, int* status,
                                  cudaStream_t stream) {
  if (rows_max == 0) return cudaSuccess;
  const int BN = pick_token_tile(capacity_hint);
  CUtensorMap tmW, tmX;
  if (!make_kmajor_map(&tmW, w, (int64_t)E * N, K, kBM) || !make_kmajor_map(&tmX, h, rows_max, K, BN))
    return cudaErrorInvalidValue;
  CombineArgs c{fc.row_token, fc.slot, fc.ids, fc.offsets, fc.gates, fc.y,
                (const uint16_t*)fc.residual, fc.out, fc.out_bf16 ? 1 : 0, fc.k, fc.E_experts,
                fc.rows_y};
  Params p{offsets, E, N, K, rows_max, bias, nullptr, status, c, nullptr, nullptr};
  return fc.dense ? launch_bn<kEpiCombineDense>(BN, tmW, tmX, p, stream, capacity_hint)
                  : launch_bn<kEpiCombineExpert>(BN, tmW, tmX, p, stream, capacity_hint);
}

bool co_gemm_supported(int64_t capacity_hint) {
  return pick_token_tile(capacity_hint) <= 128;  // two expert accumulators fit one 256-column buffer
}

cudaError_t enqueue_co_gemm_bf16(const void* xp, const int32_t* offsets, int E, int64_t rows_max,
                                 const void* w, const void* bias, void* out, int64_t capacity_hint,
                                 const void* x_dense, int64_t T, const void* w_dense,
                                 const void* bias_dense, void* out_dense, int K, int N, bool gelu,
                                 int* status, cudaStream_t stream) {
  if (T == 0 && rows_max == 0) return cudaSuccess;
  const int BN0 = pick_token_tile(capacity_hint);
  if (BN0 > 128) return cudaErrorInvalidValue;
  CUtensorMap tmW0, tmX0, tmW1, tmX1;
  // an empty expert problem still needs valid maps: point them at the dense operands (no tile
  // of problem 0 exists, so nothing is loaded through them)
  const bool no_rows = rows_max == 0;
  CUtensorMap tmX0_32, tmX0_64;  // shorter token boxes for expert tiles of few rows
  const void* x0 = no_rows ? x_dense : xp;
  const int64_t rows0 = no_rows ? T : rows_max;
  if (!make_kmajor_map(&tmW0, w, (int64_t)E * N, K, kBM) ||
      !make_kmajor_map(&tmX0, x0, rows0, K, BN0) ||
      !make_kmajor_map(&tmX0_32, x0, rows0, K, BN0 < 32 ? BN0 : 32) ||
      !make_kmajor_map(&tmX0_64, x0, rows0, K, BN0 < 64 ? BN0 : 64) ||
      !make_kmajor_map(&tmW1, w_dense, N, K, kBM) ||
      !make_kmajor_map(&tmX1, x_dense, T, K, kCoBN1))
    return cudaErrorInvalidValue;
  Params p0{offsets, E, N, K, rows_max, bias, out, status, CombineArgs{}, nullptr, nullptr};
  p0.w_read_once = gelu ? weights_read_once(capacity_hint, BN0) : 0;  // layer 1 only (measured)
  Params p1{nullptr, 1, N, K, T, bias_dense, out_dense, status, CombineArgs{}, nullptr, nullptr};
  auto go = [&](auto tag) -> cudaError_t {
    constexpr int EPI = decltype(tag)::value;
    switch (BN0) {
      case 16: return launch_co<16, EPI>(tmW0, tmX0, tmW1, tmX1, tmX0_32, tmX0_64, p0, p1, stream);
      case 32: return launch_co<32, EPI>(tmW0, tmX0, tmW1, tmX1, tmX0_32, tmX0_64, p0, p1, stream);
      case 64: return launch_co<64, EPI>(tmW0, tmX0, tmW1, tmX1, tmX0_32, tmX0_64, p0, p1, stream);
      default: return launch_co<128, EPI>(tmW0, tmX0, tmW1, tmX1, tmX0_32, tmX0_64, p0, p1, stream);
    }
  };
  return gelu ? go(std::integral_constant<int, kEpiGeluBf16>{})
              : go(std::integral_constant<int, kEpiF32>{});
}

cudaError_t enqueue_selftest_bounded_wait(void* scratch, uint64_t wait_limit_ns, int* status,
                                         cudaStream_t stream) {
  // one expert of 128 features x 64 K and one 16-row token tile, maps over the scratch (nothing
  // is copied: the TMA role is told to issue no copy)
  uint8_t* b = static_cast<uint8_t*>(scratch);
  CUtensorMap tmW, tmX;
  if (!make_kmajor_map(&tmW, b, kBM, kBK, kBM) || !make_kmajor_map(&tmX, b, 16, kBK, 16))
    return cudaErrorInvalidValue;
  Params p{nullptr, 1, kBM, kBK, 16, nullptr, b, status, CombineArgs{}, nullptr, nullptr};
  p.selftest_no_copies = 1;
  p.wait_limit_ns = wait_limit_ns;
  return launch_one<16, kEpiF32, false, 1>(tmW, tmX, p, stream);
}

cudaError_t enqueue_expert_ffn_bf16(const void* x_packed, const int32_t* offsets, int E,
                                    int64_t rows_max, int d, int d_ff, const void* w1,
                                    const void* b1, const void* w2, const void* b2, void* h_packed,
                                    float* y_packed, int64_t capacity_hint, int* status,
                                    cudaStream_t stream) {
  cudaError_t e = enqueue_grouped_gemm_bf16(x_packed, offsets, E, rows_max, d, d_ff, w1, b1, true,
                                            h_packed, capacity_hint, status, stream);
  if (e != cudaSuccess) return e;
  return enqueue_grouped_gemm_bf16(h_packed, offsets, E, rows_max, d_ff, d, w2, b2, false, y_packed,
                                   capacity_hint, status, stream);
}

}  // namespace moe
