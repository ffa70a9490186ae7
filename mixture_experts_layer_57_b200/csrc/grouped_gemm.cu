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
  static constexpr int kTmemCols = (2 * FT * BN) < 32 ? 32 : (2 * FT * BN);
  static_assert(2 * FT * BN <= 512, "two buffers of FT accumulators must fit TMEM");
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
  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[S + s]); };
  auto tfull_bar = [&](int a) { return smem_u32(&bars[2 * S + a]); };
  auto tempty_bar = [&](int a) { return smem_u32(&bars[2 * S + 2 + a]); };
  const uint32_t drain_bar = smem_u32(&bars[2 * S + 4]);

  // ------------------------------------------------------------ prologue
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), kEpiWarps * 32);
    }
    mbar_init(drain_bar, 1);
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
  if (warp == 2) {
    // Tile list: prefix[e] = first tile of expert e; validates the device offsets.
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total_tiles = prefix[p.E];
  const int n_kb = (p.K + kBK - 1) / kBK;

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
        const Tile tl = decode_tile<BN, FT>(t, prefix, seg, p.E, n_ftiles);
        const int w_row = tl.e * p.n_out + tl.f0;
        bool ok = true;
        for (int kb = 0; kb < n_kb; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const uint32_t sa = base_addr + stage * C::kStageBytes;
          mbar_arrive_expect_tx(full_bar(stage), C::kStageBytes);
#pragma unroll
          for (int i = 0; i < FT; ++i) {
            const uint32_t sai = sa + i * (kBM * kBK * 2);
            if constexpr (A_MN) {
              const int k_row = tl.e * p.K + kb * kBK;
              tma_load_2d(sai, &tmW, tl.f0 + i * kBM, k_row, full_bar(stage));
              tma_load_2d(sai + kBM * kBK, &tmW, tl.f0 + i * kBM + 64, k_row, full_bar(stage));
            } else {
              // rows past this expert's n_out (odd tile count) belong to the next expert or are
              // out of range; the epilogue masks those features
              tma_load_2d(sai, &tmW, kb * kBK, w_row + i * kBM, full_bar(stage));
            }
          }
          tma_load_2d(sa + C::kABytes, &tmX, kb * kBK, tl.row0, full_bar(stage));
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      // drain: the last min(issued, S) loads may still be landing
      for (int i = max(0, issued - S); i < issued; ++i)
        mbar_wait_drain(full_bar(i % S), (uint32_t)((i / S) & 1), p.status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const Tile tl = decode_tile<BN, FT>(t, prefix, seg, p.E, n_ftiles);
        if (!mbar_wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * FT * BN);
        const int n_mma = max(16, (tl.n_valid + 15) & ~15);
        const uint32_t idesc = idesc_bf16_f32_major(kBM, n_mma, A_MN, false);
        for (int kb = 0; kb < n_kb; ++kb) {
          if (!mbar_wait_bounded(full_bar(stage), phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base_addr + stage * C::kStageBytes;
          const uint64_t bdesc = smem_desc_sw128(sa + C::kABytes);
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
      // drain every MMA this thread issued before TMEM is released
      tc_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0, p.status);
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
      const Tile tl = decode_tile<BN, FT>(t, prefix, seg, p.E, n_ftiles);
      if (!mbar_wait_bounded_warp(tfull_bar(acc), acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
#pragma unroll 1
      for (int fi = 0; fi < FT; ++fi) {
      const int fw = tl.f0 + fi * kBM + quarter * 32;  // first feature of this warp
      const int f = fw + lane;
      const bool f_ok = f < p.n_out;
      const float bv = (p.bias != nullptr && f_ok)
                           ? bf16_to_f32(reinterpret_cast<const uint16_t*>(p.bias)[(int64_t)tl.e * p.n_out + f])
                           : 0.0f;
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) +
                             (uint32_t)(acc * FT * BN + fi * BN);
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
      }  // feature tiles
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
      if (++acc == 2) {
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
