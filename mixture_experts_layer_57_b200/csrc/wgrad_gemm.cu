// Weight-gradient GEMM on sm_100a tensor cores (tcgen05 + TMEM + TMA), for the backward pass of
// the expert layers: for every expert e and its packed rows r in [offsets[e], offsets[e+1]),
//     dW[e][m][n] = sum_r A[r][m] * B[r][n]
// (dW2[e] = dY^T h with A = dY, B = h; dW1[e] = dZ^T x with A = dZ, B = x_packed). The
// contraction runs over the expert's token rows, so both operands are read MN-major straight
// from the token-major activations: TMA boxes of 64 (M or N, contiguous) x 64 (rows) with
// 128-byte swizzle, no transposed copies. The rows of a segment are ragged: the last K block of
// an expert holds rows of the next expert (or out-of-range zeros), so the MMA warp clears the
// rows past the segment, up to the next multiple of 16, in shared memory and issues only the
// MMAs (K = 16 each) that cover the segment.
//
// Schedule: persistent CTAs walk output tiles (expert, 128-row M tile, BN-column N tile).
// Roles per CTA: warp 0 TMA producer (STAGES-deep ring), warp 1 TMEM allocation and the MMA
// issue (one thread) with the tail clearing (whole warp), warps 2..9 the epilogue: tcgen05.ld of
// 32 accumulator columns for the warp's 32 rows, staged in shared memory, then stored as whole
// 128-byte row segments (8 lanes per row, four rows per instruction).
// Two accumulators alternate so the epilogue of one tile overlaps the MMAs of the next. Every
// wait is bounded (about 2 s) as in the forward GEMM.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;          // rows per stage
constexpr int kUmmaK = 16;
constexpr int kThreads = 320;
constexpr int kEpiWarps = 8;
constexpr int kBoxBytes = 64 * kBK * 2;  // one 64 x 64 bf16 box
constexpr int kEpiRowFloats = 36;        // 32 columns + 4 pad (16-byte aligned rows)

template <int BN>
struct WCfg {
  static constexpr int kABytes = kBM * kBK * 2;  // two boxes
  static constexpr int kBBytes = BN * kBK * 2;   // BN / 64 boxes
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kEpiStageBytes = kEpiWarps * 32 * kEpiRowFloats * 4;
  static constexpr int kStagesFit = (200 * 1024 - kEpiStageBytes) / kStageBytes;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kBarBytes = 8 * 32;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kEpiStageBytes + kBarBytes + 16;
  static_assert(kStageBytes % 1024 == 0, "stage tiles must stay 1024-byte aligned");
  static_assert(2 * kStages + 5 <= 32, "barrier area too small");
  static_assert(kTmemCols <= 512, "two accumulators must fit TMEM");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

struct WParams {
  const int32_t* offsets;  // [E+1] or nullptr (one segment of rows_max rows)
  int E, M, N;
  int64_t rows_max;
  float* out;              // [splits][E][M][N]
  int* status;
  int splits;              // split-K: each split sums a contiguous range of the K blocks
  int64_t b_period;        // > 0: row r of A pairs with row r % b_period of B
};

__device__ __forceinline__ void seg_of(const WParams& p, int e, int* a, int* b) {
  if (p.offsets == nullptr) {
    *a = 0;
    *b = (int)p.rows_max;
    return;
  }
  *a = p.offsets[e];
  *b = p.offsets[e + 1];
  if (*a < 0 || *b < *a || (int64_t)*b > p.rows_max) {  // invalid: treated as empty
    *b = *a = 0;
  }
}

__device__ __forceinline__ void mbar_wait_drain_w(uint32_t bar, uint32_t parity, int* status) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      set_device_error(status, MOE_DEVERR_TIMEOUT);
      return;
    }
  }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    wgrad_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const WParams p) {
  using C = WCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_addr - raw_addr);
  float* epi_stage = reinterpret_cast<float*>(base + C::kStages * C::kStageBytes);
  uint8_t* aux = base + C::kStages * C::kStageBytes + C::kEpiStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(aux);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(aux + C::kBarBytes);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(aux + C::kBarBytes + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
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
      mbar_init(tempty_bar(a), kEpiWarps * 32);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  pdl_wait();
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int n_mt = (p.M + kBM - 1) / kBM;
  const int n_nt = (p.N + BN - 1) / BN;
  const int per_split = p.E * n_mt * n_nt;
  const int total = per_split * p.splits;
  // tile t -> split s, expert e, output tile (m0, n0), and the split's K blocks [kb0, kb1)
  auto decode = [&](int t, int* s, int* e, int* m0, int* n0, int* a, int* kb0, int* kb1) {
    *s = t / per_split;
    const int u = t - *s * per_split;
    *e = u / (n_mt * n_nt);
    const int rem = u - *e * n_mt * n_nt;
    *m0 = (rem / n_nt) * kBM;
    *n0 = (rem % n_nt) * BN;
    int b;
    seg_of(p, *e, a, &b);
    const int n_kb = (b - *a + kBK - 1) / kBK;
    const int per = (n_kb + p.splits - 1) / p.splits;
    *kb0 = min(n_kb, *s * per);
    *kb1 = min(n_kb, *kb0 + per);
    return b;
  };

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        int s, e, m0, n0, a, kb0, kb1;
        decode(t, &s, &e, &m0, &n0, &a, &kb0, &kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const uint32_t sa = base_addr + stage * C::kStageBytes;
          const int row = a + kb * kBK;
          const int brow = p.b_period > 0 ? (int)(row % p.b_period) : row;
          mbar_arrive_expect_tx(full_bar(stage), C::kStageBytes);
          tma_load_2d(sa, &tmA, m0, row, full_bar(stage));
          tma_load_2d(sa + kBoxBytes, &tmA, m0 + 64, row, full_bar(stage));
#pragma unroll
          for (int j = 0; j < BN / 64; ++j)
            tma_load_2d(sa + C::kABytes + j * kBoxBytes, &tmB, n0 + 64 * j, brow, full_bar(stage));
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      for (int i = max(0, issued - S); i < issued; ++i)
        mbar_wait_drain_w(full_bar(i % S), (uint32_t)((i / S) & 1), p.status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer (whole warp)
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    const uint32_t idesc = idesc_bf16_f32_major(kBM, BN, true, true);
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      int s, e, m0, n0, a, kb0, kb1;
      const int b = decode(t, &s, &e, &m0, &n0, &a, &kb0, &kb1);
      const int rows = b - a;
      if (!mbar_wait_bounded_warp(tempty_bar(acc), acc_phase ^ 1u, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_bounded_warp(full_bar(stage), phase, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = base_addr + stage * C::kStageBytes;
        uint8_t* sp = base + stage * C::kStageBytes;
        const int valid = min(kBK, rows - kb * kBK);
        const int kend = (valid + kUmmaK - 1) & ~(kUmmaK - 1);
        if (valid < kend) {
          // rows [valid, kend) of every box belong to the next segment: clear them (a row of an
          // MN-major box is 128 contiguous bytes; the swizzle permutes 16-byte chunks inside it)
          const int nbox = 2 + BN / 64;
          const int chunks = (kend - valid) * 8;  // 16-byte chunks per box
          for (int i = lane; i < nbox * chunks; i += 32) {
            const int bx = i / chunks, c = i - bx * chunks;
            *reinterpret_cast<uint4*>(sp + bx * kBoxBytes + valid * 128 + c * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
          const uint64_t adesc = smem_desc_sw128_mn(sa);
          const uint64_t bdesc = smem_desc_sw128_mn(sa + C::kABytes);
          for (int kk = 0; kk < kend / kUmmaK; ++kk)
            tc_mma_bf16(d_tmem, adesc + (uint64_t)(kk * (kMnKStepBytes >> 4)),
                        bdesc + (uint64_t)(kk * (kMnKStepBytes >> 4)), idesc,
                        (kb > kb0 || kk > 0) ? 1u : 0u);
          tc_commit(empty_bar(stage));
        }
        __syncwarp();
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(tfull_bar(acc));
      __syncwarp();
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) {
      tc_commit(drain_bar);
      mbar_wait_drain_w(drain_bar, 0, p.status);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue (warps 2..9)
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    float* st = epi_stage + (warp - 2) * 32 * kEpiRowFloats;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      int s, e, m0, n0, a, kb0, kb1;
      decode(t, &s, &e, &m0, &n0, &a, &kb0, &kb1);
      const bool empty = kb1 == kb0;  // no K block in this split: the tile is zero
      float* out_s = p.out + (int64_t)s * p.E * p.M * p.N;
      if (!mbar_wait_bounded_warp(tfull_bar(acc), acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      const int mw = m0 + quarter * 32;  // first row of this warp
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
      for (int c0 = half * 32; c0 < BN; c0 += 64) {
        uint32_t r0[16], r1[16];
        tmem_ld_32x32b_x16(taddr + (uint32_t)c0, r0);
        tmem_ld_32x32b_x16(taddr + (uint32_t)c0 + 16, r1);
        tmem_ld_wait();
        // lane = row: stage the row's 32 columns
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t* r = q < 4 ? r0 : r1;
          const int o = 4 * (q & 3);
          *reinterpret_cast<float4*>(st + lane * kEpiRowFloats + 4 * q) =
              empty ? make_float4(0.f, 0.f, 0.f, 0.f)
                    : make_float4(__uint_as_float(r[o]), __uint_as_float(r[o + 1]),
                                  __uint_as_float(r[o + 2]), __uint_as_float(r[o + 3]));
        }
        __syncwarp();
        // 8 lanes per row, 16 bytes each: every instruction writes four whole 128-byte segments
        const int sub = lane & 7;
        const int n = n0 + c0 + 4 * sub;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = 4 * i + (lane >> 3);
          const int m = mw + rr;
          if (m < p.M && n < p.N)
            *reinterpret_cast<float4*>(out_s + ((int64_t)e * p.M + m) * p.N + n) =
                *reinterpret_cast<const float4*>(st + rr * kEpiRowFloats + 4 * sub);
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

template <int BN>
cudaError_t launch_w(const CUtensorMap& tmA, const CUtensorMap& tmB, const WParams& p,
                     cudaStream_t stream) {
  auto kern = wgrad_kernel<BN>;
  static int attr_done[64] = {0};  // per device
  cudaError_t e = ensure_dynamic_smem(kern, WCfg<BN>::kSmemBytes, attr_done);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, dim3(num_sms()), dim3(kThreads), WCfg<BN>::kSmemBytes, stream, tmA,
                       tmB, p);
}

}  // namespace

cudaError_t enqueue_wgrad_bf16(const void* a, const void* b, const int32_t* offsets, int E,
                               int64_t rows_max, int M, int N, float* out, int* status,
                               cudaStream_t stream, int splits, int64_t b_period,
                               int64_t b_rows) {
  if (E <= 0 || M <= 0 || N <= 0) return cudaSuccess;
  if (splits < 1) splits = 1;
  if (rows_max == 0)  // every expert is empty
    return cudaMemsetAsync(out, 0, sizeof(float) * (size_t)splits * E * M * N, stream);
  const int64_t period = b_period > 0 ? b_period : 0;
  if (period > 0 && (period % kBK != 0 || b_rows <= 0 || b_rows > period))
    return cudaErrorInvalidValue;
  CUtensorMap tmA, tmB;
  // with a period, b's rows past b_rows (up to the period) read as zero
  if (!make_bf16_map_2d(&tmA, a, rows_max, M, 64, kBK) ||
      !make_bf16_map_2d(&tmB, b, period > 0 ? b_rows : rows_max, N, 64, kBK))
    return cudaErrorInvalidValue;
  WParams p{offsets, E, M, N, rows_max, out, status, splits, period};
  if (N <= 64) return launch_w<64>(tmA, tmB, p, stream);
  if (N <= 128) return launch_w<128>(tmA, tmB, p, stream);
  return launch_w<256>(tmA, tmB, p, stream);
}

}  // namespace moe
