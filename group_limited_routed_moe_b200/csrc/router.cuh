// router.cuh -- the router projection that feeds step 1:
//   logits[t][e] = sum_k x[t][k] W_router[k][e]   (bf16 in, fp32 accumulate, fp32 out)
// The pages name the group-limited routing kernel of the CUDA path ("Ling-3.0-
// tiny on a Qualcomm board", TensorFold issue #1247, "What it does not cover",
// first bullet); the projection of the hidden state onto the 128 experts is the
// step right before it.
//
// A tcgen05 GEMM with the weights as the 128-row operand: M = the 128 experts
// (W_router packed K-major, [128][1536]), N = 64 tokens per tile, K = 1536.  A
// tile's accumulator holds expert e in TMEM lane e, so each epilogue warp
// stores one token's 32 consecutive logits per instruction (128 contiguous
// bytes).  T = 8189 gives 128 tiles, one per SM; T <= 64 is one tile, whose
// token rows past T are zero-filled by the TMA.  Persistent CTAs walk the tiles
// round-robin (all tiles cost the same).  Warp roles: 0-3 epilogue, 4 TMA, 5-6
// MMA; 8 stages of (16 KB of W_router + 8 KB of x); 2 x 4 x 64 TMEM columns.
// Every wait is a bounded mbarrier wait.
#pragma once
#include "common.cuh"

namespace moe {
namespace router {

constexpr int BM = 128;  // experts (MMA M)
constexpr int BN = 64;   // tokens per tile (MMA N)
constexpr int BK = 64;
constexpr int KB = kH / BK;  // 24 k-blocks
constexpr int STAGES = 8;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_BYTES = BN * BK * 2;  // 8 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TILE_BYTES = STAGES * STAGE_BYTES;
// The 4 K steps of a stage go to 4 accumulator chains (summed in the
// epilogue as (c0 + c1) + (c2 + c3)), so consecutive MMAs do not wait on each
// other's accumulator: 2 buffers x 4 chains x 64 columns.
constexpr int NCH = 4;
constexpr int ACC_COLS = NCH * BN;
constexpr int TMEM_COLS = 2 * ACC_COLS;
// Two MMA-issuing warps: issuer i issues the stage's K steps of chains i and
// i + 2 (one thread's tcgen05.mma instructions follow one another at a few
// hundred cycles each, and a tile's 96 MMAs would otherwise run one by one).
constexpr int NISS = 2;
static_assert(NCH % NISS == 0, "each chain belongs to one issuer");
constexpr int THREADS = 32 * (5 + NISS);
constexpr int TMA_WARP = 4, MMA_WARP = 5;  // issuers: warps 5 .. 5 + NISS - 1
constexpr uint32_t IDESC = idesc_f32acc(BM, BN, kFmtBF16);

struct Tail {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain[NISS];
  uint32_t tmem_base;
  int abort_flag;
};
constexpr int TAIL_BYTES = (static_cast<int>(sizeof(Tail)) + 127) / 128 * 128;
constexpr int SMEM_BYTES = TILE_BYTES + TAIL_BYTES + 1024;

// packed[e][k] = w[k][e]: W_router [1536][128] -> K-major [128][1536].
__global__ void __launch_bounds__(256)
    router_pack_kernel(const uint16_t* __restrict__ w, uint16_t* __restrict__ packed) {
  __shared__ uint16_t tile[32][33];
  const int e0 = blockIdx.x * 32, k0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
#pragma unroll
  for (int i = 0; i < 32; i += 8) tile[ty + i][tx] = w[(k0 + ty + i) * kE + e0 + tx];
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 32; i += 8) packed[(e0 + ty + i) * kH + k0 + tx] = tile[tx][ty + i];
}

__global__ void __launch_bounds__(THREADS, 1)
    router_kernel(const __grid_constant__ CUtensorMap tmap_w,  // packed W_router, box 64 x 128
                  const __grid_constant__ CUtensorMap tmap_x,  // x [T][1536], box 64 x 64
                  int64_t T, float* __restrict__ logits, uint64_t timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Tail* S = reinterpret_cast<Tail*>(smem + TILE_BYTES);
  volatile int* abort_flag = &S->abort_flag;
  auto sA = [&](int s) { return smem + s * STAGE_BYTES; };
  auto sB = [&](int s) { return smem + s * STAGE_BYTES + A_BYTES; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&S->full[s], 1);
      mbar_init(&S->empty[s], NISS);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&S->tfull[a], NISS);
      mbar_init(&S->tempty[a], 4);
    }
    for (int i = 0; i < NISS; ++i) mbar_init(&S->drain[i], 1);
    S->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == TMA_WARP && lane == 0) {
    tma_prefetch_desc(&tmap_w);
    tma_prefetch_desc(&tmap_x);
  }
  if (warp == MMA_WARP) tmem_alloc(&S->tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();  // x may come from the preceding kernel

  const uint32_t tmem_base = S->tmem_base;
  const int ntiles = static_cast<int>((T + BN - 1) / BN);

  if (warp == TMA_WARP) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&S->empty[s], ph ^ 1, abort_flag, timeout_ns, kSiteFfnEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&S->full[s], A_BYTES + B_BYTES);
          tma_load_2d(smem_u32(sA(s)), &tmap_w, kb * BK, 0, &S->full[s]);
          tma_load_2d(smem_u32(sB(s)), &tmap_x, kb * BK, tile * BN, &S->full[s]);
        }
      }
      if (!ok) {
        for (int i = max(0, it - STAGES); i < it; ++i)
          mbar_wait_drain(&S->full[i % STAGES], (i / STAGES) & 1, kSiteFfnFull);
      }
    }
  } else if (warp >= MMA_WARP && warp < MMA_WARP + NISS) {
    const int iss = warp - MMA_WARP;
    if (lane == 0) {
      int it = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++tc) {
        const int a = tc & 1;
        const uint32_t use = tc >> 1;
        if (!mbar_wait(&S->tempty[a], (use & 1) ^ 1, abort_flag, timeout_ns, kSiteFfnTmemEmpty)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + a * ACC_COLS;  // chain k at d + k * BN
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&S->full[s], ph, abort_flag, timeout_ns, kSiteFfnFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc_k128(smem_u32(sA(s)));
          const uint64_t bdesc = smem_desc_k128(smem_u32(sB(s)));
          static_assert(BK / 16 == NCH, "one K step of a stage per chain");
#pragma unroll
          for (int k = iss; k < BK / 16; k += NISS)
            umma_f16(d + k * BN, adesc + 2 * k, bdesc + 2 * k, IDESC, kb != 0 ? 1u : 0u);
          umma_commit(&S->empty[s]);
        }
        if (ok) umma_commit(&S->tfull[a]);
      }
      umma_commit(&S->drain[iss]);
      mbar_wait_drain(&S->drain[iss], 0, kSiteFfnDrain);
    }
  } else if (warp < 4) {
    // ------------------------------------------------ epilogue: lane = expert 32w + lane
    int tc = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tc) {
      const int a = tc & 1;
      const uint32_t use = tc >> 1;
      if (!mbar_wait(&S->tfull[a], use & 1, abort_flag, timeout_ns, kSiteFfnTmemFull)) break;
      tc_fence_after();
      const int64_t t0 = static_cast<int64_t>(tile) * BN;
      float* dst = logits + t0 * kE + warp * 32 + lane;
#pragma unroll 1
      for (int h = 0; h < BN / 32; ++h) {
        uint32_t v[32], u[32], w2[32];
        const uint32_t acc =
            tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + a * ACC_COLS + h * 32;
        tmem_ld_2x32(acc, acc + BN, v, u);
#pragma unroll
        for (int t = 0; t < 32; ++t) v[t] = __float_as_uint(__uint_as_float(v[t]) + __uint_as_float(u[t]));
        tmem_ld_2x32(acc + 2 * BN, acc + 3 * BN, u, w2);
#pragma unroll
        for (int t = 0; t < 32; ++t)
          v[t] = __float_as_uint(__uint_as_float(v[t]) + (__uint_as_float(u[t]) + __uint_as_float(w2[t])));
#pragma unroll
        for (int t = 0; t < 32; ++t)
          if (t0 + h * 32 + t < T) dst[(h * 32 + t) * kE] = __uint_as_float(v[t]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->tempty[a]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace router
}  // namespace moe
