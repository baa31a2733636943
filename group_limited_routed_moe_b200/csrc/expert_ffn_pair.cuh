// expert_ffn_pair.cuh -- step 3 for large batches: the two grouped GEMMs of
// expert_ffn.cuh on CTA pairs (tcgen05 cta_group::2, tile M = 256).
//
// A cluster of two CTAs on neighbouring SMs computes a 256 x 256 tile of one
// expert: each CTA holds 128 token rows of A and half (128 rows) of the
// weight tile B in its shared memory, the leader CTA issues
// tcgen05.mma.cta_group::2 (M=256, N=256, K=16), and each CTA's TMEM receives
// its 128 rows x 256 columns of the accumulator.  Per SM this halves the
// weight bytes per flop relative to the single-CTA 128 x 256 tile (16 KB of A
// plus 16 KB of B per 64-deep k-block instead of 16 + 32 KB), which is what
// the single-CTA kernel was bound by, and it frees shared memory for six
// pipeline stages.
//
// Synchronisation (all waits bounded in time):
//  * full[s] lives in the leader.  Its transaction count collects the TMA
//    bytes of both CTAs (loads issued with .cta_group::2 name the leader's
//    barrier); the leader's TMA thread arrives with the pair's total.  In the
//    gate/up phase the leader's 128 gather threads arrive on it through
//    cp.async.mbarrier.arrive, and the peer's gather threads on a local
//    gfull[s] that the peer's (otherwise idle) MMA warp relays to the leader
//    with one cluster-scope arrive.
//  * empty[s], tfull[a] and drain exist in both CTAs; the leader's commits
//    are multicast to both.
//  * tempty[a] lives in the leader: 4 epilogue warps of each CTA arrive.
#pragma once
#include "common.cuh"
#include "expert_ffn.cuh"

namespace moe {
namespace pair {

constexpr int BMC = 128;  // token rows per CTA (the pair covers 256)
constexpr int BN = 256;   // output columns per tile (each CTA loads 128 weight rows)
constexpr int BK = 64;
constexpr int STAGES = 6;
constexpr int A_BYTES = BMC * BK * 2;        // 16 KB
constexpr int B_BYTES = (BN / 2) * BK * 2;   // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TILE_BYTES = STAGES * STAGE_BYTES;  // 192 KB
constexpr int TMEM_COLS = 2 * BN;
constexpr int STAGE_ROW = ffn::STAGE_ROW;
constexpr int EPI_WARP_BYTES = ffn::EPI_WARP_BYTES;

template <int PHASE>
struct PCfg;
template <>
struct PCfg<1> {
  static constexpr int KDIM = kH;
  static constexpr int NT = kI / 128;
  static constexpr int B_ROWS_PER_EXPERT = 2 * kI;
  static constexpr int OUT_COLS = kI;
  static constexpr int THREADS = 320;
  static constexpr int TMA_WARP = 8;
  static constexpr int MMA_WARP = 9;
  static constexpr int FULL_COUNT = 1 + 128 + 1;  // leader TMA + leader gather + peer relay
  static constexpr uint32_t TX = 2 * B_BYTES;     // both CTAs' weight halves
  static constexpr uint32_t IDESC = idesc_f32acc(2 * BMC, BN, kFmtBF16);
};
template <>
struct PCfg<2> {
  static constexpr int KDIM = kI;
  static constexpr int NT = kH / BN;
  static constexpr int B_ROWS_PER_EXPERT = kH;
  static constexpr int OUT_COLS = kH;
  static constexpr int THREADS = 192;
  static constexpr int TMA_WARP = 4;
  static constexpr int MMA_WARP = 5;
  static constexpr int FULL_COUNT = 1;
  static constexpr uint32_t TX = 2 * (A_BYTES + B_BYTES);
  static constexpr uint32_t IDESC = idesc_f32acc(2 * BMC, BN, kFmtF16);
};

struct Tail {
  uint64_t full[STAGES];
  uint64_t gfull[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int wsum[4];
  int tile_start[kE + 1];
  int cnt[kE];
  int off[kE];
};
constexpr int TAIL_BYTES = (static_cast<int>(sizeof(Tail)) + 127) / 128 * 128;
constexpr int SMEM_BYTES = TILE_BYTES + TAIL_BYTES + 4 * EPI_WARP_BYTES + 1024;

__device__ __forceinline__ void decode_tile(const Tail* S, int tile, int& e, int& m, int& j) {
  int lo = 0, hi = kE - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (S->tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  e = lo;
  const int rem = tile - S->tile_start[e];
  const int mt = (S->cnt[e] + 2 * BMC - 1) / (2 * BMC);
  j = rem / mt;
  m = rem - j * mt;
}

template <int PHASE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PCfg<PHASE>::THREADS, 1)
    pair_gemm_kernel(const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ CUtensorMap tmap_a,
                     const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ offsets,
                     const int32_t* __restrict__ perm_src, int64_t T,
                     uint16_t* __restrict__ out, uint64_t timeout_ns) {
  using C = PCfg<PHASE>;
  constexpr int KB = C::KDIM / BK;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Tail* S = reinterpret_cast<Tail*>(smem + TILE_BYTES);
  uint8_t* sEpi = smem + TILE_BYTES + TAIL_BYTES;
  volatile int* abort_flag = &S->abort_flag;
  auto sA = [&](int s) { return smem + s * STAGE_BYTES; };
  auto sB = [&](int s) { return smem + s * STAGE_BYTES + A_BYTES; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair_id = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  const int64_t nrows = T * kTopK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&S->full[s], C::FULL_COUNT);
      mbar_init(&S->gfull[s], 128);
      mbar_init(&S->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&S->tfull[a], 1);
      mbar_init(&S->tempty[a], 8);
    }
    mbar_init(&S->drain, 1);
    S->abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == C::TMA_WARP && lane == 0) {
    tma_prefetch_desc(&tmap_b);
    if (PHASE == 2) tma_prefetch_desc(&tmap_a);
  }

  int my_tiles = 0;
  if (threadIdx.x < kE) {
    const int e = threadIdx.x;
    const int o0 = offsets[e], o1 = offsets[e + 1];
    int c = o1 - o0;
    if (o0 < 0 || c < 0 || static_cast<int64_t>(o1) > nrows) {
      record_status(kSiteBadIndex);
      c = 0;
    }
    S->cnt[e] = c;
    S->off[e] = o0;
    my_tiles = ((c + 2 * BMC - 1) / (2 * BMC)) * C::NT;
  }
  int incl = my_tiles;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  if (threadIdx.x < kE && lane == 31) S->wsum[warp] = incl;
  if (warp == C::MMA_WARP) tmem_alloc_pair(&S->tmem_base, TMEM_COLS);
  __syncthreads();
  if (threadIdx.x < kE) {
    int base = 0;
    for (int w = 0; w < warp; ++w) base += S->wsum[w];
    S->tile_start[threadIdx.x] = base + incl - my_tiles;
    if (threadIdx.x == kE - 1) S->tile_start[kE] = base + incl;
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers are initialised before anyone signals the other
  tc_fence_after();

  const uint32_t tmem_base = S->tmem_base;
  const int total_tiles = S->tile_start[kE];
  const uint32_t leader_full0 = mapa_shared(smem_u32(&S->full[0]), 0);
  const uint32_t leader_tempty0 = mapa_shared(smem_u32(&S->tempty[0]), 0);

  if (warp == C::TMA_WARP) {
    // ------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = pair_id; ok && tile < total_tiles; tile += num_pairs) {
        int e, m, j;
        decode_tile(S, tile, e, m, j);
        const int brow = e * C::B_ROWS_PER_EXPERT + j * BN + static_cast<int>(rank) * (BN / 2);
        const int arow = S->off[e] + m * 2 * BMC + static_cast<int>(rank) * BMC;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&S->empty[s], ph ^ 1, abort_flag, timeout_ns, kSiteFfnEmpty)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&S->full[s], C::TX);
          const uint32_t fb = leader_full0 + s * 8;
          if (PHASE == 2) tma_load_2d_pair(smem_u32(sA(s)), &tmap_a, kb * BK, arow, fb);
          tma_load_2d_pair(smem_u32(sB(s)), &tmap_b, kb * BK, brow, fb);
        }
      }
      if (!ok) {  // give copies already issued time to land before the block can exit
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) {
        }
      }
    }
  } else if (warp == C::MMA_WARP) {
    if (leader) {
      // ---------------------------------------------- MMA issuer (leader only)
      if (lane == 0) {
        int it = 0, tc = 0;
        bool ok = true;
        for (int tile = pair_id; ok && tile < total_tiles; tile += num_pairs, ++tc) {
          const int a = tc & 1;
          const uint32_t use = tc >> 1;
          if (!mbar_wait_cluster(&S->tempty[a], (use & 1) ^ 1, abort_flag, timeout_ns,
                                 kSiteFfnTmemEmpty)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + a * BN;
          for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1;
            if (!mbar_wait_cluster(&S->full[s], ph, abort_flag, timeout_ns, kSiteFfnFull)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t adesc = smem_desc_k128(smem_u32(sA(s)));
            const uint64_t bdesc = smem_desc_k128(smem_u32(sB(s)));
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_f16_pair(d, adesc + 2 * k, bdesc + 2 * k, C::IDESC, (kb | k) != 0 ? 1u : 0u);
            umma_commit_pair(&S->empty[s], 0x3);
          }
          if (ok) umma_commit_pair(&S->tfull[a], 0x3);
        }
        umma_commit_pair(&S->drain, 0x3);
        mbar_wait(&S->drain, 0, abort_flag, timeout_ns, kSiteFfnDrain);
      }
    } else if (PHASE == 1 && lane == 0) {
      // ---------------------------------------------- relay (peer only): gathered rows ready
      int it = 0;
      bool ok = true;
      for (int tile = pair_id; ok && tile < total_tiles; tile += num_pairs) {
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&S->gfull[s], ph, abort_flag, timeout_ns, kSiteFfnFull)) {
            ok = false;
            break;
          }
          mbar_arrive_remote(leader_full0 + s * 8);
        }
      }
      mbar_wait(&S->drain, 0, abort_flag, timeout_ns, kSiteFfnDrain);
    } else if (lane == 0) {
      mbar_wait(&S->drain, 0, abort_flag, timeout_ns, kSiteFfnDrain);
    }
  } else if (PHASE == 1 && warp >= 4 && warp < 8) {
    // ------------------------------------------------ A gather (both CTAs)
    // eight threads per row: each warp instruction moves four whole 128-byte rows
    const int t = threadIdx.x - 128;
    const int chunk = t & 7, rsub = t >> 3;
    const uint32_t slot = static_cast<uint32_t>((chunk ^ (rsub & 7)) << 4);
    uint64_t* arrive_bar0 = leader ? S->full : S->gfull;
    int it = 0;
    bool ok = true;
    for (int tile = pair_id; ok && tile < total_tiles; tile += num_pairs) {
      int e, m, j;
      decode_tile(S, tile, e, m, j);
      const char* src[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        src[i] = nullptr;
        const int row_in_e = m * 2 * BMC + static_cast<int>(rank) * BMC + rsub + 16 * i;
        if (row_in_e < S->cnt[e]) {
          const int p = perm_src[S->off[e] + row_in_e];
          if (p >= 0 && static_cast<int64_t>(p) < nrows)
            src[i] = reinterpret_cast<const char*>(x + static_cast<int64_t>(p >> 3) * kH) + chunk * 16;
        }
      }
      for (int kb = 0; kb < KB; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait(&S->empty[s], ph ^ 1, abort_flag, timeout_ns, kSiteFfnEmpty)) {
          ok = false;
          break;
        }
        const uint32_t base = smem_u32(sA(s)) + rsub * 128 + slot;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (src[i] != nullptr) cp_async_16(base + i * 16 * 128, src[i] + kb * BK * 2, 16);
        cp_async_arrive_noinc(&arrive_bar0[s]);
      }
    }
    cp_async_wait_all();
  } else if (warp < 4) {
    // ------------------------------------------------ epilogue (both CTAs)
    bool range_bad = false;
    int tc = 0;
    for (int tile = pair_id; tile < total_tiles; tile += num_pairs, ++tc) {
      int e, m, j;
      decode_tile(S, tile, e, m, j);
      const int a = tc & 1;
      const uint32_t use = tc >> 1;
      if (!mbar_wait(&S->tfull[a], use & 1, abort_flag, timeout_ns, kSiteFfnTmemFull)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + a * BN;
      const int row0 = m * 2 * BMC + static_cast<int>(rank) * BMC + warp * 32;
      const int nvalid = min(32, max(0, S->cnt[e] - row0));
      const uint32_t stage = smem_u32(sEpi + warp * EPI_WARP_BYTES);
      uint16_t* g0 = out + (static_cast<int64_t>(S->off[e]) + row0) * C::OUT_COLS;
      bool bad = false;
      if (PHASE == 1) {
        g0 += j * 128;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t g[32], u[32];
          tmem_ld_2x32(tbase + c * 32, tbase + 128 + c * 32, g, u);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_f16x2(ffn::silu_mul(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                               ffn::silu_mul(__uint_as_float(g[2 * i + 1]),
                                             __uint_as_float(u[2 * i + 1])),
                               bad);
          if (nvalid > 0) ffn::store_block_32x32(pk, stage, g0 + c * 32, C::OUT_COLS, nvalid, lane);
        }
      } else {
        g0 += j * BN;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v0[32], v1[32];
          tmem_ld_2x32(tbase + c * 64, tbase + c * 64 + 32, v0, v1);
          uint32_t p0[16], p1[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            p0[i] = pack_f16x2(__uint_as_float(v0[2 * i]), __uint_as_float(v0[2 * i + 1]), bad);
            p1[i] = pack_f16x2(__uint_as_float(v1[2 * i]), __uint_as_float(v1[2 * i + 1]), bad);
          }
          if (nvalid > 0) {
            ffn::store_block_32x32(p0, stage, g0 + c * 64, C::OUT_COLS, nvalid, lane);
            ffn::store_block_32x32(p1, stage, g0 + c * 64 + 32, C::OUT_COLS, nvalid, lane);
          }
        }
      }
      range_bad |= bad && lane < nvalid;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(leader_tempty0 + a * 8);
    }
    if (range_bad) record_status(kSiteFp16Range);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's shared memory and TMEM stay live until the leader is done
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace pair
}  // namespace moe
