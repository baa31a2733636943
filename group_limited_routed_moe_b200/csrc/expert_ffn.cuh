// expert_ffn.cuh -- step 3: the grouped SwiGLU expert FFN as two persistent
// tcgen05 GEMMs over the permuted rows.
//
// Every expert has gate, up and down matrices ("HelloSun/ling30tiny", table
// 模型與路由, row on expert weights) and no SwiGLU clamp ("Ling-3.0-tiny on a
// Qualcomm board", TensorFold issue #1247, first comment: "null SwiGLU limit
// lists").  The same issue names the missing piece this replaces: the bf16
// experts there have "no grouped kernel" and run a per-expert row loop.
//
//   phase 1 (gate/up):  h[r]      = silu(x[tok(r)] W_gate[e]) * (x[tok(r)] W_up[e])
//                       M_e x N 1024 x K 1536 per expert, N tiled by 256 =
//                       128 gate + 128 up columns, SwiGLU in the epilogue.
//                       bf16 x bf16 -> fp32 accumulate -> fp16 h.
//   phase 2 (down):     y_perm[r] = h[r] W_down[e]
//                       M_e x N 1536 x K 512 per expert, N tiled by 256.
//                       fp16 x fp16 (W_down packed as fp16, exact for bf16
//                       weights in the fp16 normal range) -> fp32 -> fp16 y.
// The two intermediates are fp16 rather than bf16: same bytes and the same
// tensor-core rate, 8x smaller rounding error.  A value outside the fp16 range
// sets the device status word (kSiteFp16Range) instead of passing silently.
//
// Work is cut into tiles (expert e, n-tile j, m-tile m) of 128 rows x 256
// columns; tile ids run expert-major, then j, then m, so CTAs that run at the
// same time share an expert's weight tile through L2.  A persistent grid of
// one CTA per SM takes tile ids from a global counter (the first one too),
// so that CTAs held up by slow tiles take fewer of them; static round-robin
// left some CTAs up to 1.5x longer than the median.  The tile table is built
// by each CTA from the device-side expert offsets, so the host never reads
// them.
//
// Warp roles inside a CTA (one CTA per SM: ~205 KB of shared memory, all 512
// TMEM columns):
//   warps 0-3  epilogue: TMEM -> registers (tcgen05.ld), SwiGLU, fp16 stores
//   warps 4-11 (phase 1) A producers: gather the tile's token rows of x with
//              cp.async into the 128B-swizzled operand layout, eight threads
//              per row so that each warp instruction moves whole 128-byte
//              lines (16-byte-per-row access touched every L2 sector twice
//              and cost ~40% of the gate/up time at T=8189); each thread
//              signals the stage's barrier through cp.async.mbarrier.arrive,
//              so the gather keeps all stages in flight.  Eight warps of 4
//              rows a thread issue the 1024 copies of a k-block faster than
//              four warps of 8 (gate/up 199 -> 191 us at T=8189).  Rows past the
//              expert's count are not loaded (a row of A only reaches the
//              same, never stored, accumulator row).  With ZERO_PAD they are
//              kept at zero by a zero-fill cp.async, issued only when the
//              slot last held data (start-up, valid -> padding change): when
//              most rows are padding (small batches) the gate/up GEMM ran up
//              to 2x slower with stale bits there than with zeros, while with
//              few padding rows (large batches) leaving them stale was ~15%
//              faster.  The host picks ZERO_PAD for T <= 4096.
//   next warp  TMA producer: weight tiles (and, in phase 2, h tiles)
//   next warp  MMA issuer: tcgen05.mma 128x256x16, accumulator in TMEM,
//              double-buffered (2 x 256 columns) so the epilogue of tile i
//              overlaps the MMAs of tile i+1.
// Shared-memory ring: 4 stages of (A 128x64 + B 256x64) 16-bit elements.
// The epilogue transposes each warp's 32 x 32 fp16 block through a padded
// shared tile so that global stores are whole 64-byte row segments.
#pragma once
#include "common.cuh"

namespace moe {
namespace ffn {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;  // one 128-byte swizzle row of 16-bit elements
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int TILE_BYTES = STAGES * (A_BYTES + B_BYTES);
constexpr int TMEM_COLS = 2 * BN;
constexpr int STAGE_ROW = 80;                      // padded 64-byte row of the epilogue tile
constexpr int EPI_WARP_BYTES = 32 * STAGE_ROW;     // one warp's 32 x 32 fp16 block

// Per-phase constants (phase 1: gate/up, phase 2: down).
__host__ __device__ constexpr int nt_of(int phase) { return phase == 1 ? kI / 128 : kH / BN; }  // n-tiles
__host__ __device__ constexpr int kb_of(int phase) { return (phase == 1 ? kH : kI) / BK; }  // k-blocks
__host__ __device__ constexpr int brows_of(int phase) { return phase == 1 ? 2 * kI : kH; }  // packed rows
constexpr uint32_t kIdesc1 = idesc_f32acc(BM, BN, kFmtBF16);  // bf16 x bf16
constexpr uint32_t kIdesc2 = idesc_f32acc(BM, BN, kFmtF16);   // fp16 x fp16
// Increments a gate/up tile makes when its h rows are stored (its 4 epilogue
// warps): a down tile of expert e waits for kDoneStep * 4 n-tiles * mtiles(e).
constexpr int kDoneStep = 4;

// MODE 1: gate/up only, 2: down only, 3: both in one launch (gate/up tile ids
// first, then down).
template <int MODE>
struct Cfg {
  static constexpr bool HAS1 = MODE != 2, HAS2 = MODE != 1;
  static constexpr int GATHER_WARP0 = 4;                // warps 4-11 when HAS1
  static constexpr int TMA_WARP = HAS1 ? 12 : 4;
  static constexpr int MMA_WARP = TMA_WARP + 1;
  static constexpr int THREADS = 32 * (MMA_WARP + 1);   // 448 or 192
  static constexpr int FULL_COUNT = HAS1 ? 1 + 256 : 1; // TMA arrive (+ 256 gather threads)
};

struct SmemTail {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  TileQueue tq;
  uint32_t tmem_base;
  int abort_flag;
  int wsum[4];
  int segbase[kMaxSeg + 1];     // exclusive prefix of the segments' m-tile counts
  int mstart[kMaxSeg][kE + 1];  // per segment: exclusive prefix of the experts' 128-row m-tiles
  int cnt[kMaxSeg][kE];
  int off[kMaxSeg][kE];
};
constexpr int TAIL_BYTES = (static_cast<int>(sizeof(SmemTail)) + 127) / 128 * 128;
constexpr int SMEM_BYTES = TILE_BYTES + TAIL_BYTES + 4 * EPI_WARP_BYTES + 1024;

// Tile u of a phase with NT n-tiles per expert, over all segments: segment g,
// expert e, m-tile m, n-tile j (segment-major, then expert, then j, then m).
__device__ __forceinline__ void decode_tile(const SmemTail* S, int nseg, int u, int NT, int& g,
                                            int& e, int& m, int& j) {
  g = 0;
  while (g + 1 < nseg && S->segbase[g + 1] * NT <= u) ++g;
  u -= S->segbase[g] * NT;
  const int* ms = S->mstart[g];
  int lo = 0, hi = kE - 1;  // largest e with mstart[e] * NT <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ms[mid] * NT <= u) lo = mid; else hi = mid - 1;
  }
  e = lo;
  const int rem = u - ms[e] * NT;
  const int mt = (S->cnt[g][e] + BM - 1) / BM;
  j = rem / mt;
  m = rem - j * mt;
}

struct TileInfo {
  int phase, g, e, m, j;
};
template <int MODE>
__device__ __forceinline__ TileInfo tile_info(const SmemTail* S, int nseg, int tile, int total1) {
  TileInfo t;
  t.phase = MODE == 3 ? (tile < total1 ? 1 : 2) : MODE;
  const int u = (MODE == 3 && t.phase == 2) ? tile - total1 : tile;
  decode_tile(S, nseg, u, nt_of(t.phase), t.g, t.e, t.m, t.j);
  return t;
}

// silu(g) * u = g / (1 + exp(-g)) * u.  The fast division (2 ulp of fp32) is
// far below the fp16 rounding of h that follows; for very negative g the
// denominator overflows and the result is 0, the limit of silu.
__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

// Stores one warp's 32 rows x 32 fp16 columns (lane = row, 16 packed pairs in
// registers) as row segments of 64 bytes: written to the warp's padded shared
// tile, read back 4 lanes per row, stored 16 bytes per lane.  Rows >= nvalid
// are skipped.  g0 points at (row 0, first column); ld is the row stride.
__device__ __forceinline__ void store_block_32x32(const uint32_t (&pk)[16], uint32_t stage,
                                                  uint16_t* g0, int64_t ld, int nvalid, int lane) {
  const uint32_t mine = stage + lane * STAGE_ROW;
#pragma unroll
  for (int q = 0; q < 4; ++q) st_shared_v4(mine + q * 16, pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = i * 8 + (lane >> 2), ch = lane & 3;
    const uint4 v = ld_shared_v4(stage + row * STAGE_ROW + ch * 16);
    if (row < nvalid) st_global_v4(g0 + row * ld + ch * 8, v.x, v.y, v.z, v.w);
  }
  __syncwarp();
}

template <int MODE, bool ZERO_PAD>
__global__ void __launch_bounds__(Cfg<MODE>::THREADS, 1)
    ffn_gemm_kernel(const __grid_constant__ SegMaps maps,  // w1: packed W_gate/W_up, w2: W_down, h
                    const __grid_constant__ SegPtrs seg, const __nv_bfloat16* __restrict__ x,
                    int64_t T, int* __restrict__ sched, uint64_t timeout_ns,
                    uint64_t* __restrict__ trace) {
  using C = Cfg<MODE>;
  const int nseg = seg.n;
  // segment g's per-expert done counters (single-launch form only)
  auto done_of = [&](int g) { return const_cast<int*>(seg.offsets[g]) + kDoneWord; };

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;                       // STAGES x 16 KB
  uint8_t* sB = smem + STAGES * A_BYTES;    // STAGES x 32 KB
  SmemTail* S = reinterpret_cast<SmemTail*>(smem + TILE_BYTES);
  uint8_t* sEpi = smem + TILE_BYTES + TAIL_BYTES;  // 4 x 2.5 KB
  volatile int* abort_flag = &S->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nrows = T * kTopK;
  griddep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&S->full[s], C::FULL_COUNT);
      mbar_init(&S->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&S->tfull[a], 1);
      mbar_init(&S->tempty[a], 4);
    }
    mbar_init(&S->drain, 1);
    tileq_init(&S->tq, (C::HAS1 ? 8 : 0) + 1 + 4);  // gather warps, MMA thread, epilogue warps
    S->abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == C::TMA_WARP && lane == 0) {
    for (int g = 0; g < nseg; ++g) {
      if (C::HAS1) tma_prefetch_desc(&maps.w1[g]);
      if (C::HAS2) {
        tma_prefetch_desc(&maps.w2[g]);
        tma_prefetch_desc(&maps.h[g]);
      }
    }
  }

  // tile table: m-tiles of expert e = ceil(count_e / 128), exclusive prefix
  griddep_wait();  // offsets, perm_src and (down alone) h come from the preceding kernels
  // The producer takes its first tile id from the counter too (issued here so
  // that the atomic's round trip overlaps the tile-table set-up below).
  if (trace != nullptr && threadIdx.x == 0) trace[3 * blockIdx.x] = global_timer_ns();
  int first_tile = 0;
  if (threadIdx.x == C::TMA_WARP * 32) first_tile = atomicAdd(sched, 1);
  if (C::HAS1) {
    // Start the A ring at zero: rows past an expert's count are never loaded,
    // and with whatever the previous kernel left in shared memory there the
    // tensor cores ran measurably slower than with zeros or stale x rows.
    for (int i = threadIdx.x; i < STAGES * A_BYTES / 16; i += blockDim.x)
      st_shared_v4(smem_u32(sA) + i * 16, 0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  if (warp == C::MMA_WARP) tmem_alloc(&S->tmem_base, TMEM_COLS);
  // per segment: the experts' row counts and first rows, and the prefix of
  // their 128-row m-tiles
  for (int g = 0; g < nseg; ++g) {
    int my_mt = 0;
    if (threadIdx.x < kE) {
      const int e = threadIdx.x;
      const int32_t* offsets = seg.offsets[g];
      const int o0 = offsets[e], o1 = offsets[e + 1];
      int c = o1 - o0;
      if (o0 < 0 || c < 0 || static_cast<int64_t>(o1) > nrows) {
        record_status(kSiteBadIndex);
        c = 0;
      }
      S->cnt[g][e] = c;
      S->off[g][e] = o0;
      my_mt = (c + BM - 1) / BM;
    }
    int incl = my_mt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    if (threadIdx.x < kE && lane == 31) S->wsum[warp] = incl;
    __syncthreads();
    if (threadIdx.x < kE) {
      int base = 0;
      for (int w = 0; w < warp; ++w) base += S->wsum[w];
      S->mstart[g][threadIdx.x] = base + incl - my_mt;
      if (threadIdx.x == kE - 1) S->mstart[g][kE] = base + incl;
    }
    __syncthreads();  // wsum is reused by the next segment
  }
  if (threadIdx.x == 0) {
    S->segbase[0] = 0;
    for (int g = 0; g < nseg; ++g) S->segbase[g + 1] = S->segbase[g] + S->mstart[g][kE];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = S->tmem_base;
  const int mtiles = S->segbase[nseg];
  const int total1 = C::HAS1 ? mtiles * nt_of(1) : 0;
  const int total_tiles = total1 + (C::HAS2 ? mtiles * nt_of(2) : 0);

  if (warp == C::TMA_WARP) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int it = 0, n = 0;
      bool ok = true;
      int tile = first_tile;
      while (ok) {
        const int pub = tile < total_tiles ? tile : -1;
        if (!tileq_push(&S->tq, n++, pub, abort_flag, timeout_ns)) {
          ok = false;
          break;
        }
        if (pub < 0) break;
        const int next = atomicAdd(sched, 1);  // used after the loads
        const TileInfo ti = tile_info<MODE>(S, nseg, tile, total1);
        if (MODE == 3 && ti.phase == 2) {
          // every gate/up tile of expert e has stored its h rows
          const int need = kDoneStep * nt_of(1) * ((S->cnt[ti.g][ti.e] + BM - 1) / BM);
          if (!wait_count(done_of(ti.g) + ti.e, need, abort_flag, timeout_ns, kSiteFfnDone)) {
            ok = false;
            break;
          }
        }
        const int brow = ti.e * brows_of(ti.phase) + ti.j * BN;
        const int arow = S->off[ti.g][ti.e] + ti.m * BM;
        for (int kb = 0; kb < kb_of(ti.phase); ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&S->empty[s], ph ^ 1, abort_flag, timeout_ns, kSiteFfnEmpty)) {
            ok = false;
            break;
          }
          if (ti.phase == 2) {
            mbar_arrive_expect_tx(&S->full[s], A_BYTES + B_BYTES);
            tma_load_2d(smem_u32(sA + s * A_BYTES), &maps.h[ti.g], kb * BK, arow, &S->full[s]);
            tma_load_2d(smem_u32(sB + s * B_BYTES), &maps.w2[ti.g], kb * BK, brow, &S->full[s]);
          } else {
            mbar_arrive_expect_tx(&S->full[s], B_BYTES);
            tma_load_2d(smem_u32(sB + s * B_BYTES), &maps.w1[ti.g], kb * BK, brow, &S->full[s]);
          }
        }
        tile = next;
      }
      if (trace != nullptr) trace[3 * blockIdx.x + 2] = static_cast<uint64_t>(n - 1);  // tiles
      if (!ok) {
        // let the copies already issued land before the block can exit
        for (int i = max(0, it - STAGES); i < it; ++i)
          mbar_wait_drain(&S->full[i % STAGES], (i / STAGES) & 1, kSiteFfnFull);
      }
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, tc = 0;
      bool ok = true;
      for (;; ++tc) {
        const int tile = tileq_pop(&S->tq, tc, true, abort_flag, timeout_ns);
        if (tile < 0) {
          ok = tile == -1;
          break;
        }
        const int phase = MODE == 3 ? (tile < total1 ? 1 : 2) : MODE;
        const uint32_t idesc = phase == 1 ? kIdesc1 : kIdesc2;
        const int a = tc & 1;
        const uint32_t use = tc >> 1;
        if (!mbar_wait(&S->tempty[a], (use & 1) ^ 1, abort_flag, timeout_ns, kSiteFfnTmemEmpty)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + a * BN;
        for (int kb = 0; kb < kb_of(phase); ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(&S->full[s], ph, abort_flag, timeout_ns, kSiteFfnFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc_k128(smem_u32(sA + s * A_BYTES));
          const uint64_t bdesc = smem_desc_k128(smem_u32(sB + s * B_BYTES));
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_f16(d, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit(&S->empty[s]);
        }
        if (ok) umma_commit(&S->tfull[a]);
      }
      // every MMA this thread issued must be complete before TMEM is freed
      umma_commit(&S->drain);
      mbar_wait_drain(&S->drain, 0, kSiteFfnDrain);
    }
  } else if (C::HAS1 && warp >= C::GATHER_WARP0 && warp < C::GATHER_WARP0 + 8) {
    // ------------------------------------------------ A gather producers (gate/up tiles)
    // Thread t copies 16-byte chunk (t & 7) of rows (t >> 3) + 32 i, i < 4, so a
    // warp instruction moves four whole 128-byte rows (full L2 lines).  The
    // swizzled chunk slot (chunk ^ (row & 7)) is the same for all of a
    // thread's rows because the row stride is 32.  For a down tile (single
    // launch) the TMA brings A; the gather threads only keep the stage
    // barriers' arrival count.
    const int t = threadIdx.x - 32 * C::GATHER_WARP0;
    const int chunk = t & 7, rsub = t >> 3;  // rsub < 32: rows rsub + 32 i, i < 4
    const uint32_t slot = static_cast<uint32_t>((chunk ^ (rsub & 7)) << 4);
    uint32_t dirty = 0u;  // bit 4*s + i: row rsub+32i of stage s may be non-zero (ring starts zeroed)
    // The row sources of the next gate/up tile, read a few stages before it
    // starts (once the producer has published it), so that a new tile's first
    // copies do not wait for perm_src to come from memory.
    int pf_tile = -1;
    int pf_p[4];
    auto load_rows = [&](const TileInfo& tj, int (&pv)[4]) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row_in_e = tj.m * BM + rsub + 32 * i;
        pv[i] = row_in_e < S->cnt[tj.g][tj.e] ? seg.perm_src[tj.g][S->off[tj.g][tj.e] + row_in_e] : -1;
      }
    };
    int it = 0, n = 0;
    bool ok = true;
    while (ok) {
      const int tile = tileq_pop(&S->tq, n++, lane == 0, abort_flag, timeout_ns);
      if (tile < 0) break;
      const TileInfo ti = tile_info<MODE>(S, nseg, tile, total1);
      if (ti.phase == 2) {
        for (int kb = 0; kb < kb_of(2); ++kb, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(&S->empty[s], ((it / STAGES) & 1) ^ 1, abort_flag, timeout_ns,
                         kSiteFfnEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive(&S->full[s]);
        }
        continue;
      }
      int pv[4];
      if (pf_tile == tile) {
#pragma unroll
        for (int i = 0; i < 4; ++i) pv[i] = pf_p[i];
      } else {
        load_rows(ti, pv);
      }
      pf_tile = -1;
      const char* src[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        src[i] = nullptr;
        if (pv[i] >= 0 && static_cast<int64_t>(pv[i]) < nrows)
          src[i] = reinterpret_cast<const char*>(x + static_cast<int64_t>(pv[i] >> 3) * kH) + chunk * 16;
      }
      for (int kb = 0; kb < kb_of(1); ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (kb >= kb_of(1) - STAGES && pf_tile < 0) {  // the next tile, once it is published
          const int nx = tileq_peek(&S->tq, n);
          if (nx >= 0) {
            const TileInfo tn = tile_info<MODE>(S, nseg, nx, total1);
            if (tn.phase == 1) {
              load_rows(tn, pf_p);
              pf_tile = nx;
            }
          }
        }
        if (!mbar_wait(&S->empty[s], ph ^ 1, abort_flag, timeout_ns, kSiteFfnEmpty)) {
          ok = false;
          break;
        }
        const uint32_t base = smem_u32(sA + s * A_BYTES) + rsub * 128 + slot;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t bit = 1u << (4 * s + i);
          if (src[i] != nullptr) {
            cp_async_16(base + i * 32 * 128, src[i] + kb * BK * 2, 16);
            dirty |= bit;
          } else if (ZERO_PAD && (dirty & bit)) {
            cp_async_16(base + i * 32 * 128, x, 0);
            dirty &= ~bit;
          }
        }
        cp_async_arrive_noinc(&S->full[s]);
      }
    }
    cp_async_wait_all();
  } else if (warp < 4) {
    // ------------------------------------------------ epilogue
    bool range_bad = false;  // thread (warp w, lane l) owns row 32w + l == TMEM lane
    for (int tc = 0;; ++tc) {
      const int tile = tileq_pop(&S->tq, tc, lane == 0, abort_flag, timeout_ns);
      if (tile < 0) break;
      const TileInfo ti = tile_info<MODE>(S, nseg, tile, total1);
      const int g = ti.g, e = ti.e, m = ti.m, j = ti.j;
      const int a = tc & 1;
      const uint32_t use = tc >> 1;
      if (!mbar_wait(&S->tfull[a], use & 1, abort_flag, timeout_ns, kSiteFfnTmemFull)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + a * BN;
      const int nvalid = min(32, max(0, S->cnt[g][e] - (m * BM + warp * 32)));
      const uint32_t stage = smem_u32(sEpi + warp * EPI_WARP_BYTES);
      bool bad = false;  // range check of this thread's row; rows >= nvalid hold garbage
      const int64_t row0 = static_cast<int64_t>(S->off[g][e]) + m * BM + warp * 32;
      uint16_t* const h_out = seg.h_out[g];
      uint16_t* const y_out = seg.y_out[g];
      // A warp whose 32 rows are all padding has nothing to read or store (at
      // T=2048 with skewed routing that was a fifth of the gate/up time).
      if (nvalid == 0) {
      } else if (ti.phase == 1) {
        uint16_t* g0 = h_out + row0 * kI + j * 128;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t g[32], u[32];
          tmem_ld_2x32(tbase + c * 32, tbase + 128 + c * 32, g, u);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_f16x2(silu_mul(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                               silu_mul(__uint_as_float(g[2 * i + 1]),
                                        __uint_as_float(u[2 * i + 1])),
                               bad);
          store_block_32x32(pk, stage, g0 + c * 32, kI, nvalid, lane);
        }
      } else {
        uint16_t* g0 = y_out + row0 * kH + j * BN;
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
          store_block_32x32(p0, stage, g0 + c * 64, kH, nvalid, lane);
          store_block_32x32(p1, stage, g0 + c * 64 + 32, kH, nvalid, lane);
        }
      }
      range_bad |= bad && lane < nvalid;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->tempty[a]);
      if (MODE == 3 && ti.phase == 1) {
        // publish: this warp's h rows of the tile are stored (a down tile's TMA reads them)
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(done_of(g) + e, 1);
      }
    }
    if (range_bad) record_status(kSiteFp16Range);
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    if (trace != nullptr) trace[3 * blockIdx.x + 1] = global_timer_ns();
    const bool last = tileq_retire(sched, MODE == 3 ? done_of(0) : nullptr, MODE == 3 ? kE : 0);
    if (MODE == 3 && last)  // the other segments' done counters too
      for (int g = 1; g < nseg; ++g)
        for (int i = 0; i < kE; ++i) atomicExch(done_of(g) + i, 0);
  }
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace ffn
}  // namespace moe
