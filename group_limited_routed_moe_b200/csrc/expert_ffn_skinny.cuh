// expert_ffn_skinny.cuh -- step 3 for small batches: the same two grouped
// GEMMs as expert_ffn.cuh with the operands swapped, so that the weights are
// the 128-row MMA operand and the few tokens of an expert are the narrow one.
//
// At decode an expert sees one or two of a batch's tokens.  A 128-row token
// tile would spend 127 rows of tensor work on padding; here a tile is 128
// weight rows x 32 tokens (tcgen05.mma M=128, N=32), each pipeline stage holds
// 16 KB of weights and 4 KB of token rows, and ten stages keep 160 KB of
// weights in flight per SM, so the kernel streams the selected experts'
// weights at HBM speed (the layer's bound at small batches).
//
//   phase 1: D[f][t] = sum_k W_gu[f][k] x[tok(t)][k] over 128 weight rows f =
//            64 gate rows + the 64 matching up rows (two TMA boxes), so that
//            h[t][f] = silu(D_gate) * D_up pairs TMEM lanes f and f+64; the up
//            half is handed to the gate half through a padded shared tile.
//   phase 2: D[n][t] = sum_k W_down[n][k] h[t][k] over 128 output columns n.
// Tiles are (expert, 128-row weight block, 32-token chunk), chunk fastest, so
// the CTAs that share a weight block run together and read it from L2 once.
//
// One launch can run both phases (MODE 3, used by moe_layer and
// moe_expert_ffn): all gate/up tiles come first in the tile order, then the
// down tiles.  A down tile of expert e needs all of e's h rows, so the TMA
// producer waits (bounded) until a per-expert counter says every gate/up tile
// of e has stored its h values; the gate/up epilogue makes its stores visible
// to the TMA (async proxy) and then increments the counter with release
// semantics.  Every tile id, a CTA's first included, comes from one global
// counter, so the gate/up tiles a waiting producer depends on were all handed
// out before, to CTAs that were running and run them without waiting: the
// wait ends however many CTAs of the grid are resident.  SMs that finish their last
// gate/up tile go straight on to down tiles of experts that are ready instead
// of idling until the slowest gate/up tile ends and a second launch ramps up.
// For a single token the layer's combine also runs in this launch: the CTA
// whose retirement completes the grid's count has every y row behind it and
// writes the layer's output, one kernel boundary fewer on the decode path.
//
// Warp roles: 0-3 epilogue (TMEM lanes 32w..32w+31), 4 token gather (phase 1:
// cp.async of x rows by perm_src, barrier-tracked; padding rows kept at zero),
// 5 TMA producer, 6-7 MMA issuers.  Accumulators: 2 buffers x 2 chains x 32
// TMEM columns (each tile's K steps go round-robin to the 2 chains, one per
// issuer).  Every wait, including the up -> gate hand-off, is a bounded
// mbarrier wait.
//
// Block-FP8 weights (WQ = true, MODE 3 only): the weight stream is 8-bit E4M3
// codes, half the bytes.  A stage covers K = 128 (one scale block): the TMA
// brings 128 rows x 128 codes (16 KB, 128-byte swizzle) into an 8-stage ring
// that also takes the stage's token rows (two 64-wide SW128 tiles, gathered x
// or TMA'd h, as above).  Converter warps, one thread per weight row,
// dequantise a row's 128 codes with the block's scale and store the 64
// columns of bf16 (gate/up) or fp16 (down) pairs straight into tensor memory,
// in one of 4 operand slots; the MMA then reads A from tensor memory and B
// (the token rows) from the ring, 8 instructions per stage.  The weights never
// make a second trip through shared memory, no proxy fence sits between the
// converters and the tensor core, and the single issuing thread handles half
// as many stages per weight byte as with 64-wide stages (its per-stage
// barrier round trips, not the MMAs, bound a skinny GEMM).
//
// NVFP4 weights (WQ = 2, MODE 3 only): the same ring and operand slots with
// 4-bit E2M1 codes.  A K = 128 stage holds 128 rows x 64 bytes of codes (two
// 64-row TMA boxes, 64-byte swizzle: 16-byte chunk j of row r at chunk
// j ^ ((r / 2) % 4)), the token rows, and the 2 KB of the stage's 16-bit block
// multipliers (one per 16 codes of a row, see fp4.cuh), loaded by one bulk
// copy; a converter thread turns 64 codes of its row into 32 columns of
// bf16 (gate/up) or fp16 (down) pairs with the integer route of fp4.cuh.
#pragma once
#include "combine.cuh"
#include "common.cuh"
#include "expert_ffn.cuh"
#include "fp4.cuh"
#include "fp8.cuh"

namespace moe {
namespace skinny {

constexpr int BMW = 128;  // weight rows per tile (MMA M)
constexpr int BNT = 32;   // tokens per tile (MMA N)
constexpr int BK = 64;
constexpr int STAGES = 10;
constexpr int A_BYTES = BMW * BK * 2;  // 16 KB
constexpr int B_BYTES = BNT * BK * 2;  // 4 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TILE_BYTES = STAGES * STAGE_BYTES;
// Accumulator chains per tile: the tile's K steps (16 each) go round-robin to
// NCH accumulators of BNT columns, one per MMA-issuing warp, summed in the
// epilogue as chain 0 + chain 1.  One thread's issue rate, not the
// accumulator dependency, sets the pace (four chains, two per issuer,
// measured no faster), and the epilogue reads half as many columns.
constexpr int NCH = 2;
constexpr int ACC_COLS = NCH * BNT;  // one accumulator buffer (all chains)
constexpr int XSTRIDE = BNT + 1;  // floats per row of the up-value exchange tile
constexpr int XCHG_BYTES = 64 * XSTRIDE * 4;
// MMA-issuing warps.  One thread's tcgen05.mma instructions follow one
// another at a few hundred cycles each (measured: about 170 cycles per
// M = 128, N = 32 MMA from one thread; two warps issuing at once halve that per
// MMA, four quarter it), and a weight tile's stages go through the MMAs one
// after another, so a single issuing thread set how fast one CTA streams a
// tile.  Issuer i issues the MMAs of the accumulator chains c with
// c % NISS == i, for every stage; each commits to the stage's empty barrier
// and to the tile's accumulator-full barrier, which count NISS arrivals.
constexpr int NISS = 2;
constexpr int THREADS = 32 * (6 + NISS);
constexpr int GATHER_WARP = 4, TMA_WARP = 5, MMA_WARP = 6;  // issuers: warps 6 .. 6 + NISS - 1
constexpr int CONV_WARP0 = 6 + NISS;  // quantised weights: converter warps from here
static_assert(NCH == NISS, "each issuer owns one accumulator chain");
constexpr int kConvGroups = 2;  // block-FP8: converter warps per tensor-memory lane quarter

// Ring geometry (WQ: 0 bf16, 1 block-FP8, 2 NVFP4 weights).  bf16 weights:
// STAGES x (16 KB weights + 4 KB tokens) of K = 64, two 32-column
// accumulators in tensor memory.  Quantised weights: RSTAGES x (codes, 16 KB
// FP8 or 8 KB FP4, + 8 KB tokens + the block scales, 1 KB reserved for the
// FP8 tile's, 2 KB for the FP4 stage's multipliers) of K = 128 in the same
// 200 KB, and tensor memory also holds NA dequantised 128 x 128 weight tiles
// (64 columns each) after the accumulators.
constexpr int kMaxStages = 10;
template <int WQ>
struct Ring {
  static constexpr int KS = WQ ? 128 : BK;                  // K per stage
  static constexpr int RA_BYTES = WQ == 2 ? BMW * KS / 2 : WQ ? BMW * KS : A_BYTES;  // codes or operands
  static constexpr int RB_BYTES = BNT * KS * 2;             // token rows
  static constexpr int RSC_BYTES = WQ == 2 ? fp4::kStageMultBytes : WQ ? 1024 : 0;  // block scales
  static constexpr int RSTAGE_BYTES = RA_BYTES + RB_BYTES + RSC_BYTES;
  static constexpr int RSTAGES = WQ ? 8 : STAGES;
  static constexpr int BYTES = RSTAGES * RSTAGE_BYTES;
  static constexpr int NA = WQ ? 4 : 0;
  static constexpr int A_COLS = KS / 2;  // 32-bit columns of one operand slot
  static constexpr int A_COL0 = 2 * ACC_COLS;             // after two accumulator buffers
  static constexpr int TMEM_COLS = WQ ? 512 : 2 * ACC_COLS;
  static constexpr int NCONV = WQ ? 4 * kConvGroups : 0;
  static constexpr int THREADS = skinny::THREADS + 32 * NCONV;
};
static_assert(Ring<1>::BYTES <= TILE_BYTES && Ring<2>::BYTES <= TILE_BYTES,
              "the quantised rings must fit the bf16 ring's space");
static_assert(Ring<0>::RSTAGES <= kMaxStages && Ring<1>::RSTAGES <= kMaxStages &&
                  Ring<2>::RSTAGES <= kMaxStages, "stages");
static_assert(Ring<1>::RSTAGE_BYTES % 1024 == 0 && Ring<1>::RA_BYTES % 1024 == 0 &&
                  Ring<2>::RSTAGE_BYTES % 1024 == 0 && Ring<2>::RA_BYTES % 1024 == 0,
              "swizzled tiles must stay 1024-byte aligned in the ring");
static_assert(Ring<1>::A_COL0 + Ring<1>::A_COLS * Ring<1>::NA <= Ring<1>::TMEM_COLS,
              "operand slots must fit the tensor-memory allocation");
static_assert(Ring<1>::RSTAGES % Ring<1>::NA == 0 && Ring<2>::RSTAGES % Ring<2>::NA == 0,
              "slot reuse follows the ring");
static_assert(kConvGroups == 2 && kH / Ring<1>::KS % 2 == 0 && kI / Ring<1>::KS % 2 == 0,
              "quantised stages go in pairs, one per converter group, never across a tile");
static_assert(Ring<2>::KS == fp4::kStageK, "an NVFP4 stage is one run of multipliers");

// Per-phase constants.  Phase 1: 8 weight blocks per 32-token chunk (4 pairs
// x 2 halves of 64 gate + 64 up rows), K = 1536; phase 2: 12 blocks, K = 512.
__host__ __device__ constexpr int fblk(int phase) { return phase == 1 ? 8 : kH / BMW; }
__host__ __device__ constexpr int kblocks(int phase, int ks = BK) {
  return (phase == 1 ? kH : kI) / ks;
}
constexpr uint32_t kIdesc1 = idesc_f32acc(BMW, BNT, kFmtBF16);
constexpr uint32_t kIdesc2 = idesc_f32acc(BMW, BNT, kFmtF16);
// Counter increments a gate/up tile makes when its h values are stored (one per
// storing warp): a down tile of expert e waits for kDoneStep * 8 * chunks(e).
constexpr int kDoneStep = 2;

struct Tail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t apair[2];  // block-FP8: the operand slots of a pair of stages written
  uint64_t xfull;   // up half written to the exchange tile (64 lane arrivals)
  uint64_t xempty;  // gate half done reading it (64 lane arrivals)
  uint64_t drain[NISS];
  TileQueue tq;
  uint32_t tmem_base;
  int abort_flag;
  int last_cta;  // this CTA retired last (it runs the fused combine)
  int wsum[4];
  int segbase[kMaxSeg + 1];       // exclusive prefix of the segments' chunk counts
  int cstart[kMaxSeg][kE + 1];    // per segment: exclusive prefix of the experts' 32-token chunks
  int cnt[kMaxSeg][kE];
  int off[kMaxSeg][kE];
};
constexpr int TAIL_BYTES = (static_cast<int>(sizeof(Tail)) + 127) / 128 * 128;
constexpr int SMEM_BYTES = TILE_BYTES + TAIL_BYTES + XCHG_BYTES + 1024;

// Tile u of a phase whose experts have FBLK weight blocks per chunk, over all
// segments: segment g, expert e, weight block f, chunk c.
__device__ __forceinline__ void decode_tile(const Tail* S, int nseg, int u, int FBLK, int& g,
                                            int& e, int& f, int& c) {
  g = 0;
  while (g + 1 < nseg && S->segbase[g + 1] * FBLK <= u) ++g;
  u -= S->segbase[g] * FBLK;
  const int* cs = S->cstart[g];
  int lo = 0, hi = kE - 1;  // largest e with cstart[e] * FBLK <= u
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cs[mid] * FBLK <= u) lo = mid; else hi = mid - 1;
  }
  e = lo;
  const int rem = u - cs[e] * FBLK;
  const int nch = (S->cnt[g][e] + BNT - 1) / BNT;
  f = rem / nch;
  c = rem - f * nch;
}

// Phase and coordinates of tile id `tile` of a launch in mode MODE (1: gate/up,
// 2: down, 3: both, gate/up tile ids first).
struct TileInfo {
  int phase, g, e, f, c;
};
template <int MODE>
__device__ __forceinline__ TileInfo tile_info(const Tail* S, int nseg, int tile, int total1) {
  TileInfo t;
  t.phase = MODE == 3 ? (tile < total1 ? 1 : 2) : MODE;
  const int u = (MODE == 3 && t.phase == 2) ? tile - total1 : tile;
  decode_tile(S, nseg, u, fblk(t.phase), t.g, t.e, t.f, t.c);
  return t;
}

template <int MODE, int WQ = 0>
__global__ void __launch_bounds__(Ring<WQ>::THREADS, 1)
    skinny_gemm_kernel(const __grid_constant__ SegMaps maps, const __grid_constant__ SegPtrs seg,
                       const __nv_bfloat16* __restrict__ x, int64_t T, int* __restrict__ sched,
                       const void* __restrict__ wscale,  // FP8 scales (SGU, SD) or FP4 MGU, MD
                       uint64_t timeout_ns,
                       uint64_t* __restrict__ trace,  // NULL, or 3 words per CTA (see ffn_trace)
                       const __grid_constant__ FusedCombine cmb) {
  constexpr bool HAS1 = MODE != 2, HAS2 = MODE != 1;
  const int nseg = seg.n;
  // segment g's per-expert done counters (single-launch form only)
  auto done_of = [&](int g) { return const_cast<int*>(seg.offsets[g]) + kDoneWord; };
  static_assert(!WQ || MODE == 3, "quantised weights only in the single-launch form");
  using R = Ring<WQ>;
  constexpr int RST = R::RSTAGES;
  constexpr int NA = R::NA > 0 ? R::NA : 1;
  constexpr int KS = R::KS;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Tail* S = reinterpret_cast<Tail*>(smem + TILE_BYTES);
  float* xchg = reinterpret_cast<float*>(smem + TILE_BYTES + TAIL_BYTES);
  volatile int* abort_flag = &S->abort_flag;
  uint64_t* fullb = S->full;
  uint64_t* emptyb = S->empty;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nrows = T * kTopK;
  griddep_launch_dependents();
  auto sA = [&](int s) { return smem + s * R::RSTAGE_BYTES; };
  auto sB = [&](int s) { return smem + s * R::RSTAGE_BYTES + R::RA_BYTES; };
  auto sC = [&](int s) { return sB(s) + R::RB_BYTES; };  // quantised: block scales

  if (threadIdx.x == 0) {
    for (int s = 0; s < RST; ++s) {
      mbar_init(&fullb[s], HAS1 ? 1 + 32 : 1);  // TMA arrive (+ 32 gather lanes)
      mbar_init(&emptyb[s], NISS);               // one MMA commit per issuer
    }
    // every converter warp arrives once per stage, two stages per pair
    for (int p = 0; p < 2; ++p) mbar_init(&S->apair[p], 2 * R::NCONV);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&S->tfull[a], NISS);
      mbar_init(&S->tempty[a], 4);
    }
    mbar_init(&S->xfull, 64);
    mbar_init(&S->xempty, 64);
    for (int i = 0; i < NISS; ++i) mbar_init(&S->drain[i], 1);
    // gather warp, MMA thread, epilogue warps, converter warps
    tileq_init(&S->tq, (HAS1 ? 1 : 0) + NISS + 4 + R::NCONV);
    S->abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == TMA_WARP && lane == 0) {
    for (int g = 0; g < nseg; ++g) {
      if (HAS1) tma_prefetch_desc(&maps.w1[g]);
      if (HAS2) {
        tma_prefetch_desc(&maps.w2[g]);
        tma_prefetch_desc(&maps.h[g]);
      }
    }
  }

  griddep_wait();  // offsets, perm_src and (down alone) h come from the preceding kernels
  // The producer takes its first tile id from the counter too (issued here so
  // that the atomic's round trip overlaps the tile-table set-up below).
  if (trace != nullptr && threadIdx.x == 0) trace[3 * blockIdx.x] = global_timer_ns();
  int first_tile = 0;
  if (threadIdx.x == TMA_WARP * 32) first_tile = atomicAdd(sched, 1);
  if (warp == MMA_WARP) tmem_alloc(&S->tmem_base, R::TMEM_COLS);
  // per segment: the experts' row counts and first rows, and the prefix of
  // their 32-token chunks
  for (int g = 0; g < nseg; ++g) {
    int my_chunks = 0;
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
      my_chunks = (c + BNT - 1) / BNT;
    }
    int incl = my_chunks;
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
      S->cstart[g][threadIdx.x] = base + incl - my_chunks;
      if (threadIdx.x == kE - 1) S->cstart[g][kE] = base + incl;
    }
    __syncthreads();  // wsum is reused by the next segment
  }
  if (threadIdx.x == 0) {
    S->segbase[0] = 0;
    for (int g = 0; g < nseg; ++g) S->segbase[g + 1] = S->segbase[g] + S->cstart[g][kE];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = S->tmem_base;
  const int nchunks = S->segbase[nseg];
  const int total1 = HAS1 ? nchunks * fblk(1) : 0;
  const int total_tiles = total1 + (HAS2 ? nchunks * fblk(2) : 0);

  if (warp == TMA_WARP) {
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
        const int next = atomicAdd(sched, 1);
        const TileInfo ti = tile_info<MODE>(S, nseg, tile, total1);
        const int g = ti.g, e = ti.e, f = ti.f, c = ti.c;
        if (MODE == 3 && ti.phase == 2) {
          // every gate/up tile of expert e has stored its h values
          const int need = kDoneStep * fblk(1) * ((S->cnt[g][e] + BNT - 1) / BNT);
          if (!wait_count(done_of(g) + e, need, abort_flag, timeout_ns, kSiteFfnDone)) {
            ok = false;
            break;
          }
        }
        int wrow0, wrow1 = 0;
        if (ti.phase == 1) {  // pair j = f/2, half = f%2: gate rows then the matching up rows
          const int j = f >> 1, half = f & 1;
          wrow0 = e * 2 * kI + 256 * j + 64 * half;
          wrow1 = wrow0 + 128;
        } else {
          wrow0 = e * kH + f * BMW;
        }
        const int hrow = S->off[g][e] + c * BNT;
        const CUtensorMap* tmap_w1 = &maps.w1[g];
        const CUtensorMap* tmap_w2 = &maps.w2[g];
        const CUtensorMap* tmap_h = &maps.h[g];
        const int KB = kblocks(ti.phase, KS);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % RST;
          const uint32_t ph = (it / RST) & 1;
          if (!mbar_wait(&emptyb[s], ph ^ 1, abort_flag, timeout_ns, kSiteFfnEmpty)) {
            ok = false;
            break;
          }
          if (WQ) {  // codes: two 64-row boxes (128 or 64 bytes); in phase 2 two 64-wide h tiles
            const int r1 = ti.phase == 1 ? wrow1 : wrow0 + 64;
            const CUtensorMap* tw = ti.phase == 1 ? tmap_w1 : tmap_w2;
            const void* scl;
            uint32_t scl_bytes;
            int kx;  // x coordinate of the code boxes, in bytes
            if constexpr (WQ == 2) {  // this stage's multipliers, one contiguous run
              scl = static_cast<const uint8_t*>(wscale) + fp4::stage_mult_offset(ti.phase, e, f, kb);
              scl_bytes = fp4::kStageMultBytes;
              kx = kb * KS / 2;
            } else {  // the tile's block scales: 12 gate + 12 up (phase 1) or 4 (phase 2)
              const float* sf = static_cast<const float*>(wscale);
              scl = ti.phase == 1 ? sf + fp8::sgu_index(e, 256 * (f >> 1), 0)
                                  : sf + kE * fp8::kSguPerExpert + fp8::sd_index(e, f * BMW, 0);
              scl_bytes = ti.phase == 1 ? 96 : 16;
              kx = kb * KS;
            }
            mbar_arrive_expect_tx(&fullb[s], R::RA_BYTES + (ti.phase == 2 ? R::RB_BYTES : 0) +
                                                 scl_bytes);
            bulk_load(smem_u32(sC(s)), scl, scl_bytes, &fullb[s]);
            tma_load_2d(smem_u32(sA(s)), tw, kx, wrow0, &fullb[s]);
            tma_load_2d(smem_u32(sA(s)) + R::RA_BYTES / 2, tw, kx, r1, &fullb[s]);
            if (ti.phase == 2) {
              tma_load_2d(smem_u32(sB(s)), tmap_h, kb * KS, hrow, &fullb[s]);
              tma_load_2d(smem_u32(sB(s)) + B_BYTES, tmap_h, kb * KS + BK, hrow, &fullb[s]);
            }
          } else if (ti.phase == 1) {
            mbar_arrive_expect_tx(&fullb[s], A_BYTES);
            tma_load_2d(smem_u32(sA(s)), tmap_w1, kb * BK, wrow0, &fullb[s]);
            tma_load_2d(smem_u32(sA(s)) + A_BYTES / 2, tmap_w1, kb * BK, wrow1, &fullb[s]);
          } else {
            mbar_arrive_expect_tx(&fullb[s], A_BYTES + B_BYTES);
            tma_load_2d(smem_u32(sA(s)), tmap_w2, kb * BK, wrow0, &fullb[s]);
            tma_load_2d(smem_u32(sB(s)), tmap_h, kb * BK, hrow, &fullb[s]);
          }
        }
        tile = next;
      }
      if (trace != nullptr) trace[3 * blockIdx.x + 2] = static_cast<uint64_t>(n - 1);  // tiles
      if (!ok) {  // the loads already issued land before the CTA exits (bounded)
        for (int i = max(0, it - RST); i < it; ++i)
          mbar_wait_drain(&fullb[i % RST], (i / RST) & 1, kSiteFfnFull);
      }
    }
  } else if (warp >= MMA_WARP && warp < MMA_WARP + NISS) {
    // ------------------------------------------------ MMA issuers
    const int iss = warp - MMA_WARP;  // this thread issues chains iss, iss + NISS, ...
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
        const int KB = kblocks(phase, KS);
        const uint32_t idesc = phase == 1 ? kIdesc1 : kIdesc2;
        const int a = tc & 1;
        const uint32_t use = tc >> 1;
        if (!mbar_wait(&S->tempty[a], (use & 1) ^ 1, abort_flag, timeout_ns, kSiteFfnTmemEmpty)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + a * ACC_COLS;  // chain c at d + c * BNT
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = it % RST;
          const uint32_t ph = (it / RST) & 1;
          const uint64_t bdesc = smem_desc_k128(smem_u32(sB(s)));
          if constexpr (WQ) {
            // A: the dequantised tile in operand slot it % NA of tensor memory;
            // B: two 64-wide SW128 token tiles.  Stages go in pairs (it even):
            // one wait covers both, since any shared-memory access of this
            // thread after tcgen05 work costs a few hundred cycles.  The
            // converters waited for the stages' loads before they arrived, so
            // that wait orders the token rows too.
            if ((it & 1) == 0) {
              if (!mbar_wait(&S->apair[(it >> 1) & 1], (it >> 2) & 1, abort_flag, timeout_ns,
                             kSiteFfnFull)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            const int a = it % NA;
            const uint32_t at = tmem_base + R::A_COL0 + R::A_COLS * a;
#pragma unroll
            for (int k = iss; k < 8; k += NISS) {  // K step k of the stage into chain k % NCH
              const uint64_t b = (k < 4 ? bdesc : bdesc + (B_BYTES >> 4)) + 2 * (k & 3);
              umma_f16_ta(d + (k % NCH) * BNT, at + 8 * k, b, idesc,
                          (kb != 0 || k >= NCH) ? 1u : 0u);
            }
            // frees the ring stage and, for the converters, operand slot a
            umma_commit(&emptyb[s]);
          } else {
            if (!mbar_wait(&fullb[s], ph, abort_flag, timeout_ns, kSiteFfnFull)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t adesc = smem_desc_k128(smem_u32(sA(s)));
#pragma unroll
            for (int k = iss; k < BK / 16; k += NISS)  // K step k of the stage into chain k % NCH
              umma_f16(d + (k % NCH) * BNT, adesc + 2 * k, bdesc + 2 * k, idesc,
                       (kb != 0 || k >= NCH) ? 1u : 0u);
            umma_commit(&emptyb[s]);
          }
        }
        if (ok) umma_commit(&S->tfull[a]);
      }
      umma_commit(&S->drain[iss]);
      mbar_wait_drain(&S->drain[iss], 0, kSiteFfnDrain);
    }
  } else if (HAS1 && warp == GATHER_WARP) {
    // ------------------------------------------------ token gather (phase 1)
    const uint32_t swz = static_cast<uint32_t>(lane & 7);
    uint32_t dirty = (1u << RST) - 1;  // stage slots whose row `lane` may hold non-zero data
    int it = 0, n = 0;
    bool ok = true;
    while (ok) {
      const int tile = tileq_pop(&S->tq, n++, lane == 0, abort_flag, timeout_ns);
      if (tile < 0) break;
      const TileInfo ti = tile_info<MODE>(S, nseg, tile, total1);
      if (ti.phase == 2) {
        // down tile: the TMA brings the h rows; only keep the stage barriers' count
        for (int kb = 0; kb < kblocks(2, KS); ++kb, ++it) {
          const int s = it % RST;
          const uint32_t ph = (it / RST) & 1;
          if (!mbar_wait(&emptyb[s], ph ^ 1, abort_flag, timeout_ns, kSiteFfnEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive(&fullb[s]);
        }
        continue;
      }
      const int row_in_e = ti.c * BNT + lane;
      const char* src = nullptr;
      if (row_in_e < S->cnt[ti.g][ti.e]) {
        const int p = seg.perm_src[ti.g][S->off[ti.g][ti.e] + row_in_e];
        if (p >= 0 && static_cast<int64_t>(p) < nrows)
          src = reinterpret_cast<const char*>(x + static_cast<int64_t>(p >> 3) * kH);
      }
      for (int kb = 0; kb < kblocks(1, KS); ++kb, ++it) {
        const int s = it % RST;
        const uint32_t ph = (it / RST) & 1;
        if (!mbar_wait(&emptyb[s], ph ^ 1, abort_flag, timeout_ns, kSiteFfnEmpty)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int t2 = 0; t2 < KS / BK; ++t2) {  // 64-wide SW128 token tiles of the stage
          const uint32_t dst = smem_u32(sB(s)) + t2 * B_BYTES + lane * 128;
          if (src != nullptr) {
            const char* g = src + (kb * KS + t2 * BK) * 2;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              cp_async_16(dst + ((static_cast<uint32_t>(q) ^ swz) << 4), g + q * 16, 16);
          } else if (dirty & (1u << s)) {
#pragma unroll
            for (int q = 0; q < 8; ++q) cp_async_16(dst + q * 16, x, 0);
          }
        }
        if (src != nullptr)
          dirty |= 1u << s;
        else
          dirty &= ~(1u << s);
        cp_async_arrive_noinc(&fullb[s]);
      }
    }
    cp_async_wait_all();
  } else if (WQ && warp >= CONV_WARP0) {
    // ------------------------------------------------ converters (block-FP8, NVFP4)
    // One thread per weight row: warp w may only access tensor-memory lanes
    // 32 (w % 4) .. 32 (w % 4) + 31, so it takes those rows.  The converter
    // warps form kConvGroups groups of four (one per lane quarter); in every
    // stage group g converts the g-th 64 of a row's 128 codes, which halves
    // the time from a stage's arrival to its hand-off to the MMA (the ring's
    // cycle, not the converters' throughput, bounds the weight stream).  The
    // TMA wrote each 128-byte row of
    // codes with the 128-byte swizzle (16-byte chunk j of row r at chunk
    // j ^ (r % 8)), which spreads a warp's reads of one chunk over all banks.
    // Operand slot it % NA is free again once the MMA of stage it - NA is done,
    // which the ring's own empty barrier of that stage says.
    const int quarter = warp & 3;
    const int cgroup = (warp - CONV_WARP0) >> 2;
    const int row = 32 * quarter + lane;
    const uint32_t rsw = static_cast<uint32_t>(row & 7);
    const bool up_rows = quarter >= 2;  // rows 64..127 of a gate/up tile are up rows
    const uint32_t a_lane = static_cast<uint32_t>(32 * quarter) << 16;
    int it = 0, n = 0;
    bool ok = true;
    while (ok) {
      const int tile = tileq_pop(&S->tq, n++, lane == 0, abort_flag, timeout_ns);
      if (tile < 0) break;
      const TileInfo ti = tile_info<MODE>(S, nseg, tile, total1);
      for (int kb = 0; kb < kblocks(ti.phase, KS); ++kb, ++it) {
        const int s = it % RST;
        const uint32_t ph = (it / RST) & 1;
        const int a = it % NA;
        bool got = mbar_wait(&fullb[s], ph, abort_flag, timeout_ns, kSiteFfnFull);
        if (got && it >= NA) {
          const int prev = it - NA;  // the stage that last used slot a
          got = mbar_wait(&emptyb[prev % RST], (prev / RST) & 1, abort_flag, timeout_ns,
                          kSiteFfnEmpty);
        }
        if (!got) {
          ok = false;
          break;
        }
        const uint32_t dst = tmem_base + a_lane + R::A_COL0 + R::A_COLS * a;
        if constexpr (WQ == 2) {
          // NVFP4: this group's 64 codes are chunks 2g, 2g + 1 of the row's
          // four (64-byte swizzle), its 4 block multipliers bytes 8g.. of the
          // row's 16 in the stage's multiplier run
          const uint32_t src = smem_u32(sA(s)) + row * 64;
          const uint32_t msw = static_cast<uint32_t>((row >> 1) & 3);
          const uint2 mm = fp4::ld_shared_v2(smem_u32(sC(s)) + row * 16 + 8 * cgroup);
          const uint32_t mv[4] = {__byte_perm(mm.x, 0, 0x1010), __byte_perm(mm.x, 0, 0x3232),
                                  __byte_perm(mm.y, 0, 0x1010), __byte_perm(mm.y, 0, 0x3232)};
          uint32_t v[32];
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const uint4 c4 = ld_shared_v4(src + (((2 * static_cast<uint32_t>(cgroup) + q) ^ msw) << 4));
            const uint32_t w[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (ti.phase == 1)
                fp4::dequant8<false>(w[i], mv[2 * q + (i >> 1)], v + 16 * q + 4 * i);
              else
                fp4::dequant8<true>(w[i], mv[2 * q + (i >> 1)], v + 16 * q + 4 * i);
            }
          }
          tmem_st_x32(dst + 32 * cgroup, v);
        } else {
          // this stage's block scale, from the tile's scales the TMA brought with
          // the stage: 12 gate then 12 up (phase 1), or 4 (phase 2), one per k block
          const float sc = reinterpret_cast<const float*>(
              sC(s))[(ti.phase == 1 && up_rows ? 12 : 0) + kb];
          const uint32_t src = smem_u32(sA(s)) + row * 128;
          uint32_t v[32];
          {
            const int h2 = cgroup;  // this group's 64 codes -> 32 columns
            if (ti.phase == 1) {
              const uint32_t mult = fp8::pow2_multiplier<false>(sc);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                uint32_t o[8];
                const uint32_t jj = static_cast<uint32_t>(4 * h2 + j);
                fp8::dequant16<false>(ld_shared_v4(src + ((jj ^ rsw) << 4)), sc, mult, o);
#pragma unroll
                for (int i = 0; i < 8; ++i) v[8 * j + i] = o[i];
              }
            } else {
              const uint32_t mult = fp8::pow2_multiplier<true>(sc);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                uint32_t o[8];
                const uint32_t jj = static_cast<uint32_t>(4 * h2 + j);
                fp8::dequant16<true>(ld_shared_v4(src + ((jj ^ rsw) << 4)), sc, mult, o);
#pragma unroll
                for (int i = 0; i < 8; ++i) v[8 * j + i] = o[i];
              }
            }
            tmem_st_x32(dst + 32 * h2, v);
          }
        }
        tmem_wait_st();
        tc_fence_before();  // operand stores -> the MMA thread's tcgen05.mma
        __syncwarp();
        if (lane == 0) mbar_arrive(&S->apair[(it >> 1) & 1]);
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------ epilogue
    bool range_bad = false;
    int n1 = 0;  // gate/up tiles seen so far (exchange-tile phase)
    for (int tc = 0;; ++tc) {
      const int tile = tileq_pop(&S->tq, tc, lane == 0, abort_flag, timeout_ns);
      if (tile < 0) break;
      const TileInfo ti = tile_info<MODE>(S, nseg, tile, total1);
      const int g = ti.g, e = ti.e, f = ti.f, c = ti.c;
      const int a = tc & 1;
      const uint32_t use = tc >> 1;
      if (!mbar_wait(&S->tfull[a], use & 1, abort_flag, timeout_ns, kSiteFfnTmemFull)) break;
      tc_fence_after();
      uint32_t v[32];
      {  // chain 0 + chain 1
        static_assert(NCH == 2, "the epilogue sums two chains");
        const uint32_t acc = tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + a * ACC_COLS;
        uint32_t u[32];
        tmem_ld_2x32(acc, acc + BNT, v, u);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(u[i]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->tempty[a]);  // accumulator copied out: MMA may reuse it
      const int ntok = min(BNT, S->cnt[g][e] - c * BNT);
      const int64_t row0 = static_cast<int64_t>(S->off[g][e]) + c * BNT;
      uint16_t* const h_out = seg.h_out[g];
      uint16_t* const y_out = seg.y_out[g];
      if (ti.phase == 1) {
        const uint32_t xph = static_cast<uint32_t>(n1++) & 1;
        if (warp >= 2) {  // up half: hand the values to the gate half
          if (!mbar_wait(&S->xempty, xph ^ 1, abort_flag, timeout_ns, kSiteFfnTmemEmpty)) break;
          float* xr = xchg + ((warp - 2) * 32 + lane) * XSTRIDE;
#pragma unroll
          for (int t = 0; t < BNT; ++t) xr[t] = __uint_as_float(v[t]);
          mbar_arrive(&S->xfull);
        } else {
          if (!mbar_wait(&S->xfull, xph, abort_flag, timeout_ns, kSiteFfnTmemFull)) break;
          const int j = f >> 1, half = f & 1;
          const int col = 128 * j + 64 * half + warp * 32 + lane;  // h column (intermediate feature)
          const float* xr = xchg + (warp * 32 + lane) * XSTRIDE;
          float up[BNT];
#pragma unroll
          for (int t = 0; t < BNT; ++t) up[t] = xr[t];
          mbar_arrive(&S->xempty);  // exchange tile free for the next tile
#pragma unroll
          for (int t = 0; t < BNT; ++t) {
            if (t < ntok) {
              const float hv = ffn::silu_mul(__uint_as_float(v[t]), up[t]);
              range_bad |= !(fabsf(hv) <= 65504.f);
              st_global_b16(h_out + (row0 + t) * kI + col, __half_as_ushort(__float2half_rn(hv)));
            }
          }
          if (MODE == 3) {
            // publish: this warp's h values of the tile are stored (TMA reads them later)
            asm volatile("fence.proxy.async.global;" ::: "memory");
            __threadfence();
            __syncwarp();
            if (lane == 0) atomicAdd(done_of(g) + e, 1);
          }
        }
      } else {
        const int col = f * BMW + warp * 32 + lane;  // y column (model feature)
#pragma unroll
        for (int t = 0; t < BNT; ++t) {
          if (t < ntok) {
            const float yv = __uint_as_float(v[t]);
            range_bad |= !(fabsf(yv) <= 65504.f);
            st_global_b16(y_out + (row0 + t) * kH + col, __half_as_ushort(__float2half_rn(yv)));
          }
        }
      }
    }
    if (range_bad) record_status(kSiteFp16Range);
  }

  // Fused combine: every storing thread fences its y stores before the CTA
  // counts itself retired, the last CTA fences after seeing the final count,
  // so it reads every CTA's y rows.
  const bool fuse = MODE == 3 && cmb.out != nullptr;
  if (fuse && warp < 4) __threadfence();
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    if (trace != nullptr) trace[3 * blockIdx.x + 1] = global_timer_ns();
    const bool last = tileq_retire(sched, MODE == 3 ? done_of(0) : nullptr, MODE == 3 ? kE : 0);
    if (MODE == 3 && last)  // the other segments' done counters too
      for (int g = 1; g < nseg; ++g)
        for (int i = 0; i < kE; ++i) atomicExch(done_of(g) + i, 0);
    if (fuse && last) __threadfence();
    S->last_cta = last;
  }
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, R::TMEM_COLS);
  }
  if (fuse) {
    __syncthreads();
    if (S->last_cta) {
      const uint16_t* y_shared = cmb.n_shared > 0 ? seg.y_out[1] : nullptr;
      const int64_t nvec = T * kCombineThreads;
      for (int64_t v = threadIdx.x; v < nvec; v += blockDim.x) {
        const int64_t t = v / kCombineThreads;
        const int col = static_cast<int>(v - t * kCombineThreads) * 8;
        combine_token_vec<kTopK, true>(seg.y_out[0], cmb.topk_w, cmb.inv_perm, T, t, col,
                                       cmb.residual, cmb.out, y_shared, cmb.n_shared);
      }
    }
  }
}

}  // namespace skinny
}  // namespace moe
