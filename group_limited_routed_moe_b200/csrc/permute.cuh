// permute.cuh -- step 2: device-side stable counting sort of the T*8
// (token, slot) items by expert.
//
// Each expert must run on exactly the rows that picked it; in the GB10 path of
// "Ling-3.0-tiny on a Qualcomm board" (TensorFold issue #1247, "What it does
// not cover", bullet on bf16 experts) finding those rows costs a host sync per
// layer.  Here the row sets are built on the device and never leave it.
//
// Because a token picks an expert at most once, the rank of item (t, slot)
// inside expert e is the number of earlier tokens that picked e.  A bitmap
// [expert][token] answers that with popcounts, so the sort needs no atomics on
// global memory and its output is deterministic:
//   row(t, slot) = offsets[e] + (tokens before this block that picked e)
//                             + popcount(bitmap[e][tokens of this block before t]).
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kPermSmallMaxT = 1024;   // single-block path up to this many tokens
// A slot holding this id is empty: it gets no row (inv_perm = -1) and is not
// counted.  A token's slots may mix experts and empty slots; the expert-parallel
// receiver uses it for the slots of a row whose expert lives on another rank.
constexpr int kEmptySlot = -1;
// Tokens per block on the multi-block path: 64 while the fused scan + scatter
// covers the batch (up to kPermSmallBlocksMaxT tokens: twice the blocks in
// flight as with 128, for latency-bound kernels), 128 above (fewer histogram
// rows for the separate scan).
constexpr int kPermBlockTokens = 128;
constexpr int kPermBlockTokensSmall = 64;
constexpr int64_t kPermSmallBlocksMaxT = 16384;

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xFFFFFFFFu, v, off);
    if (lane >= off) v += o;
  }
  return v;
}

// Walks down one expert's column of a per-block histogram hist[b][e] (row
// length ld), issuing kHistBatch independent loads before summing them, so
// the walk does not rely on the compiler to overlap its L2 round trips.  A
// thread walks 32 blocks in the fused scan + scatter at T=8189 (the same time
// as a plain loop there) and up to 4096 in the separate scan of the largest
// batches.  Integer sums, so the order changes nothing.
constexpr int kHistBatch = 8;

// tot += hist[b][e] and, for b < lim, bef += hist[b][e], over b = b0, b0 +
// step, ... < b1.
__device__ __forceinline__ void hist_column_sum(const int32_t* __restrict__ hist, int ld, int e,
                                                int b0, int b1, int step, int lim, int& tot,
                                                int& bef) {
  int b = b0;
  for (; b + (kHistBatch - 1) * step < b1; b += kHistBatch * step) {
    int v[kHistBatch];
#pragma unroll
    for (int u = 0; u < kHistBatch; ++u) v[u] = hist[static_cast<int64_t>(b + u * step) * ld + e];
#pragma unroll
    for (int u = 0; u < kHistBatch; ++u) {
      tot += v[u];
      if (b + u * step < lim) bef += v[u];
    }
  }
  for (; b < b1; b += step) {
    const int v = hist[static_cast<int64_t>(b) * ld + e];
    tot += v;
    if (b < lim) bef += v;
  }
}

// hist[b][e] <- run, then run += its old value, for b = b0 .. b1 - 1 in order
// (the column's exclusive prefix sum from run); returns the final run.
__device__ __forceinline__ int hist_column_exclusive(int32_t* __restrict__ hist, int ld, int e,
                                                     int b0, int b1, int run) {
  int b = b0;
  for (; b + kHistBatch <= b1; b += kHistBatch) {
    int v[kHistBatch];
#pragma unroll
    for (int u = 0; u < kHistBatch; ++u) v[u] = hist[static_cast<int64_t>(b + u) * ld + e];
#pragma unroll
    for (int u = 0; u < kHistBatch; ++u) {
      hist[static_cast<int64_t>(b + u) * ld + e] = run;
      run += v[u];
    }
  }
  for (; b < b1; ++b) {
    const int64_t i = static_cast<int64_t>(b) * ld + e;
    const int v = hist[i];
    hist[i] = run;
    run += v;
  }
  return run;
}

// Exclusive scan of cnt[0..127] into off[0..128], run by warp 0 only.
__device__ __forceinline__ void scan_experts_warp0(const int* cnt, int* off, int lane) {
  const int c0 = cnt[4 * lane], c1 = cnt[4 * lane + 1], c2 = cnt[4 * lane + 2],
            c3 = cnt[4 * lane + 3];
  const int loc = c0 + c1 + c2 + c3;
  const int incl = warp_incl_scan(loc, lane);
  const int base = incl - loc;
  off[4 * lane] = base;
  off[4 * lane + 1] = base + c0;
  off[4 * lane + 2] = base + c0 + c1;
  off[4 * lane + 3] = base + c0 + c1 + c2;
  if (lane == 31) off[kE] = incl;
}

// ---- single block, T <= 1024: bitmap of 128 experts x 1024 tokens ---------
__global__ void __launch_bounds__(1024)
    permute_small_kernel(const int32_t* __restrict__ idx, int T, int32_t* __restrict__ counts,
                         int32_t* __restrict__ offsets, int32_t* __restrict__ perm_src,
                         int32_t* __restrict__ inv_perm) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ uint32_t bm[kE][32];
  __shared__ uint32_t pre[kE][32];
  __shared__ int cnt[kE];
  __shared__ int off[kE + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int words = (T + 31) >> 5;

  for (int i = tid; i < kE * 32; i += blockDim.x) (&bm[0][0])[i] = 0u;
  __syncthreads();
  const int n = T * kTopK;
  for (int p = tid; p < n; p += blockDim.x) {
    const int e = idx[p];
    if (static_cast<unsigned>(e) >= static_cast<unsigned>(kE)) {
      if (e != kEmptySlot) record_status(kSiteBadIndex);
      continue;
    }
    const int t = p >> 3;
    atomicOr(&bm[e][t >> 5], 1u << (t & 31));
  }
  __syncthreads();
  for (int e = warp; e < kE; e += 32) {
    const int c = lane < words ? __popc(bm[e][lane]) : 0;
    const int incl = warp_incl_scan(c, lane);
    pre[e][lane] = incl - c;
    if (lane == 31) cnt[e] = incl;
  }
  __syncthreads();
  if (warp == 0) scan_experts_warp0(cnt, off, lane);
  __syncthreads();
  if (tid < kE) {
    counts[tid] = cnt[tid];
    offsets[tid] = off[tid];
  }
  if (tid == 0) offsets[kE] = off[kE];
  if (tid < kOffsetsLen - kSchedWord) offsets[kSchedWord + tid] = 0;  // GEMM tile counters
  for (int p = tid; p < n; p += blockDim.x) {
    const int e = idx[p];
    if (static_cast<unsigned>(e) >= static_cast<unsigned>(kE)) {
      inv_perm[p] = -1;  // an empty slot (or a bad id, reported above) has no row
      continue;
    }
    const int t = p >> 3;
    const int r = off[e] + pre[e][t >> 5] + __popc(bm[e][t >> 5] & ((1u << (t & 31)) - 1u));
    perm_src[r] = p;
    inv_perm[p] = r;
  }
}

// ---- multi-block path -----------------------------------------------------
// (a) per-block expert histogram hist[b][e]
template <int BT>
__global__ void __launch_bounds__(256)
    permute_count_kernel(const int32_t* __restrict__ idx, int64_t T, int32_t* __restrict__ hist) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ uint32_t bm[kE][BT / 32];
  const int tid = threadIdx.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * BT;
  const int nt = static_cast<int>((T - t0) < BT ? (T - t0) : BT);
  for (int i = tid; i < kE * (BT / 32); i += blockDim.x) (&bm[0][0])[i] = 0u;
  __syncthreads();
  for (int q = tid; q < nt * kTopK; q += blockDim.x) {
    const int e = idx[t0 * kTopK + q];
    if (static_cast<unsigned>(e) >= static_cast<unsigned>(kE)) {
      if (e != kEmptySlot) record_status(kSiteBadIndex);
      continue;
    }
    const int tl = q >> 3;
    atomicOr(&bm[e][tl >> 5], 1u << (tl & 31));
  }
  __syncthreads();
  if (tid < kE) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < BT / 32; ++w) c += __popc(bm[tid][w]);
    hist[static_cast<int64_t>(blockIdx.x) * kE + tid] = c;
  }
}

// (b) column scans: hist[b][e] <- rows of e in blocks before b; counts, offsets.
//     One block of 1024 threads: thread (part, e) owns a contiguous range of blocks.
__global__ void __launch_bounds__(1024)
    permute_scan_kernel(int32_t* __restrict__ hist, int nb, int32_t* __restrict__ counts,
                        int32_t* __restrict__ offsets) {
  griddep_launch_dependents();
  griddep_wait();
  constexpr int kParts = 1024 / kE;  // 8
  __shared__ int part_sum[kParts][kE];
  __shared__ int cnt[kE];
  __shared__ int off[kE + 1];
  const int tid = threadIdx.x, e = tid % kE, part = tid / kE, lane = tid & 31;
  const int per = (nb + kParts - 1) / kParts;
  const int b0 = min(nb, part * per), b1 = min(nb, b0 + per);
  int s = 0, unused = 0;
  hist_column_sum(hist, kE, e, b0, b1, 1, 0, s, unused);
  part_sum[part][e] = s;
  __syncthreads();
  int run = 0;
  for (int p = 0; p < part; ++p) run += part_sum[p][e];
  if (part == kParts - 1) cnt[e] = run + s;
  hist_column_exclusive(hist, kE, e, b0, b1, run);
  __syncthreads();
  if (tid < 32) scan_experts_warp0(cnt, off, lane);
  __syncthreads();
  if (tid < kE) {
    counts[tid] = cnt[tid];
    offsets[tid] = off[tid];
  }
  if (tid == 0) offsets[kE] = off[kE];
  if (tid < kOffsetsLen - kSchedWord) offsets[kSchedWord + tid] = 0;  // GEMM tile counters
}

// (b') fused scan + scatter for up to kPermFusedMaxBlocks blocks: every block
//      re-derives the expert offsets and its own bases from the histogram
//      (nb x 128 reads per block, split over kPermScanParts threads per
//      expert), so no separate scan launch is needed.
constexpr int kPermFusedMaxBlocks = 256;
constexpr int kPermScanParts = 4;
constexpr int kPermScanThreads = kPermScanParts * kE;  // 512

template <int BT>
__global__ void __launch_bounds__(kPermScanThreads)
    permute_scan_scatter_kernel(const int32_t* __restrict__ idx, int64_t T,
                                const int32_t* __restrict__ hist, int nb,
                                int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                int32_t* __restrict__ perm_src, int32_t* __restrict__ inv_perm) {
  griddep_launch_dependents();
  griddep_wait();
  constexpr int W = BT / 32;
  __shared__ uint32_t bm[kE][W];
  __shared__ int part[kPermScanParts][kE];
  __shared__ int before_s[kPermScanParts][kE];
  __shared__ int cnt[kE];
  __shared__ int off[kE + 1];
  __shared__ int base[kE];
  const int tid = threadIdx.x, lane = tid & 31;
  const int b = blockIdx.x;
  const int64_t t0 = static_cast<int64_t>(b) * BT;
  const int nt = static_cast<int>((T - t0) < BT ? (T - t0) : BT);
  for (int i = tid; i < kE * W; i += blockDim.x) (&bm[0][0])[i] = 0u;
  {  // column sums: thread (h, e) sums blocks h, h + kPermScanParts, ...
    const int e = tid & (kE - 1), h = tid >> 7;
    int tot = 0, bef = 0;
    hist_column_sum(hist, kE, e, h, nb, kPermScanParts, b, tot, bef);
    part[h][e] = tot;
    before_s[h][e] = bef;
  }
  __syncthreads();
  if (tid < kE) {
    int c = 0;
#pragma unroll
    for (int h = 0; h < kPermScanParts; ++h) c += part[h][tid];
    cnt[tid] = c;
  }
  __syncthreads();
  if (tid < 32) scan_experts_warp0(cnt, off, lane);
  __syncthreads();
  if (tid < kE) {
    int bef = 0;
#pragma unroll
    for (int h = 0; h < kPermScanParts; ++h) bef += before_s[h][tid];
    base[tid] = off[tid] + bef;
  }
  if (b == 0) {
    if (tid < kE) {
      counts[tid] = cnt[tid];
      offsets[tid] = off[tid];
    }
    if (tid == 0) offsets[kE] = off[kE];
    if (tid < kOffsetsLen - kSchedWord) offsets[kSchedWord + tid] = 0;  // GEMM tile counters
  }
  for (int q = tid; q < nt * kTopK; q += blockDim.x) {
    const int e = idx[t0 * kTopK + q];
    if (static_cast<unsigned>(e) >= static_cast<unsigned>(kE)) continue;
    const int tl = q >> 3;
    atomicOr(&bm[e][tl >> 5], 1u << (tl & 31));
  }
  __syncthreads();
  for (int q = tid; q < nt * kTopK; q += blockDim.x) {
    const int e = idx[t0 * kTopK + q];
    if (static_cast<unsigned>(e) >= static_cast<unsigned>(kE)) {
      inv_perm[t0 * kTopK + q] = -1;  // an empty slot (or a bad id) has no row
      continue;
    }
    const int tl = q >> 3, w = tl >> 5;
    int rank = __popc(bm[e][w] & ((1u << (tl & 31)) - 1u));
    for (int v = 0; v < w; ++v) rank += __popc(bm[e][v]);
    const int64_t p = t0 * kTopK + q;
    const int r = base[e] + rank;
    perm_src[r] = static_cast<int32_t>(p);
    inv_perm[p] = r;
  }
}

// (c) stable scatter of the block's items
__global__ void __launch_bounds__(256)
    permute_scatter_kernel(const int32_t* __restrict__ idx, int64_t T,
                           const int32_t* __restrict__ before, const int32_t* __restrict__ offsets,
                           int32_t* __restrict__ perm_src, int32_t* __restrict__ inv_perm) {
  griddep_launch_dependents();
  griddep_wait();
  constexpr int W = kPermBlockTokens / 32;
  __shared__ uint32_t bm[kE][W];
  __shared__ int base[kE];
  const int tid = threadIdx.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kPermBlockTokens;
  const int nt = static_cast<int>((T - t0) < kPermBlockTokens ? (T - t0) : kPermBlockTokens);
  for (int i = tid; i < kE * W; i += blockDim.x) (&bm[0][0])[i] = 0u;
  if (tid < kE) base[tid] = offsets[tid] + before[static_cast<int64_t>(blockIdx.x) * kE + tid];
  __syncthreads();
  for (int q = tid; q < nt * kTopK; q += blockDim.x) {
    const int e = idx[t0 * kTopK + q];
    if (static_cast<unsigned>(e) >= static_cast<unsigned>(kE)) continue;
    const int tl = q >> 3;
    atomicOr(&bm[e][tl >> 5], 1u << (tl & 31));
  }
  __syncthreads();
  for (int q = tid; q < nt * kTopK; q += blockDim.x) {
    const int e = idx[t0 * kTopK + q];
    if (static_cast<unsigned>(e) >= static_cast<unsigned>(kE)) {
      inv_perm[t0 * kTopK + q] = -1;  // an empty slot (or a bad id) has no row
      continue;
    }
    const int tl = q >> 3, w = tl >> 5;
    int rank = __popc(bm[e][w] & ((1u << (tl & 31)) - 1u));
    for (int v = 0; v < w; ++v) rank += __popc(bm[e][v]);
    const int64_t p = t0 * kTopK + q;
    const int r = base[e] + rank;
    perm_src[r] = static_cast<int32_t>(p);
    inv_perm[p] = r;
  }
}

}  // namespace moe
