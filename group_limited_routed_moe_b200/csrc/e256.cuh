// e256.cuh -- routing and row permutation for the second MoE shape: 256
// experts top-6 ("Add TML Inkling architecture", llama.cpp PR #25731, model
// description: "256 experts top-6 plus 2 shared").  The pages give no group
// structure for it; tiny's rule is scaled to 8 groups of 32 experts, 4 kept.
// Scores, ties and combine weights follow route.cuh (same keys, same shifted
// weight ratio).
//
// The expert FFN of this shape reuses the 128-expert grouped kernels
// unchanged, on two packs (experts 0..127 and 128..255): the permutation below
// is one stable counting sort over all 256 experts, and each half gets its own
// 264-word offsets array whose 129 offsets are absolute rows of the shared
// perm_src / h / y_perm buffers.  Items keep the 8-slot numbering t*8 + slot
// of the 128-expert path (slots 6 and 7 unused), so the kernels' token index
// perm_src >> 3 and the combine's inv_perm stride stay as they are.
#pragma once
#include "common.cuh"
#include "permute.cuh"
#include "route.cuh"

namespace moe {
namespace e256 {

constexpr int kE2 = 256, kG2 = 8, kGS2 = 32, kKeep2 = 4, kTopK2 = 6;
constexpr int kPerLane = kE2 / 32;        // 8 experts per lane, 4 lanes per group
constexpr int kBlockTokens = 128;         // tokens per block of the counting sort
constexpr int kRouteWarps2 = 8;           // tokens (warps) per route block

// Routes one token with the whole warp.  Lane l owns experts 8l .. 8l+7
// (group l / 4); lane k < 6 receives the k-th chosen expert in sel and its
// combine weight in w (other lanes: sel = -1, w = 0).
__device__ __forceinline__ void route_token_e256(const float* __restrict__ row,
                                                 const float* __restrict__ bias, int lane,
                                                 int& sel, float& w) {
  const unsigned FULL = 0xFFFFFFFFu;
  const int grp = lane >> 2;
  float lg[kPerLane], bs[kPerLane];
  {
    const float4* src = reinterpret_cast<const float4*>(row + kPerLane * lane);
    const float4* bsrc = reinterpret_cast<const float4*>(bias + kPerLane * lane);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float4 v = __ldg(src + q);
      lg[4 * q] = v.x; lg[4 * q + 1] = v.y; lg[4 * q + 2] = v.z; lg[4 * q + 3] = v.w;
      const float4 b = bias != nullptr ? __ldg(bsrc + q) : make_float4(0.f, 0.f, 0.f, 0.f);
      bs[4 * q] = b.x; bs[4 * q + 1] = b.y; bs[4 * q + 2] = b.z; bs[4 * q + 3] = b.w;
    }
  }
  // keys, and this lane's two best (key, z)
  unsigned long long key[kPerLane];
  unsigned long long k1 = 0ull, k2 = 0ull;
  float l1 = 0.f, b1 = 0.f, l2 = 0.f, b2 = 0.f;
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    key[i] = route_key_lb(lg[i], bs[i]);
    if (key[i] > k1) {
      k2 = k1; l2 = l1; b2 = b1; k1 = key[i]; l1 = lg[i]; b1 = bs[i];
    } else if (key[i] > k2) {
      k2 = key[i]; l2 = lg[i]; b2 = bs[i];
    }
  }
  double z1 = static_cast<double>(l1) + static_cast<double>(b1);
  double z2 = static_cast<double>(l2) + static_cast<double>(b2);
  // the group's two best over its 4 lanes
#pragma unroll
  for (int off = 1; off <= 2; off <<= 1) {
    const unsigned long long o1 = __shfl_xor_sync(FULL, k1, off);
    const unsigned long long o2 = __shfl_xor_sync(FULL, k2, off);
    const double y1 = __shfl_xor_sync(FULL, z1, off);
    const double y2 = __shfl_xor_sync(FULL, z2, off);
    // merge the sorted pairs (k1 >= k2) and (o1 >= o2)
    if (o1 > k1) {
      if (k1 > o2) { k2 = k1; z2 = z1; } else { k2 = o2; z2 = y2; }
      k1 = o1; z1 = y1;
    } else if (o1 > k2) {
      k2 = o1; z2 = y1;
    }
  }
  const double gscore = sigmoid_f64(z1) + sigmoid_f64(z2);
  // rank of this lane's group among the 8 (ties: lower index first)
  int rank = 0;
#pragma unroll
  for (int j = 0; j < kG2; ++j) {
    const double gj = __shfl_sync(FULL, gscore, 4 * j);
    rank += (gj > gscore) || (gj == gscore && j < grp);
  }
  if (rank >= kKeep2) {
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) key[i] = 0ull;
  }
  sel = -1;  // lane k ends up holding the k-th chosen expert
#pragma unroll 1
  for (int k = 0; k < kTopK2; ++k) {
    unsigned long long bk = key[0];
    int bi = 0;
#pragma unroll
    for (int i = 1; i < kPerLane; ++i)
      if (key[i] > bk) { bk = key[i]; bi = i; }  // strict: lower index on ties
    // the warp's largest key, lowest expert id among equal keys (three warp
    // reductions, as in route_token_warp)
    const uint32_t hi = static_cast<uint32_t>(bk >> 32), lo = static_cast<uint32_t>(bk);
    const uint32_t mh = __reduce_max_sync(FULL, hi);
    const uint32_t ml = __reduce_max_sync(FULL, hi == mh ? lo : 0u);
    const int be = static_cast<int>(__reduce_min_sync(
        FULL, (hi == mh && lo == ml) ? static_cast<uint32_t>(kPerLane * lane + bi) : 0xFFFFFFFFu));
    if (lane == k) sel = be;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i)
      if (kPerLane * lane + i == be) key[i] = 0ull;
  }
  // combine weights over the 6 chosen, as route.cuh
  const bool mine = lane < kTopK2;
  const double l = mine ? static_cast<double>(__ldg(row + sel)) : -INFINITY;
  double m = l;
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) m = fmax(m, __shfl_xor_sync(FULL, m, off));
  double r = 0.0;
  if (mine)
    r = m >= 0.0 ? sigmoid_f64(l) / sigmoid_f64(m) : exp(l - m) * (1.0 + exp(m)) / (1.0 + exp(l));
  double tot = r;
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) tot += __shfl_xor_sync(FULL, tot, off);
  w = mine ? static_cast<float>(r / tot) : 0.f;
}

// One warp per token.
__global__ void __launch_bounds__(kRouteWarps2 * 32)
    route_e256_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
                      int64_t T, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kRouteWarps2 + (threadIdx.x >> 5);
  if (t >= T) return;  // whole warp
  int sel;
  float w;
  route_token_e256(logits + t * kE2, bias, lane, sel, w);
  if (lane < kTopK2) {
    topk_idx[t * kTopK2 + lane] = sel;
    topk_w[t * kTopK2 + lane] = w;
  }
}

// Writes the two halves' 264-word offsets arrays from the 257 expert offsets
// (absolute rows; work counters zeroed).  Thread e < 256 of the block.
__device__ __forceinline__ void write_halves(int e, const int* off, int32_t* __restrict__ off_lo,
                                             int32_t* __restrict__ off_hi) {
  const int half = e >> 7, j = e & 127;
  int32_t* dst = half ? off_hi : off_lo;
  dst[j] = off[e];
  if (j == 127) dst[128] = off[e + 1];
  for (int i = 129 + j; i < kOffsetsLen; i += 128) dst[i] = 0;
}

// Small batches (T <= kSmallMaxT): routing and the counting sort in one block,
// as route_permute_small_kernel does for 128 experts.  Each warp routes a token
// at a time; the block keeps every token's 6 expert ids in shared memory,
// builds a 64-token bitmap per expert, counts, scans and scatters.  Outputs as
// route_e256_kernel followed by the three counting-sort kernels.
constexpr int kSmallMaxT = 64;
constexpr int kSmallThreads = 512;
__global__ void __launch_bounds__(kSmallThreads, 1)
    route_sort_small_e256_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
                                 int T, int32_t* __restrict__ topk_idx,
                                 float* __restrict__ topk_w, int32_t* __restrict__ counts,
                                 int32_t* __restrict__ offsets, int32_t* __restrict__ off_lo,
                                 int32_t* __restrict__ off_hi, int32_t* __restrict__ perm_src,
                                 int32_t* __restrict__ inv_perm) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ int sidx[kSmallMaxT * kTopK2];
  __shared__ uint32_t bm[kE2][2];  // bm[e][t / 32] bit t % 32: token t chose expert e
  __shared__ int wsum[kE2 / 32];
  __shared__ int off[kE2 + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kE2 * 2; i += blockDim.x) (&bm[0][0])[i] = 0u;
  for (int t = warp; t < T; t += kSmallThreads / 32) {
    int sel;
    float w;
    route_token_e256(logits + static_cast<int64_t>(t) * kE2, bias, lane, sel, w);
    if (lane < kTopK2) {
      topk_idx[t * kTopK2 + lane] = sel;
      topk_w[t * kTopK2 + lane] = w;
      sidx[t * kTopK2 + lane] = sel;
    }
  }
  __syncthreads();
  for (int p = tid; p < T * kTopK2; p += blockDim.x) {
    const int e = sidx[p], t = p / kTopK2;
    atomicOr(&bm[e][t >> 5], 1u << (t & 31));
  }
  __syncthreads();
  // counts and their exclusive scan over the 256 experts (threads 0..255)
  int c = 0, incl = 0;
  if (tid < kE2) {
    c = __popc(bm[tid][0]) + __popc(bm[tid][1]);
    incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
  }
  __syncthreads();
  if (tid < kE2) {
    int base = 0;
    for (int j = 0; j < warp; ++j) base += wsum[j];
    off[tid] = base + incl - c;
    if (tid == kE2 - 1) off[kE2] = base + incl;
    counts[tid] = c;
  }
  __syncthreads();
  if (tid < kE2) {
    offsets[tid] = off[tid];
    if (tid == kE2 - 1) offsets[kE2] = off[kE2];
    write_halves(tid, off, off_lo, off_hi);
  }
  // rows: the 8-slot numbering t*8 + slot (slots 6 and 7 unused)
  for (int p = tid; p < T * kTopK; p += blockDim.x) {
    const int t = p >> 3, slot = p & 7;
    if (slot >= kTopK2) {
      inv_perm[p] = -1;
      continue;
    }
    const int e = sidx[t * kTopK2 + slot], wd = t >> 5;
    const int r = off[e] + (wd ? __popc(bm[e][0]) : 0) +
                  __popc(bm[e][wd] & ((1u << (t & 31)) - 1u));
    perm_src[r] = p;
    inv_perm[p] = r;
  }
}

// Counting sort, pass 1: per block of 128 tokens, the rows each expert gets.
__global__ void __launch_bounds__(256)
    count_e256_kernel(const int32_t* __restrict__ idx, int64_t T, int32_t* __restrict__ hist) {
  __shared__ int cnt[kE2];
  griddep_launch_dependents();
  griddep_wait();
  cnt[threadIdx.x] = 0;
  __syncthreads();
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kBlockTokens;
  for (int i = threadIdx.x; i < kBlockTokens * kTopK2; i += blockDim.x) {
    const int64_t t = t0 + i / kTopK2;
    if (t < T) {
      const int e = idx[t * kTopK2 + i % kTopK2];
      if (e >= 0 && e < kE2) atomicAdd(&cnt[e], 1);
      else record_status(kSiteBadIndex);
    }
  }
  __syncthreads();
  hist[static_cast<int64_t>(blockIdx.x) * kE2 + threadIdx.x] = cnt[threadIdx.x];
}

// Pass 2 (one block, a thread per expert): expert offsets, each block's first
// row for each expert (in place of its count), and the two halves' 264-word
// offsets arrays (work counters zeroed).
__global__ void __launch_bounds__(256)
    scan_e256_kernel(int32_t* __restrict__ hist, int nb, int32_t* __restrict__ counts,
                     int32_t* __restrict__ offsets, int32_t* __restrict__ off_lo,
                     int32_t* __restrict__ off_hi) {
  __shared__ int wsum[8];
  griddep_launch_dependents();
  griddep_wait();
  const int e = threadIdx.x, lane = e & 31, w = e >> 5;
  int c = 0, unused = 0;
  hist_column_sum(hist, kE2, e, 0, nb, 1, 0, c, unused);
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[w] = incl;
  __syncthreads();
  int base = 0;
  for (int j = 0; j < w; ++j) base += wsum[j];
  const int start = base + incl - c;  // exclusive prefix
  counts[e] = c;
  offsets[e] = start;
  if (e == kE2 - 1) offsets[kE2] = start + c;
  hist_column_exclusive(hist, kE2, e, 0, nb, start);
  // halves: absolute rows, then zeroed work counters
  const int half = e >> 7, j = e & 127;
  int32_t* dst = half ? off_hi : off_lo;
  dst[j] = start;
  if (j == 127) dst[128] = start + c;
  for (int i = 129 + j; i < kOffsetsLen; i += 128) dst[i] = 0;
}

// Pass 3: rows.  Items of one block go to their expert's rows in token order:
// the rank of token t among the block's tokens that chose e is the number of
// bits below t in e's 128-bit token bitmap.
__global__ void __launch_bounds__(256)
    scatter_e256_kernel(const int32_t* __restrict__ idx, int64_t T,
                        const int32_t* __restrict__ hist, int32_t* __restrict__ perm_src,
                        int32_t* __restrict__ inv_perm) {
  __shared__ uint32_t bits[kE2][kBlockTokens / 32];
  griddep_launch_dependents();
  griddep_wait();
  for (int i = threadIdx.x; i < kE2 * (kBlockTokens / 32); i += blockDim.x)
    (&bits[0][0])[i] = 0u;
  __syncthreads();
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kBlockTokens;
  for (int i = threadIdx.x; i < kBlockTokens * kTopK2; i += blockDim.x) {
    const int tl = i / kTopK2;
    const int64_t t = t0 + tl;
    if (t < T) {
      const int e = idx[t * kTopK2 + i % kTopK2];
      if (e >= 0 && e < kE2) atomicOr(&bits[e][tl >> 5], 1u << (tl & 31));
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kBlockTokens * kTopK; i += blockDim.x) {
    const int tl = i / kTopK, slot = i % kTopK;
    const int64_t t = t0 + tl;
    if (t >= T) continue;
    if (slot >= kTopK2) {  // slots 6 and 7 of the 8-slot numbering are unused
      inv_perm[t * kTopK + slot] = -1;
      continue;
    }
    const int e = idx[t * kTopK2 + slot];
    if (e < 0 || e >= kE2) continue;
    int rank = __popc(bits[e][tl >> 5] & ((1u << (tl & 31)) - 1u));
    for (int q = 0; q < (tl >> 5); ++q) rank += __popc(bits[e][q]);
    const int row = hist[static_cast<int64_t>(blockIdx.x) * kE2 + e] + rank;
    perm_src[row] = static_cast<int32_t>(t * kTopK + slot);
    inv_perm[t * kTopK + slot] = row;
  }
}

}  // namespace e256
}  // namespace moe
