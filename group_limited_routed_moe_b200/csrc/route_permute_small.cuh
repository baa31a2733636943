// route_permute_small.cuh -- steps 1 and 2 in one launch for small batches.
//
// For a few tokens (decode), routing and the counting sort are each a short
// chain of dependent instructions on one or two SMs, so a second launch and a
// round trip of the routing through global memory are a large part of their
// cost.  One block does both: each warp routes one token at a time, the block
// keeps every token's 8 expert ids in shared memory, and after one barrier the
// same block builds counts, offsets, perm_src and inv_perm from them.
//
// The routing rule and its decisions are those of route.cuh (same keys, same
// tie rules, the same float64 arithmetic for the group scores and weights, the
// weights summed over slots in the same order), so the ids and weights equal
// route_kernel's.  Only the work split differs: a whole warp per token, lane l
// owning experts 4l..4l+3 (group l/4), so that each of the 8 selection rounds
// is a 4-key scan and three warp reductions (redux.sync).  The sort is permute.cuh's
// bitmap counting sort with T <= 64 (two 32-token words per expert).
#pragma once
#include "common.cuh"
#include "permute.cuh"
#include "route.cuh"

namespace moe {

constexpr int kFusedRoutePermMaxT = 64;
constexpr int kFusedRoutePermThreads = 1024;

// Routes one token with the whole warp.  Lane k < 8 receives the k-th selected
// expert in sel and its combine weight in w (other lanes: sel = -1).  The
// token's logits are read from global memory, or (ROW_SMEM) from shared memory.
template <bool ROW_SMEM = false>
__device__ __forceinline__ void route_token_warp(const float* __restrict__ row,
                                                 const float* __restrict__ bias, int lane,
                                                 int& sel, float& w) {
  const unsigned FULL = 0xFFFFFFFFu;
  const float4 v = ROW_SMEM ? reinterpret_cast<const float4*>(row)[lane]
                            : __ldg(reinterpret_cast<const float4*>(row) + lane);
  const float4 b = bias != nullptr ? __ldg(reinterpret_cast<const float4*>(bias) + lane)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
  const float lg[4] = {v.x, v.y, v.z, v.w};
  const float bs[4] = {b.x, b.y, b.z, b.w};

  // keys, and this lane's two best scores
  unsigned long long key[4];
  unsigned long long k1 = 0ull, k2 = 0ull;
  float l1 = 0.f, b1 = 0.f, l2 = 0.f, b2 = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    key[i] = route_key_lb(lg[i], bs[i]);
    if (key[i] > k1) {
      k2 = k1;
      l2 = l1;
      b2 = b1;
      k1 = key[i];
      l1 = lg[i];
      b1 = bs[i];
    } else if (key[i] > k2) {
      k2 = key[i];
      l2 = lg[i];
      b2 = bs[i];
    }
  }
  double z1 = static_cast<double>(l1) + static_cast<double>(b1);
  double z2 = static_cast<double>(l2) + static_cast<double>(b2);
  // the group's two best scores: merge the top-2 lists of its 4 lanes
#pragma unroll
  for (int off = 1; off <= 2; off <<= 1) {
    const unsigned long long o1 = __shfl_xor_sync(FULL, k1, off);
    const unsigned long long o2 = __shfl_xor_sync(FULL, k2, off);
    const double oz1 = __shfl_xor_sync(FULL, z1, off);
    const double oz2 = __shfl_xor_sync(FULL, z2, off);
    if (o1 > k1) {
      if (k1 > o2) {
        k2 = k1;
        z2 = z1;
      } else {
        k2 = o2;
        z2 = oz2;
      }
      k1 = o1;
      z1 = oz1;
    } else if (o1 > k2) {
      k2 = o1;
      z2 = oz1;
    }
  }
  // Equal keys mean equal float64 sigmoids (see route.cuh), so every lane of
  // the group gets the same score whichever z it kept for a tied key.
  const double gscore = sigmoid_f64(z1) + sigmoid_f64(z2);
  const int g = lane >> 2;
  int rank = 0;
#pragma unroll
  for (int j = 0; j < kG; ++j) {
    const double gj = __shfl_sync(FULL, gscore, 4 * j);
    rank += (gj > gscore) || (gj == gscore && j < g);
  }
  if (rank >= kKeep) {
#pragma unroll
    for (int i = 0; i < 4; ++i) key[i] = 0ull;
  }

  sel = -1;
#pragma unroll 1
  for (int k = 0; k < kTopK; ++k) {
    unsigned long long bk = key[0];
    int bi = 0;
#pragma unroll
    for (int i = 1; i < 4; ++i) {
      if (key[i] > bk) {  // strict: keeps the lower index on exact ties
        bk = key[i];
        bi = i;
      }
    }
    // the warp's largest key, lowest expert id among equal keys: three
    // warp reductions (high word, low word among the lanes holding the
    // largest high word, expert id among the lanes holding the largest key)
    const uint32_t hi = static_cast<uint32_t>(bk >> 32), lo = static_cast<uint32_t>(bk);
    const uint32_t mh = __reduce_max_sync(FULL, hi);
    const uint32_t ml = __reduce_max_sync(FULL, hi == mh ? lo : 0u);
    const int be = static_cast<int>(__reduce_min_sync(
        FULL, (hi == mh && lo == ml) ? static_cast<uint32_t>(4 * lane + bi) : 0xFFFFFFFFu));
    if (lane == k) sel = be;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (4 * lane + i == be) key[i] = 0ull;
  }

  // weights over lanes 0..7 (slots), in route_kernel's order: r / sum r with
  // r = sigmoid(l) / sigmoid(m), m the largest chosen logit
  const double l =
      lane < kTopK ? static_cast<double>(ROW_SMEM ? row[sel] : __ldg(row + sel)) : 0.0;
  double m = l;
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) m = fmax(m, __shfl_xor_sync(FULL, m, off, 8));
  const double r = m >= 0.0 ? sigmoid_f64(l) / sigmoid_f64(m)
                            : exp(l - m) * (1.0 + exp(m)) / (1.0 + exp(l));
  double tot = r;
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) tot += __shfl_xor_sync(FULL, tot, off, 8);
  w = static_cast<float>(r / tot);
}

// The counting sort of a block's T <= 64 tokens (ids in sidx, bm zeroed, the
// caller's threads synchronised after writing sidx): counts, offsets (and the
// zeroed GEMM counters), perm_src and inv_perm, stable in token order.
__device__ __forceinline__ void sort_small_block(const int* sidx, int T, uint32_t (*bm)[2],
                                                 int* cnt, int* off, int32_t* __restrict__ counts,
                                                 int32_t* __restrict__ offsets,
                                                 int32_t* __restrict__ perm_src,
                                                 int32_t* __restrict__ inv_perm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = T * kTopK;
  for (int p = tid; p < n; p += blockDim.x) {
    const int e = sidx[p], t = p >> 3;
    atomicOr(&bm[e][t >> 5], 1u << (t & 31));
  }
  __syncthreads();
  if (tid < kE) cnt[tid] = __popc(bm[tid][0]) + __popc(bm[tid][1]);
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
    const int e = sidx[p], t = p >> 3, wd = t >> 5;
    const int r = off[e] + (wd ? __popc(bm[e][0]) : 0) +
                  __popc(bm[e][wd] & ((1u << (t & 31)) - 1u));
    perm_src[r] = p;
    inv_perm[p] = r;
  }
}

// T <= kFusedRoutePermMaxT tokens, one block of kFusedRoutePermThreads threads.
// Outputs as route_kernel followed by permute_small_kernel.
__global__ void __launch_bounds__(kFusedRoutePermThreads, 1)
    route_permute_small_kernel(const float* __restrict__ logits, const float* __restrict__ bias,
                               int T, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                               int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                               int32_t* __restrict__ perm_src, int32_t* __restrict__ inv_perm) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ int sidx[kFusedRoutePermMaxT * kTopK];
  __shared__ uint32_t bm[kE][2];  // bm[e][t / 32] bit t % 32: token t picked expert e
  __shared__ int cnt[kE];
  __shared__ int off[kE + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kE * 2; i += blockDim.x) (&bm[0][0])[i] = 0u;

  for (int t = warp; t < T; t += kFusedRoutePermThreads / 32) {
    int sel;
    float w;
    route_token_warp(logits + static_cast<int64_t>(t) * kE, bias, lane, sel, w);
    if (lane < kTopK) {
      topk_idx[t * kTopK + lane] = sel;
      topk_w[t * kTopK + lane] = w;
      sidx[t * kTopK + lane] = sel;
    }
  }
  __syncthreads();
  // counting sort of the T*8 items by expert, stable in token order
  sort_small_block(sidx, T, bm, cnt, off, counts, offsets, perm_src, inv_perm);
}

}  // namespace moe
