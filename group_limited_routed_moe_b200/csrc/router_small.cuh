// router_small.cuh -- the router projection, routing and the counting sort in
// one launch for the smallest batches (T <= kRouterFusedMaxT), so that a
// decode layer routed from its own activations costs no launch more than one
// given its logits.
//
//   logits[t][e] = sum_k x[t][k] W_router[k][e]   (bf16 in, fp32 accumulate)
// then steps 1 and 2 exactly as route_permute_small_kernel runs them.
//
// The projection is the step right before the group-limited routing kernel of
// the CUDA path ("Ling-3.0-tiny on a Qualcomm board", TensorFold issue #1247,
// "What it does not cover", first bullet).  At decode it is 128 x T dot
// products of length 1536 over 393 KB of router weights: too little work for
// the tensor cores' tile and too many bytes for one SM.  So one cluster of 8
// CTAs splits the experts (16 per CTA, 48 KB of weights each); every CTA
// computes its experts' logits for all tokens on the CUDA cores and stores
// them into the first CTA's shared memory through the cluster's distributed
// shared memory; after one cluster barrier that CTA routes and sorts exactly
// as route_permute_small_kernel does, reading the logits from its own shared
// memory.  Each logit is one warp's dot product in a fixed order (lane l sums
// 16-byte chunks l, l + 32, ... of the row in order, then a 5-level xor
// shuffle tree), so the result does not depend on T or on the work split.
// The router weights do not depend on the preceding kernel, so each CTA
// prefetches its slice into L2 before waiting for it.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"
#include "permute.cuh"
#include "route_permute_small.cuh"

namespace moe {
namespace rsmall {

constexpr int kCluster = 8;
constexpr int kExpertsPerCta = kE / kCluster;  // 16
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
// Above this many tokens the CUDA-core dot products cost more than the
// tensor-core router's launch (measured: the one-launch kernel takes 12.3 us
// at T = 1, 22.6 us at T = 16 and 57 us at T = 64, against 13.4 + 12.3 us for
// the router and routing kernels at any of them).
constexpr int kMaxT = 8;
constexpr int kChunks = kH * 2 / 16;        // 16-byte chunks per row: 192
constexpr int kChunksPerLane = kChunks / 32;  // 6

__device__ __forceinline__ float dot8_bf16(const uint4 a, const uint4 b, float acc) {
  const uint32_t pa[4] = {a.x, a.y, a.z, a.w};
  const uint32_t pb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc = fmaf(bf16_lo(pa[i]), bf16_lo(pb[i]), acc);
    acc = fmaf(bf16_hi(pa[i]), bf16_hi(pb[i]), acc);
  }
  return acc;
}

// One cluster of kCluster CTAs x kThreads threads.  logits_out (optional) gets
// the [T][128] fp32 logits; counts == nullptr skips the sort (routing only).
__global__ void __launch_bounds__(kThreads, 1)
    router_route_permute_small_kernel(const __nv_bfloat16* __restrict__ x,
                                      const __nv_bfloat16* __restrict__ packed_router,
                                      const float* __restrict__ bias, int T,
                                      float* __restrict__ logits_out,
                                      int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                                      int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                      int32_t* __restrict__ perm_src,
                                      int32_t* __restrict__ inv_perm) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int e0 = crank * kExpertsPerCta;

  // the leader's copy of all logits, T x 128 floats (dynamic: a few KB, so
  // that the cluster's CTAs fit beside a resident expert-FFN CTA)
  extern __shared__ __align__(16) float slog[];
  __shared__ int sidx[kMaxT * kTopK];
  __shared__ uint32_t bm[kE][2];
  __shared__ int cnt[kE];
  __shared__ int off[kE + 1];

  griddep_launch_dependents();
  {  // this CTA's 48 KB of router weights into L2 while the predecessor finishes
    const char* wbase = reinterpret_cast<const char*>(packed_router + static_cast<int64_t>(e0) * kH);
    constexpr int kLines = kExpertsPerCta * kH * 2 / 128;
    for (int i = tid; i < kLines; i += kThreads)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(wbase + 128 * i));
  }
  // every CTA of the cluster must be running before any stores into the
  // leader's shared memory: arrive now, wait just before the first store
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  griddep_wait();  // x comes from the preceding kernel

  // warp w: token (w / split) [+ kWarps / split for T > 32], experts of part (w % split)
  int split = 1;
  while (split < kExpertsPerCta && split * 2 * T <= kWarps) split *= 2;
  const int per = kExpertsPerCta / split;
  const int part = warp % split;
  float* leader = cluster.map_shared_rank(slog, 0);
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  for (int t = warp / split; t < T; t += kWarps / split) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * kH);
    uint4 xv[kChunksPerLane];
#pragma unroll
    for (int c = 0; c < kChunksPerLane; ++c) xv[c] = __ldg(xr + lane + 32 * c);
    for (int j = part * per; j < (part + 1) * per; ++j) {
      const int e = e0 + j;
      const uint4* wr = reinterpret_cast<const uint4*>(packed_router + static_cast<int64_t>(e) * kH);
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < kChunksPerLane; ++c) acc = dot8_bf16(xv[c], __ldg(wr + lane + 32 * c), acc);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
      if (lane == 0) {
        leader[t * kE + e] = acc;
        if (logits_out != nullptr) logits_out[static_cast<int64_t>(t) * kE + e] = acc;
      }
    }
  }
  cluster.sync();  // every CTA's logits are in the leader's shared memory
  if (crank != 0) return;

  for (int i = tid; i < kE * 2; i += kThreads) (&bm[0][0])[i] = 0u;
  for (int t = warp; t < T; t += kWarps) {
    int sel;
    float w;
    route_token_warp<true>(slog + t * kE, bias, lane, sel, w);
    if (lane < kTopK) {
      topk_idx[t * kTopK + lane] = sel;
      topk_w[t * kTopK + lane] = w;
      sidx[t * kTopK + lane] = sel;
    }
  }
  if (counts == nullptr) return;
  __syncthreads();
  sort_small_block(sidx, T, bm, cnt, off, counts, offsets, perm_src, inv_perm);
}

}  // namespace rsmall
}  // namespace moe
