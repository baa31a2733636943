// route.cuh -- step 1: group-limited top-8 routing, one warp per token.
//
// Layer facts: 128 experts in 8 groups of 16, 4 groups kept ("Ling-3.0-tiny
// on a Qualcomm board", TensorFold issue #1247, first comment, opening
// paragraph); 8 experts per token ("HelloSun/ling30tiny", table 模型與路由).
// Score rule: s = sigmoid(logit + bias); group score = sum of the group's two
// best s; keep the 4 best groups (ties to the lower group index); take the 8
// best s inside them (ties to the lower expert index) in descending order;
// weights sigmoid(logit) renormalised over the 8.
//
// The selection keys are float64, so that the decisions match a float64
// evaluation of the same rule (a near-tie would have to be closer than about
// 1e-16 to flip).  Lane l owns experts 4l..4l+3, so group j is lanes 4j..4j+3
// and the group top-2 merge needs two shuffles.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kRouteWarps = 8;  // tokens per block

__device__ __forceinline__ double sigmoid_f64(double z) { return 1.0 / (1.0 + exp(-z)); }

__global__ void __launch_bounds__(kRouteWarps * 32)
    route_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int64_t T,
                 int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  const unsigned FULL = 0xFFFFFFFFu;
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kRouteWarps + (threadIdx.x >> 5);
  if (t >= T) return;  // uniform per warp

  const float4 lg = __ldg(reinterpret_cast<const float4*>(logits + t * kE) + lane);
  float4 bs = make_float4(0.f, 0.f, 0.f, 0.f);
  if (bias != nullptr) bs = __ldg(reinterpret_cast<const float4*>(bias) + lane);

  double s[4];
  s[0] = sigmoid_f64(static_cast<double>(lg.x) + static_cast<double>(bs.x));
  s[1] = sigmoid_f64(static_cast<double>(lg.y) + static_cast<double>(bs.y));
  s[2] = sigmoid_f64(static_cast<double>(lg.z) + static_cast<double>(bs.z));
  s[3] = sigmoid_f64(static_cast<double>(lg.w) + static_cast<double>(bs.w));

  // top-2 values of the lane's four scores
  double a1 = fmax(s[0], s[1]), a2 = fmin(s[0], s[1]);
#pragma unroll
  for (int i = 2; i < 4; ++i) {
    if (s[i] > a1) {
      a2 = a1;
      a1 = s[i];
    } else if (s[i] > a2) {
      a2 = s[i];
    }
  }
  // merge with the other three lanes of the group
#pragma unroll
  for (int off = 1; off <= 2; off <<= 1) {
    const double b1 = __shfl_xor_sync(FULL, a1, off);
    const double b2 = __shfl_xor_sync(FULL, a2, off);
    if (a1 >= b1) {
      a2 = fmax(a2, b1);
    } else {
      a2 = fmax(b2, a1);
      a1 = b1;
    }
  }
  const double gscore = a1 + a2;
  const int my_group = lane >> 2;

  // rank of this lane's group among the 8 (ties: lower index ranks first)
  int rank = 0;
#pragma unroll
  for (int j = 0; j < kG; ++j) {
    const double gj = __shfl_sync(FULL, gscore, 4 * j);
    rank += (gj > gscore) || (gj == gscore && j < my_group);
  }
  const bool kept = rank < kKeep;

  // Candidates: kept experts' scores.  A score s lies in [0, 1], and the bit
  // pattern of a non-negative double orders exactly like its value, so the
  // key (hi word + 2^30, lo word) compares candidates exactly; 0 marks an
  // excluded or already-taken expert.  Each round takes the warp maximum of
  // the high words, then of the low words among lanes holding that high
  // word, then the lowest expert index among exact ties.
  uint32_t khi[4], klo[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(s[i]));
    khi[i] = kept ? static_cast<uint32_t>(b >> 32) + 0x40000000u : 0u;
    klo[i] = kept ? static_cast<uint32_t>(b) : 0u;
  }

  int sel = -1;  // lane k (k < 8) ends up holding the k-th selected expert
#pragma unroll 1
  for (int k = 0; k < kTopK; ++k) {
    // lane-local best (ties: lower index, i.e. first)
    uint32_t bh = khi[0], bl = klo[0];
    int bi = 0;
#pragma unroll
    for (int i = 1; i < 4; ++i) {
      if (khi[i] > bh || (khi[i] == bh && klo[i] > bl)) {
        bh = khi[i];
        bl = klo[i];
        bi = i;
      }
    }
    const uint32_t mh = __reduce_max_sync(FULL, bh);
    const uint32_t ml = __reduce_max_sync(FULL, bh == mh ? bl : 0u);
    const bool mine = (bh == mh) && (bl == ml);
    const uint32_t be = __reduce_min_sync(FULL, mine ? static_cast<uint32_t>(4 * lane + bi) : 0xFFFFFFFFu);
    if (lane == k) sel = static_cast<int>(be);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (static_cast<uint32_t>(4 * lane + i) == be) khi[i] = klo[i] = 0u;
  }

  // combine weights: sigmoid of the raw logit, renormalised over the 8
  double sig = 0.0;
  if (lane < kTopK) sig = sigmoid_f64(static_cast<double>(__ldg(logits + t * kE + sel)));
  double tot = sig;
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) tot += __shfl_xor_sync(FULL, tot, off);
  if (lane < kTopK) {
    topk_idx[t * kTopK + lane] = sel;
    topk_w[t * kTopK + lane] = static_cast<float>(sig / tot);
  }
}

}  // namespace moe
