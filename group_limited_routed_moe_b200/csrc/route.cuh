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

  // candidates: scores of kept experts, -1 (below any sigmoid) otherwise
  double c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = kept ? s[i] : -1.0;

  int sel = -1;  // lane k (k < 8) ends up holding the k-th selected expert
#pragma unroll 1
  for (int k = 0; k < kTopK; ++k) {
    double bv = c[0];
    int bi = 0;
#pragma unroll
    for (int i = 1; i < 4; ++i) {
      if (c[i] > bv) {
        bv = c[i];
        bi = i;
      }
    }
    int be = 4 * lane + bi;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const double ov = __shfl_xor_sync(FULL, bv, off);
      const int oe = __shfl_xor_sync(FULL, be, off);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if (lane == k) sel = be;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (be == 4 * lane + i) c[i] = -2.0;
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
