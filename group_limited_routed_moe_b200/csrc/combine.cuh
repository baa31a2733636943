// combine.cuh -- step 4: weighted combine of the 8 expert outputs of every
// token, back in token order.
//
// out[t] = bf16( residual[t] + sum_{slot} w[t,slot] * y_perm[inv_perm[8t+slot]]
//                 + sum_{s < n_shared} y_shared[s*T + t] )
// with y_perm and y_shared in fp16 (the down GEMMs' outputs) and the residual
// in bf16; the shared experts' rows (weight 1) follow the routed slots.
// The "real MoE routing + weighted layer" of "HelloSun/ling30tiny" (section
// 數值檢查摘要) is this sum.  It is done in gather form: each token reads its 8
// rows, adds them in fp32 in slot order and rounds once, so the result is
// deterministic (no atomics) and independent of how tokens are ordered.
// One thread owns 8 consecutive columns (one 16-byte vector) of one token.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kCombineThreads = kH / 8;  // 192

// The combine run at the end of a single-launch expert FFN by the CTA that
// retires last, in place of a combine launch: up to kFusedCombineMaxT tokens.
// One token's 192 output vectors are one pass of one CTA, and the layer is
// about 1 us faster than with the combine launch; two tokens (two passes)
// measured slower than the launch.  y_perm is segment 0's y rows, the shared
// rows (n_shared > 0) segment 1's.  out == nullptr: no combine in the launch.
constexpr int kFusedCombineMaxT = 1;
struct FusedCombine {
  const float* topk_w;
  const int32_t* inv_perm;
  const __nv_bfloat16* residual;
  __nv_bfloat16* out;
  int n_shared;
};

// out[t][col .. col + 7] for token t (one thread, one 16-byte vector), the
// arithmetic of the whole file comment.  NS: slots a token uses (8, or 6 in the
// 256-expert shape); topk_w has NS entries per token, inv_perm always kTopK
// (slots NS .. 7 unused).  L2_ONLY: y_perm was written by the calling kernel
// itself (and so were the shared rows), so both are read around the
// non-coherent cache.
template <int NS, bool L2_ONLY = false>
__device__ __forceinline__ void combine_token_vec(const uint16_t* __restrict__ y_perm,
                                                  const float* __restrict__ topk_w,
                                                  const int32_t* __restrict__ inv_perm, int64_t T,
                                                  int64_t t, int col, const __nv_bfloat16* residual,
                                                  __nv_bfloat16* out,
                                                  const uint16_t* __restrict__ y_shared,
                                                  int n_shared) {
  const int64_t nrows = T * kTopK;
  uint4 v[NS];
  float w[NS];
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    const int64_t r = __ldg(inv_perm + t * kTopK + s);
    w[s] = __ldg(topk_w + t * NS + s);
    if (r >= 0 && r < nrows) {
      const uint4* src = reinterpret_cast<const uint4*>(y_perm + r * kH + col);
      v[s] = L2_ONLY ? __ldcg(src) : __ldg(src);
    } else {
      v[s] = make_uint4(0u, 0u, 0u, 0u);
      w[s] = 0.f;
    }
  }
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    const uint32_t q[4] = {v[s].x, v[s].y, v[s].z, v[s].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = fmaf(w[s], f16_lo(q[i]), acc[2 * i]);
      acc[2 * i + 1] = fmaf(w[s], f16_hi(q[i]), acc[2 * i + 1]);
    }
  }
  for (int s = 0; s < n_shared; ++s) {
    const uint4* src = reinterpret_cast<const uint4*>(y_shared + (s * T + t) * kH + col);
    const uint4 sv = L2_ONLY ? __ldcg(src) : __ldg(src);
    const uint32_t q[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += f16_lo(q[i]);
      acc[2 * i + 1] += f16_hi(q[i]);
    }
  }
  if (residual != nullptr) {
    const uint4 rv = *reinterpret_cast<const uint4*>(residual + t * kH + col);
    const uint32_t q[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += bf16_lo(q[i]);
      acc[2 * i + 1] += bf16_hi(q[i]);
    }
  }
  uint4 o;
  o.x = pack_bf16x2(acc[0], acc[1]);
  o.y = pack_bf16x2(acc[2], acc[3]);
  o.z = pack_bf16x2(acc[4], acc[5]);
  o.w = pack_bf16x2(acc[6], acc[7]);
  *reinterpret_cast<uint4*>(out + t * kH + col) = o;
}

template <int NS>
__global__ void __launch_bounds__(kCombineThreads)
    combine_kernel(const uint16_t* __restrict__ y_perm, const float* __restrict__ topk_w,
                   const int32_t* __restrict__ inv_perm, int64_t T,
                   const __nv_bfloat16* residual, __nv_bfloat16* out,
                   const uint16_t* __restrict__ y_shared, int n_shared) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t t = blockIdx.x;
  if (t >= T) return;
  combine_token_vec<NS>(y_perm, topk_w, inv_perm, T, t, threadIdx.x * 8, residual, out,
                        y_shared, n_shared);
}

}  // namespace moe

namespace moe {

// The shared experts' row set: every token is one row of every shared expert,
// expert s (< n_shared) owning rows s*T .. s*T + T-1 in token order, in the
// offsets / perm_src form of the routed permutation (perm_src = 8t: token t,
// slot 0).  Also zeroes the work counters offsets[129 ..] of the expert FFN.
__global__ void __launch_bounds__(256)
    shared_rows_kernel(int64_t T, int n_shared, int32_t* __restrict__ offsets,
                       int32_t* __restrict__ perm_src) {
  griddep_launch_dependents();
  griddep_wait();
  const int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
  if (i < kOffsetsLen)
    offsets[i] = i <= kE ? static_cast<int32_t>(T * (i < n_shared ? i : n_shared)) : 0;
  if (i < n_shared * T) perm_src[i] = static_cast<int32_t>((i % T) * kTopK);
}

}  // namespace moe
