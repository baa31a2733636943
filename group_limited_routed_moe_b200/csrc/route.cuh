// route.cuh -- step 1: group-limited top-8 routing.
//
// Layer facts: 128 experts in 8 groups of 16, 4 groups kept ("Ling-3.0-tiny
// on a Qualcomm board", TensorFold issue #1247, first comment, opening
// paragraph); 8 experts per token ("HelloSun/ling30tiny", table 模型與路由).
// Score rule: s = sigmoid(logit + bias); group score = sum of the group's two
// best s; keep the 4 best groups (ties to the lower group index); take the 8
// best s inside them (ties to the lower expert index) in descending order;
// weights sigmoid(logit) renormalised over the 8.
//
// Eight lanes route one token (four tokens per warp): lane g of the segment
// owns group g, so the group's top-2 is lane-local, the group ranking is eight
// segment shuffles, and each of the 8 selection rounds is a lane-local scan
// plus three shuffle levels.
//
// The sigmoid is strictly increasing, so "the two largest s of a group" and
// "the 8 largest s among kept experts" are decided on z = logit + bias (float64)
// instead of on s: this is the exact order of the scores.  A float64 sigmoid
// can only add ties, between two z closer than about one ulp of s divided by
// s'(z); such a pair has a float64 score margin of at most an ulp, the same
// size as the difference between two float64 exp implementations.  Where s
// saturates to 1 (z > 10) or underflows (z < -700), many z share one float64
// s, so there the key is the float64 sigmoid itself, in a tier that sorts
// above or below the middle one, and those ties are exactly the float64 ones.
// Only the 2 best scores of each group (the group score) and the 8 chosen
// experts' weights need a float64 sigmoid: 24 per token, not 136.
// Keys are unsigned 64-bit integers; 0 marks an excluded or taken expert.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kRouteTokensPerWarp = 4;
constexpr int kRouteWarps = 8;
constexpr int kRouteTokensPerBlock = kRouteTokensPerWarp * kRouteWarps;  // 32

__device__ __forceinline__ double sigmoid_f64(double z) { return 1.0 / (1.0 + exp(-z)); }

// Order-preserving 64-bit key of a score given its z (see above); always >= 1.
__device__ __forceinline__ unsigned long long route_key(double z) {
  if (z > 10.0) {  // s in (0.99995, 1]: float64 sigmoid bits, above every middle key
    const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(sigmoid_f64(z)));
    return 0xD000000000000000ull + (b - 0x3FE0000000000000ull);
  }
  if (z < -700.0)  // s below 1e-304: float64 sigmoid bits (may be 0), below every middle key
    return static_cast<unsigned long long>(__double_as_longlong(sigmoid_f64(z))) + 1ull;
  // middle: z itself, mapped to unsigned order (negative doubles bit-flipped)
  const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(z));
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// Order bits of an fp32 value: unsigned order equals the value order (for
// non-NaN values; +0 and -0 differ, which the caller removes).
__device__ __forceinline__ uint32_t ord32(float x) {
  const uint32_t b = __float_as_uint(x);
  return (b >> 31) ? ~b : (b | 0x80000000u);
}

// The middle tier's key of a float64 z in [-700, 10] as two fp32 words: the
// pair (s, r) = (fl32(z), z - fl32(z)) represents z exactly (r is an fp32
// value: see route_key_lb), and s ordered first, then r, is z's order.  -0 is
// made +0 first (z = -0 and z = +0 are one score).  These keys lie between
// ord32(-700) << 32 and ord32(10) << 32 | 0xFFFFFFFF, inside route_key's
// middle range, so they sort against its tier keys as its own middle keys do.
__device__ __forceinline__ unsigned long long middle_key(float s, float r) {
  return (static_cast<unsigned long long>(ord32(__fadd_rn(s, 0.f))) << 32) |
         ord32(__fadd_rn(r, 0.f));
}

// route_key for z = l + b, the float64 sum of an fp32 logit and bias, giving
// every z the same order as route_key(z) without float64 arithmetic in the
// usual case.  Knuth's two-sum gives s = fl32(l + b) and e = (l + b) - s, both
// fp32 and exact.  When the exponents of s and e are less than 30 apart, l + b
// has at most 53 significant bits, so the float64 sum is s + e exactly and
// (s, e) is middle_key's pair.  Otherwise (a bias or logit more than 2^29
// times smaller than the other) the float64 sum rounds, and the key is taken
// from that sum: its pair (fl32(z), z - fl32(z)) is still exact, because z -
// fl32(z) is then the smaller operand cut to the float64 grid, at most 24
// significant bits.  The tiers (z > 10, z < -700) and a NaN take route_key.
__device__ __forceinline__ unsigned long long route_key_lb(float l, float b) {
  const float s = __fadd_rn(l, b);
  const float bb = __fsub_rn(s, l);
  const float e = __fadd_rn(__fsub_rn(l, __fsub_rn(s, bb)), __fsub_rn(b, bb));
  const int gap = static_cast<int>((__float_as_uint(s) >> 23) & 0xFFu) -
                  static_cast<int>((__float_as_uint(e) >> 23) & 0xFFu);
  if ((e == 0.f || gap < 30) && s > -700.f && s < 10.f) return middle_key(s, e);
  const double z = static_cast<double>(l) + static_cast<double>(b);
  if (!(z >= -700.0 && z <= 10.0)) return route_key(z);  // tiers and NaN
  const float s64 = static_cast<float>(z);
  return middle_key(s64, static_cast<float>(z - static_cast<double>(s64)));
}

__global__ void __launch_bounds__(kRouteWarps * 32)
    route_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int64_t T,
                 int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  const unsigned FULL = 0xFFFFFFFFu;
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int g = lane & 7;  // group owned by this lane; also its slot in the segment
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kRouteTokensPerBlock +
                    (threadIdx.x >> 5) * kRouteTokensPerWarp + (lane >> 3);
  const bool active = t < T;  // the whole segment agrees; inactive lanes still shuffle

  // this lane's 16 logits and biases (the segment reads the token's 512 bytes)
  float lg[16], bs[16];
  {
    const float4* src = reinterpret_cast<const float4*>(logits + (active ? t : 0) * kE + g * kGS);
    const float4* bsrc = reinterpret_cast<const float4*>(bias + g * kGS);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = __ldg(src + q);
      lg[4 * q] = v.x;
      lg[4 * q + 1] = v.y;
      lg[4 * q + 2] = v.z;
      lg[4 * q + 3] = v.w;
      const float4 b = bias != nullptr ? __ldg(bsrc + q) : make_float4(0.f, 0.f, 0.f, 0.f);
      bs[4 * q] = b.x;
      bs[4 * q + 1] = b.y;
      bs[4 * q + 2] = b.z;
      bs[4 * q + 3] = b.w;
    }
  }

  // keys, and the group's two best scores (found on the keys, evaluated in float64)
  unsigned long long key[16];
  unsigned long long k1 = 0ull, k2 = 0ull;
  float l1 = 0.f, b1 = 0.f, l2 = 0.f, b2 = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
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
  const double z1 = static_cast<double>(l1) + static_cast<double>(b1);
  const double z2 = static_cast<double>(l2) + static_cast<double>(b2);
  const double gscore = sigmoid_f64(z1) + sigmoid_f64(z2);

  // rank of this group among the token's 8 (ties: lower index ranks first)
  int rank = 0;
#pragma unroll
  for (int j = 0; j < kG; ++j) {
    const double gj = __shfl_sync(FULL, gscore, j, 8);
    rank += (gj > gscore) || (gj == gscore && j < g);
  }
  if (rank >= kKeep) {
#pragma unroll
    for (int i = 0; i < 16; ++i) key[i] = 0ull;
  }

  int sel = -1;  // segment lane k ends up holding the k-th selected expert
#pragma unroll 1
  for (int k = 0; k < kTopK; ++k) {
    unsigned long long bk = key[0];
    int bi = 0;
#pragma unroll
    for (int i = 1; i < 16; ++i) {
      if (key[i] > bk) {  // strict: keeps the lower index on exact ties
        bk = key[i];
        bi = i;
      }
    }
    int be = g * kGS + bi;
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1) {
      const unsigned long long ok = __shfl_xor_sync(FULL, bk, off, 8);
      const int oe = __shfl_xor_sync(FULL, be, off, 8);
      if (ok > bk || (ok == bk && oe < be)) {
        bk = ok;
        be = oe;
      }
    }
    if (g == k) sel = be;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (g * kGS + i == be) key[i] = 0ull;
  }

  // combine weights: sigmoid of the raw logit, renormalised over the 8, as
  // r / sum r with r = sigmoid(l) / sigmoid(m), m the largest chosen logit;
  // for m < 0, r = exp(l - m) (1 + exp(m)) / (1 + exp(l)) keeps the ratio
  // finite when every sigmoid underflows.
  const double l = active ? static_cast<double>(__ldg(logits + t * kE + sel)) : 0.0;
  double m = l;
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) m = fmax(m, __shfl_xor_sync(FULL, m, off, 8));
  const double r = m >= 0.0 ? sigmoid_f64(l) / sigmoid_f64(m)
                            : exp(l - m) * (1.0 + exp(m)) / (1.0 + exp(l));
  double tot = r;
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) tot += __shfl_xor_sync(FULL, tot, off, 8);
  if (active) {
    topk_idx[t * kTopK + g] = sel;
    topk_w[t * kTopK + g] = static_cast<float>(r / tot);
  }
}

}  // namespace moe
