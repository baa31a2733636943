// fp8.cuh -- block-FP8 expert weights: packing, dequantisation arithmetic and
// the expansion of a packed FP8 layer into the bf16/fp16 packed layout.
//
// The CUDA path of "Ling-3.0-tiny on a Qualcomm board" (TensorFold issue
// #1247, first comment, "What it does not cover", third bullet) reads experts
// in bf16, block FP8 and NVFP4.  Block FP8 here: every weight an FP8 E4M3 code,
// every 128 x 128 block of a matrix one fp32 scale, weight = value(code) *
// scale.  The kernels dequantise a weight as fp32(value(code) * scale) rounded
// once to the MMA operand type: bf16 for gate/up, fp16 for down.  An E4M3 value
// has 4 significant bits, so with a power-of-two scale the product is exact in
// fp32 and again in bf16 (same exponent range) or fp16 (when it lies in the
// fp16 range; the pack kernel checks), and the layer computes exactly what the
// bf16 layer computes on the dequantised weights.
//
// Two dequantisation routes, chosen per 128 x 128 block:
//   - power-of-two scale (the UE8M0-style scales of current block-FP8
//     checkpoints): the operand bits are assembled from the code bits with
//     integer operations (3.5 per pair of codes) and one packed 16-bit
//     multiply by the scale rescales them; exact, and no conversion
//     instruction is involved (those run on a quarter-rate pipe that bounds
//     a converter otherwise);
//   - any other fp32 scale: hardware E4M3 -> fp16 conversion, fp32 multiply,
//     rounding to the operand type.
// Both give fp32(value * scale) rounded once, so the choice never changes a
// result.
//
// Packed FP8 layer (bytes, every region 128-byte aligned):
//   GU8 [128 experts][1024 rows][1536]  codes, rows as in the bf16 pack: row
//                                       256j + r is gate column 128j + r (r < 128)
//                                       or up column 128j + r - 128
//   D8  [128][1536 rows][512]           codes, row n = output column n of W_down
// Inside every aligned group of 4 codes along k the bytes hold the elements in
// the order (k+2, k, k+3, k+1): the integer route then yields the operand
// pairs (k, k+1) and (k+2, k+3) from bytes (1, 3) and (0, 2) directly.
//   SGU [128][4 (j)][2 (gate, up)][12 (k block)]  fp32 scales, GEMM order
//   SD  [128][12 (n block)][4 (k block)]          fp32 scales
#pragma once
#include <cuda_fp8.h>

#include "common.cuh"
#include "pack.cuh"

namespace moe {
namespace fp8 {

constexpr int kBlk = 128;
constexpr int64_t kGuBytes = int64_t(kE) * 1024 * kH;
constexpr int64_t kDBytes = int64_t(kE) * kH * kI;
constexpr int kSguPerExpert = (kI / kBlk) * 2 * (kH / kBlk);  // 96
constexpr int kSdPerExpert = (kH / kBlk) * (kI / kBlk);       // 48
constexpr int64_t kSguOff = kGuBytes + kDBytes;
constexpr int64_t kSdOff = kSguOff + int64_t(kE) * kSguPerExpert * 4;
constexpr int64_t kPackedBytes = kSdOff + int64_t(kE) * kSdPerExpert * 4;
static_assert(kSguOff % 128 == 0 && kSdOff % 128 == 0, "packed regions must stay aligned");

// Scale index of gate/up packed row `row` (0..1023) and 128-wide k block kb.
__host__ __device__ constexpr int sgu_index(int e, int row, int kb) {
  return ((e * 4 + (row >> 8)) * 2 + ((row >> 7) & 1)) * (kH / kBlk) + kb;
}
// Scale index of down packed row n (output column, 0..1535) and k block kb.
__host__ __device__ constexpr int sd_index(int e, int n, int kb) {
  return (e * (kH / kBlk) + (n >> 7)) * (kI / kBlk) + kb;
}

// Position of element k (mod 4) inside its packed group of 4 codes.
__host__ __device__ constexpr int code_slot(int k) { return (0x2031 >> (4 * (k & 3))) & 0xF; }

// Two E4M3 codes (low byte first) -> their values as a float pair.  The
// hardware conversion to fp16 is exact (every E4M3 value is an fp16 value).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two_codes) {
  const __half2_raw r =
      __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes & 0xFFFFu), __NV_E4M3);
  return __half22float2(__half2(r));
}

// Multiplier of the integer route for a power-of-two scale 2^e, in both
// halves of a 32-bit word, or 0 when the scale is not a power of two or the
// route cannot represent it.  The integer route builds, from a code of value
// v, the bf16 pattern of v * 2^-120 (or the fp16 pattern of v * 2^-8): the
// seven exponent and mantissa bits of the code land in the operand's exponent
// and mantissa fields, subnormal codes included.  The multiplier is then
// 2^(e + 120) as a bf16 (e <= 7), or 2^(e + 8) as a normal fp16 (-22 <= e <= 7).
template <bool F16>
__device__ __forceinline__ uint32_t pow2_multiplier(float scale) {
  const uint32_t b = __float_as_uint(scale);
  const uint32_t E = (b >> 23) & 0xFFu;  // biased exponent; sign must be clear
  if ((b & 0x807FFFFFu) != 0 || E == 0) return 0;
  uint32_t h;
  if constexpr (F16) {
    if (E < 105 || E > 134) return 0;
    h = (E - 104) << 10;
  } else {
    if (E > 134) return 0;
    h = (E + 120) << 7;
  }
  return h | (h << 16);
}

// The conversion route of dequant16 (scales that are not powers of two).
template <bool F16>
__device__ __forceinline__ void dequant16_cvt(const uint4 q, const float scale, uint32_t (&o)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      // pair (k, k+1) sits in bytes (1, 3), pair (k+2, k+3) in bytes (0, 2)
      const float2 f = e4m3x2_to_float2(__byte_perm(w[i], 0, h == 0 ? 0x0031 : 0x0020));
      const float x0 = f.x * scale, x1 = f.y * scale;
      if constexpr (F16) {
        __half2 v = __floats2half2_rn(x0, x1);
        o[2 * i + h] = *reinterpret_cast<uint32_t*>(&v);
      } else {
        o[2 * i + h] = pack_bf16x2(x0, x1);
      }
    }
  }
}

// 16 codes (one packed 16-byte chunk) times `scale`, each product rounded once
// from fp32 to the operand type: fp16 if F16, else bf16.  Eight 32-bit words
// out, two values each, in element order.  mult: pow2_multiplier<F16>(scale);
// when non-zero the integer route runs, else the conversion route.
template <bool F16>
__device__ __forceinline__ void dequant16(const uint4 q, const float scale, const uint32_t mult,
                                          uint32_t (&o)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  if (mult != 0) {
    constexpr int R = F16 ? 1 : 4;  // exponent width of the operand type minus that of E4M3
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t a = w[i], b = w[i] << 8;
      const uint32_t lo = (a & 0x80008000u) | ((a & 0x7F007F00u) >> R);  // bytes 1, 3
      const uint32_t hi = (b & 0x80008000u) | ((b & 0x7F007F00u) >> R);  // bytes 0, 2
      if constexpr (F16) {
        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o[2 * i]) : "r"(lo), "r"(mult));
        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o[2 * i + 1]) : "r"(hi), "r"(mult));
      } else {
        asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(o[2 * i]) : "r"(lo), "r"(mult));
        asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(o[2 * i + 1]) : "r"(hi), "r"(mult));
      }
    }
    return;
  }
  dequant16_cvt<F16>(q, scale, o);
}

// dst[e][map(n)][k] = src[e][k][n] for one [K][N] code matrix, 32 x 32 byte
// tiles through shared memory; mode 0 gate, 1 up, 2 down (row mapping as in
// pack_transpose_kernel).  For down, a weight whose dequantised value leaves
// the fp16 range sets the status word; so does a NaN code in any matrix (the
// integer dequantisation route would read it as a finite value).
__global__ void __launch_bounds__(256)
    pack_fp8_transpose_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int K,
                              int N, int mode, const float* __restrict__ s_down) {
  __shared__ uint8_t tile[32][33];
  const int e = blockIdx.z;
  const int n0 = blockIdx.x * 32, k0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  const uint8_t* s = src + static_cast<int64_t>(e) * K * N;
#pragma unroll
  for (int i = 0; i < 32; i += 8) tile[ty + i][tx] = s[static_cast<int64_t>(k0 + ty + i) * N + n0 + tx];
  __syncthreads();
  uint8_t* d;
  int64_t row_len;
  if (mode == 2) {
    d = dst + kGuBytes + static_cast<int64_t>(e) * kH * kI;
    row_len = kI;
  } else {
    d = dst + static_cast<int64_t>(e) * 1024 * kH;
    row_len = kH;
  }
  bool bad = false, nan = false;
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    const int n = n0 + ty + i, k = k0 + tx;
    int64_t row = n;
    if (mode != 2) row = 256 * (n >> 7) + (n & 127) + (mode == 1 ? 128 : 0);
    const uint8_t c = tile[tx][ty + i];
    nan |= (c & 0x7F) == 0x7F;
    if (mode == 2) {
      // s_down[e][k block][n block], the caller's [4][12] order
      const float sc = s_down[(e * (kI / kBlk) + (k >> 7)) * (kH / kBlk) + (n >> 7)];
      const float v = e4m3x2_to_float2(c).x * sc;
      bad |= !(fabsf(v) <= 65504.f);
    }
    d[row * row_len + (k & ~3) + code_slot(k)] = c;
  }
  if (nan) record_status(kSiteFp8Nan);
  if (bad) record_status(kSiteFp16Range);
}

// Scales from the caller's order (s_gate/s_up [e][12][4], s_down [e][4][12])
// into the GEMM order of SGU and SD.
__global__ void __launch_bounds__(256)
    pack_fp8_scales_kernel(const float* __restrict__ s_gate, const float* __restrict__ s_up,
                           const float* __restrict__ s_down, float* __restrict__ sgu,
                           float* __restrict__ sd) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  constexpr int nkb1 = kH / kBlk, nj = kI / kBlk;  // 12, 4
  if (i < kE * kSguPerExpert) {
    const int kb = i % nkb1, g = (i / nkb1) % 2, j = (i / (2 * nkb1)) % nj, e = i / kSguPerExpert;
    sgu[i] = (g ? s_up : s_gate)[(e * nkb1 + kb) * nj + j];
  } else if (i < kE * (kSguPerExpert + kSdPerExpert)) {
    const int t = i - kE * kSguPerExpert;
    const int kb = t % nj, f = (t / nj) % nkb1, e = t / kSdPerExpert;
    sd[t] = s_down[(e * nj + kb) * nkb1 + f];
  }
}

// Packed FP8 layer -> packed bf16/fp16 layer (the layout moe_pack_weights
// writes): every 16-byte chunk of codes becomes 32 bytes of operands.
__global__ void __launch_bounds__(256)
    dequant_fp8_kernel(const uint8_t* __restrict__ packed8, uint16_t* __restrict__ packed) {
  const float* sgu = reinterpret_cast<const float*>(packed8 + kSguOff);
  const float* sd = reinterpret_cast<const float*>(packed8 + kSdOff);
  constexpr int64_t n_gu = kGuBytes / 16, n_all = (kGuBytes + kDBytes) / 16;
  for (int64_t c = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; c < n_all;
       c += int64_t(gridDim.x) * blockDim.x) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(packed8) + c);
    uint32_t o[8];
    if (c < n_gu) {
      const int64_t el = c * 16;
      const int k = static_cast<int>(el % kH);
      const int64_t rg = el / kH;  // e * 1024 + row
      const float sc = sgu[sgu_index(static_cast<int>(rg >> 10), static_cast<int>(rg & 1023), k >> 7)];
      dequant16<false>(q, sc, pow2_multiplier<false>(sc), o);
    } else {
      const int64_t el = (c - n_gu) * 16;
      const int k = static_cast<int>(el % kI);
      const int64_t rn = el / kI;  // e * 1536 + n
      const int e = static_cast<int>(rn / kH), n = static_cast<int>(rn % kH);
      const float sc = sd[sd_index(e, n, k >> 7)];
      dequant16<true>(q, sc, pow2_multiplier<true>(sc), o);
    }
    uint4* dst = reinterpret_cast<uint4*>(packed) + 2 * c;
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace fp8
}  // namespace moe
