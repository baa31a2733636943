// fp4.cuh -- NVFP4 expert weights: packing, dequantisation arithmetic and the
// expansion of a packed NVFP4 layer into the bf16/fp16 packed layout.
//
// The CUDA path of "Ling-3.0-tiny on a Qualcomm board" (TensorFold issue
// #1247, first comment, "What it does not cover", third bullet) reads ModelOpt
// NVFP4 experts.  The format of a linear weight [out, in]: 4-bit E2M1 codes
// (sign, 2-bit exponent with bias 1, 1-bit mantissa; magnitudes 0, 0.5, 1,
// 1.5, 2, 3, 4, 6), two per byte along the input dimension with the even
// element in the low nibble; one FP8 E4M3 block scale per 16 consecutive
// weights along the input dimension; one fp32 tensor scale per matrix.
// weight = value(code) * value(block scale) * tensor scale.
//
// Dequantisation (integer route, no conversion instruction): a code's three
// magnitude bits placed in bits 8..6 of a bf16 (bits 11..9 of an fp16) and its
// sign in bit 15 give the bf16 pattern of value * 2^-126 (the fp16 pattern of
// value * 2^-14), the subnormal codes 0 and 0.5 included.  One packed 16-bit
// multiply by the block's multiplier M = block scale * tensor scale * 2^126 as
// a bf16 (gate/up) or * 2^14 as an fp16 (down) gives the weight, rounded once
// to the operand type.  M is computed at pack time in fp32 and rounded to the
// operand type: exact when the tensor scale is a power of two (an E4M3 value
// has 4 significant bits) and M is a normal number of that type, which the
// pack kernel checks; the product then has at most 6 significant bits and is
// exact wherever it is a normal value.  With any other tensor scale M carries
// one rounding (relative 2^-9 in bf16, 2^-11 in fp16).
//
// Packed NVFP4 layer (bytes, every region 128-byte aligned):
//   GU4 [128 experts][1024 rows][768]   codes; rows as in the bf16 pack: row
//                                       256j + r is gate column 128j + r (r < 128)
//                                       or up column 128j + r - 128
//   D4  [128][1536 rows][256]           codes; row n = output column n of W_down
// Inside every 32-bit word (8 consecutive k from k0) nibble i holds element
// k0 + 2i for i < 4 and k0 + 2(i - 4) + 1 for i >= 4: the word shifted right by
// 4t has the pair (k0 + 2t, k0 + 2t + 1) in bits 3..0 and 19..16.
//   MGU [128][8 tiles][12 k stages][128 tile rows][8] 16-bit multipliers
//       (bf16), in the skinny kernel's tile order: tile f is pair j = f / 2,
//       half h = f % 2, tile rows 0..63 are gate columns 128j + 64h + r and
//       rows 64..127 the matching up columns; stage kb covers k in
//       [128 kb, 128 kb + 128), 8 blocks of 16
//   MD  [128][12 tiles][4 k stages][128 tile rows][8] multipliers (fp16):
//       tile f row r is output column 128f + r
// so that a 128-row x 128-k stage of codes has its 2 KB of multipliers in one
// contiguous run.
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {
namespace fp4 {

// Status site: a NaN block-scale code, a non-finite tensor scale, or a block
// multiplier outside the normal range of its operand type.
constexpr unsigned kSiteFp4Scale = 24;

constexpr int kBlk = 16;                                     // weights per block scale
constexpr int kStageK = 128;                                 // k per skinny stage
constexpr int kGuRowBytes = kH / 2, kDRowBytes = kI / 2;     // 768, 256
constexpr int64_t kGuBytes = int64_t(kE) * 1024 * kGuRowBytes;
constexpr int64_t kDBytes = int64_t(kE) * kH * kDRowBytes;
constexpr int kStageMultBytes = 128 * (kStageK / kBlk) * 2;  // 2 KB: 128 rows x 8 multipliers
constexpr int kGuTiles = 8, kGuStages = kH / kStageK;        // 8 tiles x 12 stages
constexpr int kDTiles = kH / 128, kDStages = kI / kStageK;   // 12 tiles x 4 stages
constexpr int64_t kMguOff = kGuBytes + kDBytes;
constexpr int64_t kMguBytes = int64_t(kE) * kGuTiles * kGuStages * kStageMultBytes;
constexpr int64_t kMdOff = kMguOff + kMguBytes;
constexpr int64_t kMdBytes = int64_t(kE) * kDTiles * kDStages * kStageMultBytes;
constexpr int64_t kPackedBytes = kMdOff + kMdBytes;
static_assert(kMguOff % 128 == 0 && kMdOff % 128 == 0, "packed regions must stay aligned");

// Byte offset, from MGU, of the multipliers of stage kb of skinny tile f of
// expert e (phase 1: gate/up, else down).
__host__ __device__ constexpr int64_t stage_mult_offset(int phase, int e, int f, int kb) {
  return phase == 1 ? ((int64_t(e) * kGuTiles + f) * kGuStages + kb) * kStageMultBytes
                    : kMguBytes + ((int64_t(e) * kDTiles + f) * kDStages + kb) * kStageMultBytes;
}

// Multiplier index (16-bit units, from MGU) of gate/up packed row `row`
// (0..1023) and 16-wide k block b (0..95).
__host__ __device__ constexpr int64_t mgu_index(int e, int row, int b) {
  return (stage_mult_offset(1, e, 2 * (row >> 8) + ((row & 127) >> 6), b >> 3) >> 1) +
         (((row & 255) >= 128 ? 64 : 0) + (row & 63)) * 8 + (b & 7);
}
// Multiplier index of down packed row n (0..1535) and k block b (0..31).
__host__ __device__ constexpr int64_t md_index(int e, int n, int b) {
  return (stage_mult_offset(2, e, n >> 7, b >> 3) >> 1) + (n & 127) * 8 + (b & 7);
}

__device__ __forceinline__ uint2 ld_shared_v2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
  return v;
}

// 8 codes of one packed word -> 4 operand pairs in element order, each times
// the multiplier m2 (in both halves).  F16: fp16 operands, else bf16.
template <bool F16>
__device__ __forceinline__ void dequant8(uint32_t w, uint32_t m2, uint32_t* o) {
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint32_t x = w >> (4 * t);
    const uint32_t p = ((x & 0x00070007u) << (F16 ? 9 : 6)) | ((x & 0x00080008u) << 12);
    if constexpr (F16)
      asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o[t]) : "r"(p), "r"(m2));
    else
      asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(o[t]) : "r"(p), "r"(m2));
  }
}

// ---------------------------------------------------------------- packing

// One word of the caller's codes (bytes of 2 codes, low nibble first) -> the
// packed word order above: even elements to the low half, odd to the high.
__device__ __forceinline__ uint32_t reorder_word(uint32_t u) {
  uint32_t r = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    r |= ((u >> (8 * b)) & 0xFu) << (4 * b);
    r |= ((u >> (8 * b + 4)) & 0xFu) << (16 + 4 * b);
  }
  return r;
}

// Codes of one matrix kind for all experts: src [E][N][K/2] (the caller's
// [out, in] form), mode 0 gate, 1 up (N = 512, K = 1536), 2 down (N = 1536,
// K = 512).  One thread per 32-bit word; rows are copied whole, so reads and
// writes are both coalesced.
__global__ void __launch_bounds__(256)
    pack_fp4_codes_kernel(const uint32_t* __restrict__ src, uint8_t* __restrict__ dst, int mode) {
  const int N = mode == 2 ? kH : kI, wpr = (mode == 2 ? kI : kH) / 8;  // words per row
  const int64_t total = int64_t(kE) * N * wpr;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int kw = static_cast<int>(i % wpr);
    const int64_t en = i / wpr;
    const int e = static_cast<int>(en / N), n = static_cast<int>(en % N);
    uint32_t* d;
    if (mode == 2) {
      d = reinterpret_cast<uint32_t*>(dst + kGuBytes) + (int64_t(e) * kH + n) * wpr;
    } else {
      const int row = 256 * (n >> 7) + (n & 127) + (mode == 1 ? 128 : 0);
      d = reinterpret_cast<uint32_t*>(dst) + (int64_t(e) * 1024 + row) * wpr;
    }
    d[kw] = reorder_word(__ldg(src + i));
  }
}

// The 16-bit multiplier of one block: F16 -> fp16(scale * g * 2^14), else
// bf16(scale * g * 2^126).  `bad` is set when the block scale is a NaN code
// or the multiplier of a non-zero scale is not a normal number of the type.
template <bool F16>
__device__ __forceinline__ uint16_t block_multiplier(uint8_t scale_code, float g, bool& bad) {
  const __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(scale_code), __NV_E4M3);
  const float s = __half2float(__half(hr));
  if ((scale_code & 0x7F) == 0x7F || !isfinite(g)) bad = true;
  const float m = s * g * (F16 ? 16384.0f : 0x1p126f);
  uint16_t bits;
  if constexpr (F16) {
    const __half h = __float2half_rn(m);
    bits = *reinterpret_cast<const uint16_t*>(&h);
    if (s != 0.0f && g != 0.0f && ((bits & 0x7C00u) == 0 || (bits & 0x7C00u) == 0x7C00u)) bad = true;
  } else {
    const __nv_bfloat16 b = __float2bfloat16_rn(m);
    bits = *reinterpret_cast<const uint16_t*>(&b);
    if (s != 0.0f && g != 0.0f && ((bits & 0x7F80u) == 0 || (bits & 0x7F80u) == 0x7F80u)) bad = true;
  }
  return bits;
}

// Multipliers of every block, from the caller's block scales (s_gate, s_up
// [E][512][96], s_down [E][1536][32], E4M3 codes) and tensor scales (g_* [E]),
// written in the MGU / MD order.  One thread per multiplier.
__global__ void __launch_bounds__(256)
    pack_fp4_mult_kernel(const uint8_t* __restrict__ s_gate, const uint8_t* __restrict__ s_up,
                         const uint8_t* __restrict__ s_down, const float* __restrict__ g_gate,
                         const float* __restrict__ g_up, const float* __restrict__ g_down,
                         uint16_t* __restrict__ mult) {
  constexpr int64_t n_gu = kMguBytes / 2, n_all = (kMguBytes + kMdBytes) / 2;
  bool bad = false;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n_all;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int slot = static_cast<int>(i & 7), trow = static_cast<int>((i >> 3) & 127);
    const int64_t st = i >> 10;  // stage index (1024 multipliers per stage)
    if (i < n_gu) {
      const int kb = static_cast<int>(st % kGuStages), f = static_cast<int>((st / kGuStages) % kGuTiles);
      const int e = static_cast<int>(st / (kGuStages * kGuTiles));
      const bool up = trow >= 64;
      const int n = 128 * (f >> 1) + 64 * (f & 1) + (trow & 63);  // gate / up output column
      const int b = kb * 8 + slot;
      const uint8_t code = (up ? s_up : s_gate)[(int64_t(e) * kI + n) * (kH / kBlk) + b];
      mult[i] = block_multiplier<false>(code, (up ? g_up : g_gate)[e], bad);
    } else {
      const int64_t sd = st - n_gu / 1024;
      const int kb = static_cast<int>(sd % kDStages), f = static_cast<int>((sd / kDStages) % kDTiles);
      const int e = static_cast<int>(sd / (kDStages * kDTiles));
      const int n = 128 * f + trow, b = kb * 8 + slot;
      const uint8_t code = s_down[(int64_t(e) * kH + n) * (kI / kBlk) + b];
      mult[i] = block_multiplier<true>(code, g_down[e], bad);
    }
  }
  if (bad) record_status(kSiteFp4Scale);
}

// Packed NVFP4 layer -> packed bf16/fp16 layer (the layout moe_pack_weights
// writes): every 8 bytes of codes (one block) become 32 bytes of operands.
__global__ void __launch_bounds__(256)
    dequant_fp4_kernel(const uint8_t* __restrict__ packed4, uint16_t* __restrict__ packed) {
  const uint16_t* mult = reinterpret_cast<const uint16_t*>(packed4 + kMguOff);
  constexpr int64_t n_gu = kGuBytes / 8, n_all = (kGuBytes + kDBytes) / 8;
  for (int64_t c = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; c < n_all;
       c += int64_t(gridDim.x) * blockDim.x) {
    const uint2 q = __ldg(reinterpret_cast<const uint2*>(packed4) + c);
    uint32_t o[8];
    if (c < n_gu) {
      const int b = static_cast<int>(c % (kH / kBlk));
      const int64_t rg = c / (kH / kBlk);  // e * 1024 + row
      const uint32_t m = __ldg(mult + mgu_index(static_cast<int>(rg >> 10), static_cast<int>(rg & 1023), b));
      dequant8<false>(q.x, m * 0x10001u, o);
      dequant8<false>(q.y, m * 0x10001u, o + 4);
    } else {
      const int64_t cd = c - n_gu;
      const int b = static_cast<int>(cd % (kI / kBlk));
      const int64_t rn = cd / (kI / kBlk);  // e * 1536 + n
      const uint32_t m = __ldg(mult + md_index(static_cast<int>(rn / kH), static_cast<int>(rn % kH), b));
      dequant8<true>(q.x, m * 0x10001u, o);
      dequant8<true>(q.y, m * 0x10001u, o + 4);
    }
    uint4* dst = reinterpret_cast<uint4*>(packed) + 2 * c;
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace fp4
}  // namespace moe
