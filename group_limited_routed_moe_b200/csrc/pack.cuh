// pack.cuh -- one-time re-layout of a layer's expert weights into the
// operand order of the grouped GEMMs.
//
// The tensor cores read both GEMM operands K-major.  The layer computes
// x @ W_gate[e] with W_gate[e] stored [1536 (K)][512 (N)], so the packed form
// is the transpose, [N][K].  Gate and up are interleaved in blocks of 128
// output columns (gate cols 128j..128j+127, then up cols 128j..128j+127) so
// that one 256-wide accumulator tile holds matching gate and up columns and
// the SwiGLU can be applied in the epilogue.
//
// Packed layout of one layer (16-bit elements):
//   region GU: [128 experts][1024 rows][1536] bf16  row 256j + r: r < 128 -> gate col 128j + r
//                                                                r >= 128 -> up col 128j + r - 128
//   region D : [128 experts][1536 rows][512]  fp16  row n = output column n of W_down[e]
// W_down is stored as fp16 so that the down GEMM multiplies the fp16 h by an
// operand of the same type.  Every bf16 value in the fp16 normal range
// (magnitudes 2^-14 .. 65504) converts exactly; a smaller magnitude is rounded
// to the nearest fp16 subnormal, an absolute error of at most 2^-25 (about
// 0.2% of N(0, 0.02) weights fall there); a weight beyond the fp16 range sets
// the status word.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int64_t kPackGuPerExpert = 1024LL * kH;  // elements
constexpr int64_t kPackDPerExpert = static_cast<int64_t>(kH) * kI;
constexpr int64_t kPackGuElems = kE * kPackGuPerExpert;
constexpr int64_t kPackElems = kPackGuElems + kE * kPackDPerExpert;

// dst[e][map(n)][k] = src[e][k][n] for a [K][N] source, 32x32 tiles through
// shared memory.  mode 0: gate (rows 256*(n/128) + n%128, row length 1536),
// mode 1: up (+128), mode 2: down (row n, row length 512) in the region that
// starts d_off elements into dst (after all experts' gate/up rows).
__global__ void __launch_bounds__(256)
    pack_transpose_kernel(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst, int K,
                          int N, int mode, int64_t d_off) {
  __shared__ uint16_t tile[32][33];
  const int e = blockIdx.z;
  const int n0 = blockIdx.x * 32, k0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  bool bad = false;
  const uint16_t* s = src + static_cast<int64_t>(e) * K * N;
#pragma unroll
  for (int i = 0; i < 32; i += 8) tile[ty + i][tx] = s[static_cast<int64_t>(k0 + ty + i) * N + n0 + tx];
  __syncthreads();
  uint16_t* d;
  int64_t row_len;
  if (mode == 2) {
    d = dst + d_off + static_cast<int64_t>(e) * kPackDPerExpert;
    row_len = kI;
  } else {
    d = dst + static_cast<int64_t>(e) * kPackGuPerExpert;
    row_len = kH;
  }
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    const int n = n0 + ty + i;
    int64_t row = n;
    if (mode != 2) row = 256 * (n >> 7) + (n & 127) + (mode == 1 ? 128 : 0);
    uint16_t v = tile[tx][ty + i];
    if (mode == 2) {
      const float f = __uint_as_float(static_cast<uint32_t>(v) << 16);
      bad |= !(fabsf(f) <= 65504.f);
      v = __half_as_ushort(__float2half_rn(f));
    }
    d[row * row_len + k0 + tx] = v;
  }
  if (bad) record_status(kSiteFp16Range);
}

}  // namespace moe
