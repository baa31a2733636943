// moe.cu -- libmoe: the C ABI declared in include/moe.h.
//
// Host code here only validates arguments, encodes TMA descriptors and
// launches kernels; it never allocates, synchronises or reads device memory
// (moe_get_device_status() excepted, which copies one status word).
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/moe.h"
#include "combine.cuh"
#include "common.cuh"
#include "expert_ffn.cuh"
#include "expert_ffn_skinny.cuh"
#include "e256.cuh"
#include "fp4.cuh"
#include "fp8.cuh"
#include "pack.cuh"
#include "permute.cuh"
#include "route.cuh"
#include "route_permute_small.cuh"
#include "router.cuh"
#include "router_small.cuh"

using namespace moe;

namespace {

constexpr int kAbiVersion = 6;
constexpr int64_t kMaxTokens = int64_t(1) << 22;
constexpr int kMaxDevices = 64;
constexpr int64_t kZeroPadMaxT = 1024;  // gate/up keeps padding rows of A zeroed up to this T
constexpr int64_t kSkinnyMaxT = 256;    // weights-as-M (skinny) GEMMs up to this T

thread_local char g_err[512] = "";
std::atomic<uint64_t> g_timeout_ns{2000000000ull};

// Per-CTA timing record of the expert-FFN launches (moe_set_ffn_trace); NULL
// when off.  A launch of `ctas` CTAs records only if the buffer holds them all.
std::atomic<uint64_t*> g_trace{nullptr};
std::atomic<int64_t> g_trace_cap{0};
uint64_t* ffn_trace(int ctas) {
  uint64_t* p = g_trace.load();
  return (p != nullptr && g_trace_cap.load() >= ctas) ? p : nullptr;
}

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define MOE_CUDA(call, what)                    \
  do {                                          \
    cudaError_t e_ = (call);                    \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ---- per-device setup (once): SM count, arch check, kernel attributes -------
struct DeviceInfo {
  int sms = 0;
  int status = -1;  // -1 unset, otherwise moe_status
  char msg[256] = "";
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int device_setup(int* dev_out, int* sms_out) {
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.status < 0) {
    cudaDeviceProp prop;
    cudaError_t e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
    if (prop.major != 10 || prop.minor != 0) {
      d.status = MOE_ERR_UNSUPPORTED;
      snprintf(d.msg, sizeof(d.msg), "libmoe is built for sm_100a (B200); device %d is sm_%d%d",
               dev, prop.major, prop.minor);
    } else {
      d.sms = prop.multiProcessorCount;
      e = cudaFuncSetAttribute(ffn::ffn_gemm_kernel<1, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, ffn::SMEM_BYTES);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ffn::ffn_gemm_kernel<1, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, ffn::SMEM_BYTES);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ffn::ffn_gemm_kernel<2, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, ffn::SMEM_BYTES);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ffn::ffn_gemm_kernel<3, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, ffn::SMEM_BYTES);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ffn::ffn_gemm_kernel<3, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, ffn::SMEM_BYTES);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(skinny::skinny_gemm_kernel<1>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, skinny::SMEM_BYTES);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(skinny::skinny_gemm_kernel<2>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, skinny::SMEM_BYTES);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(skinny::skinny_gemm_kernel<3>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, skinny::SMEM_BYTES);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(skinny::skinny_gemm_kernel<3, 1>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, skinny::SMEM_BYTES);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(skinny::skinny_gemm_kernel<3, 2>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, skinny::SMEM_BYTES);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(router::router_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, router::SMEM_BYTES);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
      if (g_encode == nullptr) {
        cudaDriverEntryPointQueryResult q;
        void* fn = nullptr;
        e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr)
          return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found");
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
      }
      d.status = MOE_OK;
    }
  }
  if (d.status != MOE_OK) return fail(d.status, "%s", d.msg);
  if (dev_out) *dev_out = dev;
  if (sms_out) *sms_out = d.sms;
  return MOE_OK;
}

// 2-D tensor map of 16-bit elements: `rows` rows of `cols` elements, box of
// 64 x box_rows, 128-byte swizzle (the UMMA K-major SW128 operand layout).
int make_tmap(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
              CUtensorMapDataType dtype) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, dtype, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return MOE_OK;
}

// 2-D tensor map of 8-bit codes: `rows` rows of `cols` bytes, box of 128 x 64,
// 128-byte swizzle (the converter warps read each row's eight 16-byte chunks;
// the swizzle keeps a warp's reads free of bank conflicts).
// Byte rows of codes in boxes of 64 rows x box_bytes (128: 128-byte swizzle,
// 64: 64-byte swizzle).
int make_tmap_u8(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                 uint32_t box_bytes = 128) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {box_bytes, 64};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        box_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (u8) failed (%d)", int(r));
  return MOE_OK;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int check_T(int64_t T) {
  if (T < 0 || T > kMaxTokens)
    return fail(MOE_ERR_INVALID_ARG, "T=%lld outside [0, %lld]", static_cast<long long>(T),
                static_cast<long long>(kMaxTokens));
  return MOE_OK;
}

#define REQUIRE(cond, ...)                                         \
  do {                                                             \
    if (!(cond)) return fail(MOE_ERR_INVALID_ARG, __VA_ARGS__);    \
  } while (0)

// Launch with programmatic stream serialisation (see griddep_wait).
template <typename... KArgs, typename... Args>
int launch_pdl(const char* what, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
               cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return MOE_OK;
}

int launch_check(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return MOE_OK;
}

// ---- step launchers (arguments already validated) ----------------------------
int do_route(const float* logits, const float* bias, int64_t T, int32_t* idx, float* w,
             cudaStream_t s) {
  const int64_t blocks = (T + kRouteTokensPerBlock - 1) / kRouteTokensPerBlock;
  return launch_pdl("route_kernel launch", route_kernel, dim3(static_cast<unsigned>(blocks)),
                    dim3(kRouteWarps * 32), 0, s, logits, bias, T, idx, w);
}

// Tokens per block of the multi-block counting sort at T.
int perm_block_tokens(int64_t T) {
  return T <= kPermSmallBlocksMaxT ? kPermBlockTokensSmall : kPermBlockTokens;
}

size_t permute_ws_bytes(int64_t T) {
  if (T <= kPermSmallMaxT) return 0;
  const int bt = perm_block_tokens(T);
  const int64_t nb = (T + bt - 1) / bt;
  return align_up(static_cast<size_t>(nb) * kE * sizeof(int32_t), 256);
}

int do_permute(const int32_t* idx, int64_t T, int32_t* counts, int32_t* offsets, int32_t* perm_src,
               int32_t* inv_perm, void* ws, cudaStream_t s) {
  if (T <= kPermSmallMaxT) {
    return launch_pdl("permute_small_kernel launch", permute_small_kernel, dim3(1), dim3(1024), 0,
                      s, idx, static_cast<int>(T), counts, offsets, perm_src, inv_perm);
  }
  int32_t* hist = static_cast<int32_t*>(ws);
  if (perm_block_tokens(T) == kPermBlockTokensSmall) {  // count, then the fused scan + scatter
    constexpr int bt = kPermBlockTokensSmall;
    const int64_t nb = (T + bt - 1) / bt;
    static_assert((kPermSmallBlocksMaxT + bt - 1) / bt <= kPermFusedMaxBlocks,
                  "64-token blocks only where the fused scan + scatter covers the batch");
    int rc = launch_pdl("permute_count_kernel launch", permute_count_kernel<bt>,
                        dim3(static_cast<unsigned>(nb)), dim3(256), 0, s, idx, T, hist);
    if (rc) return rc;
    return launch_pdl("permute_scan_scatter_kernel launch", permute_scan_scatter_kernel<bt>,
                      dim3(static_cast<unsigned>(nb)), dim3(kPermScanThreads), 0, s, idx, T,
                      static_cast<const int32_t*>(hist), static_cast<int>(nb), counts, offsets,
                      perm_src, inv_perm);
  }
  const int64_t nb = (T + kPermBlockTokens - 1) / kPermBlockTokens;
  int rc = launch_pdl("permute_count_kernel launch", permute_count_kernel<kPermBlockTokens>,
                      dim3(static_cast<unsigned>(nb)), dim3(256), 0, s, idx, T, hist);
  if (rc) return rc;
  if (nb <= kPermFusedMaxBlocks) {
    return launch_pdl("permute_scan_scatter_kernel launch",
                      permute_scan_scatter_kernel<kPermBlockTokens>, dim3(static_cast<unsigned>(nb)),
                      dim3(kPermScanThreads), 0, s, idx, T, static_cast<const int32_t*>(hist),
                      static_cast<int>(nb), counts, offsets, perm_src, inv_perm);
  }
  rc = launch_pdl("permute_scan_kernel launch", permute_scan_kernel, dim3(1), dim3(1024), 0, s,
                  hist, static_cast<int>(nb), counts, offsets);
  if (rc) return rc;
  return launch_pdl("permute_scatter_kernel launch", permute_scatter_kernel,
                    dim3(static_cast<unsigned>(nb)), dim3(256), 0, s, idx, T,
                    static_cast<const int32_t*>(hist), static_cast<const int32_t*>(offsets),
                    perm_src, inv_perm);
}

// Router projection: logits [T][128] fp32 from x and the packed router.
int do_router(const moe_bf16* x, const moe_bf16* packed_router, int64_t T, float* logits, int sms,
              cudaStream_t s) {
  CUtensorMap tw, tx;
  int rc = make_tmap(&tw, packed_router, kH, kE, router::BM, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  if (!rc)
    rc = make_tmap(&tx, x, kH, static_cast<uint64_t>(T), router::BN, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  if (rc) return rc;
  const int64_t ntiles = (T + router::BN - 1) / router::BN;
  const unsigned grid = static_cast<unsigned>(ntiles < sms ? ntiles : sms);
  return launch_pdl("router_kernel launch", router::router_kernel, dim3(grid),
                    dim3(router::THREADS), router::SMEM_BYTES, s, tw, tx, T, logits,
                    g_timeout_ns.load());
}

// Router projection + routing (+ the counting sort when counts != nullptr) in
// one launch of one 8-CTA cluster, for T <= rsmall::kMaxT.
int do_router_route_small(const moe_bf16* x, const moe_bf16* packed_router, const float* bias,
                          int64_t T, float* logits, int32_t* idx, float* w, int32_t* counts,
                          int32_t* offsets, int32_t* perm_src, int32_t* inv_perm,
                          cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rsmall::kCluster);
  cfg.blockDim = dim3(rsmall::kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(T) * kE * sizeof(float);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = rsmall::kCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(
      &cfg, rsmall::router_route_permute_small_kernel,
      reinterpret_cast<const __nv_bfloat16*>(x), reinterpret_cast<const __nv_bfloat16*>(packed_router),
      bias, static_cast<int>(T), logits, idx, w, counts, offsets, perm_src, inv_perm);
  if (e != cudaSuccess) return cuda_fail(e, "router_route_permute_small_kernel launch");
  return MOE_OK;
}

// Steps 1 and 2 as moe_layer runs them: one fused block for a few tokens.
int do_route_permute(const float* logits, const float* bias, int64_t T, int32_t* idx, float* w,
                     int32_t* counts, int32_t* offsets, int32_t* perm_src, int32_t* inv_perm,
                     void* perm_ws, cudaStream_t s) {
  if (T <= kFusedRoutePermMaxT) {
    return launch_pdl("route_permute_small_kernel launch", route_permute_small_kernel, dim3(1),
                      dim3(kFusedRoutePermThreads), 0, s, logits, bias, static_cast<int>(T), idx,
                      w, counts, offsets, perm_src, inv_perm);
  }
  int rc = do_route(logits, bias, T, idx, w, s);
  if (rc) return rc;
  return do_permute(idx, T, counts, offsets, perm_src, inv_perm, perm_ws, s);
}

// The GEMMs' tile counters live after the expert offsets (zeroed by the permute
// kernels, left zero by the GEMMs): words kSchedWord.. (gate/up), +2 (down).
int* sched_words(const int32_t* offsets, int phase) {
  return const_cast<int*>(offsets) + kSchedWord + 2 * (phase - 1);
}

// One weight pack's pointers for the skinny kernel (a launch of one segment).
SegPtrs one_segment(const int32_t* offsets, const int32_t* perm_src, moe_bf16* h,
                            moe_bf16* y) {
  SegPtrs p{};
  p.n = 1;
  p.offsets[0] = offsets;
  p.perm_src[0] = perm_src;
  p.h_out[0] = reinterpret_cast<uint16_t*>(h);
  p.y_out[0] = reinterpret_cast<uint16_t*>(y);
  return p;
}

int do_gate_up(const moe_bf16* x, const moe_bf16* packed, const int32_t* offsets,
               const int32_t* perm_src, int64_t T, moe_bf16* h, int sms, cudaStream_t s) {
  if (T <= kSkinnyMaxT) {
    SegMaps maps{};
    int rc = make_tmap(&maps.w1[0], packed, kH, uint64_t(kE) * 2 * kI, 64,
                       CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
    if (rc) return rc;
    return launch_pdl("skinny_gemm_kernel<1> launch", skinny::skinny_gemm_kernel<1>, dim3(sms),
                      dim3(skinny::THREADS), skinny::SMEM_BYTES, s, maps,
                      one_segment(offsets, perm_src, h, nullptr),
                      reinterpret_cast<const __nv_bfloat16*>(x), T, sched_words(offsets, 1),
                      static_cast<const void*>(nullptr), g_timeout_ns.load(), ffn_trace(sms),
                      FusedCombine{});
  }
  SegMaps maps{};
  int rc = make_tmap(&maps.w1[0], packed, kH, uint64_t(kE) * 2 * kI, ffn::BN,
                     CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  if (rc) return rc;
  return launch_pdl("ffn_gemm_kernel<1> launch",
                    T <= kZeroPadMaxT ? ffn::ffn_gemm_kernel<1, true> : ffn::ffn_gemm_kernel<1, false>,
                    dim3(sms), dim3(ffn::Cfg<1>::THREADS), ffn::SMEM_BYTES, s, maps,
                    one_segment(offsets, perm_src, h, nullptr),
                    reinterpret_cast<const __nv_bfloat16*>(x), T, sched_words(offsets, 1),
                    g_timeout_ns.load(), ffn_trace(sms));
}

int do_down(const moe_bf16* h, const moe_bf16* packed, const int32_t* offsets, int64_t T,
            moe_bf16* y, int sms, cudaStream_t s) {
  const uint64_t rows = static_cast<uint64_t>(T) * kTopK;
  if (T <= kSkinnyMaxT) {
    SegMaps maps{};
    int rc = make_tmap(&maps.w2[0], packed + kPackGuElems, kI, uint64_t(kE) * kH, skinny::BMW,
                       CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    if (!rc) rc = make_tmap(&maps.h[0], h, kI, rows, skinny::BNT, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    if (rc) return rc;
    return launch_pdl("skinny_gemm_kernel<2> launch", skinny::skinny_gemm_kernel<2>, dim3(sms),
                      dim3(skinny::THREADS), skinny::SMEM_BYTES, s, maps,
                      one_segment(offsets, nullptr, nullptr, y),
                      static_cast<const __nv_bfloat16*>(nullptr), T, sched_words(offsets, 2),
                      static_cast<const void*>(nullptr), g_timeout_ns.load(), ffn_trace(sms),
                      FusedCombine{});
  }
  SegMaps maps{};
  int rc = make_tmap(&maps.w2[0], packed + kPackGuElems, kI, uint64_t(kE) * kH, ffn::BN,
                     CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  if (!rc) rc = make_tmap(&maps.h[0], h, kI, rows, ffn::BM, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  if (rc) return rc;
  return launch_pdl("ffn_gemm_kernel<2> launch", ffn::ffn_gemm_kernel<2, false>, dim3(sms),
                    dim3(ffn::Cfg<2>::THREADS), ffn::SMEM_BYTES, s, maps,
                    one_segment(offsets, nullptr, nullptr, y),
                    static_cast<const __nv_bfloat16*>(nullptr), T, sched_words(offsets, 2),
                    g_timeout_ns.load(), ffn_trace(sms));
}

// Tensor maps of segment g of a skinny launch: a bf16 pack of n_exp experts
// (its down region from element d_off) and its h buffer of h_rows rows (a
// chunk's box past the last row reads zeros, never past the buffer).
int skinny_maps(SegMaps* maps, int g, const moe_bf16* packed, int n_exp, int64_t d_off,
                const moe_bf16* h, int64_t h_rows) {
  int rc = make_tmap(&maps->w1[g], packed, kH, uint64_t(n_exp) * 2 * kI, 64,
                     CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  if (!rc) rc = make_tmap(&maps->w2[g], packed + d_off, kI, uint64_t(n_exp) * kH, skinny::BMW,
                          CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  if (!rc) rc = make_tmap(&maps->h[g], h, kI, static_cast<uint64_t>(h_rows), skinny::BNT,
                          CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  return rc;
}

// Tensor maps of segment g of a wide launch: as skinny_maps, with the wide
// kernel's boxes (256 weight rows, 128 h rows).
int wide_maps(SegMaps* maps, int g, const moe_bf16* packed, int n_exp, int64_t d_off,
              const moe_bf16* h, int64_t h_rows) {
  int rc = make_tmap(&maps->w1[g], packed, kH, uint64_t(n_exp) * 2 * kI, ffn::BN,
                     CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  if (!rc) rc = make_tmap(&maps->w2[g], packed + d_off, kI, uint64_t(n_exp) * kH, ffn::BN,
                          CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  if (!rc) rc = make_tmap(&maps->h[g], h, kI, static_cast<uint64_t>(h_rows), ffn::BM,
                          CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  return rc;
}

// The maps of segment g for the kernel that runs T tokens.
int ffn_maps(SegMaps* maps, int g, const moe_bf16* packed, int n_exp, int64_t d_off,
             const moe_bf16* h, int64_t h_rows, int64_t T) {
  return T <= kSkinnyMaxT ? skinny_maps(maps, g, packed, n_exp, d_off, h, h_rows)
                          : wide_maps(maps, g, packed, n_exp, d_off, h, h_rows);
}

// The single-launch expert FFN over the segments p (maps from ffn_maps); the
// tile counters are segment 0's.  cmb.out != nullptr (T <= kFusedCombineMaxT
// only): the launch also runs the layer's combine.
int do_ffn_segments(const SegMaps& maps, const SegPtrs& p, const moe_bf16* x, int64_t T, int sms,
                    cudaStream_t s, const FusedCombine& cmb = FusedCombine{}) {
  const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  if (T <= kSkinnyMaxT)
    return launch_pdl("skinny_gemm_kernel<3> launch", skinny::skinny_gemm_kernel<3>, dim3(sms),
                      dim3(skinny::THREADS), skinny::SMEM_BYTES, s, maps, p, xb, T,
                      sched_words(p.offsets[0], 1), static_cast<const void*>(nullptr),
                      g_timeout_ns.load(), ffn_trace(sms), cmb);
  return launch_pdl("ffn_gemm_kernel<3> launch",
                    T <= kZeroPadMaxT ? ffn::ffn_gemm_kernel<3, true> : ffn::ffn_gemm_kernel<3, false>,
                    dim3(sms), dim3(ffn::Cfg<3>::THREADS), ffn::SMEM_BYTES, s, maps, p, xb, T,
                    sched_words(p.offsets[0], 1), g_timeout_ns.load(), ffn_trace(sms));
}

// n_exp: experts in the pack (128, or the shared experts' count), d_off: start
// of its down region in elements; only experts with rows in `offsets` are read.
// h_rows: rows of the h buffer (default 8T).
int do_expert_ffn(const moe_bf16* x, const moe_bf16* packed, const int32_t* offsets,
                  const int32_t* perm_src, int64_t T, moe_bf16* h, moe_bf16* y, int sms,
                  cudaStream_t s, int n_exp = kE, int64_t d_off = kPackGuElems,
                  int64_t h_rows = -1, const FusedCombine& cmb = FusedCombine{}) {
  if (h_rows < 0) h_rows = T * kTopK;
  // both GEMMs in one launch (see expert_ffn_skinny.cuh, expert_ffn.cuh)
  SegMaps maps{};
  int rc = ffn_maps(&maps, 0, packed, n_exp, d_off, h, h_rows, T);
  if (rc) return rc;
  return do_ffn_segments(maps, one_segment(offsets, perm_src, h, y), x, T, sms, s, cmb);
}

// Packed block-FP8 layer -> packed bf16/fp16 layer.
int do_dequant_fp8(const void* packed8, moe_bf16* packed, int sms, cudaStream_t s) {
  return launch_pdl("dequant_fp8_kernel launch", fp8::dequant_fp8_kernel, dim3(sms * 8),
                    dim3(256), 0, s, static_cast<const uint8_t*>(packed8),
                    reinterpret_cast<uint16_t*>(packed));
}

// Expert FFN with block-FP8 weights.  Up to kSkinnyMaxT tokens the skinny
// single-launch kernel dequantises each weight tile in shared memory (half
// the weight bytes from HBM); above it, where the GEMMs are bound by the
// tensor cores rather than by the weight stream, the layer is expanded into
// `dq` (moe_packed_weight_bytes) and run by the bf16 kernel.
int do_expert_ffn_fp8(const moe_bf16* x, const void* packed8, const int32_t* offsets,
                      const int32_t* perm_src, int64_t T, moe_bf16* h, moe_bf16* y, moe_bf16* dq,
                      int sms, cudaStream_t s, const FusedCombine& cmb = FusedCombine{}) {
  if (T > kSkinnyMaxT) {
    int rc = do_dequant_fp8(packed8, dq, sms, s);
    if (rc) return rc;
    return do_expert_ffn(x, dq, offsets, perm_src, T, h, y, sms, s);
  }
  const uint8_t* p8 = static_cast<const uint8_t*>(packed8);
  SegMaps maps{};
  int rc = make_tmap_u8(&maps.w1[0], p8, kH, uint64_t(kE) * 2 * kI);
  if (!rc) rc = make_tmap_u8(&maps.w2[0], p8 + fp8::kGuBytes, kI, uint64_t(kE) * kH);
  if (!rc) rc = make_tmap(&maps.h[0], h, kI, static_cast<uint64_t>(T) * kTopK, skinny::BNT,
                          CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  if (rc) return rc;
  return launch_pdl("skinny_gemm_kernel<3, fp8> launch", skinny::skinny_gemm_kernel<3, 1>,
                    dim3(sms), dim3(skinny::Ring<1>::THREADS), skinny::SMEM_BYTES, s, maps,
                    one_segment(offsets, perm_src, h, y),
                    reinterpret_cast<const __nv_bfloat16*>(x), T, sched_words(offsets, 1),
                    static_cast<const void*>(p8 + fp8::kSguOff), g_timeout_ns.load(), ffn_trace(sms),
                    cmb);
}

// Packed NVFP4 layer -> packed bf16/fp16 layer.
int do_dequant_fp4(const void* packed4, moe_bf16* packed, int sms, cudaStream_t s) {
  return launch_pdl("dequant_fp4_kernel launch", fp4::dequant_fp4_kernel, dim3(sms * 8),
                    dim3(256), 0, s, static_cast<const uint8_t*>(packed4),
                    reinterpret_cast<uint16_t*>(packed));
}

// Expert FFN with NVFP4 weights: as do_expert_ffn_fp8, with 4-bit codes and
// per-16 block multipliers in the skinny kernel up to kSkinnyMaxT tokens.
int do_expert_ffn_fp4(const moe_bf16* x, const void* packed4, const int32_t* offsets,
                      const int32_t* perm_src, int64_t T, moe_bf16* h, moe_bf16* y, moe_bf16* dq,
                      int sms, cudaStream_t s, const FusedCombine& cmb = FusedCombine{}) {
  if (T > kSkinnyMaxT) {
    int rc = do_dequant_fp4(packed4, dq, sms, s);
    if (rc) return rc;
    return do_expert_ffn(x, dq, offsets, perm_src, T, h, y, sms, s);
  }
  const uint8_t* p4 = static_cast<const uint8_t*>(packed4);
  SegMaps maps{};
  int rc = make_tmap_u8(&maps.w1[0], p4, fp4::kGuRowBytes, uint64_t(kE) * 2 * kI, 64);
  if (!rc)
    rc = make_tmap_u8(&maps.w2[0], p4 + fp4::kGuBytes, fp4::kDRowBytes, uint64_t(kE) * kH, 64);
  if (!rc) rc = make_tmap(&maps.h[0], h, kI, static_cast<uint64_t>(T) * kTopK, skinny::BNT,
                          CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  if (rc) return rc;
  return launch_pdl("skinny_gemm_kernel<3, nvfp4> launch", skinny::skinny_gemm_kernel<3, 2>,
                    dim3(sms), dim3(skinny::Ring<2>::THREADS), skinny::SMEM_BYTES, s, maps,
                    one_segment(offsets, perm_src, h, y),
                    reinterpret_cast<const __nv_bfloat16*>(x), T, sched_words(offsets, 1),
                    static_cast<const void*>(p4 + fp4::kMguOff), g_timeout_ns.load(), ffn_trace(sms),
                    cmb);
}

int do_combine(const moe_bf16* y, const float* w, const int32_t* inv, int64_t T,
               const moe_bf16* residual, moe_bf16* out, cudaStream_t s,
               const moe_bf16* y_shared = nullptr, int n_shared = 0) {
  return launch_pdl("combine_kernel launch", combine_kernel<kTopK>, dim3(static_cast<unsigned>(T)),
                    dim3(kCombineThreads), 0, s, reinterpret_cast<const uint16_t*>(y), w, inv, T,
                    reinterpret_cast<const __nv_bfloat16*>(residual),
                    reinterpret_cast<__nv_bfloat16*>(out),
                    reinterpret_cast<const uint16_t*>(y_shared), n_shared);
}

// The shared experts' FFN: their row set (every token, once per shared
// expert), then the grouped FFN on the shared pack.
constexpr int kMaxShared = kTopK;  // n_shared * T rows fit the routed buffers' bounds
int do_shared_rows(int n_shared, int64_t T, int32_t* offsets, int32_t* perm_src, cudaStream_t s) {
  const int64_t n = std::max<int64_t>(kOffsetsLen, n_shared * T);
  return launch_pdl("shared_rows_kernel launch", shared_rows_kernel,
                    dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, s, T, n_shared,
                    offsets, perm_src);
}

int do_shared_ffn(const moe_bf16* x, const moe_bf16* packed_shared, int n_shared, int64_t T,
                  int32_t* offsets, int32_t* perm_src, moe_bf16* h, moe_bf16* y, int sms,
                  cudaStream_t s) {
  int rc = do_shared_rows(n_shared, T, offsets, perm_src, s);
  if (rc) return rc;
  return do_expert_ffn(x, packed_shared, offsets, perm_src, T, h, y, sms, s, n_shared,
                       int64_t(n_shared) * kPackGuPerExpert, int64_t(n_shared) * T);
}

// workspace carve-up of moe_layer
struct LayerWs {
  size_t idx, w, counts, offsets, perm_src, inv_perm, perm_ws, h, y, logits, dq;
  size_t sh_offsets, sh_perm, sh_h, sh_y, total;
};
// quant: a quantised (block-FP8 or NVFP4) layer, which above kSkinnyMaxT tokens
// also needs room for the expanded bf16/fp16 layer; n_shared: shared experts'
// rows and results.
LayerWs layer_ws(int64_t T, bool quant = false, int n_shared = 0) {
  LayerWs L{};
  const size_t n = static_cast<size_t>(T) * kTopK;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 1024);
    return at;
  };
  L.idx = take(n * 4);
  L.w = take(n * 4);
  L.counts = take(kE * 4);
  L.offsets = take(kOffsetsLen * 4);
  L.perm_src = take(n * 4);
  L.inv_perm = take(n * 4);
  L.perm_ws = take(permute_ws_bytes(T));
  L.h = take(n * kI * 2);
  L.y = take(n * kH * 2);
  L.logits = take(static_cast<size_t>(T) * kE * 4);  // used by moe_layer_routed
  L.dq = take(quant && T > kSkinnyMaxT ? static_cast<size_t>(kPackElems) * 2 : 0);
  const size_t ns = static_cast<size_t>(n_shared) * static_cast<size_t>(T);
  L.sh_offsets = take(n_shared ? kOffsetsLen * 4 : 0);
  L.sh_perm = take(ns * 4);
  L.sh_h = take(ns * kI * 2);
  L.sh_y = take(ns * kH * 2);
  L.total = o;
  return L;
}

}  // namespace

// =============================================================================
extern "C" {

int moe_abi_version(void) { return kAbiVersion; }
int64_t moe_max_tokens(void) { return kMaxTokens; }
const char* moe_last_error_string(void) { return g_err; }

int moe_get_device_status(int device) {
  int prev = 0;
  MOE_CUDA(cudaGetDevice(&prev), "cudaGetDevice");
  MOE_CUDA(cudaSetDevice(device), "cudaSetDevice");
  unsigned v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_status, sizeof(v));
  const unsigned zero = 0;
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_status, &zero, sizeof(zero));
  cudaSetDevice(prev);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  if (v == 0) return MOE_OK;
  if ((v & 0x7FFFFFFFu) == kSiteBadIndex)
    return fail(MOE_ERR_INVALID_ARG, "a kernel met an out-of-range index (status 0x%08x)", v);
  if ((v & 0x7FFFFFFFu) == kSiteFp16Range)
    return fail(MOE_ERR_RANGE, "a value of h, y_perm or W_down exceeded the fp16 range");
  if ((v & 0x7FFFFFFFu) == kSiteFp8Nan)
    return fail(MOE_ERR_RANGE, "a block-FP8 expert weight is a NaN code");
  if ((v & 0x7FFFFFFFu) == fp4::kSiteFp4Scale)
    return fail(MOE_ERR_RANGE,
                "an NVFP4 block scale is a NaN code, a tensor scale is not finite, or a block "
                "multiplier leaves the normal range of its operand type");
  return fail(MOE_ERR_TIMEOUT, "a bounded device wait ran out (status 0x%08x, site %u)", v,
              v & 0x7FFFFFFFu);
}

int moe_set_ffn_trace(uint64_t* buf, int64_t capacity_ctas) {
  if (buf == nullptr) {
    g_trace.store(nullptr);
    g_trace_cap.store(0);
    return MOE_OK;
  }
  REQUIRE(aligned(buf, 8), "trace buffer must be 8-byte aligned");
  REQUIRE(capacity_ctas > 0, "trace capacity must be positive");
  g_trace_cap.store(capacity_ctas);
  g_trace.store(buf);
  return MOE_OK;
}

int moe_set_wait_timeout_ns(uint64_t ns) {
  if (ns < 1000ull) return fail(MOE_ERR_INVALID_ARG, "timeout below 1 us");
  g_timeout_ns.store(ns);
  return MOE_OK;
}

size_t moe_packed_weight_bytes(void) { return static_cast<size_t>(kPackElems) * 2; }

int moe_pack_weights(const moe_bf16* w_gate, const moe_bf16* w_up, const moe_bf16* w_down,
                     moe_bf16* packed, moe_stream_t stream) {
  REQUIRE(w_gate && w_up && w_down && packed, "null pointer");
  REQUIRE(aligned(packed, 128), "packed must be 128-byte aligned");
  int rc = device_setup(nullptr, nullptr);
  if (rc) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const dim3 ggu(kI / 32, kH / 32, kE), gd(kH / 32, kI / 32, kE);
  pack_transpose_kernel<<<ggu, 256, 0, s>>>(w_gate, packed, kH, kI, 0, kPackGuElems);
  pack_transpose_kernel<<<ggu, 256, 0, s>>>(w_up, packed, kH, kI, 1, kPackGuElems);
  pack_transpose_kernel<<<gd, 256, 0, s>>>(w_down, packed, kI, kH, 2, kPackGuElems);
  return launch_check("pack_transpose_kernel launch");
}

int moe_route(const float* logits, const float* bias, int64_t T, int32_t* topk_idx, float* topk_w,
              moe_stream_t stream) {
  int rc = check_T(T);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  REQUIRE(logits && topk_idx && topk_w, "null pointer");
  REQUIRE(aligned(logits, 16) && (!bias || aligned(bias, 16)) && aligned(topk_idx, 16) &&
              aligned(topk_w, 16),
          "pointers must be 16-byte aligned");
  rc = device_setup(nullptr, nullptr);
  if (rc) return rc;
  return do_route(logits, bias, T, topk_idx, topk_w, reinterpret_cast<cudaStream_t>(stream));
}

size_t moe_permute_workspace_bytes(int64_t T) {
  if (T < 0 || T > kMaxTokens) return 0;
  return permute_ws_bytes(T);
}

int moe_permute(const int32_t* topk_idx, int64_t T, int32_t* counts, int32_t* offsets,
                int32_t* perm_src, int32_t* inv_perm, void* workspace, size_t workspace_bytes,
                moe_stream_t stream) {
  int rc = check_T(T);
  if (rc) return rc;
  REQUIRE(counts && offsets, "null pointer");
  if (T > 0) REQUIRE(topk_idx && perm_src && inv_perm, "null pointer");
  const size_t need = permute_ws_bytes(T);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return fail(MOE_ERR_WORKSPACE, "permute workspace needs %zu bytes, got %zu", need,
                workspace ? workspace_bytes : size_t(0));
  if (need > 0) REQUIRE(aligned(workspace, 16), "workspace must be 16-byte aligned");
  rc = device_setup(nullptr, nullptr);
  if (rc) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {
    MOE_CUDA(cudaMemsetAsync(counts, 0, kE * sizeof(int32_t), s), "cudaMemsetAsync");
    MOE_CUDA(cudaMemsetAsync(offsets, 0, kOffsetsLen * sizeof(int32_t), s), "cudaMemsetAsync");
    return MOE_OK;
  }
  return do_permute(topk_idx, T, counts, offsets, perm_src, inv_perm, workspace, s);
}

int moe_expert_ffn(const moe_bf16* x, const moe_bf16* packed_w, const int32_t* offsets,
                   const int32_t* perm_src, int64_t T, moe_bf16* h, moe_bf16* y_perm,
                   moe_stream_t stream) {
  int rc = check_T(T);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  REQUIRE(x && packed_w && offsets && perm_src && h && y_perm, "null pointer");
  REQUIRE(aligned(x, 128) && aligned(packed_w, 128) && aligned(h, 128),
          "x, packed_w and h must be 128-byte aligned");
  REQUIRE(aligned(y_perm, 16) && aligned(offsets, 16) && aligned(perm_src, 16),
          "pointers must be 16-byte aligned");
  int sms = 0;
  rc = device_setup(nullptr, &sms);
  if (rc) return rc;
  return do_expert_ffn(x, packed_w, offsets, perm_src, T, h, y_perm, sms,
                       reinterpret_cast<cudaStream_t>(stream));
}

int moe_expert_gate_up(const moe_bf16* x, const moe_bf16* packed_w, const int32_t* offsets,
                       const int32_t* perm_src, int64_t T, moe_bf16* h, moe_stream_t stream) {
  int rc = check_T(T);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  REQUIRE(x && packed_w && offsets && perm_src && h, "null pointer");
  REQUIRE(aligned(x, 128) && aligned(packed_w, 128) && aligned(h, 128),
          "x, packed_w and h must be 128-byte aligned");
  REQUIRE(aligned(offsets, 16) && aligned(perm_src, 16), "pointers must be 16-byte aligned");
  int sms = 0;
  rc = device_setup(nullptr, &sms);
  if (rc) return rc;
  return do_gate_up(x, packed_w, offsets, perm_src, T, h, sms,
                    reinterpret_cast<cudaStream_t>(stream));
}

int moe_expert_down(const moe_bf16* h, const moe_bf16* packed_w, const int32_t* offsets,
                    int64_t T, moe_bf16* y_perm, moe_stream_t stream) {
  int rc = check_T(T);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  REQUIRE(h && packed_w && offsets && y_perm, "null pointer");
  REQUIRE(aligned(packed_w, 128) && aligned(h, 128), "packed_w and h must be 128-byte aligned");
  REQUIRE(aligned(y_perm, 16) && aligned(offsets, 16), "pointers must be 16-byte aligned");
  int sms = 0;
  rc = device_setup(nullptr, &sms);
  if (rc) return rc;
  return do_down(h, packed_w, offsets, T, y_perm, sms, reinterpret_cast<cudaStream_t>(stream));
}

int moe_combine(const moe_bf16* y_perm, const float* topk_w, const int32_t* inv_perm, int64_t T,
                const moe_bf16* residual, moe_bf16* out, moe_stream_t stream) {
  int rc = check_T(T);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  REQUIRE(y_perm && topk_w && inv_perm && out, "null pointer");
  REQUIRE(aligned(y_perm, 16) && aligned(topk_w, 16) && aligned(inv_perm, 16) &&
              aligned(out, 16) && (!residual || aligned(residual, 16)),
          "pointers must be 16-byte aligned");
  rc = device_setup(nullptr, nullptr);
  if (rc) return rc;
  return do_combine(y_perm, topk_w, inv_perm, T, residual, out,
                    reinterpret_cast<cudaStream_t>(stream));
}

size_t moe_layer_workspace_bytes(int64_t T) {
  if (T < 0 || T > kMaxTokens) return 0;
  return layer_ws(T).total;
}

}  // extern "C"

namespace {
// The layer from given router logits, or (packed_router != NULL) from the
// router projection of x computed into the workspace first.
// With packed_q != NULL the experts are the quantised layer it points to,
// block-FP8 (qfmt 1) or NVFP4 (qfmt 2); packed_w is then ignored.
int layer_impl(const char* fn, const moe_bf16* x, const float* logits,
               const moe_bf16* packed_router, const float* bias, const moe_bf16* packed_w,
               int64_t T, const moe_bf16* residual, moe_bf16* out, int32_t* topk_idx_out,
               float* topk_w_out, void* workspace, size_t workspace_bytes, moe_stream_t stream,
               const void* packed_q = nullptr, const moe_bf16* packed_shared = nullptr,
               int n_shared = 0, int qfmt = 1) {
  int rc = check_T(T);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  const bool quant = packed_q != nullptr;
  if (quant) packed_w = static_cast<const moe_bf16*>(packed_q);
  REQUIRE(x && (logits || packed_router) && packed_w && out && workspace, "null pointer");
  REQUIRE(aligned(x, 128) && aligned(packed_w, 128) && (!packed_router || aligned(packed_router, 128)),
          "x, the packed weights and packed_router must be 128-byte aligned");
  REQUIRE(aligned(workspace, 1024), "workspace must be 1024-byte aligned");
  REQUIRE((!logits || aligned(logits, 16)) && (!bias || aligned(bias, 16)) && aligned(out, 16) &&
              (!residual || aligned(residual, 16)) && (!topk_idx_out || aligned(topk_idx_out, 16)) &&
              (!topk_w_out || aligned(topk_w_out, 16)),
          "pointers must be 16-byte aligned");
  REQUIRE(n_shared >= 0 && n_shared <= kMaxShared, "n_shared=%d outside [0, %d]", n_shared,
          kMaxShared);
  REQUIRE(n_shared == 0 || (packed_shared && aligned(packed_shared, 128)),
          "packed_shared must be a 128-byte aligned pointer when n_shared > 0");
  const LayerWs L = layer_ws(T, quant, n_shared);
  if (workspace_bytes < L.total)
    return fail(MOE_ERR_WORKSPACE, "%s workspace needs %zu bytes, got %zu", fn, L.total,
                workspace_bytes);
  int sms = 0;
  rc = device_setup(nullptr, &sms);
  if (rc) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  int32_t* idx = topk_idx_out ? topk_idx_out : reinterpret_cast<int32_t*>(ws + L.idx);
  float* w = topk_w_out ? topk_w_out : reinterpret_cast<float*>(ws + L.w);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* perm_src = reinterpret_cast<int32_t*>(ws + L.perm_src);
  int32_t* inv_perm = reinterpret_cast<int32_t*>(ws + L.inv_perm);
  moe_bf16* h = reinterpret_cast<moe_bf16*>(ws + L.h);
  moe_bf16* y = reinterpret_cast<moe_bf16*>(ws + L.y);

  if (packed_router != nullptr && T <= rsmall::kMaxT) {
    // router projection, routing and the sort in one launch
    rc = do_router_route_small(x, packed_router, bias, T, reinterpret_cast<float*>(ws + L.logits),
                               idx, w, counts, offsets, perm_src, inv_perm, s);
  } else {
    if (packed_router != nullptr) {
      float* lg = reinterpret_cast<float*>(ws + L.logits);
      rc = do_router(x, packed_router, T, lg, sms, s);
      logits = lg;
    }
    if (!rc)
      rc = do_route_permute(logits, bias, T, idx, w, counts, offsets, perm_src, inv_perm,
                            ws + L.perm_ws, s);
  }
  // A single token: the FFN launch runs the combine too (not with a
  // separate shared-expert launch, which the combine must follow).
  const bool fused = T <= kFusedCombineMaxT && !(quant && n_shared > 0);
  FusedCombine cmb{};
  if (fused)
    cmb = FusedCombine{w, inv_perm, reinterpret_cast<const __nv_bfloat16*>(residual),
                       reinterpret_cast<__nv_bfloat16*>(out), n_shared};
  moe_bf16* y_sh = reinterpret_cast<moe_bf16*>(ws + L.sh_y);
  int32_t* sh_offsets = reinterpret_cast<int32_t*>(ws + L.sh_offsets);
  int32_t* sh_perm = reinterpret_cast<int32_t*>(ws + L.sh_perm);
  moe_bf16* sh_h = reinterpret_cast<moe_bf16*>(ws + L.sh_h);
  if (!rc && !quant && n_shared > 0) {
    // the routed experts and the shared experts as two segments of one launch
    rc = do_shared_rows(n_shared, T, sh_offsets, sh_perm, s);
    SegMaps maps{};
    SegPtrs p{};
    p.n = 2;
    if (!rc) rc = ffn_maps(&maps, 0, packed_w, kE, kPackGuElems, h, T * kTopK, T);
    if (!rc)
      rc = ffn_maps(&maps, 1, packed_shared, n_shared, int64_t(n_shared) * kPackGuPerExpert,
                    sh_h, int64_t(n_shared) * T, T);
    p.offsets[0] = offsets;
    p.perm_src[0] = perm_src;
    p.h_out[0] = reinterpret_cast<uint16_t*>(h);
    p.y_out[0] = reinterpret_cast<uint16_t*>(y);
    p.offsets[1] = sh_offsets;
    p.perm_src[1] = sh_perm;
    p.h_out[1] = reinterpret_cast<uint16_t*>(sh_h);
    p.y_out[1] = reinterpret_cast<uint16_t*>(y_sh);
    if (!rc) rc = do_ffn_segments(maps, p, x, T, sms, s, cmb);
  } else {
    if (!rc) {
      if (quant && qfmt == 2)
        rc = do_expert_ffn_fp4(x, packed_q, offsets, perm_src, T, h, y,
                               reinterpret_cast<moe_bf16*>(ws + L.dq), sms, s, cmb);
      else if (quant)
        rc = do_expert_ffn_fp8(x, packed_q, offsets, perm_src, T, h, y,
                               reinterpret_cast<moe_bf16*>(ws + L.dq), sms, s, cmb);
      else
        rc = do_expert_ffn(x, packed_w, offsets, perm_src, T, h, y, sms, s, kE, kPackGuElems, -1,
                           cmb);
    }
    if (!rc && n_shared > 0)
      rc = do_shared_ffn(x, packed_shared, n_shared, T, sh_offsets, sh_perm, sh_h, y_sh, sms, s);
  }
  if (!rc && !fused) rc = do_combine(y, w, inv_perm, T, residual, out, s, y_sh, n_shared);
  return rc;
}
}  // namespace

extern "C" {

int moe_layer(const moe_bf16* x, const float* logits, const float* bias, const moe_bf16* packed_w,
              int64_t T, const moe_bf16* residual, moe_bf16* out, int32_t* topk_idx_out,
              float* topk_w_out, void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  if (T > 0 && logits == nullptr) return fail(MOE_ERR_INVALID_ARG, "null pointer");
  return layer_impl("moe_layer", x, logits, nullptr, bias, packed_w, T, residual, out,
                    topk_idx_out, topk_w_out, workspace, workspace_bytes, stream);
}

int moe_layer_routed(const moe_bf16* x, const moe_bf16* packed_router, const float* bias,
                     const moe_bf16* packed_w, int64_t T, const moe_bf16* residual,
                     moe_bf16* out, int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                     size_t workspace_bytes, moe_stream_t stream) {
  if (T > 0 && packed_router == nullptr) return fail(MOE_ERR_INVALID_ARG, "null pointer");
  return layer_impl("moe_layer_routed", x, nullptr, packed_router, bias, packed_w, T, residual,
                    out, topk_idx_out, topk_w_out, workspace, workspace_bytes, stream);
}

// ---- the layer from host buffers --------------------------------------------------
namespace {
struct HostWs {
  size_t x, logits, out, layer, total;
};
HostWs host_ws(int64_t T, int fmt) {
  HostWs H{};
  size_t o = 0;
  auto take = [&](size_t bytes, size_t align) {
    o = align_up(o, align);
    const size_t at = o;
    o += bytes;
    return at;
  };
  H.x = take(static_cast<size_t>(T) * kH * 2, 1024);
  H.logits = take(static_cast<size_t>(T) * kE * 4, 1024);
  H.out = take(static_cast<size_t>(T) * kH * 2, 1024);
  H.layer = take(layer_ws(T, fmt != 0).total, 1024);
  H.total = align_up(o, 1024);
  return H;
}
}  // namespace

size_t moe_layer_host_workspace_bytes(int64_t T, int weight_format) {
  if (T < 0 || T > kMaxTokens || weight_format < 0 || weight_format > 2) return 0;
  return host_ws(T, weight_format).total;
}

int moe_layer_host(const moe_bf16* x_host, const float* logits_host, const float* bias,
                   const void* packed, int weight_format, int64_t T, moe_bf16* out_host,
                   void* workspace, size_t workspace_bytes, void* wait_event, void* done_event,
                   moe_stream_t stream) {
  int rc = check_T(T);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  REQUIRE(weight_format >= 0 && weight_format <= 2, "weight_format=%d outside [0, 2]",
          weight_format);
  REQUIRE(x_host && logits_host && packed && out_host && workspace, "null pointer");
  REQUIRE(aligned(workspace, 1024), "workspace must be 1024-byte aligned");
  const HostWs H = host_ws(T, weight_format);
  if (workspace_bytes < H.total)
    return fail(MOE_ERR_WORKSPACE, "moe_layer_host workspace needs %zu bytes, got %zu", H.total,
                workspace_bytes);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  auto* x = reinterpret_cast<moe_bf16*>(ws + H.x);
  auto* lg = reinterpret_cast<float*>(ws + H.logits);
  auto* out = reinterpret_cast<moe_bf16*>(ws + H.out);
  // one copy per buffer; host memory should be page-locked for the copies to
  // overlap other work
  MOE_CUDA(cudaMemcpyAsync(x, x_host, static_cast<size_t>(T) * kH * 2, cudaMemcpyHostToDevice, s),
           "cudaMemcpyAsync (x)");
  MOE_CUDA(cudaMemcpyAsync(lg, logits_host, static_cast<size_t>(T) * kE * 4,
                           cudaMemcpyHostToDevice, s),
           "cudaMemcpyAsync (logits)");
  if (wait_event != nullptr)
    MOE_CUDA(cudaStreamWaitEvent(s, static_cast<cudaEvent_t>(wait_event), 0), "cudaStreamWaitEvent");
  const size_t lbytes = H.total - H.layer;
  if (weight_format == 0)
    rc = layer_impl("moe_layer_host", x, lg, nullptr, bias, static_cast<const moe_bf16*>(packed), T,
                    nullptr, out, nullptr, nullptr, ws + H.layer, lbytes, stream);
  else
    rc = layer_impl("moe_layer_host", x, lg, nullptr, bias, nullptr, T, nullptr, out, nullptr,
                    nullptr, ws + H.layer, lbytes, stream, packed, nullptr, 0, weight_format);
  if (rc) return rc;
  if (done_event != nullptr)
    MOE_CUDA(cudaEventRecord(static_cast<cudaEvent_t>(done_event), s), "cudaEventRecord");
  MOE_CUDA(cudaMemcpyAsync(out_host, out, static_cast<size_t>(T) * kH * 2, cudaMemcpyDeviceToHost,
                           s),
           "cudaMemcpyAsync (out)");
  return MOE_OK;
}

size_t moe_router_packed_bytes(void) { return static_cast<size_t>(kE) * kH * 2; }

int moe_pack_router(const moe_bf16* w_router, moe_bf16* packed_router, moe_stream_t stream) {
  REQUIRE(w_router && packed_router, "null pointer");
  REQUIRE(aligned(packed_router, 128), "packed_router must be 128-byte aligned");
  int rc = device_setup(nullptr, nullptr);
  if (rc) return rc;
  router::router_pack_kernel<<<dim3(kE / 32, kH / 32), 256, 0,
                               reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint16_t*>(w_router), reinterpret_cast<uint16_t*>(packed_router));
  return launch_check("router_pack_kernel launch");
}

int moe_router(const moe_bf16* x, const moe_bf16* packed_router, int64_t T, float* logits,
               moe_stream_t stream) {
  int rc = check_T(T);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  REQUIRE(x && packed_router && logits, "null pointer");
  REQUIRE(aligned(x, 128) && aligned(packed_router, 128), "x and packed_router must be 128-byte aligned");
  REQUIRE(aligned(logits, 16), "logits must be 16-byte aligned");
  int sms = 0;
  rc = device_setup(nullptr, &sms);
  if (rc) return rc;
  return do_router(x, packed_router, T, logits, sms, reinterpret_cast<cudaStream_t>(stream));
}

int moe_route_from_x(const moe_bf16* x, const moe_bf16* packed_router, const float* bias,
                     int64_t T, float* logits, int32_t* topk_idx, float* topk_w,
                     moe_stream_t stream) {
  int rc = check_T(T);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  REQUIRE(x && packed_router && logits && topk_idx && topk_w, "null pointer");
  REQUIRE(aligned(x, 128) && aligned(packed_router, 128),
          "x and packed_router must be 128-byte aligned");
  REQUIRE(aligned(logits, 16) && (!bias || aligned(bias, 16)) && aligned(topk_idx, 16) &&
              aligned(topk_w, 16),
          "pointers must be 16-byte aligned");
  int sms = 0;
  rc = device_setup(nullptr, &sms);
  if (rc) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T <= rsmall::kMaxT)
    return do_router_route_small(x, packed_router, bias, T, logits, topk_idx, topk_w, nullptr,
                                 nullptr, nullptr, nullptr, s);
  rc = do_router(x, packed_router, T, logits, sms, s);
  if (rc) return rc;
  return do_route(logits, bias, T, topk_idx, topk_w, s);
}

// ---- block-FP8 experts ---------------------------------------------------------
size_t moe_packed_fp8_bytes(void) { return static_cast<size_t>(fp8::kPackedBytes); }

int moe_pack_weights_fp8(const uint8_t* q_gate, const float* s_gate, const uint8_t* q_up,
                         const float* s_up, const uint8_t* q_down, const float* s_down,
                         void* packed_fp8, moe_stream_t stream) {
  REQUIRE(q_gate && s_gate && q_up && s_up && q_down && s_down && packed_fp8, "null pointer");
  REQUIRE(aligned(packed_fp8, 128), "packed_fp8 must be 128-byte aligned");
  REQUIRE(aligned(s_gate, 4) && aligned(s_up, 4) && aligned(s_down, 4),
          "scales must be 4-byte aligned");
  int rc = device_setup(nullptr, nullptr);
  if (rc) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* p8 = static_cast<uint8_t*>(packed_fp8);
  const dim3 ggu(kI / 32, kH / 32, kE), gd(kH / 32, kI / 32, kE);
  fp8::pack_fp8_transpose_kernel<<<ggu, 256, 0, s>>>(q_gate, p8, kH, kI, 0, s_down);
  fp8::pack_fp8_transpose_kernel<<<ggu, 256, 0, s>>>(q_up, p8, kH, kI, 1, s_down);
  fp8::pack_fp8_transpose_kernel<<<gd, 256, 0, s>>>(q_down, p8, kI, kH, 2, s_down);
  constexpr int n_sc = kE * (fp8::kSguPerExpert + fp8::kSdPerExpert);
  fp8::pack_fp8_scales_kernel<<<(n_sc + 255) / 256, 256, 0, s>>>(
      s_gate, s_up, s_down, reinterpret_cast<float*>(p8 + fp8::kSguOff),
      reinterpret_cast<float*>(p8 + fp8::kSdOff));
  return launch_check("pack_fp8 kernels launch");
}

int moe_dequant_fp8(const void* packed_fp8, moe_bf16* packed, moe_stream_t stream) {
  REQUIRE(packed_fp8 && packed, "null pointer");
  REQUIRE(aligned(packed_fp8, 128) && aligned(packed, 128),
          "packed_fp8 and packed must be 128-byte aligned");
  int sms = 0;
  int rc = device_setup(nullptr, &sms);
  if (rc) return rc;
  return do_dequant_fp8(packed_fp8, packed, sms, reinterpret_cast<cudaStream_t>(stream));
}

size_t moe_expert_ffn_fp8_workspace_bytes(int64_t T) {
  if (T < 0 || T > kMaxTokens) return 0;
  return T > kSkinnyMaxT ? static_cast<size_t>(kPackElems) * 2 : 0;
}

int moe_expert_ffn_fp8(const moe_bf16* x, const void* packed_fp8, const int32_t* offsets,
                       const int32_t* perm_src, int64_t T, moe_f16* h, moe_f16* y_perm,
                       void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  int rc = check_T(T);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  REQUIRE(x && packed_fp8 && offsets && perm_src && h && y_perm, "null pointer");
  REQUIRE(aligned(x, 128) && aligned(packed_fp8, 128) && aligned(h, 128),
          "x, packed_fp8 and h must be 128-byte aligned");
  REQUIRE(aligned(y_perm, 16) && aligned(offsets, 16) && aligned(perm_src, 16),
          "pointers must be 16-byte aligned");
  const size_t need = moe_expert_ffn_fp8_workspace_bytes(T);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return fail(MOE_ERR_WORKSPACE, "moe_expert_ffn_fp8 workspace needs %zu bytes, got %zu", need,
                workspace ? workspace_bytes : size_t(0));
  if (need > 0) REQUIRE(aligned(workspace, 128), "workspace must be 128-byte aligned");
  int sms = 0;
  rc = device_setup(nullptr, &sms);
  if (rc) return rc;
  return do_expert_ffn_fp8(x, packed_fp8, offsets, perm_src, T, h, y_perm,
                           static_cast<moe_bf16*>(workspace), sms,
                           reinterpret_cast<cudaStream_t>(stream));
}

size_t moe_layer_fp8_workspace_bytes(int64_t T) {
  if (T < 0 || T > kMaxTokens) return 0;
  return layer_ws(T, true).total;
}

int moe_layer_fp8(const moe_bf16* x, const float* logits, const float* bias,
                  const void* packed_fp8, int64_t T, const moe_bf16* residual, moe_bf16* out,
                  int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                  size_t workspace_bytes, moe_stream_t stream) {
  if (T > 0 && (logits == nullptr || packed_fp8 == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "null pointer");
  return layer_impl("moe_layer_fp8", x, logits, nullptr, bias, nullptr, T, residual, out,
                    topk_idx_out, topk_w_out, workspace, workspace_bytes, stream, packed_fp8);
}

// ---- NVFP4 experts ---------------------------------------------------------------
size_t moe_packed_nvfp4_bytes(void) { return static_cast<size_t>(fp4::kPackedBytes); }

int moe_pack_weights_nvfp4(const uint8_t* q_gate, const uint8_t* s_gate, const float* g_gate,
                           const uint8_t* q_up, const uint8_t* s_up, const float* g_up,
                           const uint8_t* q_down, const uint8_t* s_down, const float* g_down,
                           void* packed_nvfp4, moe_stream_t stream) {
  REQUIRE(q_gate && s_gate && g_gate && q_up && s_up && g_up && q_down && s_down && g_down &&
              packed_nvfp4,
          "null pointer");
  REQUIRE(aligned(packed_nvfp4, 128), "packed_nvfp4 must be 128-byte aligned");
  REQUIRE(aligned(q_gate, 4) && aligned(q_up, 4) && aligned(q_down, 4) && aligned(g_gate, 4) &&
              aligned(g_up, 4) && aligned(g_down, 4),
          "codes and tensor scales must be 4-byte aligned");
  int sms = 0;
  int rc = device_setup(nullptr, &sms);
  if (rc) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* p4 = static_cast<uint8_t*>(packed_nvfp4);
  const dim3 grid(sms * 8), block(256);
  fp4::pack_fp4_codes_kernel<<<grid, block, 0, s>>>(reinterpret_cast<const uint32_t*>(q_gate), p4, 0);
  fp4::pack_fp4_codes_kernel<<<grid, block, 0, s>>>(reinterpret_cast<const uint32_t*>(q_up), p4, 1);
  fp4::pack_fp4_codes_kernel<<<grid, block, 0, s>>>(reinterpret_cast<const uint32_t*>(q_down), p4, 2);
  fp4::pack_fp4_mult_kernel<<<grid, block, 0, s>>>(s_gate, s_up, s_down, g_gate, g_up, g_down,
                                                   reinterpret_cast<uint16_t*>(p4 + fp4::kMguOff));
  return launch_check("pack_fp4 kernels launch");
}

int moe_dequant_nvfp4(const void* packed_nvfp4, moe_bf16* packed, moe_stream_t stream) {
  REQUIRE(packed_nvfp4 && packed, "null pointer");
  REQUIRE(aligned(packed_nvfp4, 128) && aligned(packed, 128),
          "packed_nvfp4 and packed must be 128-byte aligned");
  int sms = 0;
  int rc = device_setup(nullptr, &sms);
  if (rc) return rc;
  return do_dequant_fp4(packed_nvfp4, packed, sms, reinterpret_cast<cudaStream_t>(stream));
}

size_t moe_expert_ffn_nvfp4_workspace_bytes(int64_t T) {
  return moe_expert_ffn_fp8_workspace_bytes(T);
}

int moe_expert_ffn_nvfp4(const moe_bf16* x, const void* packed_nvfp4, const int32_t* offsets,
                         const int32_t* perm_src, int64_t T, moe_f16* h, moe_f16* y_perm,
                         void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  int rc = check_T(T);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  REQUIRE(x && packed_nvfp4 && offsets && perm_src && h && y_perm, "null pointer");
  REQUIRE(aligned(x, 128) && aligned(packed_nvfp4, 128) && aligned(h, 128),
          "x, packed_nvfp4 and h must be 128-byte aligned");
  REQUIRE(aligned(y_perm, 16) && aligned(offsets, 16) && aligned(perm_src, 16),
          "pointers must be 16-byte aligned");
  const size_t need = moe_expert_ffn_nvfp4_workspace_bytes(T);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need))
    return fail(MOE_ERR_WORKSPACE, "moe_expert_ffn_nvfp4 workspace needs %zu bytes, got %zu",
                need, workspace ? workspace_bytes : size_t(0));
  if (need > 0) REQUIRE(aligned(workspace, 128), "workspace must be 128-byte aligned");
  int sms = 0;
  rc = device_setup(nullptr, &sms);
  if (rc) return rc;
  return do_expert_ffn_fp4(x, packed_nvfp4, offsets, perm_src, T, h, y_perm,
                           static_cast<moe_bf16*>(workspace), sms,
                           reinterpret_cast<cudaStream_t>(stream));
}

size_t moe_layer_nvfp4_workspace_bytes(int64_t T) { return moe_layer_fp8_workspace_bytes(T); }

int moe_layer_nvfp4(const moe_bf16* x, const float* logits, const float* bias,
                    const void* packed_nvfp4, int64_t T, const moe_bf16* residual, moe_bf16* out,
                    int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                    size_t workspace_bytes, moe_stream_t stream) {
  if (T > 0 && (logits == nullptr || packed_nvfp4 == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "null pointer");
  return layer_impl("moe_layer_nvfp4", x, logits, nullptr, bias, nullptr, T, residual, out,
                    topk_idx_out, topk_w_out, workspace, workspace_bytes, stream, packed_nvfp4,
                    nullptr, 0, 2);
}

// ---- shared experts --------------------------------------------------------------
size_t moe_packed_shared_bytes(int n_shared) {
  if (n_shared < 0 || n_shared > kMaxShared) return 0;
  return static_cast<size_t>(n_shared) * (kPackGuPerExpert + kPackDPerExpert) * 2;
}

int moe_pack_shared(const moe_bf16* w_gate, const moe_bf16* w_up, const moe_bf16* w_down,
                    int n_shared, moe_bf16* packed_shared, moe_stream_t stream) {
  REQUIRE(n_shared >= 1 && n_shared <= kMaxShared, "n_shared=%d outside [1, %d]", n_shared,
          kMaxShared);
  REQUIRE(w_gate && w_up && w_down && packed_shared, "null pointer");
  REQUIRE(aligned(packed_shared, 128), "packed_shared must be 128-byte aligned");
  int rc = device_setup(nullptr, nullptr);
  if (rc) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t d_off = int64_t(n_shared) * kPackGuPerExpert;
  const dim3 ggu(kI / 32, kH / 32, n_shared), gd(kH / 32, kI / 32, n_shared);
  pack_transpose_kernel<<<ggu, 256, 0, s>>>(w_gate, packed_shared, kH, kI, 0, d_off);
  pack_transpose_kernel<<<ggu, 256, 0, s>>>(w_up, packed_shared, kH, kI, 1, d_off);
  pack_transpose_kernel<<<gd, 256, 0, s>>>(w_down, packed_shared, kI, kH, 2, d_off);
  return launch_check("pack_transpose_kernel launch (shared)");
}

// ---- a slice of a layer's experts (expert parallelism) ---------------------------
size_t moe_packed_experts_bytes(int n_experts) {
  if (n_experts < 1 || n_experts > kE) return 0;
  return static_cast<size_t>(n_experts) * (kPackGuPerExpert + kPackDPerExpert) * 2;
}

int moe_pack_experts(const moe_bf16* w_gate, const moe_bf16* w_up, const moe_bf16* w_down,
                     int n_experts, moe_bf16* packed, moe_stream_t stream) {
  REQUIRE(n_experts >= 1 && n_experts <= kE, "n_experts=%d outside [1, %d]", n_experts, kE);
  REQUIRE(w_gate && w_up && w_down && packed, "null pointer");
  REQUIRE(aligned(packed, 128), "packed must be 128-byte aligned");
  int rc = device_setup(nullptr, nullptr);
  if (rc) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t d_off = int64_t(n_experts) * kPackGuPerExpert;
  const dim3 ggu(kI / 32, kH / 32, n_experts), gd(kH / 32, kI / 32, n_experts);
  pack_transpose_kernel<<<ggu, 256, 0, s>>>(w_gate, packed, kH, kI, 0, d_off);
  pack_transpose_kernel<<<ggu, 256, 0, s>>>(w_up, packed, kH, kI, 1, d_off);
  pack_transpose_kernel<<<gd, 256, 0, s>>>(w_down, packed, kI, kH, 2, d_off);
  return launch_check("pack_transpose_kernel launch (expert slice)");
}

int moe_expert_ffn_slice(const moe_bf16* x, const moe_bf16* packed, int n_experts,
                         const int32_t* offsets, const int32_t* perm_src, int64_t T, moe_bf16* h,
                         moe_bf16* y_perm, moe_stream_t stream) {
  int rc = check_T(T);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  REQUIRE(n_experts >= 1 && n_experts <= kE, "n_experts=%d outside [1, %d]", n_experts, kE);
  REQUIRE(x && packed && offsets && perm_src && h && y_perm, "null pointer");
  REQUIRE(aligned(x, 128) && aligned(packed, 128) && aligned(h, 128),
          "x, packed and h must be 128-byte aligned");
  REQUIRE(aligned(y_perm, 16) && aligned(offsets, 16) && aligned(perm_src, 16),
          "pointers must be 16-byte aligned");
  int sms = 0;
  rc = device_setup(nullptr, &sms);
  if (rc) return rc;
  return do_expert_ffn(x, packed, offsets, perm_src, T, h, y_perm, sms,
                       reinterpret_cast<cudaStream_t>(stream), n_experts,
                       int64_t(n_experts) * kPackGuPerExpert);
}

size_t moe_layer_shared_workspace_bytes(int64_t T, int n_shared, int fp8_routed) {
  if (T < 0 || T > kMaxTokens || n_shared < 0 || n_shared > kMaxShared) return 0;
  return layer_ws(T, fp8_routed != 0, n_shared).total;
}

int moe_layer_shared(const moe_bf16* x, const float* logits, const float* bias,
                     const moe_bf16* packed_w, const void* packed_fp8,
                     const moe_bf16* packed_shared, int n_shared, int64_t T,
                     const moe_bf16* residual, moe_bf16* out, int32_t* topk_idx_out,
                     float* topk_w_out, void* workspace, size_t workspace_bytes,
                     moe_stream_t stream) {
  if (T > 0 && (logits == nullptr || (packed_w == nullptr) == (packed_fp8 == nullptr)))
    return fail(MOE_ERR_INVALID_ARG,
                "moe_layer_shared needs logits and exactly one of packed_w, packed_fp8");
  return layer_impl("moe_layer_shared", x, logits, nullptr, bias, packed_w, T, residual, out,
                    topk_idx_out, topk_w_out, workspace, workspace_bytes, stream, packed_fp8,
                    packed_shared, n_shared);
}

int moe_layer_shared_nvfp4(const moe_bf16* x, const float* logits, const float* bias,
                           const void* packed_nvfp4, const moe_bf16* packed_shared, int n_shared,
                           int64_t T, const moe_bf16* residual, moe_bf16* out,
                           int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                           size_t workspace_bytes, moe_stream_t stream) {
  if (T > 0 && (logits == nullptr || packed_nvfp4 == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "null pointer");
  return layer_impl("moe_layer_shared_nvfp4", x, logits, nullptr, bias, nullptr, T, residual,
                    out, topk_idx_out, topk_w_out, workspace, workspace_bytes, stream,
                    packed_nvfp4, packed_shared, n_shared, 2);
}

}  // extern "C"

// ---- second MoE shape: 256 experts top-6 ------------------------------------------
namespace {
struct E256Ws {
  size_t idx, w, counts, offsets, off_lo, off_hi, perm_src, inv_perm, hist, h, y;
  size_t sh_offsets, sh_perm, sh_h, sh_y, total;
};
E256Ws e256_ws(int64_t T, int n_shared) {
  E256Ws L{};
  const size_t n = static_cast<size_t>(T) * kTopK;  // 8-slot numbering, 6 used
  const size_t nb = static_cast<size_t>((T + e256::kBlockTokens - 1) / e256::kBlockTokens);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 1024);
    return at;
  };
  L.idx = take(static_cast<size_t>(T) * e256::kTopK2 * 4);
  L.w = take(static_cast<size_t>(T) * e256::kTopK2 * 4);
  L.counts = take(e256::kE2 * 4);
  L.offsets = take((e256::kE2 + 1) * 4);
  L.off_lo = take(kOffsetsLen * 4);
  L.off_hi = take(kOffsetsLen * 4);
  L.perm_src = take(n * 4);
  L.inv_perm = take(n * 4);
  L.hist = take(nb * e256::kE2 * 4);
  L.h = take(n * kI * 2);
  L.y = take(n * kH * 2);
  const size_t ns = static_cast<size_t>(n_shared) * static_cast<size_t>(T);
  L.sh_offsets = take(n_shared ? kOffsetsLen * 4 : 0);
  L.sh_perm = take(ns * 4);
  L.sh_h = take(ns * kI * 2);
  L.sh_y = take(ns * kH * 2);
  L.total = o;
  return L;
}

int do_route_e256(const float* logits, const float* bias, int64_t T, int32_t* idx, float* w,
                  cudaStream_t s) {
  const int64_t blocks = (T + e256::kRouteWarps2 - 1) / e256::kRouteWarps2;
  return launch_pdl("route_e256_kernel launch", e256::route_e256_kernel,
                    dim3(static_cast<unsigned>(blocks)), dim3(e256::kRouteWarps2 * 32), 0, s,
                    logits, bias, T, idx, w);
}
}  // namespace

extern "C" {

int moe_route_e256(const float* logits, const float* bias, int64_t T, int32_t* topk_idx,
                   float* topk_w, moe_stream_t stream) {
  int rc = check_T(T);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  REQUIRE(logits && topk_idx && topk_w, "null pointer");
  REQUIRE(aligned(logits, 16) && (!bias || aligned(bias, 16)) && aligned(topk_idx, 16) &&
              aligned(topk_w, 16),
          "pointers must be 16-byte aligned");
  rc = device_setup(nullptr, nullptr);
  if (rc) return rc;
  return do_route_e256(logits, bias, T, topk_idx, topk_w, reinterpret_cast<cudaStream_t>(stream));
}

size_t moe_layer_e256_workspace_bytes(int64_t T, int n_shared) {
  if (T < 0 || T > kMaxTokens || n_shared < 0 || n_shared > kMaxShared) return 0;
  return e256_ws(T, n_shared).total;
}

int moe_layer_e256(const moe_bf16* x, const float* logits, const float* bias,
                   const moe_bf16* packed_lo, const moe_bf16* packed_hi,
                   const moe_bf16* packed_shared, int n_shared, int64_t T,
                   const moe_bf16* residual, moe_bf16* out, int32_t* topk_idx_out,
                   float* topk_w_out, void* workspace, size_t workspace_bytes,
                   moe_stream_t stream) {
  int rc = check_T(T);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  REQUIRE(x && logits && packed_lo && packed_hi && out && workspace, "null pointer");
  REQUIRE(n_shared >= 0 && n_shared <= kMaxShared, "n_shared=%d outside [0, %d]", n_shared,
          kMaxShared);
  REQUIRE(n_shared == 0 || (packed_shared && aligned(packed_shared, 128)),
          "packed_shared must be a 128-byte aligned pointer when n_shared > 0");
  REQUIRE(aligned(x, 128) && aligned(packed_lo, 128) && aligned(packed_hi, 128),
          "x and the packed weights must be 128-byte aligned");
  REQUIRE(aligned(workspace, 1024), "workspace must be 1024-byte aligned");
  REQUIRE(aligned(logits, 16) && (!bias || aligned(bias, 16)) && aligned(out, 16) &&
              (!residual || aligned(residual, 16)) && (!topk_idx_out || aligned(topk_idx_out, 16)) &&
              (!topk_w_out || aligned(topk_w_out, 16)),
          "pointers must be 16-byte aligned");
  const E256Ws L = e256_ws(T, n_shared);
  if (workspace_bytes < L.total)
    return fail(MOE_ERR_WORKSPACE, "moe_layer_e256 workspace needs %zu bytes, got %zu", L.total,
                workspace_bytes);
  int sms = 0;
  rc = device_setup(nullptr, &sms);
  if (rc) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  int32_t* idx = topk_idx_out ? topk_idx_out : reinterpret_cast<int32_t*>(ws + L.idx);
  float* w = topk_w_out ? topk_w_out : reinterpret_cast<float*>(ws + L.w);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + L.hist);
  int32_t* off_lo = reinterpret_cast<int32_t*>(ws + L.off_lo);
  int32_t* off_hi = reinterpret_cast<int32_t*>(ws + L.off_hi);
  int32_t* perm_src = reinterpret_cast<int32_t*>(ws + L.perm_src);
  int32_t* inv_perm = reinterpret_cast<int32_t*>(ws + L.inv_perm);
  moe_bf16* h = reinterpret_cast<moe_bf16*>(ws + L.h);
  moe_bf16* y = reinterpret_cast<moe_bf16*>(ws + L.y);
  const int nb = static_cast<int>((T + e256::kBlockTokens - 1) / e256::kBlockTokens);

  if (T <= e256::kSmallMaxT) {  // routing and the counting sort in one block
    rc = launch_pdl("route_sort_small_e256_kernel launch", e256::route_sort_small_e256_kernel,
                    dim3(1), dim3(e256::kSmallThreads), 0, s, logits, bias, static_cast<int>(T), idx,
                    w, reinterpret_cast<int32_t*>(ws + L.counts),
                    reinterpret_cast<int32_t*>(ws + L.offsets), off_lo, off_hi, perm_src, inv_perm);
  } else {
    rc = do_route_e256(logits, bias, T, idx, w, s);
    if (!rc)
      rc = launch_pdl("count_e256_kernel launch", e256::count_e256_kernel, dim3(nb), dim3(256), 0,
                      s, static_cast<const int32_t*>(idx), T, hist);
    if (!rc)
      rc = launch_pdl("scan_e256_kernel launch", e256::scan_e256_kernel, dim3(1), dim3(256), 0, s,
                      hist, nb, reinterpret_cast<int32_t*>(ws + L.counts),
                      reinterpret_cast<int32_t*>(ws + L.offsets), off_lo, off_hi);
    if (!rc)
      rc = launch_pdl("scatter_e256_kernel launch", e256::scatter_e256_kernel, dim3(nb), dim3(256),
                      0, s, static_cast<const int32_t*>(idx), T, static_cast<const int32_t*>(hist),
                      perm_src, inv_perm);
  }
  moe_bf16* y_sh = reinterpret_cast<moe_bf16*>(ws + L.sh_y);
  int32_t* sh_offsets = reinterpret_cast<int32_t*>(ws + L.sh_offsets);
  int32_t* sh_perm = reinterpret_cast<int32_t*>(ws + L.sh_perm);
  moe_bf16* sh_h = reinterpret_cast<moe_bf16*>(ws + L.sh_h);
  {
    // one launch over experts 0..127, 128..255 and the shared experts (three
    // segments: each pack, its offsets, its rows)
    if (!rc && n_shared > 0) rc = do_shared_rows(n_shared, T, sh_offsets, sh_perm, s);
    SegMaps maps{};
    SegPtrs p{};
    const moe_bf16* packs[3] = {packed_lo, packed_hi, packed_shared};
    const int32_t* offs[3] = {off_lo, off_hi, sh_offsets};
    const int32_t* perms[3] = {perm_src, perm_src, sh_perm};
    moe_bf16* hs[3] = {h, h, sh_h};
    moe_bf16* ys[3] = {y, y, y_sh};
    p.n = n_shared > 0 ? 3 : 2;
    for (int g = 0; g < p.n && !rc; ++g) {
      const bool routed = g < 2;
      rc = ffn_maps(&maps, g, packs[g], routed ? kE : n_shared,
                    routed ? kPackGuElems : int64_t(n_shared) * kPackGuPerExpert, hs[g],
                    routed ? T * kTopK : int64_t(n_shared) * T, T);
      p.offsets[g] = offs[g];
      p.perm_src[g] = perms[g];
      p.h_out[g] = reinterpret_cast<uint16_t*>(hs[g]);
      p.y_out[g] = reinterpret_cast<uint16_t*>(ys[g]);
    }
    if (!rc) rc = do_ffn_segments(maps, p, x, T, sms, s);
  }
  if (!rc)
    rc = launch_pdl("combine_kernel launch", combine_kernel<e256::kTopK2>,
                    dim3(static_cast<unsigned>(T)), dim3(kCombineThreads), 0, s,
                    reinterpret_cast<const uint16_t*>(y), static_cast<const float*>(w),
                    static_cast<const int32_t*>(inv_perm), T,
                    reinterpret_cast<const __nv_bfloat16*>(residual),
                    reinterpret_cast<__nv_bfloat16*>(out), reinterpret_cast<const uint16_t*>(y_sh),
                    n_shared);
  return rc;
}

}  // extern "C"

// ---- timeout self-test ------------------------------------------------------
namespace {
__global__ void selftest_wait_kernel(uint64_t timeout_ns, int* done_flag) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // nothing ever arrives
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(&bar, 0, &abort_flag, timeout_ns, kSiteSelftest);
    (void)ok;
  }
  __syncthreads();
}
}  // namespace

extern "C" int moe_selftest_wait_timeout(moe_stream_t stream) {
  int rc = device_setup(nullptr, nullptr);
  if (rc) return rc;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(g_timeout_ns.load(),
                                                                             nullptr);
  return launch_check("selftest_wait_kernel launch");
}

// ---- permutation with library-owned scratch ----------------------------------
// moe_permute takes its per-block histogram from a caller workspace, which the
// caller has to allocate.  Some callers cannot allocate when they permute:
//   - a serving runtime that reserves all of its device memory once at
//     start-up and hands every byte to a fixed plan, so a later request has
//     nowhere to come from;
//   - code that runs inside a memory allocator's own bookkeeping, where a
//     nested allocation would re-enter the allocator;
//   - latency-bound loops that must not pay for an allocator miss, or for the
//     device-wide synchronisation that freeing device memory implies.
// For those, the histogram lives in a file-scope device array of fixed size
// that belongs to the library, so the call allocates nothing.
namespace {
constexpr int64_t kFixedPermMaxT = 65536;
constexpr int64_t kFixedPermBlocks = (kFixedPermMaxT + kPermBlockTokens - 1) / kPermBlockTokens;
// hist[b][e] for up to 512 blocks of 128 tokens: 256 KiB per device.  The count
// kernel writes every entry that the scan and scatter kernels later read, so no
// word of it has to start at zero; the only words that must start at zero, the
// expert-FFN work counters offsets[132..263], are written by the permute
// kernels themselves.
static __device__ __align__(256) int32_t g_fixed_perm_hist[kFixedPermBlocks * kE];

int32_t* g_fixed_perm_ptr[kMaxDevices] = {};
std::mutex g_fixed_perm_mu;

// Device address of the array on the current device, looked up the first time
// a device asks for it (with that device current) and kept afterwards.
int fixed_perm_scratch(int32_t** out) {
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_fixed_perm_mu);
  if (g_fixed_perm_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_fixed_perm_hist);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(fixed permute scratch)");
    if (p == nullptr || !aligned(p, 256))
      return fail(MOE_ERR_CUDA, "fixed permute scratch has a bad device address");
    g_fixed_perm_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_fixed_perm_ptr[dev];
  return MOE_OK;
}
}  // namespace

extern "C" int64_t moe_permute_fixed_scratch_max_tokens(void) { return kFixedPermMaxT; }

extern "C" int moe_permute_fixed_scratch(const int32_t* topk_idx, int64_t T, int32_t* counts,
                                         int32_t* offsets, int32_t* perm_src, int32_t* inv_perm,
                                         moe_stream_t stream) {
  if (T < 0 || T > kFixedPermMaxT)
    return fail(MOE_ERR_INVALID_ARG,
                "T=%lld outside [0, %lld]: the fixed permute scratch holds %lld blocks of %d "
                "tokens; use moe_permute with a workspace for more",
                static_cast<long long>(T), static_cast<long long>(kFixedPermMaxT),
                static_cast<long long>(kFixedPermBlocks), kPermBlockTokens);
  REQUIRE(counts && offsets, "null pointer");
  if (T > 0) REQUIRE(topk_idx && perm_src && inv_perm, "null pointer");
  int rc = device_setup(nullptr, nullptr);
  if (rc) return rc;
  int32_t* hist = nullptr;
  rc = fixed_perm_scratch(&hist);
  if (rc) return rc;
  if (permute_ws_bytes(T) > sizeof(g_fixed_perm_hist))
    return fail(MOE_ERR_WORKSPACE, "fixed permute scratch too small for T=%lld",
                static_cast<long long>(T));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {
    MOE_CUDA(cudaMemsetAsync(counts, 0, kE * sizeof(int32_t), s), "cudaMemsetAsync");
    MOE_CUDA(cudaMemsetAsync(offsets, 0, kOffsetsLen * sizeof(int32_t), s), "cudaMemsetAsync");
    return MOE_OK;
  }
  return do_permute(topk_idx, T, counts, offsets, perm_src, inv_perm, hist, s);
}

// ---- explicit per-device set-up ----------------------------------------------
extern "C" int moe_init_device(void) {
  int rc = device_setup(nullptr, nullptr);
  if (rc) return rc;
  int32_t* hist = nullptr;
  return fixed_perm_scratch(&hist);
}
