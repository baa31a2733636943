// common.cuh -- constants and sm_100a PTX wrappers shared by the libmoe kernels.
//
// Every device-side wait goes through mbar_wait(), which is bounded in time:
// when it runs out it records the site in the per-device status word, raises
// the block's abort flag and returns false so that the caller can leave its
// loop, drain its own copies and let the block exit normally.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kH = 1536;     // hidden size
constexpr int kI = 512;      // expert intermediate size
constexpr int kE = 128;      // routed experts
constexpr int kG = 8;        // groups
constexpr int kGS = 16;      // experts per group
constexpr int kKeep = 4;     // groups kept per token
constexpr int kTopK = 8;     // experts per token

// Per-device status word.  0 = fine; otherwise bit 31 set and the low bits
// hold the site id of the first wait that ran out (or a bad-index code).
__device__ unsigned int g_status;

enum StatusSite : unsigned {
  kSiteBadIndex = 1,
  kSiteFp16Range = 2,
  kSiteFfnEmpty = 16,
  kSiteFfnFull = 17,
  kSiteFfnTmemFull = 18,
  kSiteFfnTmemEmpty = 19,
  kSiteFfnDrain = 20,
  kSiteTileQueue = 21,
  kSiteFfnDone = 22,  // a down tile waiting for its expert's gate/up tiles
  kSiteFp8Nan = 23,   // a NaN E4M3 code in packed block-FP8 weights
  kSiteSelftest = 30,
};

__device__ __forceinline__ void record_status(unsigned site) {
  atomicCAS(&g_status, 0u, 0x80000000u | site);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase of `bar` with the given parity.  `abort_flag`
// lives in shared memory and is shared by the whole block.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t timeout_ns, unsigned site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 31u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > timeout_ns) {
        record_status(site);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Waits, on the way out of a kernel, for this thread's own asynchronous work
// (a TMA copy it issued, or its MMAs through a commit) to land before the CTA
// frees its shared or tensor memory.  Bounded (10 ms), and not cut short by
// the CTA's abort flag, which is usually what sent the thread here.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, unsigned site) {
  int no_abort = 0;
  mbar_wait(bar, parity, &no_abort, 10000000ull, site);
}

// ---------------------------------------------------------------- cp.async

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed.
// The barrier's expected count includes this arrival (.noinc).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// ---------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t c0,
                                            int32_t c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// Untiled bulk copy global -> shared of `bytes` (multiple of 16, both
// addresses 16-byte aligned), completing on `bar` like a TMA load.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t* slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, 16-bit inputs (type in idesc), fp32
// accumulate, single CTA.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T: the A operand read from tensor memory
// (row i of A in lane i, consecutive K elements packed two per 32-bit column),
// B from a shared-memory descriptor; 16-bit inputs, fp32 accumulate.
__device__ __forceinline__ void umma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor: K-major operand stored as rows of 128 bytes
// (64 bf16) with the 128-byte swizzle, 8-row groups 1024 bytes apart.
// Fields: start address >> 4 [0,14), leading offset [16,30) (unused by the
// swizzled K-major form, set to 1), stride offset >> 4 [32,46) = 1024 B,
// descriptor version 1 at [46,48), swizzle mode 2 (128 B) at [61,64).
__device__ __forceinline__ uint64_t smem_desc_k128(uint32_t smem_addr) {
  return static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu) | (uint64_t(1) << 16) |
         (uint64_t(1024 >> 4) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Instruction descriptor for kind::f16: fp32 accumulator, A and B of the same
// 16-bit type (ab_format 0 = fp16, 1 = bf16), both K-major, M x N tile.
__host__ __device__ constexpr uint32_t idesc_f32acc(int M, int N, uint32_t ab_format) {
  return (1u << 4) | (ab_format << 7) | (ab_format << 10) | (uint32_t(N >> 3) << 17) |
         (uint32_t(M >> 4) << 24);
}
constexpr uint32_t kFmtF16 = 0, kFmtBF16 = 1;

// Two loads of 32 consecutive fp32 columns of the calling warp's 32 TMEM
// lanes (one row per thread), completed before returning.
__device__ __forceinline__ void tmem_ld_2x32(uint32_t taddr0, uint32_t taddr1, uint32_t (&a)[32],
                                             uint32_t (&b)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]),
        "=r"(a[7]), "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]),
        "=r"(a[14]), "=r"(a[15]), "=r"(a[16]), "=r"(a[17]), "=r"(a[18]), "=r"(a[19]),
        "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]), "=r"(a[24]), "=r"(a[25]),
        "=r"(a[26]), "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31]),
        "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]),
        "=r"(b[7]), "=r"(b[8]), "=r"(b[9]), "=r"(b[10]), "=r"(b[11]), "=r"(b[12]), "=r"(b[13]),
        "=r"(b[14]), "=r"(b[15]), "=r"(b[16]), "=r"(b[17]), "=r"(b[18]), "=r"(b[19]),
        "=r"(b[20]), "=r"(b[21]), "=r"(b[22]), "=r"(b[23]), "=r"(b[24]), "=r"(b[25]),
        "=r"(b[26]), "=r"(b[27]), "=r"(b[28]), "=r"(b[29]), "=r"(b[30]), "=r"(b[31])
      : "r"(taddr0), "r"(taddr1)
      : "memory");
}

// Stores 32 consecutive 32-bit columns of the calling warp's 32 TMEM lanes
// (one lane per thread), asynchronously: tmem_wait_st() waits for them.
__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t* a) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]),
      "r"(a[8]), "r"(a[9]), "r"(a[10]), "r"(a[11]), "r"(a[12]), "r"(a[13]), "r"(a[14]),
      "r"(a[15]), "r"(a[16]), "r"(a[17]), "r"(a[18]), "r"(a[19]), "r"(a[20]), "r"(a[21]),
      "r"(a[22]), "r"(a[23]), "r"(a[24]), "r"(a[25]), "r"(a[26]), "r"(a[27]), "r"(a[28]),
      "r"(a[29]), "r"(a[30]), "r"(a[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void st_global_b16(void* p, uint16_t v) {
  asm volatile("st.global.b16 [%0], %1;" ::"l"(p), "h"(v) : "memory");
}

// ---------------------------------------------------------------- programmatic dependent launch
// The layer's kernels are launched with programmatic stream serialisation: a
// kernel may be scheduled while its predecessor finishes, runs its prologue,
// and waits (griddep_wait) for the predecessor's completion and memory before
// touching anything the predecessor produces or reads.  Every kernel lets its
// successor launch as soon as all of its own CTAs are resident.  Launched
// without the attribute, both instructions do nothing.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- dynamic tile queue
// Persistent GEMM CTAs take every tile id, the first one included, from a
// global counter, so that a CTA that met slow tiles (weights from HBM rather
// than L2, stalls) takes fewer of them, and so that only a CTA that is
// running can own a tile: in the single-launch expert FFN a down tile waits
// for its expert's gate/up tiles, and those were handed out earlier (the
// counter only grows) to CTAs that were running then and finish them without
// waiting on anything outside the CTA.  So the wait ends however many of the
// grid's CTAs are resident at once (SMs shared with another stream's
// kernels, MPS, a green context with fewer SMs).  Inside a CTA one
// thread grabs tile ids and publishes them through a small shared-memory queue
// that every warp role reads in the same order.  The counter words live after
// the expert offsets (see kSchedWord), followed by 128 per-expert completion
// counters of the single-launch expert FFN: moe_permute zeroes them all, and
// the last CTA of every GEMM launch sets the ones it used back to zero.

constexpr int kTileQ = 4;          // queue slots
constexpr int kSchedWord = 132;    // offsets[132..135]: scheduler words (2 per GEMM phase)
constexpr int kOffsetsLen = 264;   // length of the offsets array ([136..263]: expert counters)

struct TileQueue {
  int tile[kTileQ];
  uint64_t full[kTileQ];
  uint64_t empty[kTileQ];
};

__device__ __forceinline__ void tileq_init(TileQueue* q, uint32_t consumers) {
  for (int i = 0; i < kTileQ; ++i) {
    mbar_init(&q->full[i], 1);
    mbar_init(&q->empty[i], consumers);
  }
}

// Producer side (one thread): publish tile id `tile` (or -1 = no more work) as
// the n-th entry.  Returns false if the wait for a free slot ran out.
__device__ __forceinline__ bool tileq_push(TileQueue* q, int n, int tile, volatile int* abort_flag,
                                           uint64_t timeout_ns) {
  const int slot = n % kTileQ;
  const uint32_t ph = (n / kTileQ) & 1;
  if (!mbar_wait(&q->empty[slot], ph ^ 1, abort_flag, timeout_ns, kSiteTileQueue)) return false;
  reinterpret_cast<volatile int*>(q->tile)[slot] = tile;
  mbar_arrive(&q->full[slot]);
  return true;
}

// Consumer side: the n-th tile id (-1: no more work, -2: wait ran out).  Every
// lane of a consuming warp calls this; lane 0 (or the single consuming
// thread) releases the slot after the whole warp has read it.
__device__ __forceinline__ int tileq_pop(TileQueue* q, int n, bool release,
                                         volatile int* abort_flag, uint64_t timeout_ns) {
  const int slot = n % kTileQ;
  const uint32_t ph = (n / kTileQ) & 1;
  if (!mbar_wait(&q->full[slot], ph, abort_flag, timeout_ns, kSiteTileQueue)) return -2;
  const int tile = reinterpret_cast<volatile int*>(q->tile)[slot];
  __syncwarp(__activemask());
  if (release) mbar_arrive(&q->empty[slot]);
  return tile;
}

// Non-blocking look at the n-th tile id: returns it if the producer has
// published it already, else -3.  The slot is not released (tileq_pop does
// that when its turn comes).
__device__ __forceinline__ int tileq_peek(TileQueue* q, int n) {
  const int slot = n % kTileQ;
  const uint32_t ph = (n / kTileQ) & 1;
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(&q->full[slot])), "r"(ph)
      : "memory");
  return ok ? reinterpret_cast<volatile int*>(q->tile)[slot] : -3;
}

// End of a launch: the last CTA to finish zeroes the two counter words (and
// the n_extra words at `extra`, if any).
// Returns true in the CTA that retired last (the one that reset the words).
__device__ __forceinline__ bool tileq_retire(int* sched, int* extra = nullptr, int n_extra = 0) {
  __threadfence();
  const int fin = atomicAdd(sched + 1, 1);
  if (fin == static_cast<int>(gridDim.x) - 1) {
    atomicExch(sched, 0);
    atomicExch(sched + 1, 0);
    for (int i = 0; i < n_extra; ++i) atomicExch(extra + i, 0);
    return true;
  }
  return false;
}

constexpr int kDoneWord = kSchedWord + 4;  // offsets[136 .. 263]: per-expert done counters

// Weight packs of one expert-FFN launch ("segments"): up to kMaxSeg packs of
// up to 128 experts each, every one with its own offsets array (the down
// tiles' done counters live in it), row sources and h / y_perm rows.  The
// 256-expert shape runs its two halves and its shared experts as three
// segments of one launch, the shared experts of the 128-expert shape run as a
// second segment beside the routed pack; every other call is one segment.
// Tile ids run over all segments' gate/up tiles, then all segments' down
// tiles.
constexpr int kMaxSeg = 3;
struct SegMaps {
  CUtensorMap w1[kMaxSeg];  // gate/up weights (phase 1)
  CUtensorMap w2[kMaxSeg];  // down weights (phase 2)
  CUtensorMap h[kMaxSeg];   // h rows (phase 2)
};
struct SegPtrs {
  int n;                             // segments in the launch, 1 .. kMaxSeg
  const int32_t* offsets[kMaxSeg];   // offsets array (129 offsets, then the work counters)
  const int32_t* perm_src[kMaxSeg];  // row sources (8t + slot)
  uint16_t* h_out[kMaxSeg];
  uint16_t* y_out[kMaxSeg];
};


// Waits until *counter >= need (acquire), bounded in time; then orders the
// async proxy (TMA) after it.
__device__ __forceinline__ bool wait_count(const int* counter, int need, volatile int* abort_flag,
                                           uint64_t timeout_ns, unsigned site) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t n = 0;; ++n) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
    if (v >= need) break;
    if (*abort_flag) return false;
    if ((n & 15u) == 15u && global_timer_ns() - t0 > timeout_ns) {
      record_status(site);
      *abort_flag = 1;
      return false;
    }
    __nanosleep(64);
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

// ---------------------------------------------------------------- misc

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// fp16 pair with round-to-nearest-even; `bad` collects values outside the
// fp16 range (or NaN), which the caller reports instead of storing infinities
// silently.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi, bool& bad) {
  bad |= !(fabsf(lo) <= 65504.f) || !(fabsf(hi) <= 65504.f);
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float f16_lo(uint32_t v) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(v & 0xFFFFu)));
}
__device__ __forceinline__ float f16_hi(uint32_t v) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(v >> 16)));
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ void st_global_v4(void* p, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

}  // namespace moe
