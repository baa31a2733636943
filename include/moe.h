/*
 * moe.h -- C ABI of libmoe, the B200 (sm_100a) routed-expert MoE layer of
 * Ling-3.0-tiny: group-limited top-k routing, token-to-expert permutation,
 * grouped SwiGLU expert FFN on tcgen05 tensor cores, weighted combine.
 *
 * Layer shape, as the pages state it:
 *   - 128 routed experts per layer in 8 groups of 16, 4 groups kept per
 *     token, hidden size 1536: "Ling-3.0-tiny on a Qualcomm board" (TensorFold
 *     issue #1247), first comment, opening paragraph.
 *   - 8 experts active per token: "HelloSun/ling30tiny", table 模型與路由
 *     (model and routing), row on experts active per token.
 *   - experts with gate, up and down matrices (a SwiGLU FFN), no SwiGLU
 *     clamp ("null SwiGLU limit lists"): same table, row on expert weights;
 *     issue #1247, opening paragraph.  Intermediate size 512.
 *
 * Conventions shared by every entry point
 *   - Return value: a moe_status code.  No C++ exception crosses the ABI.
 *     moe_last_error_string() describes the last failure of the calling
 *     thread.
 *   - Pointers are caller-owned DEVICE memory unless stated otherwise.  The
 *     library never allocates, frees or reads device memory from the host,
 *     and never synchronises a stream; every call is asynchronous on
 *     `stream` (a cudaStream_t; NULL means the legacy default stream).
 *   - Arrays are dense row-major.  Every pointer must be 16-byte aligned;
 *     bf16 matrices read by the tensor-memory-accelerator (x, packed weights,
 *     the h workspace) must be 128-byte aligned.
 *   - T (tokens) is int64_t; 0 <= T <= moe_max_tokens().  T == 0 is a valid
 *     no-op.  Invalid arguments return MOE_ERR_INVALID_ARG before anything is
 *     launched.  Internal address arithmetic is 64-bit ("Add TML Inkling
 *     architecture", llama.cpp PR #25731, description: int64 indices because
 *     large MoEs overflow 32-bit ones).
 *   - bf16 values are passed as raw 16-bit patterns (moe_bf16).
 *   - Device-side waits inside the kernels are bounded in time.  A wait that
 *     runs out sets a per-device error word and makes the kernel return;
 *     moe_get_device_status() reports it as MOE_ERR_TIMEOUT.
 *   - The first call of the library on a device sets that device up: it
 *     queries its properties, raises the kernels' shared-memory limits
 *     (cudaFuncSetAttribute) and resolves the tensor-map encoder.  Those
 *     calls are not stream operations, so make the first call on each device
 *     outside stream capture (moe_init_device() does the set-up alone); later
 *     calls only launch kernels and can be captured into a CUDA graph.
 *   - Calls on different streams may run at the same time on one device (they
 *     share nothing but the device status word), provided they do not share
 *     a workspace or an offsets array.  The persistent expert-FFN kernels
 *     hand out every tile, the first included, from a global counter, so a
 *     kernel that gets fewer SMs than its grid (another stream's kernels, MPS
 *     or a green context) still finishes: only running CTAs own work.
 */
#ifndef MOE_B200_MOE_H
#define MOE_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* cudaStream_t */
typedef uint16_t moe_bf16;                /* raw bfloat16 bits */
typedef uint16_t moe_f16;                 /* raw IEEE binary16 bits */

enum {
  MOE_HIDDEN = 1536,     /* H: model width */
  MOE_INTER = 512,       /* I: expert intermediate size */
  MOE_EXPERTS = 128,     /* E: routed experts per layer */
  MOE_GROUPS = 8,        /* expert groups */
  MOE_GROUP_SIZE = 16,   /* experts per group */
  MOE_KEEP_GROUPS = 4,   /* groups kept per token */
  MOE_TOPK = 8,          /* experts used per token */
  MOE_OFFSETS_LEN = 264  /* int32 words of the offsets array (129 offsets + scratch) */
};

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* bad size, null or misaligned pointer */
  MOE_ERR_WORKSPACE = 2,   /* workspace smaller than the query says */
  MOE_ERR_CUDA = 3,        /* a CUDA runtime / driver call failed */
  MOE_ERR_TIMEOUT = 4,     /* a bounded device-side wait ran out */
  MOE_ERR_UNSUPPORTED = 5, /* device is not sm_100 */
  MOE_ERR_RANGE = 6        /* an fp16 intermediate (h, y_perm, packed W_down)
                              left the fp16 range, a block-FP8 weight is a
                              NaN code, or an NVFP4 block multiplier is out
                              of range; reported by moe_get_device_status() */
} moe_status;

/* ---- library information ------------------------------------------------ */

/* ABI version of this header (bumped on any signature change). */
int moe_abi_version(void);

/* Largest T accepted by every entry point. */
int64_t moe_max_tokens(void);

/* Text of the calling thread's last error ("" when none).  The pointer stays
 * valid until the next call on that thread. */
const char* moe_last_error_string(void);

/* Reads and clears the error word of `device` that the kernels set: a bounded
 * wait that ran out (MOE_ERR_TIMEOUT), an fp16 intermediate out of range
 * (MOE_ERR_RANGE) or an out-of-range index in caller data
 * (MOE_ERR_INVALID_ARG).  MOE_OK when clean; MOE_ERR_CUDA if the query failed.
 * This is the one call that synchronises: it copies 4 bytes to the host. */
int moe_get_device_status(int device);

/* Sets the current device up for the library (the set-up that the first call
 * on a device does otherwise): checks that it is an sm_100 device, raises the
 * kernels' shared-memory limits, resolves the tensor-map encoder and looks up
 * the device address of moe_permute_fixed_scratch's scratch array.  Call it
 * once per device, with that device current, before capturing any library
 * call into a CUDA graph.  Idempotent; MOE_ERR_UNSUPPORTED on other devices. */
int moe_init_device(void);

/* Time limit of every bounded device-side wait, in nanoseconds (default 2e9).
 * Applies to launches issued after the call. */
int moe_set_wait_timeout_ns(uint64_t ns);

/* Diagnostics with no counterpart in the pages: a per-CTA timing record of
 * the persistent expert-FFN launches, for measuring how evenly their tiles
 * spread over the SMs (the tail of a grouped GEMM whose experts hold very
 * different row counts).  While set, every expert-FFN launch of at most
 * `capacity_ctas` CTAs writes, for CTA b:
 *   buf[3b]     the device clock (%globaltimer, ns) when b started work, after
 *               the preceding kernel's results became visible;
 *   buf[3b + 1] the device clock when b had finished its last tile;
 *   buf[3b + 2] the number of tiles b ran.
 * Each launch overwrites the record of the one before (so the record is that
 * of the last expert-FFN launch).  buf: device memory of 3 * capacity_ctas
 * uint64 words, 8-byte aligned, caller-owned; NULL turns the record off (the
 * default).  A launch with more CTAs than capacity_ctas records nothing. */
int moe_set_ffn_trace(uint64_t* buf, int64_t capacity_ctas);

/* Launches one block whose bounded wait on a barrier that nothing completes
 * must run out after the current limit: a self-test of the timeout path.  The
 * kernel returns normally and leaves the context usable; afterwards
 * moe_get_device_status() returns MOE_ERR_TIMEOUT. */
int moe_selftest_wait_timeout(moe_stream_t stream);

/* ---- weights ------------------------------------------------------------ */

/* Bytes of one layer's packed expert weights (604 MB). */
size_t moe_packed_weight_bytes(void);

/* One-time re-layout of one layer's expert weights into the tensor-core
 * operand order used by moe_expert_ffn.  W_down is converted to fp16: exact
 * for bf16 values in the fp16 normal range [2^-14, 65504]; a magnitude below
 * 2^-14 is rounded to the nearest fp16 subnormal (an absolute error of at
 * most 2^-25 per weight); a magnitude above 65504 is flagged (MOE_ERR_RANGE
 * from moe_get_device_status()).
 *   w_gate, w_up : [128][1536][512] bf16, the layer computes x @ W_gate[e]
 *   w_down       : [128][512][1536] bf16, the layer computes h @ W_down[e]
 *   packed       : moe_packed_weight_bytes() bytes, 128-byte aligned, output.
 * Packed layout: per expert, W_gate/W_up transposed to K-major [512][1536] and
 * interleaved in blocks of 128 output columns (gate block j, up block j, ...),
 * followed (after all experts' gate/up blocks, 128 x 1024 x 1536 elements)
 * by every expert's W_down transposed to [1536][512] in fp16.  Inputs must not
 * alias `packed`. */
int moe_pack_weights(const moe_bf16* w_gate, const moe_bf16* w_up,
                     const moe_bf16* w_down, moe_bf16* packed,
                     moe_stream_t stream);

/* ---- the four steps ----------------------------------------------------- */

/* Step 1: group-limited top-8 routing.  Up to 64 tokens one warp works on
 * each token (moe_layer fuses this with step 2 in one block); above that, 8
 * lanes share a token, one per group, which needs half the instructions per
 * token at large T.  Group-limited routing runs as its own kernel in the GB10 CUDA path of issue
 * #1247 ("What it does not cover", bullet on the CUDA C kernels); the score
 * rule used here:
 *   s_e = sigmoid(logit[t,e] + bias[e])                 (float64)
 *   group score = sum of the two largest s_e of the group
 *   keep the 4 best groups (ties: lower group index)
 *   topk_idx[t,0..7] = the 8 largest s_e inside kept groups, in descending
 *                      order (ties: lower expert index)
 *   topk_w[t,i] = sigmoid(logit[t,e_i]) / sum_j sigmoid(logit[t,e_j])
 *   logits : [T][128] fp32          bias : [128] fp32, or NULL for zeros
 *   topk_idx : [T][8] int32 (out)   topk_w : [T][8] fp32 (out)  */
int moe_route(const float* logits, const float* bias, int64_t T,
              int32_t* topk_idx, float* topk_w, moe_stream_t stream);

/* Scratch bytes moe_permute needs for T tokens (0 when T <= 1024). */
size_t moe_permute_workspace_bytes(int64_t T);

/* Step 2: device-side stable counting sort of the T*8 (token, slot) items by
 * expert, so that each expert runs on exactly the rows that picked it with no
 * host round trip (issue #1247, "What it does not cover", bullet on bf16
 * experts: the per-expert row loop there needs a host sync per layer).
 *   topk_idx : [T][8] int32 (from moe_route); an id of -1 marks an empty
 *              slot, which gets no row (the expert-parallel receiver's rows
 *              carry only the slots whose experts it owns)
 *   counts   : [128] int32 (out)  rows per expert
 *   offsets  : [MOE_OFFSETS_LEN] int32 (out): [0..128] exclusive prefix of counts,
 *              offsets[128] = the number of non-empty slots (8T when none is
 *              empty); [132..263] zeroed work counters that the expert-FFN
 *              kernels use and leave at zero (words 129..131 unused)
 *   perm_src : [8T] int32 (out)   permuted row r holds item t*8+slot; rows are
 *                                 expert-major, token-ascending inside an expert
 *   inv_perm : [8T] int32 (out)   item t*8+slot sits at row inv_perm[t*8+slot]
 *                                 (-1 for an empty slot; moe_combine skips it)
 *   workspace: moe_permute_workspace_bytes(T) bytes (may be NULL when 0). */
int moe_permute(const int32_t* topk_idx, int64_t T, int32_t* counts,
                int32_t* offsets, int32_t* perm_src, int32_t* inv_perm,
                void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* Step 3: grouped SwiGLU expert FFN over the permuted rows, persistent
 * tcgen05 GEMMs (the grouped kernel that issue #1247 names as missing):
 *   h[r]      = silu(x[t] W_gate[e]) * (x[t] W_up[e])   (bf16 in, fp32 accumulate, fp16 out)
 *   y_perm[r] = h[r] W_down[e]                          (fp16 in, fp32 accumulate, fp16 out)
 * for every permuted row r = offsets[e] + i, i < counts[e], t = perm_src[r]/8.
 *   x        : [T][1536] bf16, 128-byte aligned
 *   packed_w : from moe_pack_weights
 *   offsets, perm_src : from moe_permute (the work counters in offsets[132..263]
 *                       are updated during the call and are zero again after it;
 *                       two calls sharing one offsets array must not overlap)
 *   h        : [8T][512] fp16 workspace (out), 128-byte aligned
 *   y_perm   : [8T][1536] fp16 (out)
 * Both GEMMs run in one persistent launch at every T: a down tile starts as
 * soon as every gate/up tile of its expert has stored h.  Up to 256 tokens
 * the weights are the 128-row MMA operand (128 weight rows x 32 tokens per
 * tile); above, the tokens are (128 rows x 256 output columns per tile). */
int moe_expert_ffn(const moe_bf16* x, const moe_bf16* packed_w,
                   const int32_t* offsets, const int32_t* perm_src, int64_t T,
                   moe_f16* h, moe_f16* y_perm, moe_stream_t stream);

/* Step 4: weighted combine back into token order ("HelloSun/ling30tiny",
 * section 數值檢查摘要: routing plus the weighted layer):
 *   out[t] = bf16( residual[t] + sum_{slot 0..7} topk_w[t,slot] * y_perm[inv_perm[8t+slot]] )
 * summed in fp32 in slot order and rounded once (deterministic, no atomics).
 *   y_perm   : [8T][1536] fp16 (from moe_expert_ffn / moe_expert_down)
 *   residual : [T][1536] bf16 or NULL (then 0).  `out` may alias `residual`. */
int moe_combine(const moe_f16* y_perm, const float* topk_w,
                const int32_t* inv_perm, int64_t T, const moe_bf16* residual,
                moe_bf16* out, moe_stream_t stream);

/* Step 3, first half alone: h[r] = silu(x[t] W_gate[e]) * (x[t] W_up[e]),
 * arguments as in moe_expert_ffn (one persistent tcgen05 GEMM launch). */
int moe_expert_gate_up(const moe_bf16* x, const moe_bf16* packed_w,
                       const int32_t* offsets, const int32_t* perm_src, int64_t T,
                       moe_f16* h, moe_stream_t stream);

/* Step 3, second half alone: y_perm[r] = h[r] W_down[e] (one persistent
 * tcgen05 GEMM launch).  h: [8T][512] fp16 from moe_expert_gate_up. */
int moe_expert_down(const moe_f16* h, const moe_bf16* packed_w,
                    const int32_t* offsets, int64_t T, moe_f16* y_perm,
                    moe_stream_t stream);

/* ---- router projection (the step before routing) ----------------------- */

/* The pages name the group-limited routing kernel of the CUDA path ("Ling-3.0-
 * tiny on a Qualcomm board", TensorFold issue #1247, "What it does not cover",
 * first bullet); its input is the projection of the hidden state onto the 128
 * experts, computed here as
 *   logits[t][e] = sum_k x[t][k] W_router[k][e]   (bf16 in, fp32 accumulate, fp32 out)
 * on the tensor cores.  The routing rule's bias is added afterwards by moe_route. */

/* Bytes of the packed router matrix (128 x 1536 bf16). */
size_t moe_router_packed_bytes(void);

/* One-time re-layout of W_router [1536][128] bf16 into the K-major [128][1536]
 * operand order of moe_router.  packed_router: moe_router_packed_bytes()
 * bytes, 128-byte aligned, caller-owned. */
int moe_pack_router(const moe_bf16* w_router, moe_bf16* packed_router, moe_stream_t stream);

/* logits [T][128] fp32 (out) = x [T][1536] bf16 (128-byte aligned) times the
 * packed router.  One persistent tcgen05 GEMM launch (64 tokens per tile). */
int moe_router(const moe_bf16* x, const moe_bf16* packed_router, int64_t T, float* logits,
               moe_stream_t stream);

/* Router projection and routing from x: logits [T][128] fp32 (out), then
 * moe_route on them (topk_idx, topk_w out).  Up to 8 tokens both run in one
 * launch: a cluster of 8 CTAs, each computing 16 experts' logits for every
 * token on the CUDA cores (one warp per dot product, in a fixed order) and
 * storing them into the first CTA's shared memory, which then routes.  Above
 * 8 tokens: moe_router (tensor cores), then moe_route.  The two projections
 * sum in different orders; each is within the fp32 accumulation bound of the
 * exact product. */
int moe_route_from_x(const moe_bf16* x, const moe_bf16* packed_router, const float* bias,
                     int64_t T, float* logits, int32_t* topk_idx, float* topk_w,
                     moe_stream_t stream);

/* ---- the fused layer ---------------------------------------------------- */

/* Workspace bytes moe_layer needs for T tokens. */
size_t moe_layer_workspace_bytes(int64_t T);

/* The whole layer: route -> permute -> expert FFN -> combine, back to back on
 * `stream` with no host synchronisation.  For a single token the combine
 * runs at the end of the expert-FFN launch (by its CTA that retires last, with
 * the arithmetic of moe_combine, bit for bit), one launch fewer.  The same
 * holds for moe_layer_routed, moe_layer_fp8, moe_layer_nvfp4, moe_layer_host
 * and moe_layer_shared with bf16 routed experts; moe_layer_e256 and the
 * quantised layers with shared experts keep the combine launch.
 * Arguments as in the steps above;
 *   residual   : NULL, or [T][1536] bf16 added before the final rounding
 *                (a stack layer computes h <- bf16(h + moe(h)) with
 *                residual = x = out allowed)
 *   topk_idx_out, topk_w_out : optional [T][8] copies of the routing (NULL to skip)
 *   workspace  : moe_layer_workspace_bytes(T) bytes of device memory, 1024-byte aligned. */
int moe_layer(const moe_bf16* x, const float* logits, const float* bias,
              const moe_bf16* packed_w, int64_t T, const moe_bf16* residual,
              moe_bf16* out, int32_t* topk_idx_out, float* topk_w_out,
              void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* moe_layer with the router projection in front: the logits are computed
 * from x into the workspace (same workspace size as moe_layer), then route ->
 * permute -> expert FFN -> combine as above.  Up to 8 tokens the projection,
 * routing and the sort are one launch (as in moe_route_from_x), so the layer
 * is as many launches as moe_layer (two for one token, three up to 8);
 * above, moe_router's tensor-core projection runs first. */
int moe_layer_routed(const moe_bf16* x, const moe_bf16* packed_router, const float* bias,
                     const moe_bf16* packed_w, int64_t T, const moe_bf16* residual,
                     moe_bf16* out, int32_t* topk_idx_out, float* topk_w_out,
                     void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* ---- the layer from host buffers ---------------------------------------- */

/* Workspace bytes of moe_layer_host (weight_format 0 bf16, 1 block FP8, 2
 * NVFP4); 0 for an invalid argument. */
size_t moe_layer_host_workspace_bytes(int64_t T, int weight_format);

/* One layer from HOST buffers, the call a serving loop makes per batch: the
 * token rows and their router logits are copied host -> device into the
 * workspace, the layer runs on those copies (moe_layer, moe_layer_fp8 or
 * moe_layer_nvfp4 by weight_format), and its output is copied device -> host,
 * all asynchronously on `stream`, one cudaMemcpyAsync per buffer.
 *   x_host      : [T][1536] bf16, host memory (page-locked for the copies to
 *                 overlap other work)
 *   logits_host : [T][128] fp32, host memory
 *   bias        : [128] fp32 device memory, or NULL
 *   packed      : the device-resident packed layer of that format
 *   out_host    : [T][1536] bf16, host memory; complete once the stream has
 *                 reached the end of the call (synchronise before reading)
 *   workspace   : moe_layer_host_workspace_bytes(T, weight_format) bytes of
 *                 device memory, 1024-byte aligned
 *   wait_event  : NULL, or a cudaEvent_t the layer waits for after the input
 *                 copies (so that calls on several streams can overlap one
 *                 call's copies with another's layer while the layers
 *                 themselves run one after another)
 *   done_event  : NULL, or a cudaEvent_t recorded when the layer has finished
 *                 (before the output copy) */
int moe_layer_host(const moe_bf16* x_host, const float* logits_host, const float* bias,
                   const void* packed, int weight_format, int64_t T, moe_bf16* out_host,
                   void* workspace, size_t workspace_bytes, void* wait_event, void* done_event,
                   moe_stream_t stream);

/* ---- block-FP8 experts ---------------------------------------------------- */

/* The CUDA path of issue #1247 reads experts in bf16, block FP8 and NVFP4
 * ("What it does not cover", third bullet); the pages do not spell the block-
 * FP8 format out.  Read here as the usual block-FP8 checkpoint form: every
 * weight an FP8 E4M3 code (OCP 8-bit float, no infinities, 0x7F/0xFF NaN,
 * largest finite 448) and every 128 x 128 block of a matrix one fp32 scale,
 *   weight = value(code) * scale.
 * The kernels dequantise each weight to the tensor-core operand type as
 * fp32(value * scale) rounded once to bf16 (gate/up) or fp16 (down).  With
 * power-of-two scales that is exact, and moe_layer_fp8 returns bit for bit
 * what moe_layer returns on the dequantised weights; other scales add one
 * rounding per weight (relative 2^-9 for bf16, 2^-12 for fp16). */

/* Bytes of one layer's packed block-FP8 experts (302 MB: codes, then scales). */
size_t moe_packed_fp8_bytes(void);

/* One-time re-layout of one layer's block-FP8 experts.
 *   q_gate, q_up : [128][1536][512] uint8 E4M3 codes (the layer computes x @ W)
 *   s_gate, s_up : [128][12][4] fp32: scale of rows 128i..128i+127 (of 1536) and
 *                  columns 128j..128j+127 (of 512) at [e][i][j]
 *   q_down       : [128][512][1536] codes;  s_down : [128][4][12] fp32
 *   packed_fp8   : moe_packed_fp8_bytes() bytes, 128-byte aligned, output:
 *                  codes in the operand order of moe_pack_weights (K-major,
 *                  gate/up interleaved in 128-column blocks), then the scales
 *                  reordered to match.
 * Within every aligned group of 4 codes along k the packed bytes hold the
 * elements in the order k+2, k, k+3, k+1 (the dequantisation reads them so).
 * A down weight whose dequantised value lies outside the fp16 range, or a
 * NaN code (0x7F, 0xFF) in any matrix, sets the device error word
 * (moe_get_device_status(): MOE_ERR_RANGE); the packed bytes are written
 * regardless, and the layer's results on such weights are unspecified. */
int moe_pack_weights_fp8(const uint8_t* q_gate, const float* s_gate, const uint8_t* q_up,
                         const float* s_up, const uint8_t* q_down, const float* s_down,
                         void* packed_fp8, moe_stream_t stream);

/* Expands a packed block-FP8 layer into the packed bf16/fp16 layer that
 * moe_pack_weights writes (packed: moe_packed_weight_bytes() bytes, 128-byte
 * aligned, output).  With power-of-two scales it equals moe_pack_weights of
 * the dequantised weights, byte for byte. */
int moe_dequant_fp8(const void* packed_fp8, moe_bf16* packed, moe_stream_t stream);

/* Scratch bytes moe_expert_ffn_fp8 needs: 0 for T <= 256, else
 * moe_packed_weight_bytes() (the expanded layer). */
size_t moe_expert_ffn_fp8_workspace_bytes(int64_t T);

/* Step 3 with block-FP8 experts: moe_expert_ffn's arguments, with packed_fp8
 * (from moe_pack_weights_fp8) in place of packed_w, plus a scratch workspace
 * of moe_expert_ffn_fp8_workspace_bytes(T) bytes (128-byte aligned; may be
 * NULL when that is 0).  Up to 256 tokens one persistent launch streams the
 * codes and dequantises each weight tile in shared memory; above, the layer
 * is expanded into the workspace and the bf16 expert FFN runs on it. */
int moe_expert_ffn_fp8(const moe_bf16* x, const void* packed_fp8, const int32_t* offsets,
                       const int32_t* perm_src, int64_t T, moe_f16* h, moe_f16* y_perm,
                       void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* Workspace bytes moe_layer_fp8 needs for T tokens: moe_layer's, plus room
 * for the expanded layer (moe_packed_weight_bytes()) when T > 256. */
size_t moe_layer_fp8_workspace_bytes(int64_t T);

/* moe_layer with block-FP8 experts (packed_fp8 from moe_pack_weights_fp8),
 * other arguments as in moe_layer.  For T <= 256 the single-launch expert FFN
 * streams the 8-bit codes and dequantises every weight tile on its way to the
 * tensor cores (half the weight bytes of the bf16 layer); above, the layer is
 * first expanded into the workspace (moe_dequant_fp8) and the bf16 expert FFN
 * runs on it.  A caller with the HBM to spare can expand once with
 * moe_dequant_fp8 and call moe_layer on the result, which gives the same
 * output. */
int moe_layer_fp8(const moe_bf16* x, const float* logits, const float* bias,
                  const void* packed_fp8, int64_t T, const moe_bf16* residual,
                  moe_bf16* out, int32_t* topk_idx_out, float* topk_w_out,
                  void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* ---- NVFP4 experts ---------------------------------------------------------- */

/* The third expert format of the same bullet: ModelOpt NVFP4.  For a weight
 * matrix in a linear layer's [out, in] orientation:
 *   - every weight a 4-bit E2M1 code (sign, 2-bit exponent with bias 1, 1-bit
 *     mantissa; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), two codes per byte
 *     along the input dimension, the even element in the low nibble;
 *   - every 16 consecutive weights along the input dimension one FP8 E4M3
 *     block scale (0x7F/0xFF are NaN);
 *   - the matrix one fp32 tensor scale;
 *   weight = value(code) * value(block scale) * tensor scale.
 * The kernels dequantise each weight as value * M rounded once to bf16
 * (gate/up) or fp16 (down), where M, block scale * tensor scale, is rounded to
 * that type at pack time.  With a power-of-two tensor scale M is exact, and
 * moe_layer_nvfp4 returns bit for bit what moe_layer returns on the
 * dequantised weights; other tensor scales add one rounding of M (relative
 * 2^-9 for bf16, 2^-11 for fp16). */

/* Bytes of one layer's packed NVFP4 experts (189 MB: codes, then the block
 * multipliers). */
size_t moe_packed_nvfp4_bytes(void);

/* One-time re-layout of one layer's NVFP4 experts ([out, in] orientation, the
 * transposes of moe_pack_weights' matrices).
 *   q_gate, q_up : [128][512][768] uint8, two codes per byte (4-byte aligned)
 *   s_gate, s_up : [128][512][96] uint8 E4M3 block scales: [e][n][b] scales
 *                  inputs 16b .. 16b+15 of output n
 *   g_gate, g_up : [128] fp32 tensor scales
 *   q_down       : [128][1536][256];  s_down : [128][1536][32];  g_down : [128]
 *   packed_nvfp4 : moe_packed_nvfp4_bytes() bytes, 128-byte aligned, output:
 *                  codes in the row order of moe_pack_weights (gate/up
 *                  interleaved in 128-column blocks), then every block's
 *                  16-bit multiplier in the order the kernels read them.
 * A NaN block scale, a non-finite tensor scale, or a multiplier of a non-zero
 * scale that is not a normal bf16 (gate/up: block scale * tensor scale must
 * lie in [2^-252, 4)) or fp16 (down: [2^-28, 4)) number sets the device
 * error word (moe_get_device_status(): MOE_ERR_RANGE); the packed bytes are
 * written regardless, and the layer's results on such weights are
 * unspecified. */
int moe_pack_weights_nvfp4(const uint8_t* q_gate, const uint8_t* s_gate, const float* g_gate,
                           const uint8_t* q_up, const uint8_t* s_up, const float* g_up,
                           const uint8_t* q_down, const uint8_t* s_down, const float* g_down,
                           void* packed_nvfp4, moe_stream_t stream);

/* Expands a packed NVFP4 layer into the packed bf16/fp16 layer that
 * moe_pack_weights writes (packed: moe_packed_weight_bytes() bytes, 128-byte
 * aligned, output).  With power-of-two tensor scales it equals
 * moe_pack_weights of the dequantised weights, byte for byte. */
int moe_dequant_nvfp4(const void* packed_nvfp4, moe_bf16* packed, moe_stream_t stream);

/* Scratch bytes moe_expert_ffn_nvfp4 needs: 0 for T <= 256, else
 * moe_packed_weight_bytes() (the expanded layer). */
size_t moe_expert_ffn_nvfp4_workspace_bytes(int64_t T);

/* Step 3 with NVFP4 experts: moe_expert_ffn_fp8's arguments with packed_nvfp4
 * (from moe_pack_weights_nvfp4).  Up to 256 tokens one persistent launch
 * streams the 4-bit codes and dequantises each weight tile into tensor memory
 * on its way to the tensor cores; above, the layer is expanded into the
 * workspace and the bf16 expert FFN runs on it. */
int moe_expert_ffn_nvfp4(const moe_bf16* x, const void* packed_nvfp4, const int32_t* offsets,
                         const int32_t* perm_src, int64_t T, moe_f16* h, moe_f16* y_perm,
                         void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* Workspace bytes moe_layer_nvfp4 needs for T tokens (as moe_layer_fp8). */
size_t moe_layer_nvfp4_workspace_bytes(int64_t T);

/* moe_layer with NVFP4 experts (packed_nvfp4 from moe_pack_weights_nvfp4),
 * other arguments as in moe_layer; the expert FFN as moe_expert_ffn_nvfp4.
 * Above 256 tokens every call expands the layer first (about half the time of
 * the layer at 8K tokens); a caller with the HBM to spare (604 MB per layer)
 * can expand once with moe_dequant_nvfp4 and call moe_layer on the result,
 * which gives the same output. */
int moe_layer_nvfp4(const moe_bf16* x, const float* logits, const float* bias,
                    const void* packed_nvfp4, int64_t T, const moe_bf16* residual,
                    moe_bf16* out, int32_t* topk_idx_out, float* topk_w_out,
                    void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* ---- shared experts --------------------------------------------------------- */

/* The Ling family's flash model has shared experts ("khronnuz/Ling-3.0-flash-
 * exl3", table of quants: kept at higher precision beside attention) and the
 * Inkling model "256 experts top-6 plus 2 shared" ("Add TML Inkling
 * architecture", llama.cpp PR #25731); the pages give neither their size nor
 * how they enter the sum.  Read as the usual form: each shared expert is a
 * SwiGLU FFN of the routed experts' shape (1536 -> 512 -> 1536) that every
 * token passes through with weight 1:
 *   out[t] = bf16( residual[t] + sum_slot w[t,slot] FFN_{e_slot}(x[t]) + sum_s FFN_s(x[t]) )
 * summed in fp32 in that order (routed slots, then shared experts by index)
 * and rounded once.  Shared experts stay bf16 with bf16 or FP8 routed experts. */

/* Bytes of n_shared packed shared experts (0 <= n_shared <= 8). */
size_t moe_packed_shared_bytes(int n_shared);

/* One-time re-layout of n_shared (1..8) shared experts:
 *   w_gate, w_up : [n_shared][1536][512] bf16;  w_down : [n_shared][512][1536] bf16
 *   packed_shared: moe_packed_shared_bytes(n_shared) bytes, 128-byte aligned, output;
 *                  the layout of moe_pack_weights for n_shared experts (gate/up
 *                  K-major and interleaved, then W_down in fp16). */
int moe_pack_shared(const moe_bf16* w_gate, const moe_bf16* w_up, const moe_bf16* w_down,
                    int n_shared, moe_bf16* packed_shared, moe_stream_t stream);

/* Workspace bytes moe_layer_shared needs (fp8_routed != 0: routed experts in
 * block FP8 or NVFP4, for moe_layer_shared_nvfp4 too). */
size_t moe_layer_shared_workspace_bytes(int64_t T, int n_shared, int fp8_routed);

/* moe_layer (packed_w, bf16 routed experts) or moe_layer_fp8 (packed_fp8):
 * exactly one of the two is non-NULL; plus n_shared (0..8) shared experts
 * from packed_shared.  The shared experts' rows (every token once per shared
 * expert) go through the same grouped expert-FFN kernels as the routed ones:
 * with bf16 routed experts as a second weight pack of the routed experts'
 * launch, with block-FP8 or NVFP4 routed experts in a second launch; the
 * combine adds their outputs.  With n_shared = 0 the result is bit for bit
 * that of moe_layer / moe_layer_fp8. */
int moe_layer_shared(const moe_bf16* x, const float* logits, const float* bias,
                     const moe_bf16* packed_w, const void* packed_fp8,
                     const moe_bf16* packed_shared, int n_shared, int64_t T,
                     const moe_bf16* residual, moe_bf16* out, int32_t* topk_idx_out,
                     float* topk_w_out, void* workspace, size_t workspace_bytes,
                     moe_stream_t stream);

/* moe_layer_shared with NVFP4 routed experts (packed_nvfp4 from
 * moe_pack_weights_nvfp4) and n_shared (0..8) bf16 shared experts; workspace
 * as moe_layer_shared_workspace_bytes(T, n_shared, 1).  With n_shared = 0 the
 * result is bit for bit that of moe_layer_nvfp4. */
int moe_layer_shared_nvfp4(const moe_bf16* x, const float* logits, const float* bias,
                           const void* packed_nvfp4, const moe_bf16* packed_shared, int n_shared,
                           int64_t T, const moe_bf16* residual, moe_bf16* out,
                           int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                           size_t workspace_bytes, moe_stream_t stream);

/* ---- a slice of a layer's experts (expert parallelism) --------------------- */

/* With expert parallelism every rank holds only its own experts.  The pages put
 * 128 experts in 8 groups of 16 and keep 4 groups per token ("Ling-3.0-tiny on
 * a Qualcomm board", TensorFold issue #1247, first comment, opening
 * paragraph), so with one or more whole groups per rank a token's rows go to
 * at most 4 ranks.  These calls pack and run a contiguous slice of n_experts
 * experts, renumbered 0 .. n_experts-1 (the rank's local ids).
 *
 * Bytes of a packed slice of n_experts experts (0 outside [1, 128]). */
size_t moe_packed_experts_bytes(int n_experts);

/* moe_pack_weights for a slice: w_gate, w_up [n][1536][512], w_down
 * [n][512][1536] bf16 -> packed (moe_packed_experts_bytes(n) bytes, 128-byte
 * aligned): the slice's gate/up blocks, then its W_down blocks in fp16, each
 * in moe_pack_weights' per-expert layout. */
int moe_pack_experts(const moe_bf16* w_gate, const moe_bf16* w_up, const moe_bf16* w_down,
                     int n_experts, moe_bf16* packed, moe_stream_t stream);

/* moe_expert_ffn on a packed slice: offsets and perm_src from moe_permute of
 * local ids (every id < n_experts, or -1 for an empty slot), T the rows of x. */
int moe_expert_ffn_slice(const moe_bf16* x, const moe_bf16* packed, int n_experts,
                         const int32_t* offsets, const int32_t* perm_src, int64_t T,
                         moe_f16* h, moe_f16* y_perm, moe_stream_t stream);

/* ---- second MoE shape: 256 experts, top-6 ------------------------------------- */

/* The Inkling model has "256 experts top-6 plus 2 shared" ("Add TML Inkling
 * architecture", llama.cpp PR #25731, model description); its group structure,
 * hidden and intermediate sizes are not given.  Read with tiny's rule scaled
 * to 256 experts: 8 groups of 32, 4 kept, 6 chosen, the same score, tie and
 * weight rules as moe_route; expert FFNs of tiny's shape (1536 -> 512 -> 1536). */
enum { MOE_E256_EXPERTS = 256, MOE_E256_TOPK = 6 };

/* Routing on the second shape: logits [T][256] fp32, bias [256] fp32 or NULL;
 * topk_idx [T][6] int32 and topk_w [T][6] fp32 (out), slot order = descending
 * score.  One warp per token. */
int moe_route_e256(const float* logits, const float* bias, int64_t T, int32_t* topk_idx,
                   float* topk_w, moe_stream_t stream);

/* Workspace bytes moe_layer_e256 needs. */
size_t moe_layer_e256_workspace_bytes(int64_t T, int n_shared);

/* The whole layer on the second shape: routing, a stable counting sort over
 * the 256 experts, the grouped expert FFN of experts 0..127 (packed_lo) and
 * 128..255 (packed_hi) -- each packed by moe_pack_weights from that half's
 * [128][...] weights -- and of the n_shared (0..8) shared experts of
 * packed_shared (moe_pack_shared), all three packs in one launch of the
 * 128-expert kernels, and the combine (up to 64 tokens the routing and the
 * sort are one launch):
 *   out[t] = bf16( residual[t] + sum_{slot < 6} w[t,slot] FFN_{e_slot}(x[t]) + sum_s FFN_s(x[t]) ).
 * topk_idx_out / topk_w_out: optional [T][6]. */
int moe_layer_e256(const moe_bf16* x, const float* logits, const float* bias,
                   const moe_bf16* packed_lo, const moe_bf16* packed_hi,
                   const moe_bf16* packed_shared, int n_shared, int64_t T,
                   const moe_bf16* residual, moe_bf16* out, int32_t* topk_idx_out,
                   float* topk_w_out, void* workspace, size_t workspace_bytes,
                   moe_stream_t stream);

/* ---- permutation without a caller workspace ------------------------------ */

/* The pages describe no such call: it is moe_permute for callers that cannot
 * allocate device memory at the moment they permute (a runtime whose device
 * memory is all reserved up front, code running inside an allocator, loops
 * that must not wait on an allocator).  The per-block histogram that
 * moe_permute takes from `workspace` lives instead in a fixed array of 256 KiB
 * per device owned by the library, so the call allocates nothing.
 *   Limit  : 0 <= T <= moe_permute_fixed_scratch_max_tokens() (65536);
 *            larger T returns MOE_ERR_INVALID_ARG with nothing launched.
 *   Outputs: identical, bit for bit, to moe_permute's for the same topk_idx.
 *   Set-up : the first call on a device (with that device current) looks up
 *            the array's device address, unless moe_init_device() has done so;
 *            make that first call, or moe_init_device(), before any stream
 *            capture.
 *   Races  : one array per device serves every call, so two calls whose
 *            kernels may overlap (different streams with no ordering between
 *            them, or several host threads) corrupt each other's result.
 *            Order them on one stream or with events. */
int64_t moe_permute_fixed_scratch_max_tokens(void);
int moe_permute_fixed_scratch(const int32_t* topk_idx, int64_t T, int32_t* counts,
                              int32_t* offsets, int32_t* perm_src, int32_t* inv_perm,
                              moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_MOE_H */
