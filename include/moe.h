/*
 * moe.h -- C ABI of the B200 (sm_100a) routed Mixture-of-Experts FFN.
 *
 * One layer, on one GPU:
 *
 *   route    top-k expert selection from router logits, the bias used for the
 *            selection only (flashinfer.fused_moe.MoEActivationPack,
 *            routing_input_mode FromLogits)
 *   permute  stable counting sort of the routed slots into expert-contiguous
 *            rows (Struct_mega_ffn_ep_combine_send, Args: expert_start_indices,
 *            expert_ids, a_scale_offsets, src_info, num_active_experts)
 *   ffn      grouped gate_up GEMM with the clamped-SwiGLU + re-quant epilogue,
 *            then the grouped down GEMM whose epilogue scatter-reduces every
 *            row, weighted by its router weight, into the token-ordered output
 *            (Struct_mega_ffn_ep_combine_send: gate_up_weight, down_weight,
 *            gate_up_expert_scales, down_expert_scales, c_input_scales;
 *            flashinfer.megamoe.MegaMoESymmBuffer: activation_clamp)
 *   combine  the router-weighted reduction back to token order, finalised to
 *            BF16 (DistributedEPCombine, Args: router_weights)
 *   fused    all of the above on one stream, from one call
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument named as a device buffer is a CUDA device address
 *    on the current device.  The caller owns all memory, including the
 *    workspace; the library allocates nothing per call and keeps no per-call
 *    state on the host.
 *  - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *    stream.  Every call except moe_read_status only enqueues work.
 *  - Host-side validation runs before any launch.  A failed check returns an
 *    error and launches nothing.  Unsupported combinations return
 *    MOE_ERR_UNSUPPORTED; nothing falls back silently (EPConfig,
 *    fuse_ffn_combine_send: incompatible options raise rather than degrade).
 *  - Errors found on the device (an expert id >= num_experts or < -1, a
 *    bounded wait that ran out) are recorded in a sticky status word at the
 *    start of the workspace; the affected outputs are unspecified.  Read it
 *    with moe_read_status.  No kernel traps or asserts.
 *  - topk_idx == -1 marks a skipped slot (the -1 = masked convention of
 *    expert_ids): it is not counted and contributes nothing.
 *  - num_tokens == 0 is a no-op that returns MOE_OK.
 *
 * Layouts (row-major; K-major weights as the pages give them)
 * ----------------------------------------------------------
 *  M = num_tokens, H = hidden, I = intermediate_hidden, E = num_experts,
 *  k = num_topk, R = M*k routed slots.
 *
 *  format BF16      x  bf16 [M, H]
 *                   w13 bf16 [E, 2I, H]   rows [0, I) gate (W1), [I, 2I) up (W3)
 *                   w2  bf16 [E, H, I]
 *  format FP8       x  e4m3 [M, H], x_scale fp32 [M, H/128] (token-major)
 *                   w13 e4m3 [E, 2I, H], w13_scale fp32 [E, 2I/128, H/128]
 *                   w2  e4m3 [E, H, I],  w2_scale  fp32 [E, H/128, I/128]
 *  format NVFP4     x  packed e2m1 uint8 [M, H/2] (element 2i in the low
 *                   nibble), x_scale e4m3 [M, H/16]
 *                   w13 uint8 [E, 2I, H/2], w13_scale e4m3 [E, 2I, H/16]
 *                   w2  uint8 [E, H, I/2],  w2_scale  e4m3 [E, H, I/16]
 *                   gate_up_expert_scales fp32 [E]  L1 output multiplier
 *                   down_expert_scales    fp32 [E]  L2 output multiplier
 *                   c_input_scales        fp32 [E]  re-quant dequant multiplier G
 *  format MXFP8     x  e4m3 [M, H], x_scale ue8m0 uint8 [M, H/32] (code c
 *                   is 2^(c-127); flashinfer.fused_moe.MoEActivationPack,
 *                   MXFP8 activations; the OCP MX block format)
 *                   w13 e4m3 [E, 2I, H], w13_scale ue8m0 [E, 2I, H/32]
 *                   w2  e4m3 [E, H, I],  w2_scale  ue8m0 [E, H, I/32]
 *                   the intermediate is re-quantised per 32 columns with
 *                   scale 2^(floor(log2 amax) - 8), clamped to 2^[-127, 127]
 *  format FP8 per-tensor (MoEActivationPack, FP8 per-tensor: E4M3 values
 *                   with a scalar FP32 dequantisation scale)
 *                   x  e4m3 [M, H], x_scale fp32 [1]
 *                   w13 e4m3 [E, 2I, H], w13_scale fp32 [E] (one per matrix)
 *                   w2  e4m3 [E, H, I],  w2_scale  fp32 [E]
 *                   c_input_scales fp32 [E]: the intermediate's static
 *                   re-quant scale G, q = e4m3(h * (1/G)), a dequant
 *                   multiplier of the down GEMM
 *  topk_idx int64 [M, k]; topk_weights fp32 [M, k]; output bf16 [M, H].
 *
 *  Geometry (flashinfer.megamoe.MegaMoESymmBuffer, Parameters): hidden is a
 *  multiple of 256 and intermediate_hidden a multiple of 128; NVFP4 also needs
 *  intermediate_hidden % 256 == 0 (one 128-byte K stage of the down GEMM).
 *  1 <= num_topk <= num_experts <= 1024.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* a null pointer, a bad size, a bad enum value */
  MOE_ERR_UNSUPPORTED = 2,  /* a valid but unserved combination */
  MOE_ERR_WORKSPACE = 3,    /* workspace smaller than moe_get_workspace_size */
  MOE_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, attribute) */
  MOE_ERR_BAD_INDEX = 5,    /* device: topk_idx outside [-1, num_experts) */
  MOE_ERR_TIMEOUT = 6       /* device: a bounded wait gave up */
} moe_status_t;

typedef enum {
  MOE_FMT_BF16 = 0,
  MOE_FMT_FP8_E4M3_B128 = 1,  /* E4M3 with FP32 per-128 block scales */
  MOE_FMT_NVFP4 = 2,          /* e2m1 with E4M3 per-16 block scales + per-expert FP32 */
  MOE_FMT_MXFP8 = 3,          /* E4M3 with UE8M0 (power-of-two) per-32 block scales */
  MOE_FMT_FP8_PER_TENSOR = 4  /* E4M3 with one FP32 scale per tensor / expert matrix */
} moe_format_t;

/* The problem statement, after flashinfer.megamoe.MegaMoESymmBuffer
 * (num_experts, num_topk, hidden, intermediate_hidden, activation_clamp,
 * fast_math), plus the GEMM tile regime and the shared expert.
 *
 * shared_expert = 1 (EPConfig fused_shared_expert; DistributedEPCombine
 * fused_shared_expert): the shared expert's computation is fused with the
 * routed experts'.  It is expert index num_experts, after the routed ones,
 * with their shapes and formats, and every token goes through it with
 * router weight 1 in the same grouped GEMMs.  Then:
 *   - every weight array and per-expert array holds num_experts + 1
 *     experts, the shared one last;
 *   - every per-token slot array (topk_idx, topk_weights, and the rows of
 *     the layout) has num_topk + 1 columns, the last being (num_experts,
 *     1.0): moe_route and moe_fused's in-kernel routing choose num_topk of
 *     the num_experts routed experts and write that column themselves;
 *     callers passing precomputed routing pass it too;
 *   - sizes, layouts and the tile regime are those of the problem with
 *     num_experts + 1 experts and num_topk + 1 slots. */
typedef struct {
  int64_t num_tokens;           /* M >= 0 */
  int32_t hidden;               /* H, multiple of 256 */
  int32_t intermediate_hidden;  /* I, multiple of 128 */
  int32_t num_experts;          /* E */
  int32_t num_topk;             /* k */
  float activation_clamp;       /* c of the clamped SwiGLU; +inf disables the clamp */
  int32_t format;               /* moe_format_t */
  int32_t fast_math;            /* nonzero: the SiLU uses the fast exponential */
  int32_t tile_regime;          /* moe_tile_regime_t: the grouped GEMMs' tile shape */
  int32_t shared_expert;        /* 0, or 1: a fused shared expert (above) */
  int32_t activation;           /* moe_activation_t: the L1 activation */
  float activation_alpha;       /* swigluoai: the gate's sigmoid slope (finite, > 0); else ignored */
} moe_problem_t;

/* The L1 activation, on the gate g and up u of an intermediate column, with
 * c = activation_clamp (the gate clamped from above, the up branch on both
 * sides):
 *   SWIGLU     h = min(g,c) * sigmoid(min(g,c)) * clamp(u,-c,c)
 *              (MegaMoESymmBuffer activation_clamp, the SwiGLU clamp value)
 *   SWIGLUOAI  h = min(g,c) * sigmoid(a * min(g,c)) * (clamp(u,-c,c) + 1),
 *              a = activation_alpha (Struct_mega_ffn_ep_combine_send
 *              clamp_activation: the clamped "swigluoai" activation, whose
 *              constants come from the dispatch code). */
typedef enum {
  MOE_ACT_SWIGLU = 0,
  MOE_ACT_SWIGLUOAI = 1
} moe_activation_t;

/* Tile shape of the grouped GEMMs (the tile-regime choice the pages make
 * between prefill and decode batches).  AUTO picks SMALL_M when the routed
 * rows average at most 64 per expert (num_tokens*num_topk <=
 * 64*num_experts), else LARGE_M.  LARGE_M: 128 routed rows x 256 weight rows
 * per tile.  SMALL_M: the operands swapped, 256 weight rows x 32 routed rows
 * per tile, so the tensor work follows the routed rows that exist; every
 * format (NVFP4 and MXFP8 with the routed rows' block scales as the MMA's
 * N-side scale factors).  Results agree between regimes up to FP32
 * summation order. */
typedef enum {
  MOE_TILE_AUTO = 0,
  MOE_TILE_LARGE_M = 1,
  MOE_TILE_SMALL_M = 2
} moe_tile_regime_t;

/* Activations (device).  x is 16-byte aligned and x_scale 4-byte aligned
 * (MOE_ERR_INVALID_ARG otherwise).  x_scale is NULL for BF16.  x_rowwise_scale is
 * NULL, or for NVFP4 activations quantised per token (EPConfig,
 * nvfp4_dyn_global_scales; moe_quantize_nvfp4_rowwise) the BF16 [M] rowwise
 * scales: row t dequantises as e2m1 * block scale * x_rowwise_scale[t], and
 * gate_up_expert_scales then carry the weights' global scales alone. */
typedef struct {
  const void* x;
  const void* x_scale;
  const void* x_rowwise_scale;
} moe_act_t;

/* Expert weights (device).  moe_prepare_weights takes them in the logical
 * layouts listed above.  Every other call takes w13 and w2 as the PREPARED
 * blobs that moe_prepare_weights wrote (Struct_mega_ffn_ep_combine_send:
 * "pre-permuted gate/up weights", "pre-permuted W13 scale tile"); for NVFP4
 * and MXFP8 the block scales are inside those blobs and w13_scale / w2_scale
 * are ignored; for FP8 w13_scale / w2_scale are the logical FP32 block scales,
 * for FP8 per-tensor the FP32 [E] per-matrix scales.  gate_up_expert_scales
 * and down_expert_scales are used by NVFP4 only, c_input_scales by NVFP4 and
 * FP8 per-tensor; they may be NULL otherwise. */
typedef struct {
  const void* w13;
  const void* w13_scale;
  const void* w2;
  const void* w2_scale;
  const float* gate_up_expert_scales;
  const float* down_expert_scales;
  const float* c_input_scales;
} moe_weights_t;

/* The expert-contiguous layout that moe_permute writes (device int32 arrays,
 * caller-owned):
 *   expert_counts [E]          valid slots per expert
 *   expert_start_indices [E+1] exclusive prefix sum of the counts; the last
 *                              entry is the number of valid slots R'
 *   src_info [R]               row r holds the flat slot s = t*k + j (rows
 *                              >= R' are unspecified)
 *   slot_to_row [R]            inverse of src_info; -1 for a skipped slot
 *   expert_ids [E]             active experts ascending, then -1
 *   num_active [1]             number of active experts
 *   a_scale_offsets [E+1]      first padded scale row of each expert: the
 *                              prefix sum of the counts rounded up to 128
 *   tile_offsets [E+1]         prefix sum over the active experts of their
 *                              128-row tile counts (the GEMM scheduler table)
 * Within an expert the rows ascend in flat slot index (a stable sort). */
typedef struct {
  int32_t* expert_counts;
  int32_t* expert_start_indices;
  int32_t* src_info;
  int32_t* slot_to_row;
  int32_t* expert_ids;
  int32_t* num_active;
  int32_t* a_scale_offsets;
  int32_t* tile_offsets;
} moe_layout_t;

/* moe_ffn output modes. */
#define MOE_OUT_ACCUMULATE 0  /* out: fp32 [M, H], zeroed by the call, then += w * y per slot */
#define MOE_OUT_STAGED 1      /* out: fp32 [R, H], row r = y of row r (no router weight) */

/* moe_combine input modes. */
#define MOE_IN_ACCUMULATED 0  /* in: fp32 [M, H] from MOE_OUT_ACCUMULATE; round to BF16 */
#define MOE_IN_STAGED 1       /* in: fp32 [R, H] from MOE_OUT_STAGED; weighted gather */

/* Sets the kernels' shared-memory attributes on `device` (the current device
 * is not changed).  Call once per device before capturing any call into a
 * CUDA graph (flashinfer.megamoe.MegaMoESymmBuffer, prewarm: build every
 * module the fused op can select before capture).  Idempotent. */
moe_status_t moe_init(int device);

/* Bytes of device workspace that every call with this problem needs
 * (256-byte aligned base required).  Valid for any num_tokens up to
 * problem->num_tokens. */
moe_status_t moe_get_workspace_size(const moe_problem_t* problem, size_t* bytes);

/* Zeroes the workspace header (the sticky status word).  Call once after
 * allocating a workspace and after moe_read_status reported an error. */
moe_status_t moe_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* Test hooks of the failure detection, stored in the workspace header
 * (EPConfig, fuse_ffn_combine_send: incompatible options raise rather than
 * degrade silently -- here, a CTA that never arrives must surface as an
 * error, not as a hang).  wait_limit_us > 0 makes every bounded wait of
 * later calls on this workspace give up after that many microseconds
 * instead of 2 s (0 restores the default).  skip_arrival = 1 makes CTA 0 of
 * the next moe_fused call withhold its arrival at its first grid barrier,
 * once: the other CTAs' waits run out, the call returns, the status word
 * reads MOE_ERR_TIMEOUT and the outputs are unspecified.  Nothing faults or
 * hangs.  moe_workspace_init clears both hooks and the status.  Enqueued on
 * `stream`. */
moe_status_t moe_workspace_test_hooks(void* workspace, size_t workspace_bytes, int32_t wait_limit_us,
                                      int32_t skip_arrival, void* stream);

/* The tile regime (moe_tile_regime_t, MOE_TILE_LARGE_M or MOE_TILE_SMALL_M)
 * the grouped GEMMs of this problem use once MOE_TILE_AUTO is resolved
 * (tile regimes of the pages' prefill and decode batches; host only). */
moe_status_t moe_get_tile_regime(const moe_problem_t* problem, int32_t* regime);

/* Bytes of the prepared gate_up and down weight blobs. */
moe_status_t moe_get_prepared_weights_size(const moe_problem_t* problem, size_t* w13_bytes,
                                           size_t* w2_bytes);

/* One-time re-layout of the expert weights for the GEMM kernels (per weight
 * set; "pre-permuted" weights of Struct_mega_ffn_ep_combine_send).  Reads
 * `logical` (w13 / w2 and, for NVFP4 and MXFP8, w13_scale / w2_scale in the logical
 * layouts above) and writes out_w13 / out_w2 (device, sizes from
 * moe_get_prepared_weights_size, 16-byte aligned).  The blobs hold, for
 * every (expert, n tile, 128-byte K slice), the 256 weight rows the tile
 * multiplies (gate_up tiles: 64 gate rows, the 64 matching up rows, then
 * the next 64 of each) in the 128-byte-swizzled order the tensor cores read,
 * followed for NVFP4 / MXFP8 by the slice's scales in 512-byte tiles, so each
 * pipeline stage streams one contiguous block. */
moe_status_t moe_prepare_weights(const moe_problem_t* problem, const moe_weights_t* logical,
                                 void* out_w13, void* out_w2, void* stream);

/* Routing from logits (flashinfer.fused_moe.MoEActivationPack, FromLogits).
 * logits fp32 [M, E]; bias fp32 [E] or NULL (used for the selection only).
 * Per token: score_e = logit_e + bias_e (one FP32 add); the k highest scores
 * in descending order, ties to the lower expert index, NaN scores last;
 * topk_weights = softmax over the chosen k of the UNBIASED logits.
 * Writes topk_idx int64 [M, k] and topk_weights fp32 [M, k].  The indices
 * are defined for any logits (NaN ranks last, +-inf compare as themselves);
 * the weights of a token are unspecified when one of its chosen logits is
 * not finite (+inf, -inf or NaN), since the softmax has no value there. */
moe_status_t moe_route(const moe_problem_t* problem, const float* logits, const float* bias,
                       int64_t* topk_idx, float* topk_weights, void* stream);

/* Per-token dynamic NVFP4 quantisation of BF16 activations (EPConfig,
 * nvfp4_dyn_global_scales: each token is quantised against its own global
 * scale 2688 / rowmax -- 448 * 6, the largest block scale times the largest
 * e2m1 code -- and the scale's BF16 inverse travels with the token).  Per
 * token t of x_bf16 [M, H]: rowmax = max |x[t]|, G = rowmax / 2688 (FP32);
 * per 16 values: scale = e4m3(amax / (6 G)), code = e2m1(x / (scale * G))
 * (0 where the scale is 0); rowwise_scale[t] = bf16(G).  All steps FP32,
 * round to nearest even, saturating; an all-zero token gives zeros.
 * Writes codes uint8 [M, H/2] (element 2i in the low nibble), block_scales
 * E4M3 [M, H/16] and rowwise_scales BF16 [M] -- the moe_act_t of an NVFP4
 * problem with x_rowwise_scale set.  Uses problem->num_tokens and ->hidden. */
moe_status_t moe_quantize_nvfp4_rowwise(const moe_problem_t* problem, const void* x_bf16, void* codes,
                                        void* block_scales, void* rowwise_scales, void* stream);

/* Expert-contiguous layout of the routed slots (see moe_layout_t).
 * topk_idx int64 [M, k], values in [-1, E).  Out-of-range ids set
 * MOE_ERR_BAD_INDEX in the workspace status word and are skipped. */
moe_status_t moe_permute(const moe_problem_t* problem, const int64_t* topk_idx,
                         const moe_layout_t* layout, void* workspace, size_t workspace_bytes,
                         void* stream);

/* The expert FFN over a layout from moe_permute: gathers the activation rows
 * into expert order, runs the grouped gate_up GEMM with the clamped-SwiGLU
 * and re-quant epilogue, then the grouped down GEMM whose epilogue either
 * scatter-reduces w * y into `out` (MOE_OUT_ACCUMULATE) or stores y per row
 * (MOE_OUT_STAGED).  topk_weights fp32 [M, k] (read in accumulate mode).
 * If `intermediate` is not NULL the re-quantised intermediate is ALSO kept
 * there for inspection: codes [R, I] (BF16: 2 bytes, FP8, FP8 per-tensor and
 * MXFP8: 1, NVFP4: 1/2 byte per element) at byte 0, followed at the byte
 * offset `scale_offset` of moe_get_intermediate_size by its scales (FP8:
 * fp32 [I/128][P]; NVFP4: 512-byte tiles [P/128][I/64]; MXFP8: 512-byte
 * tiles [P/128][I/128]; FP8 per-tensor: none, its scale is c_input_scales;
 * P = padded rows, a_scale_offsets[E]).
 * Size it with moe_get_intermediate_size. */
moe_status_t moe_ffn(const moe_problem_t* problem, const moe_act_t* act,
                     const moe_weights_t* weights, const moe_layout_t* layout,
                     const float* topk_weights, int32_t out_mode, void* out,
                     void* intermediate, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes needed for moe_ffn's optional `intermediate` buffer, and the byte
 * offset of its scales. */
moe_status_t moe_get_intermediate_size(const moe_problem_t* problem, size_t* bytes,
                                       size_t* scale_offset);

/* Combine back to token order, BF16 out [M, H] (DistributedEPCombine).
 * MOE_IN_ACCUMULATED: out = bf16_rn(in[t]).  MOE_IN_STAGED: out[t] =
 * bf16_rn(sum_{j<k, slot valid} w[t,j] * in[slot_to_row[t*k+j]]), summed in
 * FP32 in ascending j (deterministic).  `layout` and `topk_weights` are read
 * in staged mode only. */
moe_status_t moe_combine(const moe_problem_t* problem, const moe_layout_t* layout,
                         const float* topk_weights, const void* in, int32_t in_mode,
                         void* out_bf16, void* stream);

/* The whole layer from one call: route (when `logits` is given, else the
 * caller's topk_idx / topk_weights are used), permute, the FFN with the
 * scatter-reduce epilogue, and the BF16 finalise, enqueued on `stream`
 * without any host synchronisation.  Exactly one of (topk_idx and
 * topk_weights) or logits must be non-NULL.  The routing chosen in-kernel
 * is written into the workspace and is not returned. */
moe_status_t moe_fused(const moe_problem_t* problem, const moe_act_t* act,
                       const moe_weights_t* weights, const int64_t* topk_idx,
                       const float* topk_weights, const float* logits, const float* bias,
                       void* out_bf16, void* workspace, size_t workspace_bytes, void* stream);

/* moe_permute without a workspace and without allocating, for callers that
 * cannot call cudaMalloc: a host runtime that links this library but has no
 * device allocator of its own to hand out scratch, or a serving loop that
 * reserves all device memory once at start-up and must not allocate per
 * request (cudaMalloc can synchronise the device and can fail under memory
 * pressure).  It computes the same layout as moe_permute.  The caller still
 * passes topk_idx and the layout arrays, plus device_status: one device
 * int32 that the call sets to MOE_OK before its kernels run and that they
 * set to the first device error (MOE_ERR_BAD_INDEX for an index outside
 * [-1, num_experts)).  The pages have no counterpart of this entry point.
 *
 * Its scratch is a file-scope device array of 32768 int32 (128 KB), which
 * every GPU that loads the library holds until the process exits.  Problems
 * with more than 16384 slots or more than 256 experts keep their per-chunk
 * expert counts there, which limits them to
 * ceil(num_tokens*num_topk/1024) * num_experts <= 32768; larger problems
 * return MOE_ERR_UNSUPPORTED and launch nothing.  Smaller problems run in
 * one block and need no scratch.  The counts are rewritten in full by every
 * call, so nothing has to start at zero; the array keeps the last call's
 * contents.  The first call on each device looks up the array's device
 * address with that device current (again after a cudaDeviceReset, which
 * gives the device a new context); make that first call before any stream
 * capture.  All calls share the one array: calls that overlap on the GPU
 * (on other streams, or from other host threads) race on it.  No memory is
 * allocated or freed, by this library or any other. */
moe_status_t moe_permute_noalloc(const moe_problem_t* problem, const int64_t* topk_idx,
                                 const moe_layout_t* layout, int32_t* device_status, void* stream);

/* Where moe_fused leaves its working data inside the workspace, for
 * inspection and testing: byte offsets from the workspace base for a call
 * with this problem (the offsets depend on num_tokens, so pass the call's
 * problem).  After a moe_fused call has completed, the regions hold
 *   status               int32 sticky status word
 *   topk_idx             int64 [M, k]   routing chosen in-kernel (only when
 *   topk_weights         fp32  [M, k]   the call routed from logits)
 *   expert_counts .. tile_offsets       the layout of moe_layout_t, int32
 *   intermediate         the re-quantised intermediate [R, I] in expert
 *                        order, and at intermediate_scales its scales, in
 *                        the layout moe_ffn gives its `intermediate` buffer;
 *                        scale_rows is P, the padded scale rows
 *   accumulator          fp32 [M, H], the router-weighted sum before the
 *                        BF16 rounding
 * (Struct_mega_ffn_ep_combine_send lists these operands: expert_start_indices,
 * expert_ids, a_scale_offsets, src_info.)  Host only; nothing is launched. */
typedef struct {
  size_t status;
  size_t topk_idx;
  size_t topk_weights;
  size_t expert_counts;
  size_t expert_start_indices;
  size_t src_info;
  size_t slot_to_row;
  size_t expert_ids;
  size_t num_active;
  size_t a_scale_offsets;
  size_t tile_offsets;
  size_t intermediate;
  size_t intermediate_scales;
  int64_t scale_rows;
  size_t accumulator;
} moe_workspace_offsets_t;
moe_status_t moe_get_workspace_offsets(const moe_problem_t* problem, moe_workspace_offsets_t* offsets);

/* Per-kernel timing, for measurement.  moe_timing_enable(1, max_calls)
 * creates CUDA events for up to max_calls calls (once, on the current
 * device); from then on every moe_fused / moe_ffn / moe_permute / moe_route /
 * moe_combine call records an event pair around each kernel it launches, on
 * the call's stream (the calls then must not be captured into a CUDA graph).
 * moe_timing_read waits for the recorded events and returns, per kernel slot,
 * the summed milliseconds and the number of launches timed, then starts a
 * new window.  moe_timing_enable(0, 0) stops recording (events are kept).
 * Slots: MOE_SLOT_* below. */
#define MOE_SLOT_ROUTE 0
#define MOE_SLOT_PERMUTE 1
#define MOE_SLOT_GATHER 2
#define MOE_SLOT_GEMM1 3
#define MOE_SLOT_ZERO 4
#define MOE_SLOT_GEMM2 5
#define MOE_SLOT_FINALIZE 6
#define MOE_SLOT_COMBINE 7
#define MOE_SLOT_FUSED 8   /* the single moe_fused launch */
#define MOE_NUM_SLOTS 9
moe_status_t moe_timing_enable(int enable, int max_calls);
moe_status_t moe_timing_read(float* ms /* [MOE_NUM_SLOTS] */, int* launches /* [MOE_NUM_SLOTS] */);

/* Synchronises `stream` and returns the sticky device status recorded in the
 * workspace (MOE_OK if no device error was seen). */
moe_status_t moe_read_status(const void* workspace, void* stream);

/* A static, human-readable name for a status code. */
const char* moe_status_string(moe_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
