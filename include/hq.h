/*
 * hq.h -- C ABI of the B200 (sm_100a) quantised-weight GEMM library.
 *
 * The operations follow the Humming kernel library as described in
 * "Announcing Humming: Fast, Flexible Kernels for Quantized Inference":
 *   - section "Unified quantization representation": weight format, scale
 *     granularity, scale dtype, zero point and second-level scale are
 *     independent parameters; the activation has its own format
 *     (hq_quant_desc below);
 *   - section "Tuning & JIT per workload": parameters are validated, dims
 *     padded and tensors repacked into the kernel's layout (hq_pack_weights);
 *   - section "Performance", WnA16 and W8A8/W4A8/W4A4: dense and MoE GEMMs,
 *     MoE on "Indexed" and "Grouped" paths (hq_gemm, hq_moe_gemm);
 * and the SGLang integration digest (PR #23754, humming_moe_runner_core_run,
 * moe_permute_prepare, moe_permute / moe_unpermute, moe_fused_mul_sum) for
 * the MoE call semantics (hq_moe_permute, hq_moe_gemm,
 * hq_moe_unpermute_sum).
 *
 * Conventions for every call:
 *   - All pointers are DEVICE pointers unless stated otherwise, 16-byte
 *     aligned.  The caller allocates and owns every buffer and stream.  The
 *     library allocates no device memory.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronises.
 *   - Every call returns an hq_status and never aborts.  Argument errors are
 *     detected on the host before any launch.  Errors that can only be seen
 *     on the device (an expert id out of range, a pipeline wait that timed
 *     out) are recorded in a per-device error word read by hq_device_error().
 *   - Row-major layouts; `[a, b]` means a rows of b contiguous elements.
 *   - Tensors the library consumes are in the "standard format":
 *       INT4/UINT4 codes  int32 [E, N, K/8]: nibble j (bits 4j..4j+3) of word
 *                         w is the code of k = 8w + j; INT4 two's complement.
 *       INT4 zero points  int32 [E, N, ceil(G/8)] packed the same way along
 *                         the group axis (G = K / w_group, or 1 per channel).
 *       INT4 scales       bf16  [E, N, G].
 *       E2M1 codes        uint8 [E, N, K/2], low nibble = even k.
 *       E8M0 scales       uint8 [E, N, K/32] (MXFP4, MXINT4).
 *       UE4M3 scales      uint8 [E, N, K/16] (NVFP4) + fp32 global [E].
 *       E4M3 codes        uint8 [E, N, K] + fp32 per-channel scales [E, N]
 *                         (block-scaled: fp32 [E, ceil(N / 128), K / 128]).
 *       INT1/UINT1/INT2/UINT2/INT3/UINT3/E2M3/E3M2/E0M3 codes (b bits): uint8
 *                         [E, N, K * b / 8], a little-endian bit stream per
 *                         row (code k at bits b*k .. b*k + b - 1; for b = 4
 *                         the INT4 / E2M1 nibble order).  UINT1/2/3 zero
 *                         points: uint8 [E, N, G], one per byte.  E0M3 code:
 *                         bit 3 = sign, bits 0..2 = magnitude.
 *   - Decoded values: INT4 w = (q - z) * s (z = 0 when symmetric; MXINT4
 *     s = 2^(c - 127));
 *     MXFP4 w = e2m1 * 2^(c - 127); NVFP4 w = e2m1 * ue4m3 * g;
 *     FP8 w = e4m3 with the channel scale applied to the output.
 *   - Accumulation is fp32; outputs are bf16 (round to nearest even).
 */
#ifndef HQ_H
#define HQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define HQ_API __attribute__((visibility("default")))
#else
#define HQ_API
#endif

typedef struct CUstream_st *hq_stream_t; /* identical to cudaStream_t */

typedef enum {
  HQ_OK = 0,
  HQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer    */
  HQ_ERR_UNSUPPORTED = 2,  /* valid description, combination not built     */
  HQ_ERR_WORKSPACE = 3,    /* workspace smaller than *_workspace_bytes()   */
  HQ_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed         */
  HQ_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up           */
  HQ_ERR_DEVICE_INDEX = 6, /* an expert id outside [0, E) seen on device   */
  HQ_ERR_ARCH = 7          /* the current device is not sm_100             */
} hq_status;

/* Element formats used in hq_quant_desc. */
typedef enum {
  HQ_BF16 = 0,
  HQ_FP32 = 1,
  HQ_INT4 = 2,   /* signed 4-bit, two's complement                         */
  HQ_UINT4 = 3,  /* unsigned 4-bit (asymmetric with zero points)           */
  HQ_E2M1 = 4,   /* FP4 (OCP MX)                                           */
  HQ_E4M3 = 5,   /* FP8 (OCP "fn"); as an activation: per-token fp32 scale */
  HQ_E8M0 = 6,   /* power-of-two scale (OCP MX)                            */
  HQ_UE4M3 = 7,  /* unsigned E4M3 block scale (NVFP4)                      */
  HQ_MXFP8 = 8,  /* activation: E4M3 codes + E8M0 scale per 32 along K     */
  HQ_NVFP4 = 9,  /* activation: E2M1 codes + UE4M3 per 16 + fp32 global    */
  HQ_INT2 = 10,  /* signed 2-bit, two's complement                         */
  HQ_UINT2 = 11, /* unsigned 2-bit (with zero points)                      */
  HQ_INT3 = 12,  /* signed 3-bit, two's complement                         */
  HQ_UINT3 = 13, /* unsigned 3-bit (with zero points)                      */
  HQ_E2M3 = 14,  /* FP6 (OCP MX), with E8M0 scales: MXFP6                  */
  HQ_E3M2 = 15,  /* FP6 (OCP MX), with E8M0 scales: MXFP6                  */
  HQ_E0M3 = 16,  /* float4e0m3: sign + 3-bit magnitude, no exponent bits   */
  HQ_INT1 = 17,  /* signed 1-bit, two's complement (codes 0, -1)           */
  HQ_UINT1 = 18  /* unsigned 1-bit (with zero points)                      */
} hq_dtype;

/*
 * Unified quantisation description ("Announcing Humming", section "Unified
 * quantization representation").  Supported weight descriptions:
 *   INT4  + BF16 scales, w_group in {0 (per channel), 32, 64, 128}
 *   INT4  + E8M0 scales, w_group = 32                       (MXINT4)
 *   UINT4 + BF16 scales + zero points, w_group in {32, 64, 128}
 *   E2M1  + E8M0 scales, w_group = 32                       (MXFP4)
 *   E2M1  + UE4M3 scales, w_group = 16, w_has_global = 1    (NVFP4)
 *   E4M3  + FP32 per-channel scales, w_group = 0            (FP8)
 *   E4M3  + FP32 scales per 128 x 128 block, w_group = 128  (block-scaled
 *         FP8, only with a_dtype E4M3 and a_group 128, K a multiple of 128)
 *   INT1, INT2, INT3, E0M3 + BF16 scales, w_group in {0, 32, 64, 128}
 *   UINT1, UINT2, UINT3 + BF16 scales + zero points, w_group in {32, 64, 128}
 *   E2M3, E3M2 + E8M0 scales, w_group = 32                  (MXFP6)
 * and every one of them with a_dtype in {BF16, E4M3, MXFP8, NVFP4}.  E0M3
 * ("Announcing Humming", section "Quantization support": a float with no
 * exponent bits, whose values are the symmetric integers -7..7) is the
 * zero-exponent view of symmetric INT4 and computes as INT4.
 * a_group is the activation's scale granularity along K: 0 = the format's
 * own (E4M3: one fp32 scale per token; MXFP8: 32; NVFP4: 16); MXFP8 also
 * accepts 32 and NVFP4 16; E4M3 with a_group 128 has one fp32 scale per
 * token and 128 k (the activations of block-scaled FP8, which take no
 * other weight format).  Zero-initialise the struct.
 */
typedef struct {
  int32_t w_dtype;       /* HQ_INT4 | HQ_UINT4 | HQ_E2M1 | HQ_E4M3           */
  int32_t w_group;       /* 0 = per output channel, else group size along K */
  int32_t w_scale_dtype; /* HQ_BF16 | HQ_E8M0 | HQ_UE4M3 | HQ_FP32           */
  int32_t w_has_zero;    /* 1: UINT4 zero points, same grouping as scales   */
  int32_t w_has_global;  /* 1: FP32 second-level scale per expert (NVFP4)   */
  int32_t a_dtype;       /* HQ_BF16 | HQ_E4M3 | HQ_MXFP8 | HQ_NVFP4          */
  int32_t a_group;       /* activation scale group along K (0: the format's) */
} hq_quant_desc;

typedef enum { HQ_MOE_GROUPED = 0, HQ_MOE_INDEXED = 1 } hq_moe_mode;

/*
 * Compute options ("Announcing Humming", section "Tuning & JIT per
 * workload": the compute configuration holds the GEMM type and options such
 * as batch invariance).  Zero-initialise; unknown fields must stay zero.
 *   batch_invariant: 1 = every output row is bit-identical whatever the
 *       number of rows M of the call (and whatever the other rows hold): one
 *       fixed token tile (64 rows) and no split of K, each tile summed in k
 *       order by one CTA.  Slower at small M, where splitting K is what keeps
 *       every SM busy.  (With NVFP4 activations the caller's codes, scales and
 *       global scale are taken as given; a dynamic global scale computed over
 *       a batch is itself batch-dependent.)
 */
typedef struct {
  int32_t batch_invariant;
  int32_t reserved[7];
} hq_compute_config;

/* Text for a status code (static storage). */
HQ_API const char *hq_status_string(hq_status s);

/* Reads and clears the current device's device-side error word after
 * synchronising `stream`.  Returns HQ_OK, HQ_ERR_TIMEOUT or
 * HQ_ERR_DEVICE_INDEX. */
HQ_API hq_status hq_device_error(hq_stream_t stream);

/* Diagnostics (no counterpart in the pages): launches one warp that waits
 * on an mbarrier nothing arrives on, with the same bounded wait every GEMM
 * pipeline uses, limited to `limit_ns` (0 < limit_ns <= 1e9).  The wait
 * gives up, records HQ_ERR_TIMEOUT in the device error word (read it with
 * hq_device_error) and the kernel returns; the context stays usable.  This
 * is how the device-side failure path is tested without faulting a GPU. */
HQ_API hq_status hq_selftest_wait_timeout(unsigned long long limit_ns, hq_stream_t stream);

/* ------------------------------------------------------------------------
 * Weight repack ("Announcing Humming", section "Tuning & JIT per workload":
 * validate, pad, repack into the kernel layout).
 *
 * hq_packed_weights_bytes: size of the opaque packed buffer for E experts of
 *   N x K weights (0 if the description or sizes are unsupported).  N is
 *   padded to 128 rows and K must be a multiple of 64.
 * The packed layout depends on the whole description, the activation
 *   format included: MXFP4 weights with a_dtype MXFP8 (K a multiple of 128)
 *   and NVFP4 weights with a_dtype NVFP4 (K a multiple of 256) are stored
 *   for the block-scaled tensor-core MMA (each row's codes cut into stage
 *   chunks stored contiguously per 128-row tile, scales in the MMA's chunk
 *   order), FP8 weights with a_dtype E4M3 (K a multiple of 128) likewise as
 *   E4M3 bytes with per-row fp32 scales for the FP8 MMA; every other pair
 *   for in-kernel dequantisation.  Pack,
 *   unpack, hq_gemm and hq_moe_gemm must be given the same description.
 *   The packed buffer must be 32-byte aligned (cudaMalloc's 256 is).
 * hq_pack_weights: standard-format codes / scales / zeros (device) and, for
 *   NVFP4, `global_scale` (device fp32 [E]) -> `packed` (device,
 *   hq_packed_weights_bytes).  `zeros` must be NULL unless w_has_zero;
 *   `global_scale` NULL unless w_has_global.  Bit-exact and deterministic.
 * hq_unpack_weights: the inverse, back to the standard format (for tests).
 * ---------------------------------------------------------------------- */
HQ_API size_t hq_packed_weights_bytes(const hq_quant_desc *desc, int E, int N, int K);
HQ_API hq_status hq_pack_weights(const hq_quant_desc *desc, int E, int N, int K, const void *codes,
                          const void *scales, const void *zeros, const float *global_scale,
                          void *packed, hq_stream_t stream);
HQ_API hq_status hq_unpack_weights(const hq_quant_desc *desc, int E, int N, int K, const void *packed,
                            void *codes, void *scales, void *zeros, float *global_scale,
                            hq_stream_t stream);

/* ------------------------------------------------------------------------
 * Activation quantisation ("Announcing Humming", section "W8A8 / W4A8 /
 * W4A4" and the MoE activation override in its usage section: tokenwise
 * FP8, MXFP8, NVFP4 activations).  x: bf16 [M, K], K a multiple of 32.
 *   a_dtype == HQ_E4M3: codes uint8 [M, K], scales fp32 [M];
 *       s = amax_row / 448, q = e4m3(x / s) (s = 1 for an all-zero row).
 *       With a_group == 128: scales fp32 [M, K / 128], the same recipe on
 *       each 128-k group of a row (K a multiple of 128).
 *   a_dtype == HQ_MXFP8: codes uint8 [M, K], scales uint8 E8M0 [M, K/32];
 *       e = floor(log2(amax_blk)) - 8 clamped to [-127, 127], code e + 127,
 *       q = e4m3(x * 2^-e) (code 127 and q = 0 for an all-zero block).
 *   a_dtype == HQ_NVFP4: codes uint8 [M, K/2] (low nibble = even k),
 *       scales uint8 UE4M3 [M, K/16], global fp32 [1];
 *       g = amax_tensor / 2688 (or *static_global if non-NULL; 1 for an
 *       all-zero tensor), sb = ue4m3((amax_blk / 6) / g),
 *       d = sb * g, q = e2m1(x / d) (q = 0 when d = 0).
 * All conversions round to nearest even and saturate; fp32 IEEE steps in
 * the order written.  `global_out` receives g (NVFP4 only).
 * `workspace` (NVFP4 dynamic only): >= 16 bytes, may be NULL otherwise.
 * ---------------------------------------------------------------------- */
HQ_API hq_status hq_quant_act(const hq_quant_desc *desc, int M, int K, const void *x_bf16, void *codes,
                       void *scales, float *global_out, const float *static_global,
                       void *workspace, size_t ws_bytes, hq_stream_t stream);

/* ------------------------------------------------------------------------
 * Dense GEMM: C[M, N] (bf16) = A[M, K] . W[N, K]^T with W the packed
 * weights of one expert (E = 1) and A in desc->a_dtype:
 *   BF16:  a = bf16 [M, K], a_scales = NULL
 *   E4M3:  a = uint8 [M, K], a_scales = fp32 [M] (per token), or with
 *          a_group 128 fp32 [M, K / 128] (block-scaled FP8 weights: each
 *          128-k stage is multiplied in the tensor core and added in fp32
 *          with both scales)
 *   MXFP8: a = uint8 [M, K], a_scales = uint8 [M, K/32]
 *   NVFP4: a = uint8 [M, K/2], a_scales = uint8 [M, K/16], a_global = fp32 [1]
 * M >= 0 (M == 0 is a no-op), N >= 1, K a multiple of 64.
 * `workspace` of hq_gemm_workspace_bytes() bytes; its split-K counters must
 * be zero when first used (for example cudaMemset once after allocation);
 * every completed call leaves them zero again.
 * Block-scaled pairs (MXFP4 x MXFP8, NVFP4 x NVFP4) and FP8 x E4M3 with K a
 * multiple of 128 (see hq_pack_weights) multiply the quantised activations
 * as they are (a_scales 4-byte aligned); other quantised activations are
 * decoded exactly to bf16 in the workspace and multiplied with the
 * dequantised weights (FP8 x E4M3 otherwise: E4M3 weights and activations on
 * the FP8 MMA with the weights staged through tensor memory).
 * ---------------------------------------------------------------------- */
HQ_API size_t hq_gemm_workspace_bytes(const hq_quant_desc *desc, int M, int N, int K);
HQ_API hq_status hq_gemm(const hq_quant_desc *desc, int M, int N, int K, const void *packed_w,
                  const void *a, const void *a_scales, const float *a_global, void *c_bf16,
                  void *workspace, size_t ws_bytes, hq_stream_t stream);

/* Which kernel and tiling a call would use (host only; no device work).
 * Filled for hq_gemm / hq_gemm_config (hq_gemm_plan) and for hq_moe_gemm
 * (hq_moe_plan) with the same arguments; the CTA count follows the current
 * device's SM count (148 when no device is present). */
typedef struct {
  int32_t kernel;       /* 0: multi-stage (dequantised weights in TMEM), 1: decode (<= 32 tokens
                           per tile), 2: TMA-fed (block-scaled pairs, FP8 x FP8)               */
  int32_t layout;       /* 0: dequantisation, 1: MXFP4 x MXFP8, 2: NVFP4 x NVFP4, 3: FP8 x FP8  */
  int32_t token_tile;   /* tokens per tile (the MMA's N)                                       */
  int32_t weight_tiles; /* 128-row weight tiles                                                */
  int32_t token_tiles;  /* token tiles (MoE: an upper bound over experts)                      */
  int32_t ctas;         /* persistent CTAs launched                                            */
  int32_t reserved[2];
} hq_plan_info;
HQ_API hq_status hq_gemm_plan(const hq_quant_desc *desc, const hq_compute_config *cfg, int M, int N, int K,
                       hq_plan_info *out);
HQ_API hq_status hq_moe_plan(const hq_quant_desc *desc, int T, int topk, int E, int N, int K, int a_per_slot,
                      hq_plan_info *out);

/* hq_gemm with compute options (cfg may be NULL: the defaults, identical to
 * hq_gemm).  Same arguments and contract as hq_gemm; size the workspace with
 * hq_gemm_config_workspace_bytes for the same cfg. */
HQ_API size_t hq_gemm_config_workspace_bytes(const hq_quant_desc *desc, const hq_compute_config *cfg, int M,
                                      int N, int K);
HQ_API hq_status hq_gemm_config(const hq_quant_desc *desc, const hq_compute_config *cfg, int M, int N, int K,
                         const void *packed_w, const void *a, const void *a_scales, const float *a_global,
                         void *c_bf16, void *workspace, size_t ws_bytes, hq_stream_t stream);

/* ------------------------------------------------------------------------
 * MoE routing prepare (SGLang digest: moe_permute_prepare /
 * moe_align_block_size).  topk_ids int32 [T, topk], values in [0, E).
 * Slot s = t * topk + j.  Outputs (int32):
 *   expert_offsets [E + 1]: exclusive prefix of per-expert slot counts;
 *   perm [T * topk]: slot at each expert-sorted position (stable: slots of
 *       one expert in increasing s);
 *   inv_perm [T * topk]: position of each slot.
 * An id outside [0, E) sets HQ_ERR_DEVICE_INDEX in the device error word
 * and expert_offsets[E] = -1; hq_moe_gemm then writes nothing.
 * ---------------------------------------------------------------------- */
HQ_API hq_status hq_moe_permute(int T, int topk, int E, const int32_t *topk_ids, int32_t *expert_offsets,
                         int32_t *perm, int32_t *inv_perm, hq_stream_t stream);

/* ------------------------------------------------------------------------
 * MoE expert GEMM ("Announcing Humming", section "Performance": Indexed and
 * Grouped MoE paths; SGLang digest: humming_moe_runner_core_run with gemm
 * types "indexed" and "grouped_contiguous").  Slot s = t * topk + j of token
 * t multiplies expert e(s) = topk_ids[t, j]:  Y[s] = a_row(s) . W_e(s)^T.
 *   packed_w: hq_pack_weights output for E experts of N x K.
 *   a: activations in slot-independent token order, a_per_slot == 0: [T, K]
 *       (every slot of token t multiplies row t, the gate-up case), or
 *       a_per_slot == 1: [T * topk, K] (slot s multiplies row s, the down
 *       case).  Either bf16 (a_scales == NULL; quantised on the fly with
 *       hq_quant_act's recipe when desc->a_dtype is not BF16), or, with
 *       a_scales != NULL, codes already quantised by the caller in
 *       hq_quant_act's layout for desc->a_dtype (a_scales 4-byte aligned;
 *       NVFP4 also a_global, device fp32 [1]).
 *   Routing: expert_offsets [E + 1] and perm [T * topk] from hq_moe_permute;
 *       or both NULL and topk_ids (device int32 [T, topk]): the call then
 *       runs the routing prepare itself into the workspace.
 *   mode HQ_MOE_GROUPED: the routed rows are first copied expert-contiguous
 *       into the workspace (quantised codes as they are), and the grouped
 *       GEMM reads each token tile as one block of rows.
 *   mode HQ_MOE_INDEXED: no copy; the GEMM reads each token tile's rows
 *       straight from `a` (or from its quantised or decoded copy, which has
 *       the caller's T or T * topk rows, not the routed T * topk) through
 *       the routing index, four rows per TMA (tensor memory accelerator)
 *       gather instruction.
 *   combine == 0: out = Y bf16 [T * topk, N] in slot order.
 *   combine == 1: out bf16 [T, N],
 *       out[t] = routed_scale * sum_j topk_weights[t, j] * Y[t * topk + j]
 *       (fp32 sum over j in increasing j; Y rounded to bf16 first); N a
 *       multiple of 8.
 * Both modes give bit-identical results (the same rows in the same tiles
 * and k order).  `workspace`: hq_moe_workspace_bytes() bytes (enough for
 * on-the-fly quantisation and internal routing), 16-byte aligned.
 * ---------------------------------------------------------------------- */
HQ_API size_t hq_moe_workspace_bytes(hq_moe_mode mode, const hq_quant_desc *desc, int T, int topk, int E,
                              int N, int K, int a_per_slot, int combine);
HQ_API hq_status hq_moe_gemm(hq_moe_mode mode, const hq_quant_desc *desc, int T, int topk, int E, int N,
                      int K, const void *packed_w, const void *a, const void *a_scales,
                      const float *a_global, int a_per_slot, const int32_t *topk_ids,
                      const float *topk_weights, const int32_t *expert_offsets, const int32_t *perm,
                      int combine, float routed_scale, void *out_bf16, void *workspace, size_t ws_bytes,
                      hq_stream_t stream);

/* ------------------------------------------------------------------------
 * Gate-up GEMM with SiLU-and-mul fused into its epilogue (an addition of this
 * library; the pages name no activation, and the gated-MLP form is the
 * usual one).  For an MoE layer's gate-up weights, N2 = 2I rows per expert
 * (standard format: gate rows 0..I-1, then up rows I..2I-1), I a multiple of
 * 64:
 *   hq_pack_weights_gated / hq_unpack_weights_gated: as hq_pack_weights /
 *       hq_unpack_weights (same arguments, same hq_packed_weights_bytes), but
 *       the gate and the up row of each output column are stored side by
 *       side in the packed tiles.  Only hq_moe_gemm_gated reads this form.
 *   hq_moe_gemm_gated: hq_moe_gemm's gate-up call (one activation row per
 *       token, a_per_slot = 0; modes, activation formats, routing and
 *       workspace rules as there, hq_moe_gated_workspace_bytes) whose
 *       epilogue writes out bf16 [T * topk, I] in slot order:
 *       out[s, i] = bf16_rne(silu(g) * u), g = Y[s, i], u = Y[s, I + i] in
 *       fp32 (Y unrounded), silu(g) = g / (1 + exp(-g)).  The up-and-gate
 *       bf16 tensor [T * topk, 2I] of the unfused path never reaches HBM.
 * ---------------------------------------------------------------------- */
HQ_API hq_status hq_pack_weights_gated(const hq_quant_desc *desc, int E, int N2, int K, const void *codes,
                                       const void *scales, const void *zeros, const float *global_scale,
                                       void *packed, hq_stream_t stream);
HQ_API hq_status hq_unpack_weights_gated(const hq_quant_desc *desc, int E, int N2, int K, const void *packed,
                                         void *codes, void *scales, void *zeros, float *global_scale,
                                         hq_stream_t stream);
HQ_API size_t hq_moe_gated_workspace_bytes(hq_moe_mode mode, const hq_quant_desc *desc, int T, int topk, int E,
                                           int I, int K);
HQ_API hq_status hq_moe_gemm_gated(hq_moe_mode mode, const hq_quant_desc *desc, int T, int topk, int E, int I,
                                   int K, const void *packed_w, const void *a, const void *a_scales,
                                   const float *a_global, const int32_t *topk_ids, const int32_t *expert_offsets,
                                   const int32_t *perm, void *out_bf16, void *workspace, size_t ws_bytes,
                                   hq_stream_t stream);

/* ------------------------------------------------------------------------
 * Masked MoE expert GEMM (SGLang digest: humming_moe_runner_core_run with
 * gemm type "grouped_masked", arguments expert_num_tokens and expected_m).
 * The activations arrive already grouped per expert in fixed-size slabs:
 *   a_bf16: bf16 [E * slab, K]; expert e owns rows [e * slab, (e + 1) * slab),
 *       of which the first c_e = clamp(expert_num_tokens[e], 0, slab) are
 *       valid (the rest may hold anything, NaN included, and are ignored).
 *   expert_num_tokens: device int32 [E].
 *   expected_m: the typical c_e (a tiling hint; < 1 means slab).
 *   out_bf16: bf16 [E * slab, N]; row e * slab + i = a_row . W_e^T for
 *       i < c_e; the other rows are left as they were.
 * If desc->a_dtype is not BF16 the valid rows are quantised on the fly with
 * hq_quant_act's recipe (NVFP4: the tensor scale of the valid rows alone).
 * The result of a valid row equals hq_moe_gemm's for the same row and expert.
 * E in [1, 1024], E * slab <= 2^30, K a multiple of 64; `workspace` of
 * hq_moe_masked_workspace_bytes() bytes, 16-byte aligned.
 * ---------------------------------------------------------------------- */
HQ_API size_t hq_moe_masked_workspace_bytes(const hq_quant_desc *desc, int E, int slab, int N, int K,
                                     int expected_m);
HQ_API hq_status hq_moe_gemm_masked(const hq_quant_desc *desc, int E, int slab, int N, int K,
                             const void *packed_w, const void *a_bf16,
                             const int32_t *expert_num_tokens, int expected_m, void *out_bf16,
                             void *workspace, size_t ws_bytes, hq_stream_t stream);

/* ------------------------------------------------------------------------
 * SiLU-and-mul between an MoE layer's gate-up and down GEMMs (the gate-up
 * GEMM computes N = 2I columns per row: gate then up).  y bf16 [R, 2I],
 * out bf16 [R, I]: out[r, i] = bf16_rne(silu(g) * u) with g = y[r, i],
 * u = y[r, I + i], silu(g) = g / (1 + exp(-g)), computed in fp32.  I a
 * multiple of 8; both buffers 16-byte aligned.  (The pages name no
 * activation; this is the usual gated-MLP form, an addition of this
 * library.)
 * ---------------------------------------------------------------------- */
HQ_API hq_status hq_silu_and_mul(int R, int I, const void *y_bf16, void *out_bf16, hq_stream_t stream);

/* ------------------------------------------------------------------------
 * Fused weighted top-k sum (SGLang digest: moe_fused_mul_sum, and
 * moe_unpermute): out[t, n] = routed_scale * sum_j w[t, j] * y[r(t, j), n]
 * with r(t, j) = inv_perm[t * topk + j] if inv_perm is non-NULL (y in
 * expert-sorted order) else t * topk + j (y in slot order).  y bf16
 * [T * topk, N]; out bf16 [T, N]; the sum is fp32 in increasing j.
 * ---------------------------------------------------------------------- */
HQ_API hq_status hq_moe_unpermute_sum(int T, int topk, int N, const void *y_bf16,
                               const int32_t *inv_perm, const float *topk_weights,
                               float routed_scale, void *out_bf16, hq_stream_t stream);

/* ------------------------------------------------------------------------
 * Dense GEMM for callers that cannot allocate device memory (no counterpart
 * in the pages; an addition of this library).
 *
 * Some callers cannot call cudaMalloc when they run a GEMM: embedded
 * runtimes or allocator hooks that own all device memory, plugins that are
 * given no allocator, and code paths that must not allocate.  This call
 * computes exactly what hq_gemm computes, with the same arguments except the
 * workspace: its scratch is one fixed array of 64 MiB inside the library's
 * device image, which every GPU that loads the library holds until the
 * process exits.
 *   - Sizes whose workspace (hq_gemm_workspace_bytes) exceeds 64 MiB are
 *     rejected with HQ_ERR_WORKSPACE before anything is launched.
 *   - Arguments are checked as hq_gemm checks them; a rejected call
 *     enqueues nothing.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, a synchronous runtime query) with that device
 *     current and caches it; later calls reuse the cached address.
 *   - The call allocates nothing; it clears the part of the array that must
 *     start at zero (split-K tile counters) with cudaMemsetAsync on `stream`.
 *   - Every call shares the one array and it keeps the last call's contents:
 *     calls that overlap on the GPU (different streams, no ordering) race.
 * ---------------------------------------------------------------------- */
HQ_API hq_status hq_gemm_noalloc(const hq_quant_desc *desc, int M, int N, int K, const void *packed_w,
                                 const void *a, const void *a_scales, const float *a_global, void *c_bf16,
                                 hq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HQ_H */
