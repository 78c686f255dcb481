/*
 * hq.h -- C ABI of the B200 (sm_100a) low-bit-weight GEMM library with
 * fused dequantization.
 *
 * What it computes.  A linear layer y = x * W^T whose weights W are stored
 * in a low-bit format and are dequantized inside the GEMM kernel.  The
 * method (the Humming quantized-inference kernel library) is described on
 * news pages only:
 *   [fr]  the French edition of the Ant/vLLM Humming kernels news
 *         (news.cocoloop.cn), section "one library, many formats": WnA16 /
 *         W8A8 / W4A8 / W4A4; INT1..INT8, FP4..FP8, MXFP4, MXINT4, NVFP4;
 *         comparison-table rows "W4A16 dense, small batch", "W4A8-MXFP4,
 *         H200", "MoE W4A16, B300, large batch".
 *   [fa]  "Humming: open-source kernel library for quantized inference"
 *         (news.ditty.ir), summary paragraph 2 (one standard description in
 *         which weight, scale, zero point and the other parameters are
 *         described separately), paragraph 3 (Layer / Compute / Tuning
 *         configs: shapes+dtype+arch / GEMM type / tile, stages, MMA),
 *         paragraph 4 (MXFP4 weights converted inside the kernel),
 *         paragraph 5 (the "Grouped" MoE path).
 *   [pt]  "Ant Group e vLLM lancam a biblioteca open source Humming"
 *         (aube.news), quantization explainer (dense and MoE layers).
 *   [vi]  the Vietnamese edition of the same news (news.cocoloop.cn),
 *         section "meaning for domestic deployers" (GPTQ INT3 weights
 *         served through the library) and "one library, many formats".
 * Element formats follow the public standards the pages name: OCP MX v1.0
 * (e2m1, E8M0, 32-element blocks), OCP FP8 (E4M3), NVIDIA NVFP4 (e2m1 with
 * an E4M3 scale per 16 elements and an fp32 tensor scale).
 *
 * Conventions shared by every entry point.
 *   - A (activations) is [M, K] row-major, K contiguous.  W is logically
 *     [N, K] (K contiguous).  C is [M, N] row-major bf16.
 *   - The caller owns all memory.  The library never allocates device
 *     memory, never synchronizes a stream (except hq_check_device_status),
 *     and launches only on the caller's stream.
 *   - Arguments are validated on the host before any launch; on failure a
 *     non-OK status is returned and nothing is launched or written.
 *   - Errors found on the device (a bounded wait that ran out, offsets that
 *     are not monotone) are written to the workspace error word and read
 *     back by hq_check_device_status.
 *   - Device pointers must be 16-byte aligned; workspaces 256-byte aligned.
 *   - A workspace must be zero-filled once after allocation.  Every
 *     workspace starts with the same two parts: a 256-byte header (the
 *     error word, which hq_check_device_status clears) and a 256 KiB region
 *     of stream-K tile counters; scratch that needs no initial value
 *     follows.  Counters must start at zero, and every call that completes
 *     leaves the ones it used at zero again, so one workspace may serve any
 *     sequence of calls (of any entry points and plans) ordered on a stream.
 *   - Pointers named *_dev are device pointers; *_host are host pointers.
 *   - The GEMM kernels are launched as programmatic dependents of the
 *     previous kernel on the stream: their CTAs may start, set up and fetch
 *     the first stages of the packed weights while that kernel finishes;
 *     everything else (activations, scales, offsets, outputs, workspace) is
 *     touched only after it has completed.  So the kernel launched just
 *     before a GEMM call must not write that call's packed weights (copies
 *     and memsets are ordinary stream dependencies and are not affected),
 *     unless the call's tuning sets HQ_TUNE_NO_EARLY_WEIGHTS.
 */
#ifndef HQ_H_
#define HQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Packed-layout version written by hq_quant_desc_init and checked by every
 * call taking a descriptor (a descriptor from another layout version is
 * rejected with HQ_ERR_LAYOUT_VERSION). */
#define HQ_LAYOUT_VERSION 1

typedef struct CUstream_st* hq_stream_t; /* the same handle as cudaStream_t */

typedef enum {
  HQ_OK = 0,
  HQ_ERR_INVALID_ARG = 1,
  HQ_ERR_UNSUPPORTED = 2,
  HQ_ERR_ALIGNMENT = 3,
  HQ_ERR_WORKSPACE_TOO_SMALL = 4,
  HQ_ERR_LAYOUT_VERSION = 5,
  HQ_ERR_CUDA = 6,
  HQ_ERR_DEVICE_TIMEOUT = 7,
  HQ_ERR_DEVICE_BAD_OFFSETS = 8,
  HQ_ERR_NO_DEVICE = 9
} hq_status;

typedef enum {
  HQ_FMT_INT4 = 1,  /* unsigned INT4 codes, fp16 scale + optional uint4 zero point per group of 128 K */
  HQ_FMT_MXFP4 = 2, /* e2m1 codes, E8M0 scale per 32 K                                             */
  HQ_FMT_NVFP4 = 3, /* e2m1 codes, E4M3 scale per 16 K, fp32 tensor scale                          */
  HQ_FMT_MXFP4_A16 = 4, /* e2m1 codes, E8M0 scale per 32 K, for bf16 activations: the W4A16 entry
                           points dequantize it in registers like INT4                              */
  HQ_FMT_INT3 = 5,      /* unsigned INT3 codes, fp16 scale + optional uint3 zero point per group of
                           128 K, for bf16 activations (the W4A16 entry points)                     */
  HQ_FMT_INT2 = 6,      /* unsigned INT2 codes, fp16 scale + optional uint2 zero point per group of
                           128 K, for bf16 activations (the W4A16 entry points)                     */
  HQ_FMT_INT8 = 7,      /* unsigned INT8 codes, fp16 scale + optional uint8 zero point per group of
                           128 K, for bf16 activations (the W4A16 entry points)                     */
  HQ_FMT_MXINT4 = 8     /* two's-complement 4-bit integer codes, E8M0 scale per 32 K, for bf16
                           activations (the W4A16 entry points)                                     */
} hq_format;

/* Quantization description ([fa] paragraph 2) plus the Layer Config
 * shape fields ([fa] paragraph 3).  Fill it with hq_quant_desc_init. */
typedef struct {
  int32_t layout_version; /* HQ_LAYOUT_VERSION                                         */
  int32_t fmt;            /* hq_format                                                 */
  int32_t n;              /* output features (weight rows), per expert                 */
  int32_t k;              /* input features (reduction length)                         */
  int32_t group_size;     /* INT4, INT3, INT2: 128; MXFP4, MXFP4_A16: 32; NVFP4: 16    */
  int32_t has_zero_point; /* INT4 / INT3 / INT2: 1 = zero point per group, 0 = symmetric
                             (zero point 8 / 4 / 2)                                    */
  int32_t num_experts;    /* 1 = dense layer; >1 = MoE weights stored expert after expert */
} hq_quant_desc;

/* Execution choices (the Tuning Config of [fa] paragraph 3).  Pass NULL
 * to let the library's heuristic choose; a zero field also means "choose".
 *   tile_m   : token tile (the MMA N extent): 16, 32, 64, 128 or 256
 *   tile_n   : weight rows per tile: 128 (the only value)
 *   tile_k   : K per pipeline stage: 128 (fixed by the packed layout)
 *   stages   : pipeline stages the producer keeps in flight (each a slot
 *              of the kernel's shared-memory ring: one or two 128-K
 *              records, or one or two block-scaled boxes); 0 = the whole
 *              ring; larger than the ring = the whole ring
 *   split_k  : dense GEMMs: CTAs sharing each tile's K range (stream-K
 *              splits the whole iteration space evenly when 0).  A split
 *              plan needs a counter per output tile and epilogue warp in
 *              the workspace's counter region (up to 16384 output tiles
 *              for W4A16, 8192 for the block-scaled GEMMs); one with more
 *              tiles runs as whole tiles.
 *   cta_group: block-scaled GEMMs: 0 = the library's choice (CTA pairs
 *              for 128/256-token whole tiles when N is a multiple of
 *              256 and the pairs fill the SMs), 1 = one CTA per 128-row
 *              weight tile, 2 = CTA pairs: clusters of two CTAs run
 *              256-row weight tiles with cta_group::2 MMAs (each CTA
 *              stages its 128 weight rows and half of the token tile);
 *              needs N % 256 == 0, tile_m 0, 128 or 256, split_k 0.
 *              W4A16 (dense): 0 or 1 = one CTA per tile; 2 = CTA pairs
 *              for 256-token whole tiles (each CTA dequantizes its
 *              128 rows; N % 256 == 0, tile_m 0 or 256, split_k 0;
 *              measured slower than one CTA per tile, kept on request).
 *   variant  : W4A16 / grouped MoE: 0 = the library's choice, currently
 *              2 for token tiles of up to 64 and 1 for larger tiles
 *              (MXFP4_A16 weights: always 1).
 *              1 = weights rescaled to bf16 in the kernel: each weight is
 *              the correctly rounded bf16 of (q - z) * s (one rounding),
 *              fp32 accumulation across K.
 *              2 = for token tiles of up to 64, the exact integers (q - z)
 *              go to the tensor core and each 128-K group's scale is
 *              applied to its fp32 group sum (no rounding of w or s);
 *              larger tiles as 1.  INT4, INT3 and INT2 weights.
 *              3 = the register-path kernels (whole records staged in
 *              shared memory by bulk copies, codes read with ldmatrix into
 *              mma.sync register fragments, exact (q - z) with each group's
 *              scale applied to its fp32 sum, as 2), INT4 weights only:
 *              dense GEMMs of 1 to 16 tokens (split_k = CTAs per weight
 *              tile, 0: the library's split) and grouped MoE GEMMs in 8- or
 *              16-token units (tile_m 16 forces 16).  The library's choice
 *              for dense INT4 at 1 to 16 tokens and for grouped INT4 whose
 *              typical expert rows fit 8 tokens.  Other calls run the
 *              library's choice.
 *              Block-scaled GEMMs: 0.                                     */
typedef struct {
  int32_t tile_m, tile_n, tile_k, stages, split_k, cta_group, variant;
  int32_t flags; /* HQ_TUNE_* bits below, 0 = none                         */
} hq_tuning;

/* hq_tuning.flags: the GEMM kernels do not fetch packed weights before the
 * previous kernel on the stream has completed (see the launch-overlap rule
 * in the header comment above).  For callers whose kernel just before a
 * GEMM call writes that call's packed weights (an in-place repack or a
 * weight update); costs the overlap of the weight prefetch with that
 * kernel's tail. */
#define HQ_TUNE_NO_EARLY_WEIGHTS 1

/* A per-shape tuning table (the offline autotuner writes one): a call that
 * passes no tuning (t == NULL) runs with the tuning of the first entry
 * whose fmt, n, k and num_experts equal its descriptor's and whose
 * [m_min, m_max] holds its m (total sorted rows for MoE), and with the
 * library's rules otherwise.  The pages name heuristics that are not
 * globally optimal and an autotuner on the roadmap ([vi] "stated
 * limitations"; [fa] key points). */
typedef struct {
  int32_t fmt, n, k, num_experts;
  int32_t m_min, m_max;
  hq_tuning tuning;
} hq_tuning_entry;

/* Replaces the process-wide table with a copy of entries[0 .. count)
 * (count 0 clears it).  Every entry's tuning is checked as the matching
 * entry point would check it; on an error the table is left as it was.
 * Safe to call from any thread; calls running concurrently see the old or
 * the new table. */
hq_status hq_tuning_table_set(const hq_tuning_entry* entries, int32_t count);

/* The launch plan a call would run (tuning t, else the table, else the
 * rules), without a GPU if none is current (148 SMs assumed, as for
 * hq_workspace_size). */
typedef struct {
  int32_t kernel;      /* 1: W4A16 weights rescaled to bf16, 2: W4A16 exact weights, 3: block-scaled,
                          4: W4A16 register path (exact weights in mma.sync fragments)              */
  int32_t tile_m;      /* token tile (the register path: 8 or 16, one or two 8-token MMA tiles)       */
  int32_t grid;        /* CTAs                                                                       */
  int32_t split;       /* 0: whole tiles; >0: tiles share their K range (stream-K or a K split)      */
  int32_t whole_tiles; /* dense W4A16 split plans: tiles run whole before the shared tail            */
  int32_t stages;      /* pipeline stages in flight                                                  */
  int32_t ring_stages; /* the kernel's shared-memory ring depth                                      */
  int32_t from_table;  /* 1 when the tuning came from the table                                      */
  int32_t cta_group;   /* 2: block-scaled CTA pairs (cta_group::2 MMAs), else 1                     */
  size_t workspace_bytes;
} hq_plan;
hq_status hq_plan_describe(const hq_quant_desc* d, int32_t m, const hq_tuning* t, hq_plan* out);

/* Library and layout version. */
int hq_layout_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* hq_status_string(hq_status s);

/* Fill *d.  Returns HQ_ERR_INVALID_ARG / HQ_ERR_UNSUPPORTED for shapes or
 * formats the library cannot run:
 *   INT4 : k % 128 == 0, group_size == 128, n >= 1
 *   MXFP4: k % 128 == 0, group_size == 32, has_zero_point == 0
 *   NVFP4: k % 256 == 0, group_size == 16, has_zero_point == 0
 *   MXFP4_A16: k % 128 == 0, group_size == 32, has_zero_point == 0
 *   INT3, INT2: k % 128 == 0, group_size == 128
 *   num_experts 1..1024 for INT4, INT3, INT2 and MXFP4_A16 (MoE), 1 otherwise. */
hq_status hq_quant_desc_init(hq_quant_desc* d, int32_t fmt, int32_t n, int32_t k, int32_t group_size,
                             int32_t has_zero_point, int32_t num_experts);

/* Size in bytes of the packed weight blob for *d (0 if *d is invalid). */
size_t hq_packed_size(const hq_quant_desc* d);

/* Offline weight packer ([fa] paragraph 2: weight, scale and zero point
 * described separately -> one device layout).  Host memory in, host memory
 * out; the caller copies the result to the device.  Canonical inputs,
 * experts back to back:
 *   INT4 : codes_host  = int32 [E][N][K/8], element k in bits 4*(k%8)..+3
 *          scales_host = fp16 bits [E][N][K/128]
 *          zeros_host  = uint8 [E][N][K/128] (0..15), NULL when symmetric
 *   MXFP4: codes_host  = uint8 [N][K/2] (even k in the low nibble)
 *          scales_host = uint8 E8M0 [N][K/32]
 *   NVFP4: codes_host  = uint8 [N][K/2]; scales_host = uint8 E4M3 [N][K/16];
 *          global_scale = the fp32 tensor scale of the weights.
 *   INT3 : codes_host  = int32 [E][N][3K/32]: each row's codes as one
 *          little-endian bit stream, code k in stream bits 3k..3k+2 (stream
 *          bit b = bit b%32 of word b/32), the container of GPTQ INT3
 *          scales_host = fp16 bits [E][N][K/128]
 *          zeros_host  = uint8 [E][N][K/128] (0..7), NULL when symmetric
 *   INT2 : codes_host  = int32 [E][N][K/16], element k in bits 2*(k%16)..+1
 *          scales_host = fp16 bits [E][N][K/128]
 *          zeros_host  = uint8 [E][N][K/128] (0..3), NULL when symmetric
 *   MXFP4_A16: codes_host = uint8 [E][N][K/2] (even k in the low nibble),
 *          scales_host = uint8 E8M0 [E][N][K/32], every byte <= 252 (a
 *          larger scale would overflow bf16 weights, 255 is NaN).
 * The output layout (layout version 1) is spelled out in the header comment
 * of the packer source, hq_pack.cpp.
 * Errors: HQ_ERR_INVALID_ARG (NULL pointers, zeros given for a symmetric
 * descriptor or missing for an asymmetric one, a zero point above the
 * code range (15 / 7 / 3 for INT4 / INT3 / INT2), an MXFP4_A16 scale byte
 * > 252),
 * HQ_ERR_WORKSPACE_TOO_SMALL (out_bytes < hq_packed_size). */
hq_status hq_pack_weights(const hq_quant_desc* d, const void* codes_host, const void* scales_host,
                          const void* zeros_host, float global_scale, void* out_host, size_t out_bytes);

/* Workspace bytes that hq_gemm_w4a16 (a W4A16-family fmt: INT4, INT3, INT2, INT8,
 * MXFP4_A16 or MXINT4; num_experts 1),
 * hq_gemm_mxfp4_a8, hq_gemm_nvfp4 or hq_grouped_gemm_moe need for M rows
 * (total sorted rows for MoE) and the given tuning (NULL = heuristic). */
size_t hq_workspace_size(const hq_quant_desc* d, int32_t m, const hq_tuning* t);

/* Dense W4A16 GEMM ([fr] table row "W4A16 dense"): C = A * W_hat^T with
 * W_hat[n,k] = (q[n,k] - z[n,k/128]) * s[n,k/128] dequantized in-kernel.
 *   d            : INT4, INT3, INT2, INT8, MXFP4_A16 or MXINT4 descriptor,
 *                  num_experts == 1.
 *                  INT3 (GPTQ INT3 weights, [vi] "meaning for domestic
 *                  deployers"): W_hat = (q - z) * s with 3-bit codes and
 *                  the symmetric zero point 4, computed as for INT4.  INT2
 *                  ([fr] format list INT1..INT8) likewise, with 2-bit codes
 *                  and the symmetric zero point 2; INT8 likewise, with
 *                  8-bit codes and the symmetric zero point 128.
 *                  MXFP4_A16 (MXFP4 weights with bf16 activations; [fa]
 *                  paragraph 2 lists MXFP4 weights and bf16 activations):
 *                  W_hat[n,k] = e2m1(c[n,k]) * 2^(e[n,k/32] - 127), each
 *                  weight converted to bf16 exactly (every scale byte <= 252
 *                  keeps it finite) and accumulated in fp32; tuning variant
 *                  2 is refused with HQ_ERR_UNSUPPORTED (one scale per 32 K
 *                  leaves nothing to factor out of a 128-K group).
 *                  MXINT4 (MXINT8's element rule at 4 bits): W_hat[n,k] =
 *                  c[n,k] * 2^(e[n,k/32] - 127) with c a two's-complement
 *                  4-bit integer, as for MXFP4_A16 (variant 2 refused too).
 *   packed_w_dev : blob from hq_pack_weights (hq_packed_size bytes)
 *   a_dev        : bf16 [m][d->k]
 *   m            : rows of A (m == 0 returns HQ_OK without launching)
 *   c_dev        : bf16 [m][d->n], written
 *   ws_dev       : workspace of at least hq_workspace_size bytes */
hq_status hq_gemm_w4a16(const hq_quant_desc* d, const void* packed_w_dev, const void* a_dev, int32_t m,
                        void* c_dev, const hq_tuning* t, void* ws_dev, size_t ws_bytes, hq_stream_t stream);

/* W4A8-MXFP4 GEMM ([fr] table row "W4A8-MXFP4"; [fa] paragraph 4):
 * C[m,n] = s_m * sum_k E4M3(a[m,k]) * e2m1(w[n,k]) * 2^(e[n,k/32]-127).
 *   a_e4m3_dev : uint8 [m][k] E4M3 codes;  a_scale_dev : fp32 [m] */
hq_status hq_gemm_mxfp4_a8(const hq_quant_desc* d, const void* packed_w_dev, const void* a_e4m3_dev,
                           const float* a_scale_dev, int32_t m, void* c_dev, const hq_tuning* t, void* ws_dev,
                           size_t ws_bytes, hq_stream_t stream);

/* NVFP4 W4A4 GEMM ([fr] format list, W4A4 combination):
 * C = (g_a * g_w) * sum_k e2m1(a)*sf_a * e2m1(w)*sf_w.
 *   a_fp4_dev : uint8 [m][k/2] (even k low nibble); a_sf_dev : uint8 E4M3
 *   [m][k/16]; a_global : fp32 tensor scale of A.  g_w is in the blob.
 * Two launches on `stream`: a_sf is first copied into the workspace in the
 * order the tensor core reads block scales (k/256 chunks of 2 KB per
 * 128-token slice of each token tile), then the GEMM runs; the workspace
 * size includes that copy. */
hq_status hq_gemm_nvfp4(const hq_quant_desc* d, const void* packed_w_dev, const void* a_fp4_dev,
                        const void* a_sf_dev, float a_global, int32_t m, void* c_dev, const hq_tuning* t,
                        void* ws_dev, size_t ws_bytes, hq_stream_t stream);

/* Activation quantization for the W4A8 GEMM ([fr] W4A8 combination):
 * per row r, s_r = amax_r / 448 (1 for an all-zero row) and
 * q[r][k] = RNE_E4M3(x[r][k] / s_r), saturating, every step in fp32 (OCP FP8
 * rounding); zero results are written as +0.
 *   x_bf16_dev : bf16 [rows][k], k % 8 == 0;  q_e4m3_dev : uint8 [rows][k];
 *   scale_dev  : fp32 [rows]. */
hq_status hq_quantize_fp8_rows(const void* x_bf16_dev, int32_t rows, int32_t k, void* q_e4m3_dev,
                               float* scale_dev, hq_stream_t stream);

/* Workspace bytes hq_quantize_nvfp4 needs. */
size_t hq_quantize_nvfp4_workspace_size(int32_t rows, int32_t k);

/* Activation quantization for the W4A4 GEMM ([fr] NVFP4 type, W4A4):
 * g = amax / (448*6) over the whole tensor (1 if all zero);
 * per 16 contiguous K: sb = RNE_E4M3(amax_block / (6 g)), d = E4M3(sb) * g,
 * c = RNE_e2m1(x / d) saturating (0 when d == 0); fp32 throughout.
 *   x_bf16_dev : bf16 [rows][k], k % 16 == 0
 *   codes_dev  : uint8 [rows][k/2] (even k in the low nibble)
 *   sf_dev     : uint8 E4M3 [rows][k/16];  global_dev : fp32 [1] (g) */
hq_status hq_quantize_nvfp4(const void* x_bf16_dev, int32_t rows, int32_t k, void* codes_dev, void* sf_dev,
                            float* global_dev, void* ws_dev, size_t ws_bytes, hq_stream_t stream);

/* MoE routing ([fa] paragraph 5, "Grouped" path): top-k experts per
 * token by router logit (equal to top-k by softmax probability), ties to
 * the lower expert index, slots in descending logit order.
 *   logits_dev : fp32 [t][e];  topk_ids_dev : int32 [t][k], written
 *   1 <= k <= 16, k <= e <= 1024. */
hq_status hq_moe_topk(const float* logits_dev, int32_t t, int32_t e, int32_t k, int32_t* topk_ids_dev,
                      hq_stream_t stream);

/* hq_moe_topk plus the combine weights: the softmax probabilities (over
 * all e experts, fp32, not renormalised over the k) of the selected
 * experts, in slot order.
 *   topk_weights_dev : fp32 [t][k], written */
hq_status hq_moe_topk_softmax(const float* logits_dev, int32_t t, int32_t e, int32_t k, int32_t* topk_ids_dev,
                              float* topk_weights_dev, hq_stream_t stream);

/* Workspace bytes hq_moe_permute needs. */
size_t hq_moe_permute_workspace_size(int32_t t, int32_t k, int32_t e);

/* Expert-sorted permutation: expert_offsets = exclusive prefix sum of the
 * per-expert slot counts ([e+1], offsets[e] = t*k); sorted_src lists the
 * flattened slots t*k+j ordered by (expert, slot); when a_dev and
 * a_sorted_dev are both non-NULL, a_sorted[i] = a[sorted_src[i] / k]
 * (bf16 rows of `hidden` elements).  Ids outside [0, e) set
 * HQ_ERR_DEVICE_BAD_OFFSETS in the workspace error word. */
hq_status hq_moe_permute(const int32_t* topk_ids_dev, int32_t t, int32_t k, int32_t e, int32_t* sorted_src_dev,
                         int32_t* expert_offsets_dev, const void* a_dev, int32_t hidden, void* a_sorted_dev,
                         void* ws_dev, size_t ws_bytes, hq_stream_t stream);

/* Grouped MoE W4A16 GEMM, one launch for all experts ([fr] table row
 * "MoE W4A16"): for every expert e, rows [off[e], off[e+1]) of A_sorted
 * times W_hat_e^T.  The tile scheduler reads expert_offsets on the device
 * (no host synchronization).
 *   d              : INT4, INT3, INT2, INT8, MXFP4_A16 or MXINT4 descriptor,
 *                    num_experts = e (per-expert n, k); the other formats'
 *                    weights as for hq_gemm_w4a16
 *   packed_w_dev   : blob of all experts from hq_pack_weights
 *   a_sorted_dev   : bf16 [total_rows][k]
 *   expert_offsets_dev : int32 [e+1], monotone, offsets[e] == total_rows
 *   c_sorted_dev   : bf16 [total_rows][n], written */
hq_status hq_grouped_gemm_moe(const hq_quant_desc* d, const void* packed_w_dev, const void* a_sorted_dev,
                              const int32_t* expert_offsets_dev, int32_t total_rows, void* c_sorted_dev,
                              const hq_tuning* t, void* ws_dev, size_t ws_bytes, hq_stream_t stream);

/* Offline packer for the gate+up weights of a gated feed-forward, for
 * hq_grouped_gemm_moe_swiglu: the same canonical inputs as hq_pack_weights
 * (d->n = 2I rows: gate rows [0, I), up rows [I, 2I), per expert), packed
 * in the gated row order: in every 32-row quarter q of 128-row tile j, rows
 * 0-15 are the gate rows 64j + 16q + l and rows 16-31 the up rows
 * I + 64j + 16q + l (l < 16), so that one tile's accumulators hold matching
 * gate and up values.  Same blob size as hq_pack_weights.
 *   d : INT4, INT3, INT2, INT8, MXFP4_A16 or MXINT4 descriptor with
 *       d->n % 128 == 0.
 * Errors as hq_pack_weights; HQ_ERR_UNSUPPORTED for other formats or n. */
hq_status hq_pack_weights_gated(const hq_quant_desc* d, const void* codes_host, const void* scales_host,
                                const void* zeros_host, void* out_host, size_t out_bytes);

/* Grouped gate+up GEMM with the gated activation fused into its epilogue
 * (the layer around the "Grouped" path; [fa] paragraph 5): for every expert
 * e, rows [off[e], off[e+1]) of A_sorted times the expert's gate and up
 * weights, then h = silu(gate) * up, silu(x) = x / (1 + exp(-x)), from the
 * fp32 accumulators (no bf16 rounding of gate and up), one bf16 rounding.
 *   d              : as for hq_grouped_gemm_moe, d->n = 2I, d->n % 128 == 0
 *   packed_w_dev   : blob from hq_pack_weights_gated
 *   h_sorted_dev   : bf16 [total_rows][d->n / 2], written
 *   other arguments, tuning, workspace and errors as hq_grouped_gemm_moe. */
hq_status hq_grouped_gemm_moe_swiglu(const hq_quant_desc* d, const void* packed_w_dev, const void* a_sorted_dev,
                                     const int32_t* expert_offsets_dev, int32_t total_rows, void* h_sorted_dev,
                                     const hq_tuning* t, void* ws_dev, size_t ws_bytes, hq_stream_t stream);

/* Gated activation between the two grouped GEMMs of an MoE layer (the
 * pages leave the layer around the "Grouped" path open; this is the usual
 * gated feed-forward): h = silu(g) * u, silu(x) = x / (1 + exp(-x)), fp32
 * arithmetic, bf16 round to nearest.
 *   gate_up_dev : bf16 [rows][2*inter]: gate in columns [0, inter), up in
 *                 [inter, 2*inter) (the gate+up GEMM's output)
 *   h_dev       : bf16 [rows][inter], written (may not overlap the input)
 *   inter % 8 == 0; both pointers 16-byte aligned.  Row order is kept, so
 *   it runs on the expert-sorted rows. */
hq_status hq_moe_swiglu(const void* gate_up_dev, int32_t rows, int32_t inter, void* h_dev, hq_stream_t stream);

/* Workspace bytes hq_moe_combine needs (the error word and the inverse
 * of the sorted slot list). */
size_t hq_moe_combine_workspace_size(int32_t t, int32_t k);

/* Weighted combine after the down GEMM: for every token t,
 * out[t] = sum_j w[t][j] * y_sorted[p], where sorted_src[p] = t*k + j,
 * summed in slot order j = 0..k-1 in fp32 (no atomics: the same inputs give
 * the same bits), bf16 round to nearest.
 *   y_sorted_dev     : bf16 [t*k][hidden], expert-sorted (the down GEMM's output)
 *   sorted_src_dev   : int32 [t*k] from hq_moe_permute
 *   topk_weights_dev : fp32 [t][k] (hq_moe_topk_softmax, or the caller's)
 *   out_dev          : bf16 [t][hidden], written
 *   hidden % 8 == 0, k <= 16.  A sorted_src that is not a permutation of
 *   [0, t*k) sets HQ_ERR_DEVICE_BAD_OFFSETS in the workspace error word;
 *   nothing is read or written out of bounds. */
hq_status hq_moe_combine(const void* y_sorted_dev, const int32_t* sorted_src_dev, const float* topk_weights_dev,
                         int32_t t, int32_t k, int32_t hidden, void* out_dev, void* ws_dev, size_t ws_bytes,
                         hq_stream_t stream);

/* Synchronizes `stream`, reads the workspace error word, clears it and
 * returns it (HQ_OK when no device-side error was recorded). */
hq_status hq_check_device_status(void* ws_dev, hq_stream_t stream);

/* Test hook for the bounded-wait machinery: launches one block that waits
 * on a barrier nobody arrives on, with a limit of `limit_ns`; the wait runs
 * out and the kernel writes HQ_ERR_DEVICE_TIMEOUT to the workspace error
 * word and returns normally.  limit_ns must be <= 100 ms. */
hq_status hq_debug_timeout_probe(void* ws_dev, uint64_t limit_ns, hq_stream_t stream);

/* Dense W4A16 GEMM that allocates nothing (no counterpart in the method's
 * pages; an addition of this library).  For callers that cannot allocate
 * device memory where they run the layer -- an engine that plans all memory
 * up front and forbids allocation on its serving path, or code running inside
 * another owner's memory pool -- the scratch hq_gemm_w4a16 takes as a
 * workspace (split-K tile counters and fp32 partial sums) lives here in one
 * fixed 16 MiB array inside the library, present on every device that loads
 * it until the process exits.
 *   Same arguments and result as hq_gemm_w4a16 (INT4, INT3, INT2, INT8,
 *   MXFP4_A16 or MXINT4 weights), without ws_dev / ws_bytes.
 *   A launch plan needing more than 16 MiB of scratch is refused with
 *   HQ_ERR_WORKSPACE_TOO_SMALL before anything runs (a smaller tile_m in
 *   `t` needs less); a plan of whole tiles with a split-K tail whose partial
 *   sums would not fit runs as whole tiles instead.  The array is laid out
 *   as a workspace: its tile counters start at zero and every call that
 *   completes leaves them at zero; after a call that recorded a device-side
 *   error, hq_static_check_device_status (which reports it) zeroes them and
 *   the error word again, so check the status after an error before the
 *   next call.  All calls share the array: calls that may overlap on the GPU (unordered
 *   streams) race; calls ordered on one stream are safe.  The first call in
 *   each CUDA context looks up the array's device address
 *   (cudaGetSymbolAddress), so make it before any stream capture.
 *   A device-side error of any call (a bounded wait that ran out, after
 *   which the output may be partly written) is kept in the array until
 *   hq_static_check_device_status reads it. */
hq_status hq_gemm_w4a16_static(const hq_quant_desc* d, const void* packed_w_dev, const void* a_dev, int32_t m,
                               void* c_dev, const hq_tuning* t, hq_stream_t stream);

/* Synchronizes `stream`, then reads and returns the first device-side error
 * recorded by hq_gemm_w4a16_static calls on the current device since the
 * last such read (HQ_OK when none).  When there was one it zeroes the
 * array's error word and tile counters (and synchronizes the device).
 * Allocates nothing. */
hq_status hq_static_check_device_status(hq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HQ_H_ */
