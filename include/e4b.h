/*
 * e4b.h -- C ABI of the 4-bit routed-MoE layer forward for NVIDIA B200 (sm_100a).
 *
 * The library computes the forward of one routed Mixture-of-Experts layer
 * whose fused expert stacks [E, ...] stay packed in 4-bit, as NF4 or MXFP4,
 * plus the two standalone format kernels (MXFP4 -> bf16 decode and the NF4
 * quantiser).  Sources for what each call computes, by page and section:
 *
 *   [MX]  "How do I train and serve MoE models released in MXFP4 (gpt-oss,
 *         DeepSeek-V4)?" -- "Why it happens" (MXFP4: two E2M1 nibbles per
 *         byte, 32-value blocks sharing one E8M0 power-of-two scale) and
 *         "Two fidelity paths" (bit-exact MXFP4 decode; Experts4bit.from_float
 *         quantises a float stack to NF4).
 *   [IX]  "MoE Training & Inference Guides" (solutions index) --
 *         grouped-nf4-gemm table: the routed MoE expert GEMM on NF4 packed
 *         weights (gemm_4bit_grouped) and on E2M1/E8M0 bytes
 *         (gemm_mxfp4_grouped), one launch over all experts, fp32
 *         accumulation, no bf16 expert tensor; experts4bit-qlora table:
 *         ExpertsLoRA, a per-expert low-rank delta before each routed
 *         expert's activation.
 *   [PKG] "experts4bit-qlora" package page -- limits list: one fp32 absmax
 *         per 64 NF4 weights; the stock expert epilogue act(gate)*up with no
 *         biases or clamps; "Current measured position": routing is decided
 *         on the router logits.
 *   [MX] "Why it happens" also names what gpt-oss adds to that epilogue:
 *         per-expert biases, interleaved gate/up rows and a clamped GLU;
 *         "Which project solves it": its module de-interleaves the rows.
 *
 * Conventions for every entry point:
 *   - Device pointers are plain CUDA device addresses; the caller owns every
 *     buffer.  The library never allocates memory; scratch lives in a
 *     caller-provided workspace whose size the *_workspace_bytes queries give.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  Calls return before the GPU finishes.
 *   - Argument errors are detected on the host before anything is launched
 *     and return E4B_ERR_INVALID_ARG or E4B_ERR_UNSUPPORTED; nothing is
 *     enqueued then.  A failed launch returns E4B_ERR_CUDA.  Kernels never
 *     trap: a bounded wait that runs out records E4B_ERR_TIMEOUT in the
 *     workspace status word, which e4b_device_status() reports.
 *   - There is no fallback path: a call either runs these kernels or fails.
 *
 * Storage layouts (readings of the pages where they are silent):
 *   - Expert stacks are stored K-contiguous: gate_up as [E, 2I, H] (logical
 *     [E, H, 2I] transposed), down as [E, H, I]; the fused 2I rows are
 *     [gate rows 0..I-1 | up rows I..2I-1] (a stack released with gate/up
 *     rows interleaved is brought to this order once, by
 *     e4b_deinterleave_rows).  Quantisation blocks are runs of the flat
 *     stored stack, hence along K.
 *   - MXFP4: element 2j is the LOW nibble of byte j; scale byte b covers
 *     elements [32b, 32b+32); value = e2m1(code) * 2^(scale - 127), 0xFF = NaN.
 *   - NF4: element 2j is the HIGH nibble of byte j; absmax[b] (fp32) covers
 *     elements [64b, 64b+64); value = level[code] * absmax.
 */
#ifndef E4B_H
#define E4B_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define E4B_ABI_VERSION 3

typedef enum {
  E4B_OK = 0,
  E4B_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, workspace too small */
  E4B_ERR_UNSUPPORTED = 2,   /* shape outside what the kernels implement */
  E4B_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
  E4B_ERR_TIMEOUT = 4        /* a bounded device-side wait ran out (reported by e4b_device_status) */
} e4b_status;

/* e4b_moe_desc.format.  E4B_NF4_DQ is NF4 whose absmax is stored double-quantised
 * (e4b_nf4_dq below); the forward expands it to fp32 and runs as E4B_NF4. */
enum { E4B_NF4 = 0, E4B_MXFP4 = 1, E4B_NF4_DQ = 2 };

/*
 * Double-quantised NF4 absmax: [PKG] limits list -- bitsandbytes' nested form
 * of an NF4 stack's fp32 absmax (an offset, 8-bit codes and one fp32 per 256
 * values, about a quarter of the bytes), expanded back to fp32 just in time.
 * The pages give neither the 8-bit code table nor the expansion's rounding;
 * the table is part of the stored form here and the expansion is, for
 * absmax b,  fl32(fl32(table[codes[b]] * absmax2[b / 256]) + *offset)
 * (two roundings, no fused multiply-add).  All four are device pointers.
 */
typedef struct {
  const uint8_t* codes;    /* [n_absmax] 8-bit codes */
  const float* absmax2;    /* [ceil(n_absmax / 256)] fp32 second-level scales, 4-byte aligned */
  const float* offset;     /* [1] fp32, 4-byte aligned */
  const float* table;      /* [256] fp32 code table, 4-byte aligned */
} e4b_nf4_dq;
/* e4b_moe_desc.act.  E4B_ACT_SWIGLU: h = silu(gate) * up, silu(z) = z / (1 + e^-z).
 * E4B_ACT_CLAMPED_GLU (gpt-oss, [MX] "Why it happens"; the pages give no formula or
 * constants, so this is the library's reading, with the constants as parameters):
 *   g = min(gate, glu_limit), u = clamp(up, -glu_limit, glu_limit),
 *   h = g * sigmoid(glu_alpha * g) * (u + glu_beta).
 * The public gpt-oss release uses glu_alpha = 1.702, glu_limit = 7, glu_beta = 1. */
enum { E4B_ACT_SWIGLU = 0, E4B_ACT_CLAMPED_GLU = 1 };

/* Router gate weights (e4b_moe_desc.gating, e4b_route's gating argument).
 * E4B_GATE_SOFTMAX_TOPK: softmax over the k selected logits (they sum to 1).
 * E4B_GATE_SOFTMAX_ALL : softmax over all E logits, read at the k selected
 *                        experts without renormalising (they sum to <= 1).
 * The pages do not state the gating function; the first is the library's
 * reading for the named families, the second the other common choice. */
enum { E4B_GATE_SOFTMAX_TOPK = 0, E4B_GATE_SOFTMAX_ALL = 1 };

/* Same type as cudaStream_t. */
typedef struct CUstream_st* e4b_stream;

/* One MoE layer.  [IX] (grouped GEMMs, ExpertsLoRA), [PKG] (stock epilogue). */
typedef struct {
  int32_t E;               /* experts, 1..256 */
  int32_t H;               /* hidden size, multiple of 64 */
  int32_t I;               /* expert intermediate size, multiple of 64 */
  int32_t k;               /* experts per token, 1..min(E, 32) */
  int32_t format;          /* E4B_NF4 or E4B_MXFP4 */
  int32_t lora_rank;       /* 0 = no LoRA; else 1..16 */
  float lora_scale;        /* alpha / r, multiplies the LoRA delta */
  int32_t act;             /* E4B_ACT_SWIGLU or E4B_ACT_CLAMPED_GLU */
  int32_t tokens_per_tile; /* 0 = chosen by the library (the decode kernel when the mean number of rows
                              per routed expert is at most 12, else a tcgen05 tile); 8 = decode kernel
                              (codes decoded in registers, warp-level MMA; tokens go in chunks of 8, 16
                              or 32 by the mean rows per expert; needs the scale rows of 128 weight rows
                              of both stacks to fit in shared memory, else E4B_ERR_UNSUPPORTED);
                              32, 64, 128, 192 or 256 = tcgen05 tile width */
  float glu_alpha;         /* E4B_ACT_CLAMPED_GLU only: finite */
  float glu_limit;         /* E4B_ACT_CLAMPED_GLU only: > 0, +inf allowed (no clamp) */
  float glu_beta;          /* E4B_ACT_CLAMPED_GLU only: finite */
  int32_t gating;          /* E4B_GATE_SOFTMAX_TOPK or E4B_GATE_SOFTMAX_ALL */
} e4b_moe_desc;

/* ABI version of the loaded library (E4B_ABI_VERSION it was built with). */
int32_t e4b_abi_version(void);

/* Static, human-readable name of a status code. */
const char* e4b_status_string(int32_t status);

/* The library's 16 NF4 levels (ascending, fp32), as its kernels use them.
 * Host-only; out must hold 16 floats.  [PKG]/[IX]: NormalFloat levels. */
void e4b_nf4_codebook(float* out);

/*
 * Standalone MXFP4 -> bf16 decode.  [MX] "Two fidelity paths": exact decode
 * of the released blocks and scales.
 *   codes  : n/2 bytes, 16-byte aligned       (device, read)
 *   scales : n/32 E8M0 bytes                  (device, read)
 *   n      : element count, multiple of 32, >= 0
 *   out    : n bf16 values, 16-byte aligned   (device, written)
 * Bit-exact: out[i] = bf16(e2m1(code_i) * 2^(scales[i/32] - 127)); the
 * product is exact unless it overflows (+-inf); scale 0xFF gives NaN.
 */
e4b_status e4b_dequant_mxfp4(const uint8_t* codes, const uint8_t* scales, int64_t n,
                             uint16_t* out, e4b_stream stream);

/*
 * Standalone NF4 quantiser (Experts4bit.from_float).  [MX] "Two fidelity
 * paths"; [PKG] one fp32 absmax per 64 weights.
 *   x      : n fp32 values, 16-byte aligned   (device, read)
 *   n      : multiple of 64, >= 0
 *   codes  : n/2 bytes, packed high nibble first (device, written)
 *   absmax : n/64 fp32                        (device, written)
 * Per 64-block: a = max|x| (exact); a == 0 gives code 7 everywhere; else
 * y = x / a (IEEE fp32 division) and code = #{i : y > m_i} with the fp32
 * midpoints m_i = fl32((level_i + level_{i+1}) / 2).  NaN/Inf input is
 * outside the contract.
 */
e4b_status e4b_quantize_nf4(const float* x, int64_t n, uint8_t* codes, float* absmax,
                            e4b_stream stream);

/*
 * Double-quantised absmax -> fp32 (the read path's expansion on its own).
 *   dq  : host struct describing the device arrays (see e4b_nf4_dq)
 *   n   : absmax values, >= 0
 *   out : n fp32 (device, written), 4-byte aligned
 * Bit-exact: out[b] = fl32(fl32(table[codes[b]] * absmax2[b / 256]) + *offset).
 */
e4b_status e4b_expand_absmax_dq(const e4b_nf4_dq* dq, int64_t n, float* out, e4b_stream stream);

/*
 * gpt-oss gate_up de-interleave (load-time layout step).  [MX] "Why it
 * happens" (interleaved gate/up rows), "Which project solves it" (the gpt-oss
 * module de-interleaves them).
 *   in        : [E, 2I] rows of row_bytes bytes each, gate i at row 2i and
 *               up i at row 2i + 1                      (device, read)
 *   out       : [E, 2I] rows, gate rows 0..I-1 then up rows I..2I-1 (device,
 *               written); must not overlap `in`
 *   row_bytes : bytes per row, >= 0 (H/2 for packed codes, the scale bytes of
 *               one row, 4 for one fp32 bias per row)
 * A pure byte permutation: exact.  Any alignment is accepted (16- and 4-byte
 * aligned rows move in wider words).
 */
e4b_status e4b_deinterleave_rows(const void* in, void* out, int32_t E, int32_t I, int64_t row_bytes,
                                 e4b_stream stream);

/* Workspace bytes e4b_route needs for T tokens, E experts, k choices. */
size_t e4b_route_workspace_bytes(int32_t T, int32_t E, int32_t k);

/*
 * Top-k routing and expert permute.  [IX] (routed expert GEMM over all
 * experts in one launch), [PKG] "Current measured position" (routing is
 * defined on given logits).
 *   logits         : [T, E] bf16, row-major       (device, read)
 *   gating         : E4B_GATE_SOFTMAX_TOPK or E4B_GATE_SOFTMAX_ALL
 *   topk_ids       : [T, k] int32                 (device, written) ids by
 *                    (logit desc, id asc); -0 == +0
 *   topk_w         : [T, k] fp32                  (device, written) gate
 *                    weights as `gating` says
 *   expert_offsets : [E+1] int32                  (device, written) exclusive
 *                    prefix sum of per-expert slot counts
 *   sorted_slot    : [T*k] int32                  (device, written) slots
 *                    s = t*k + j grouped by expert, ascending s in each group
 *   ws, ws_bytes   : workspace, 256-byte aligned, >= e4b_route_workspace_bytes
 * Integer outputs are deterministic and bit-exact.  T == 0 is a no-op that
 * still writes expert_offsets (all zero).
 */
e4b_status e4b_route(const uint16_t* logits, int32_t T, int32_t E, int32_t k, int32_t gating,
                     int32_t* topk_ids, float* topk_w, int32_t* expert_offsets,
                     int32_t* sorted_slot, void* ws, size_t ws_bytes, e4b_stream stream);

/*
 * e4b_route without a caller-provided workspace.  The described system has
 * no counterpart: this entry point exists for callers that cannot allocate
 * device memory -- for instance a host runtime that owns all device memory
 * through its own pool and forbids cudaMalloc once running, or a serving loop
 * that must not risk an allocation that synchronises the device.
 *   Arguments and outputs are those of e4b_route, minus ws/ws_bytes.
 *   Scratch lives in one fixed 1 MiB device array inside the library; every
 *   GPU that loads the library holds it until the process exits.  Inputs that
 *   would need more (256 B + ceil(T / 128) x E x 4 B + T*k x 4 B, each part
 *   rounded up to 256 B; e.g. T above 26200 at E = 256, k = 8) return
 *   E4B_ERR_UNSUPPORTED before anything is looked up or launched.
 *   It allocates nothing: no cudaMalloc, cudaFree or allocating routine.
 *   The first call on each device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   The address is kept for the process: do not reset the device
 *   (cudaDeviceReset) between calls.
 *   Every call on a device shares the one array, so calls that overlap on the
 *   GPU (different streams, no ordering between them) race and corrupt each
 *   other's results: order them on one stream or with events.
 */
e4b_status e4b_route_noalloc(const uint16_t* logits, int32_t T, int32_t E, int32_t k, int32_t gating,
                             int32_t* topk_ids, float* topk_w, int32_t* expert_offsets,
                             int32_t* sorted_slot, e4b_stream stream);

/* Workspace bytes e4b_moe_forward needs for this layer at T tokens (0 on a bad desc). */
size_t e4b_moe_workspace_bytes(const e4b_moe_desc* d, int32_t T);

/*
 * Layer forward.  [IX] grouped gate_up GEMM with in-kernel dequant, optional
 * per-expert LoRA delta before the activation, [PKG] SwiGLU epilogue
 * act(gate)*up (or [MX] the gpt-oss biases and clamped GLU, per d->act and
 * the bias pointers), grouped down GEMM, then the weighted combine
 * out[t] = sum_j w[t,j] * y[t,j] in fp32, j ascending, rounded to bf16.
 *   x         : [T, H] bf16                            (device, read)
 *   logits    : [T, E] bf16                            (device, read)
 *   gu_codes  : [E, 2I, H] packed 4-bit (E*2I*H/2 bytes, 16-byte aligned)
 *   gu_scales : NF4 fp32 absmax [E*2I*H/64] or MXFP4 E8M0 bytes [E*2I*H/32]
 *               (device, 16-byte aligned); for E4B_NF4_DQ a HOST pointer to
 *               an e4b_nf4_dq describing the stack's E*2I*H/64 absmax
 *   dn_codes  : [E, H, I] packed 4-bit;  dn_scales as gu_scales for [E, H, I]
 *   lora_A    : [E, H, r] bf16 or NULL;  lora_B : [E, r, 2I] bf16 or NULL
 *               (both or neither, and r == d->lora_rank)
 *   gu_bias   : [E, 2I] fp32 as [gate | up], or NULL (no bias); added to
 *               the gate_up output before the activation
 *   dn_bias   : [E, H] fp32 or NULL; added to each expert's down output, so
 *               the combine weights scale it too
 *   out       : [T, H] bf16                            (device, written)
 *   ws        : workspace, 256-byte aligned, >= e4b_moe_workspace_bytes(d, T);
 *               its first 256 bytes hold the device status word and the decode
 *               kernel's work counters (zeroed by the route stage, left at zero
 *               by every launch that completes)
 * bf16 outputs match the fp64 definition within relative Frobenius error
 * 5e-3 and max-abs error 3e-2 * max|ref|; routing is bit-exact.
 */
e4b_status e4b_moe_forward(const e4b_moe_desc* d, int32_t T, const uint16_t* x,
                           const uint16_t* logits, const uint8_t* gu_codes, const void* gu_scales,
                           const uint8_t* dn_codes, const void* dn_scales,
                           const uint16_t* lora_A, const uint16_t* lora_B,
                           const float* gu_bias, const float* dn_bias, uint16_t* out,
                           void* ws, size_t ws_bytes, e4b_stream stream);

/*
 * QLoRA training: the layer's backward through its frozen 4-bit stacks.
 * [IX] experts4bit-qlora table: ExpertsLoRA wraps each frozen expert stack
 * with a per-expert low-rank adapter, and the fast training path runs the
 * grouped kernels with dgrad, i.e. it also takes the input gradient through
 * the frozen 4-bit weights.  The packed stacks and any biases are frozen; the
 * trainable parameters are the LoRA factors, and the layer's inputs (x and
 * the router logits) receive gradients.  The routing choice is piecewise
 * constant and carries none; only the gate weights of the chosen experts do.
 */

/* Workspace bytes of e4b_moe_forward_train + e4b_moe_backward at T tokens (0 on a bad desc). */
size_t e4b_moe_train_workspace_bytes(const e4b_moe_desc* d, int32_t T);

/*
 * e4b_moe_forward that also keeps, in its workspace, what e4b_moe_backward
 * needs: the routing, the routed rows, the down outputs and the gate_up
 * outputs before the activation (fp32, LoRA delta and bias included).
 * Arguments as e4b_moe_forward; ws must hold e4b_moe_train_workspace_bytes.
 */
e4b_status e4b_moe_forward_train(const e4b_moe_desc* d, int32_t T, const uint16_t* x,
                                 const uint16_t* logits, const uint8_t* gu_codes, const void* gu_scales,
                                 const uint8_t* dn_codes, const void* dn_scales,
                                 const uint16_t* lora_A, const uint16_t* lora_B,
                                 const float* gu_bias, const float* dn_bias, uint16_t* out,
                                 void* ws, size_t ws_bytes, e4b_stream stream);

/*
 * Gradients of sum(dout * out) for the forward last run by
 * e4b_moe_forward_train on this workspace (same desc, T, stacks, LoRA factors
 * and logits; nothing in between may reuse the workspace).  For routed row
 * r = (t, j) of expert e with gate weight w and LoRA scale s = d->lora_scale:
 *   dY_r = w dout_t;  dh = dY_r W_dn[e];  dG = act'(G) applied to dh;
 *   dxa = s dG B_e^T;  dx_t = sum_j (dG W_gu[e] + dxa A_e^T);
 *   dB_e = sum over e's rows of s (x A_e)^T dG;  dA_e = sum of x^T dxa;
 * and dw_j = <dout_t, y_r> reaches the logits through the gating softmax
 * (E4B_GATE_SOFTMAX_TOPK: w_j (dw_j - sum_i w_i dw_i) at the picks, 0
 * elsewhere; E4B_GATE_SOFTMAX_ALL: p_e ([e = id_j] dw_j - sum_i w_i dw_i)).
 * The clamps of E4B_ACT_CLAMPED_GLU pass the gradient inside their range,
 * ends included.
 *   logits  : [T, E] bf16, the forward's                    (device, read)
 *   dout    : [T, H] bf16 upstream gradient, 8-byte aligned (device, read)
 *   gu_codes, gu_scales, dn_codes, dn_scales, lora_A, lora_B: the forward's
 *             (lora_B here 16-byte aligned: its rows are read in 16-byte words)
 *   dx      : [T, H] fp32, 16-byte aligned                  (device, written)
 *   dlogits : [T, E] fp32                                   (device, written)
 *   dA      : [E, H, r] fp32, dB : [E, r, 2I] fp32, with LoRA, else NULL
 *             (device, written; experts no row is routed to get zeros)
 *   ws      : the workspace e4b_moe_forward_train filled
 * Within the forward's tolerance class: bf16 operands (dY, dG and the decoded
 * weights), fp32 accumulation.  Misaligned or missing pointers return
 * E4B_ERR_INVALID_ARG before any launch.
 */
e4b_status e4b_moe_backward(const e4b_moe_desc* d, int32_t T, const uint16_t* logits,
                            const uint16_t* dout, const uint8_t* gu_codes, const void* gu_scales,
                            const uint8_t* dn_codes, const void* dn_scales,
                            const uint16_t* lora_A, const uint16_t* lora_B, float* dx, float* dlogits,
                            float* dA, float* dB, void* ws, size_t ws_bytes, e4b_stream stream);

/* Stages of e4b_moe_forward, in order. */
enum {
  E4B_STAGE_ROUTE = 0,     /* clears the status word; top-k, histogram, stable permute */
  E4B_STAGE_GATHER = 1,    /* routed rows in expert order (+ LoRA left factor x.A_e; E4B_NF4_DQ: the
                              touched experts' absmax expanded to fp32) */
  E4B_STAGE_GATE_UP = 2,   /* grouped gate_up GEMM with dequant, LoRA delta, bias, activation -> h */
  E4B_STAGE_DOWN = 3,      /* grouped down GEMM with dequant (+ bias) -> y */
  E4B_STAGE_COMBINE = 4    /* out[t] = sum_j w[t,j] * y[t,j] */
};

/*
 * Runs one stage of e4b_moe_forward with the same arguments (for timing a
 * single kernel).  Running E4B_STAGE_ROUTE .. E4B_STAGE_COMBINE in order on
 * one stream and workspace is exactly e4b_moe_forward; a stage reads what the
 * earlier stages left in the workspace.
 */
e4b_status e4b_moe_forward_stage(int32_t stage, const e4b_moe_desc* d, int32_t T, const uint16_t* x,
                                 const uint16_t* logits, const uint8_t* gu_codes, const void* gu_scales,
                                 const uint8_t* dn_codes, const void* dn_scales,
                                 const uint16_t* lora_A, const uint16_t* lora_B,
                                 const float* gu_bias, const float* dn_bias, uint16_t* out,
                                 void* ws, size_t ws_bytes, e4b_stream stream);

/* Intermediate buffers inside a forward workspace, for inspection. */
enum {
  E4B_WS_TOPK_IDS = 0,     /* int32 [T*k] */
  E4B_WS_TOPK_W = 1,       /* fp32  [T*k] */
  E4B_WS_EXPERT_OFFSETS = 2, /* int32 [E+1] */
  E4B_WS_SORTED_SLOT = 3,  /* int32 [T*k] */
  E4B_WS_X_SORTED = 4,     /* bf16  [T*k, H] */
  E4B_WS_H = 5,            /* bf16  [T*k, I]  act(gate, up) per routed row */
  E4B_WS_Y = 6,            /* fp32  [T*k, H]  down output per routed row */
  E4B_WS_GU_ABSMAX = 7,    /* fp32  [E*2I*H/64] expanded gate_up absmax (E4B_NF4_DQ; touched experts only) */
  E4B_WS_DN_ABSMAX = 8     /* fp32  [E*H*I/64]  expanded down absmax (E4B_NF4_DQ; touched experts only) */
};

/* Byte offset and size of one intermediate of e4b_moe_forward's workspace. */
e4b_status e4b_moe_workspace_region(const e4b_moe_desc* d, int32_t T, int32_t region,
                                    size_t* offset, size_t* bytes);

/*
 * Synchronises `stream`, then reads and clears the status word at the start
 * of a workspace used by e4b_moe_forward or e4b_route.  Returns E4B_OK or the
 * first device-side error recorded since the last call (E4B_ERR_TIMEOUT when
 * a bounded wait ran out).
 */
e4b_status e4b_device_status(void* ws, e4b_stream stream);

/*
 * Test hook for the bounded-wait machinery: launches one block that waits on
 * a barrier nothing ever releases, with a limit of limit_ns nanoseconds (at
 * most 10^9), then records E4B_ERR_TIMEOUT in the workspace status word and
 * returns from the kernel.  Read the result with e4b_device_status().
 */
e4b_status e4b_debug_wait_timeout(uint32_t limit_ns, void* ws, size_t ws_bytes, e4b_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* E4B_H */
