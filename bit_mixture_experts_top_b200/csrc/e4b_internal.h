// Host-side internals shared by the library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "e4b.h"

namespace e4b {

// What the gate_up and down launches add to their fp32 accumulators.  The
// stock epilogue is silu(gate) * up with no bias.  The gpt-oss epilogue
// ("How do I train and serve MoE models released in MXFP4 (gpt-oss,
// DeepSeek-V4)?", "Why it happens": per-expert biases and a clamped GLU) adds
// a per-expert bias to each output and, on gate_up, applies
// min(gate, limit) * sigmoid(alpha * .) * (clamp(up, -limit, limit) + beta).
struct Epilogue {
  const float* bias;   // gate_up launch: [E, 2I] as [gate | up]; down launch: [E, H]; null = none
  int32_t glu;         // E4B_ACT_SWIGLU or E4B_ACT_CLAMPED_GLU
  float alpha, limit, beta;
};


constexpr size_t kAlign = 256;
constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 32;
constexpr int kMaxLoraRank = 16;
constexpr int kRouteTokensPerBlock = 128;   // tokens per histogram block of the router
constexpr int kDecodeMaxRows = 12;         // auto choice: decode kernel up to this mean rows per expert
constexpr int kStatusBytes = 256;           // status word + router done-counter at the start of a workspace
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // bounded device waits: 2 s

inline size_t align_up(size_t v, size_t a = kAlign) { return (v + a - 1) / a * a; }

// Launches a forward-path kernel with programmatic stream serialization, so it
// may begin (up to its pdl_wait()) while the previous kernel on the stream
// finishes; the launch is captured into CUDA graphs as a programmatic edge.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// 16 fp32 NF4 levels and the 15 fp32 decision midpoints, built on the host from
// the NormalFloat construction (own inverse-normal-CDF, see nf4_table.cpp).
struct Nf4Table {
  float level[16];
  float mid[15];
};
const Nf4Table& nf4_table();

// Router: status/done-counter layout inside the first kStatusBytes of a workspace.
struct RouteBuffers {
  int32_t* status;          // [2] device status word
  uint32_t* done_counter;   // last-block detection of the histogram kernel
  int32_t* topk_ids;        // [T*k]
  float* topk_w;            // [T*k]
  int32_t* expert_offsets;  // [E+1]
  int32_t* chunk_off;       // [E+1] prefix of ceil(count_e / tokens_per_tile), or null
  int32_t* block_counts;    // [nblk * E] per-block histograms, then per-block bases
  int32_t* sorted_slot;     // [T*k]
  int32_t* slot_pos;        // [T*k]
};

inline int route_blocks(int32_t T) { return (T + kRouteTokensPerBlock - 1) / kRouteTokensPerBlock; }

// Routing kernels.  status_words (kStatusBytes, or null) are zeroed before
// anything else runs: inside the single routing block for T <= 128, else by a
// memset ahead of the multi-block kernels.
cudaError_t launch_route(const uint16_t* logits, int32_t T, int32_t E, int32_t k, int32_t gating,
                         int32_t tokens_per_tile,
                         const RouteBuffers& b, int32_t* status_words, cudaStream_t s);

cudaError_t launch_dequant_mxfp4(const uint8_t* codes, const uint8_t* scales, int64_t n, uint16_t* out,
                                 cudaStream_t s);

cudaError_t launch_quantize_nf4(const float* x, int64_t n, uint8_t* codes, float* absmax, cudaStream_t s);
// absmax[b] = fl32(fl32(table[codes[b]] * absmax2[b / 256]) + *offset) for b < n; with expert_offsets,
// blocks of experts (per_expert absmax each) that no row is routed to are left unwritten.
cudaError_t launch_expand_absmax_dq(const uint8_t* codes, const float* absmax2, const float* offset,
                                    const float* table, int64_t n, int64_t per_expert,
                                    const int32_t* expert_offsets, float* out, cudaStream_t s);
cudaError_t launch_deinterleave_rows(const void* in, void* out, int32_t E, int32_t I, int64_t row_bytes,
                                     cudaStream_t s);

// x_sorted[r] = x[sorted_slot[r] / k]; with LoRA also xa[r, j] = bf16(scale * x . A_e[:, j]) (j < r, zeros to 64).
cudaError_t launch_gather(const uint16_t* x, int32_t H, int32_t k, int32_t R, const int32_t* sorted_slot,
                          const int32_t* topk_ids, int32_t E, uint16_t* x_sorted, const uint16_t* lora_A,
                          int32_t lora_rank, float lora_scale, uint16_t* xa, cudaStream_t s);

// out[t] = sum_j w[t, j] * y[slot_pos[t*k + j]], j ascending, fp32 -> bf16.
cudaError_t launch_combine(const float* y, const float* topk_w, const int32_t* slot_pos, int32_t T, int32_t k,
                           int32_t H, uint16_t* out, cudaStream_t s);

// Grouped 4-bit GEMMs on tcgen05.
struct GroupedGemmLaunch {
  int32_t mode;             // 0: gate_up + LoRA + SwiGLU -> bf16 h [R, I]; 1: down -> fp32 y [R, H]
  int32_t fmt;              // E4B_NF4 / E4B_MXFP4
  int32_t E, N, K, I;       // stack [E, N, K]; I = intermediate size (mode 0 pairing)
  int32_t R;                // routed rows
  int32_t tokens_per_tile;  // decode kernel: tokens per chunk (8, 16, 32); tcgen05: tile width (32..256)
  int32_t decode;           // 1: skinny_gemm (decode kernel), 0: grouped_gemm (tcgen05)
  const uint8_t* codes;     // [E, N, K] packed
  const void* scales;
  const uint16_t* act;      // [R, K] bf16 (x_sorted or h)
  const uint16_t* xa;       // [R, 64] bf16 LoRA left factor (mode 0) or null
  const uint16_t* lora_B;   // [E, r, 2I] or null
  int32_t lora_rank;
  const int32_t* expert_offsets;
  const int32_t* chunk_off;
  void* out;                // mode 0: bf16 [R, I]; mode 1: fp32 [R, H]
  int32_t* status;
  uint64_t wait_limit_ns;
  const float* bias;        // mode 0: [E, 2I] ([gate | up]); mode 1: [E, H]; null = none
  int32_t glu;              // E4B_ACT_SWIGLU / E4B_ACT_CLAMPED_GLU (mode 0)
  float glu_alpha, glu_limit, glu_beta;
  float* g_out;             // mode 0: the pre-activation outputs G [R, 2I] fp32 ([gate | up]) or null
};
e4b_status launch_grouped_gemm(const GroupedGemmLaunch& g, cudaStream_t s);

// Decode-sized batches: warp-level MMA with the codes decoded in registers;
// chunk_off counts chunks of tokens_per_tile (8, 16 or 32) tokens.
e4b_status launch_skinny_gemm(const GroupedGemmLaunch& g, cudaStream_t s);
bool skinny_gemm_supported(int32_t K, int32_t fmt);   // the per-unit scale buffers fit in shared memory

int device_sm_count();

// Layer backward (QLoRA): everything the training forward left in its workspace plus the
// upstream gradient; outputs dx [T, H], dlogits [T, E] and, with LoRA, dA [E, H, r], dB [E, r, 2I].
struct BackwardLaunch {
  int32_t T, k, E, H, I, fmt, gating, lora_rank;
  float lora_scale;
  Epilogue ep;
  const uint16_t* logits;       // [T, E] bf16
  const uint16_t* dout;         // [T, H] bf16
  const float* y;               // [R, H] fp32 down outputs (expert order)
  const float* topk_w;
  const int32_t *topk_ids, *slot_pos, *sorted_slot, *expert_offsets;
  const uint16_t* x_sorted;     // [R, H]
  const uint16_t* xa;           // [R, 64] bf16 s * x A_e (LoRA)
  const float* G;               // [R, 2I] fp32
  uint16_t* dY;                 // [R, H] bf16 scratch
  uint16_t* dG;                 // [R, 2I] bf16 scratch
  float* dxa;                   // [R, 16] fp32 scratch
  float* dX;                    // [R, H] fp32 scratch
  float *dx, *dlogits, *dA, *dB;
  const uint8_t *gu_codes, *dn_codes;
  const void *gu_scales, *dn_scales;   // NF4 fp32 absmax (expanded for the nested form) or MXFP4 e8m0
  const uint16_t *lora_A, *lora_B;
};
e4b_status launch_moe_backward(const BackwardLaunch& b, cudaStream_t s);

// 2-D tiled tensor map (inner dim contiguous, `row_bytes` apart) through the
// driver entry point; false when the driver refuses the description.
bool encode_tma_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);
// 3-D tiled tensor map: dims d0 (contiguous), d1 (stride1_bytes apart), d2 (stride2_bytes apart).
bool encode_tma_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t d0, uint64_t d1,
                   uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2,
                   CUtensorMapSwizzle swz);

}  // namespace e4b
