// Grouped 4-bit GEMMs for decode-sized batches: few routed rows per expert.
//
// Same contraction as grouped_gemm.cu ("MoE Training & Inference Guides",
// grouped-nf4-gemm table: packed 4-bit expert stacks, codes decoded on chip,
// fp32 accumulation, one launch over all experts; "experts4bit-qlora" limits
// list: the stock epilogue act(gate)*up; "experts4bit-qlora" index table:
// ExpertsLoRA's per-expert low-rank delta before the activation), organised
// for the case where each expert sees only a handful of tokens and the weight
// stream from HBM is the whole cost.
//
// Why a second kernel: with <= 8 tokens per expert a 128-row tcgen05 tile
// spends one UMMA (fixed issue cost, independent of N) per 1 KB of packed
// codes, and the dequantised operand must round-trip through shared or tensor
// memory with a barrier handshake per stage.  Here every warp owns its rows
// end to end: it streams the packed codes straight into registers, decodes
// them through a byte table into the A fragments of warp-level bf16 MMAs
// (m16n8k16, 8 tokens per MMA), and accumulates in registers.  No
// shared-memory operand, no cross-warp synchronisation.
//
// Work unit: (chunk of <= 8 tokens of one expert, group of MT 16-row tiles),
// full K.  chunk_off[E+1] is the router's prefix of ceil(count_e / 8).
//  * mode 0 (gate_up): tile j pairs gate rows gi..gi+7 with up rows
//    I+gi..I+gi+7 (gi = 8 * (MT * rg + j)), so each thread holds gate and up
//    of the same (token, column) and applies SwiGLU in registers;
//  * mode 1 (down): tile j covers output rows 16 * (MT * rg + j) + 0..15.
//
// Fragment/byte mapping.  Lane (g = lane / 4, c = lane % 4) loads, per 64-K
// block, the 8 code bytes [8c, 8c+8) of its two rows (g and g+8 of the tile):
// the four lanes of a quad cover one 32-byte block row, so every load
// instruction reads whole 32-byte sectors.  MMA i (i = 0..3) of the block
// takes code byte 2i (elements 16c+4i, +1) as the low K pair and byte 2i+1
// (elements 16c+4i+2, +3) as the high K pair of the A fragment; the B
// fragment (activations) is loaded with the same K permutation, so the dot
// product is unchanged.
//
// Scales.  NF4: the byte table holds the bf16-rounded codebook levels; the
// per-64 fp32 absmax multiplies the block's fp32 partial sum (one MMA chain
// per block), so the weights are never rounded after scaling.  MXFP4: exact
// bf16 e2m1 pairs times the bf16 power-of-two scale (exact).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "e4b_device.cuh"
#include "e4b_internal.h"

namespace e4b {
namespace {

constexpr int SK_WARPS = 8;
constexpr int SK_THREADS = SK_WARPS * 32;
constexpr int SK_TOK = 8;                        // tokens per chunk (MMA N)
constexpr int SK_LUT_WORDS = 256 * 32;           // byte table, one copy per lane

struct SkParams {
  int32_t E, N, K, I;
  int32_t row_groups;     // units per chunk
  int32_t lora_rank;
  const uint8_t* codes;   // [E, N, K/2]
  const void* scales;     // NF4 fp32 [E, N, K/64]; MXFP4 u8 [E, N, K/32]
  const uint16_t* act;    // [R, K] bf16
  const uint16_t* xa;     // [R, 64] bf16 (mode 0 with LoRA)
  const uint16_t* lora_B; // [E, r, 2I]
  const int32_t* expert_offsets;
  const int32_t* chunk_off;
  void* out;              // mode 0: bf16 h [R, I]; mode 1: fp32 y [R, N]
  uint32_t lut_hi[8];     // NF4: bf16 levels, two per word (level 2w low, 2w+1 high)
};

__device__ __forceinline__ uint2 ld_stream_v2(const uint8_t* p) {
  uint2 r;
  asm("ld.global.nc.L1::no_allocate.L2::256B.v2.u32 {%0, %1}, [%2];"
               : "=r"(r.x), "=r"(r.y)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ld_act_v4(const uint16_t* p) {
  uint4 r;
  asm("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// lut_l points at this lane's column of the table (entry stride 32 words).
__device__ __forceinline__ uint32_t lut_at(const uint32_t* lut_l, uint32_t word, int byte) {
  return lut_l[((word >> (8 * byte)) & 0xFFu) << 5];
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// bf16x2 of the E8M0 scale 2^(s-127) in both halves (s = 0: bf16 subnormal, 255: NaN).
__device__ __forceinline__ uint32_t e8m0_bf16x2(uint32_t s) {
  const uint32_t b = s == 0u ? 0x0040u : (s == 255u ? 0x7FC0u : (s << 7));
  return b | (b << 16);
}

__device__ __forceinline__ float e2m1_value(uint32_t nib) {
  return __uint_as_float(((nib & 8u) << 28) | ((nib & 7u) << 22)) * 0x1p126f;
}

struct Unit {
  int e, t0, m, rg;
};

// Unit u -> (expert, first token, tokens, row group), from the CTA's copies of
// chunk_off[E+1] and expert_offsets[E+1].
__device__ __forceinline__ Unit decode_unit(int u, int row_groups, int E, const int32_t* s_chunk,
                                            const int32_t* s_off) {
  const int chunk = u / row_groups;
  Unit r;
  r.rg = u - chunk * row_groups;
  int lo = 0, hi = E;                   // last e with chunk_off[e] <= chunk
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_chunk[mid] <= chunk) lo = mid; else hi = mid;
  }
  r.e = lo;
  r.t0 = s_off[lo] + SK_TOK * (chunk - s_chunk[lo]);
  const int rem = s_off[lo + 1] - r.t0;
  r.m = rem < SK_TOK ? rem : SK_TOK;
  return r;
}

template <int FMT, int MODE, int MT>
struct Slot {
  uint2 q[MT][2];                                        // code bytes of rows g, g+8 of each tile
  uint32_t s[MT][2];                                     // NF4 absmax bits / MXFP4 bf16x2 scale
  uint4 x[2];                                            // 16 activations of token g
};

// Row of the stack that lane row g of tile 0 reads (tile j, half rr add
// compile-time multiples of the row steps below).
template <int MODE, int MT>
__device__ __forceinline__ int first_row(const SkParams& p, int rg, int g) {
  return MODE == 0 ? 8 * MT * rg + g : 16 * MT * rg + g;
}

template <int FMT, int MODE, int MT>
__device__ __forceinline__ void issue_loads(const SkParams& p, const Unit& u, int b, int g, int c,
                                            Slot<FMT, MODE, MT>& sl) {
  const int row0 = first_row<MODE, MT>(p, u.rg, g);
  const int64_t rbytes = p.K >> 1;
  const int tile_rows = MODE == 0 ? 8 : 16;             // row step between tiles
  const int half_rows = MODE == 0 ? p.I : 8;            // row step from row g to row g+8 of a tile
  const int64_t er = static_cast<int64_t>(u.e) * p.N + row0;
  const uint8_t* cp = p.codes + er * rbytes + b * 32 + 8 * c;
#pragma unroll
  for (int j = 0; j < MT; ++j)
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
      sl.q[j][rr] = ld_stream_v2(cp + (static_cast<int64_t>(j) * tile_rows + rr * half_rows) * rbytes);
  if (FMT == E4B_NF4) {
    const int kb = p.K >> 6;
    const float* sp = static_cast<const float*>(p.scales) + er * kb + b;
#pragma unroll
    for (int j = 0; j < MT; ++j)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr)
        sl.s[j][rr] = __float_as_uint(__ldg(sp + (static_cast<int64_t>(j) * tile_rows + rr * half_rows) * kb));
  } else {
    const int kb = p.K >> 5;
    const uint8_t* sp = static_cast<const uint8_t*>(p.scales) + er * kb + 2 * b + (c >> 1);
#pragma unroll
    for (int j = 0; j < MT; ++j)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr)
        sl.s[j][rr] = __ldg(sp + (static_cast<int64_t>(j) * tile_rows + rr * half_rows) * kb);
  }
  if (g < u.m) {
    const uint16_t* xp = p.act + static_cast<int64_t>(u.t0 + g) * p.K + b * 64 + 16 * c;
    sl.x[0] = ld_act_v4(xp);
    sl.x[1] = ld_act_v4(xp + 8);
  } else {
    sl.x[0] = make_uint4(0, 0, 0, 0);
    sl.x[1] = make_uint4(0, 0, 0, 0);
  }
}

template <int FMT, int MODE, int MT>
__device__ __forceinline__ void compute_block(const Slot<FMT, MODE, MT>& sl, const uint32_t* lut_l, float (&acc)[MT][4]) {
  const uint32_t xw[8] = {sl.x[0].x, sl.x[0].y, sl.x[0].z, sl.x[0].w, sl.x[1].x, sl.x[1].y, sl.x[1].z, sl.x[1].w};
#pragma unroll
  for (int j = 0; j < MT; ++j) {
    float blk[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t s2[2] = {0u, 0u};
    if (FMT == E4B_MXFP4) {
      s2[0] = e8m0_bf16x2(sl.s[j][0]);
      s2[1] = e8m0_bf16x2(sl.s[j][1]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w0 = i < 2 ? sl.q[j][0].x : sl.q[j][0].y;
      const uint32_t w1 = i < 2 ? sl.q[j][1].x : sl.q[j][1].y;
      const int by = 2 * (i & 1);
      uint32_t a[4];
      a[0] = lut_at(lut_l, w0, by);
      a[1] = lut_at(lut_l, w1, by);
      a[2] = lut_at(lut_l, w0, by + 1);
      a[3] = lut_at(lut_l, w1, by + 1);
      if (FMT == E4B_MXFP4) {
        a[0] = bf16x2_mul(a[0], s2[0]);
        a[1] = bf16x2_mul(a[1], s2[1]);
        a[2] = bf16x2_mul(a[2], s2[0]);
        a[3] = bf16x2_mul(a[3], s2[1]);
        mma_bf16(acc[j], a, xw[2 * i], xw[2 * i + 1]);
      } else {
        mma_bf16(blk, a, xw[2 * i], xw[2 * i + 1]);
      }
    }
    if (FMT == E4B_NF4) {
      const float s0 = __uint_as_float(sl.s[j][0]), s1 = __uint_as_float(sl.s[j][1]);
      acc[j][0] = fmaf(s0, blk[0], acc[j][0]);
      acc[j][1] = fmaf(s0, blk[1], acc[j][1]);
      acc[j][2] = fmaf(s1, blk[2], acc[j][2]);
      acc[j][3] = fmaf(s1, blk[3], acc[j][3]);
    }
  }
}

__device__ __forceinline__ uint32_t lora_pair(const uint16_t* col, int64_t rstride, int j0, int rank) {
  const uint32_t lo = j0 < rank ? __ldg(col + j0 * rstride) : 0u;
  const uint32_t hi = j0 + 1 < rank ? __ldg(col + (j0 + 1) * rstride) : 0u;
  return lo | (hi << 16);
}

template <int MODE, int MT>
__device__ __forceinline__ void epilogue(const SkParams& p, const Unit& u, int g, int c, float (&acc)[MT][4]) {
  if (MODE == 0) {
    if (p.lora_rank > 0) {
      // LoRA step: A = B_e^T (rows n, K = rank padded to 16), B = xa (scale folded in).
      uint32_t b0 = 0u, b1 = 0u;
      if (g < u.m) {
        const uint32_t* xr = reinterpret_cast<const uint32_t*>(p.xa + static_cast<int64_t>(u.t0 + g) * 64);
        b0 = __ldg(xr + c);
        b1 = __ldg(xr + 4 + c);
      }
      const int64_t rs = 2 * static_cast<int64_t>(p.I);
      const uint16_t* Be = p.lora_B + static_cast<int64_t>(u.e) * p.lora_rank * rs;
#pragma unroll
      for (int j = 0; j < MT; ++j) {
        const int col = 8 * (MT * u.rg + j) + g;
        uint32_t a[4];
        a[0] = lora_pair(Be + col, rs, 2 * c, p.lora_rank);
        a[1] = lora_pair(Be + p.I + col, rs, 2 * c, p.lora_rank);
        a[2] = lora_pair(Be + col, rs, 2 * c + 8, p.lora_rank);
        a[3] = lora_pair(Be + p.I + col, rs, 2 * c + 8, p.lora_rank);
        mma_bf16(acc[j], a, b0, b1);
      }
    }
    __nv_bfloat16* h = static_cast<__nv_bfloat16*>(p.out);
#pragma unroll
    for (int j = 0; j < MT; ++j) {
      const int col = 8 * (MT * u.rg + j) + g;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (2 * c + t < u.m) {
          const float v = acc[j][t], w = acc[j][2 + t];
          const float sg = __fdividef(v, 1.0f + __expf(-v));
          h[static_cast<int64_t>(u.t0 + 2 * c + t) * p.I + col] = __float2bfloat16_rn(sg * w);
        }
      }
    }
  } else {
    float* y = static_cast<float*>(p.out);
#pragma unroll
    for (int j = 0; j < MT; ++j) {
      const int n = 16 * (MT * u.rg + j) + g;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (2 * c + t < u.m) {
          float* yr = y + static_cast<int64_t>(u.t0 + 2 * c + t) * p.N + n;
          yr[0] = acc[j][t];
          yr[8] = acc[j][2 + t];
        }
      }
    }
  }
}

template <int FMT, int MODE, int MT, int D>
__global__ void __launch_bounds__(SK_THREADS, 2) skinny_gemm_kernel(const __grid_constant__ SkParams p) {
  extern __shared__ uint32_t sk_smem[];
  uint32_t* lut = sk_smem;
  int32_t* s_chunk = reinterpret_cast<int32_t*>(sk_smem + SK_LUT_WORDS);
  int32_t* s_off = s_chunk + (kMaxExperts + 1);

  __shared__ uint16_t s_level[16];
  if (FMT == E4B_NF4 && threadIdx.x < 16) {
    const uint32_t w = p.lut_hi[threadIdx.x >> 1];
    s_level[threadIdx.x] = static_cast<uint16_t>(w >> (16 * (threadIdx.x & 1)));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < SK_LUT_WORDS; i += SK_THREADS) {
    const uint32_t b = static_cast<uint32_t>(i) >> 5;
    uint32_t v;
    if (FMT == E4B_NF4) {
      // element 2j sits in the high nibble: it goes to the low half
      v = static_cast<uint32_t>(s_level[b >> 4]) | (static_cast<uint32_t>(s_level[b & 15u]) << 16);
    } else {
      // element 2j sits in the low nibble: it goes to the low half
      __nv_bfloat162 t = __floats2bfloat162_rn(e2m1_value(b & 15u), e2m1_value(b >> 4));
      v = *reinterpret_cast<uint32_t*>(&t);
    }
    lut[i] = v;
  }
  for (int i = threadIdx.x; i <= p.E; i += SK_THREADS) {
    s_chunk[i] = __ldg(p.chunk_off + i);
    s_off[i] = __ldg(p.expert_offsets + i);
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const uint32_t* lut_l = lut + lane;
  const int gwarp = blockIdx.x * SK_WARPS + warp;
  const int nwarps = gridDim.x * SK_WARPS;
  const int total = s_chunk[p.E] * p.row_groups;
  if (gwarp >= total) return;
  const int KB = p.K >> 6;
  const int my_units = (total - gwarp + nwarps - 1) / nwarps;
  const int nsteps = my_units * KB;

  // load side: next step to issue, its unit and block
  int l_unit = gwarp, l_b = 0;
  Unit lu = decode_unit(l_unit, p.row_groups, p.E, s_chunk, s_off);
  // compute side
  int c_unit = gwarp, c_b = 0;
  Unit cu = lu;

  Slot<FMT, MODE, MT> slot[D];
  float acc[MT][4];
#pragma unroll
  for (int j = 0; j < MT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

  auto advance_load = [&]() {
    if (++l_b == KB) {
      l_b = 0;
      l_unit += nwarps;
      if (l_unit < total) lu = decode_unit(l_unit, p.row_groups, p.E, s_chunk, s_off);
    }
  };

#pragma unroll
  for (int d = 0; d < D; ++d) {
    if (d < nsteps) {
      issue_loads<FMT, MODE, MT>(p, lu, l_b, g, c, slot[d]);
      advance_load();
    }
  }

  for (int s0 = 0; s0 < nsteps; s0 += D) {
#pragma unroll
    for (int d = 0; d < D; ++d) {
      const int st = s0 + d;
      if (st < nsteps) {
        compute_block<FMT, MODE, MT>(slot[d], lut_l, acc);
        if (st + D < nsteps) {
          issue_loads<FMT, MODE, MT>(p, lu, l_b, g, c, slot[d]);
          advance_load();
        }
        if (++c_b == KB) {
          epilogue<MODE, MT>(p, cu, g, c, acc);
#pragma unroll
          for (int j = 0; j < MT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
          c_b = 0;
          c_unit += nwarps;
          if (c_unit < total) cu = decode_unit(c_unit, p.row_groups, p.E, s_chunk, s_off);
        }
      }
    }
  }
}

constexpr int kSmemBytes = SK_LUT_WORDS * 4 + 2 * (kMaxExperts + 1) * 4;

template <int FMT, int MODE, int MT, int D>
e4b_status launch_cfg(const SkParams& prm, cudaStream_t s) {
  auto kern = skinny_gemm_kernel<FMT, MODE, MT, D>;
  static int blocks_per_sm[64] = {0};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return E4B_ERR_CUDA;
  int bps = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (blocks_per_sm[dev] == 0) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
        return E4B_ERR_CUDA;
      int n = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, SK_THREADS, kSmemBytes) != cudaSuccess || n < 1)
        return E4B_ERR_CUDA;
      blocks_per_sm[dev] = n;
    }
    bps = blocks_per_sm[dev];
  }
  kern<<<device_sm_count() * bps, SK_THREADS, kSmemBytes, s>>>(prm);
  return cudaGetLastError() == cudaSuccess ? E4B_OK : E4B_ERR_CUDA;
}

}  // namespace

e4b_status launch_skinny_gemm(const GroupedGemmLaunch& g, cudaStream_t s) {
  if (g.R == 0) return E4B_OK;
  constexpr int MT = 2;
  SkParams prm;
  prm.E = g.E;
  prm.N = g.N;
  prm.K = g.K;
  prm.I = g.I;
  prm.row_groups = g.mode == 0 ? g.I / (8 * MT) : g.N / (16 * MT);
  prm.lora_rank = g.mode == 0 ? g.lora_rank : 0;
  prm.codes = g.codes;
  prm.scales = g.scales;
  prm.act = g.act;
  prm.xa = g.xa;
  prm.lora_B = g.lora_B;
  prm.expert_offsets = g.expert_offsets;
  prm.chunk_off = g.chunk_off;
  prm.out = g.out;
  const Nf4Table& t = nf4_table();
  for (int w = 0; w < 8; ++w) {
    const __nv_bfloat16 lo = __float2bfloat16_rn(t.level[2 * w]);
    const __nv_bfloat16 hi = __float2bfloat16_rn(t.level[2 * w + 1]);
    prm.lut_hi[w] = static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&lo)) |
                    (static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&hi)) << 16);
  }
  if ((g.mode == 0 && g.I % (8 * MT) != 0) || (g.mode == 1 && g.N % (16 * MT) != 0) || g.K % 64 != 0)
    return E4B_ERR_UNSUPPORTED;
  if (g.fmt == E4B_NF4)
    return g.mode == 0 ? launch_cfg<E4B_NF4, 0, MT, 4>(prm, s) : launch_cfg<E4B_NF4, 1, MT, 4>(prm, s);
  return g.mode == 0 ? launch_cfg<E4B_MXFP4, 0, MT, 4>(prm, s) : launch_cfg<E4B_MXFP4, 1, MT, 4>(prm, s);
}

}  // namespace e4b
