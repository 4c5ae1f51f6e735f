// Backward of the routed 4-bit MoE layer for QLoRA: gradients of the LoRA
// factors and of the layer's inputs, through the frozen packed stacks.
//
// "MoE Training & Inference Guides" (solutions index), experts4bit-qlora
// table: ExpertsLoRA wraps each frozen 4-bit expert stack with a per-expert
// low-rank adapter, and the fast training path runs the grouped kernels with
// dgrad, i.e. the input gradient is taken through the frozen 4-bit weights as
// well.  For routed row r = (t, j) of expert e with gate weight w:
//
//   dY_r = w * dout_t,  dw = <dout_t, Y_r>          (bwd_gate_kernel)
//   dh   = dY_r W_dn[e]                              (dgrad_kernel, down stack)
//   dG   = act'(G) applied to dh, [gate | up]        (its epilogue)
//   dxa  = s dG B_e^T                                (lora_dxa_kernel)
//   dX_r = dG W_gu[e] + dxa A_e^T                    (dgrad_kernel, gate_up stack)
//   dx_t = sum_j dX_(t, j)                           (dx_combine_kernel)
//   dB_e = sum_r xa_r^T dG_r,  dA_e = sum_r x_r^T dxa_r   (lora_grads_kernel)
//
// and the gate weights' gradient goes through the gating softmax into the
// logits.  The routing choice itself is piecewise constant and carries none.
//
// dgrad contracts over the STORED ROW dimension of a stack (H rows of the down
// stack [E, H, I], 2I rows of the gate_up stack [E, 2I, H]) and produces the
// K-contiguous dimension, so its weight tiles are the transpose of the
// forward's: a CTA decodes a 64-row x 64-column slab of packed codes into a
// bf16 tile in shared memory (NF4 as one rounding of level * absmax, MXFP4
// exactly) and multiplies it with warp-level MMAs, reading the slab through
// transposing matrix loads.  No transposed copy of a stack exists anywhere.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "e4b_device.cuh"
#include "e4b_internal.h"

namespace e4b {
namespace {

constexpr uint32_t kFull = 0xFFFFFFFFu;
constexpr int kDgTok = 64;       // routed rows per dgrad tile
constexpr int kDgCols = 128;     // output columns per dgrad tile
constexpr int kDgK = 64;         // stored rows (contraction) per slab
constexpr int kPad = 72;         // activation tile row pitch in bf16 (conflict-free matrix loads)
constexpr int kPadW = 136;       // weight tile row pitch in bf16
constexpr int kDgSmem = 2 * kDgK * kPadW * 2 + 2 * kDgTok * kPad * 2;   // double-buffered tiles

__device__ __forceinline__ float sigmoidf_acc(float z) { return 1.0f / (1.0f + expf(-z)); }

// d(act)/d(gate) and d(act)/d(up) at (gate, up): SwiGLU or the clamped GLU.
// The clamps pass the gradient inside their range, ends included.
__device__ __forceinline__ void act_grads(const Epilogue& ep, float gate, float up, float& dg, float& du) {
  if (ep.glu == E4B_ACT_CLAMPED_GLU) {
    const float g = fminf(gate, ep.limit);
    const float u = fminf(fmaxf(up, -ep.limit), ep.limit);
    const float sa = sigmoidf_acc(ep.alpha * g);
    const float f = g * sa;
    const float df = sa * (1.0f + ep.alpha * g * (1.0f - sa));
    dg = gate <= ep.limit ? df * (u + ep.beta) : 0.0f;
    du = (up >= -ep.limit && up <= ep.limit) ? f : 0.0f;
    return;
  }
  const float s = sigmoidf_acc(gate);
  dg = up * s * (1.0f + gate * (1.0f - s));
  du = gate * s;
}

__device__ __forceinline__ float block_sum(float v, float* s_red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  float t = 0.0f;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += s_red[w];
  return t;
}

__device__ __forceinline__ float block_max(float v, float* s_red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, off));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  float t = s_red[0];
  for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) t = fmaxf(t, s_red[w]);
  return t;
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }
__device__ __forceinline__ float bf16_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// One block per token: dw_j = <dout_t, y_(t,j)> (one warp per pick j), dY rows
// in expert order, and the logit gradient through the gating softmax (fp32).
__global__ void __launch_bounds__(256) bwd_gate_kernel(const uint16_t* __restrict__ dout, const float* __restrict__ y,
                                                       const float* __restrict__ topk_w,
                                                       const int32_t* __restrict__ topk_ids,
                                                       const int32_t* __restrict__ slot_pos,
                                                       const uint16_t* __restrict__ logits, int E, int k, int H,
                                                       int gating, uint16_t* __restrict__ dY,
                                                       float* __restrict__ dlogits) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ float s_red[8];
  __shared__ float s_dw[kMaxTopK];
  const int64_t t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint16_t* drow = dout + t * H;
  for (int j = warp; j < k; j += 8) {
    const int64_t pos = slot_pos[t * k + j];
    const float w = topk_w[t * k + j];
    const float4* yr = reinterpret_cast<const float4*>(y + pos * H);
    const uint2* dr = reinterpret_cast<const uint2*>(drow);
    uint2* dyr = reinterpret_cast<uint2*>(dY + pos * H);
    float acc = 0.0f;
    for (int c = lane; c < H / 4; c += 32) {          // four elements per lane and step
      const uint2 d = __ldg(dr + c);
      const float4 v = yr[c];
      const float d0 = bf16_to_f32(d.x & 0xFFFFu), d1 = bf16_to_f32(d.x >> 16);
      const float d2 = bf16_to_f32(d.y & 0xFFFFu), d3 = bf16_to_f32(d.y >> 16);
      acc = fmaf(d0, v.x, fmaf(d1, v.y, fmaf(d2, v.z, fmaf(d3, v.w, acc))));
      dyr[c] = make_uint2(pack_bf16x2(w * d0, w * d1), pack_bf16x2(w * d2, w * d3));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(kFull, acc, off);
    if (lane == 0) s_dw[j] = acc;
  }
  __syncthreads();
  float S = 0.0f;                                   // sum_j w_j dw_j
  for (int j = 0; j < k; ++j) S = fmaf(topk_w[t * k + j], s_dw[j], S);
  float* dl = dlogits + t * E;
  if (gating == E4B_GATE_SOFTMAX_ALL) {
    // p = softmax over all E logits; dl_e = -p_e S + [e picked] w_j dw_j  (w_j = p at pick j)
    const uint16_t* lr = logits + t * E;
    float m = -INFINITY;
    for (int e = threadIdx.x; e < E; e += blockDim.x) m = fmaxf(m, bf16_to_f32(lr[e]));
    m = block_max(m, s_red);
    float z = 0.0f;
    for (int e = threadIdx.x; e < E; e += blockDim.x) z += expf(bf16_to_f32(lr[e]) - m);
    z = block_sum(z, s_red);
    for (int e = threadIdx.x; e < E; e += blockDim.x) dl[e] = -(expf(bf16_to_f32(lr[e]) - m) / z) * S;
    __syncthreads();
    if (threadIdx.x < k) {
      const int j = threadIdx.x;
      const int e = topk_ids[t * k + j];
      dl[e] += topk_w[t * k + j] * s_dw[j];
    }
  } else {
    // softmax over the k picks: dl at pick j = w_j (dw_j - S), zero elsewhere
    for (int e = threadIdx.x; e < E; e += blockDim.x) dl[e] = 0.0f;
    __syncthreads();
    if (threadIdx.x < k) {
      const int j = threadIdx.x;
      dl[topk_ids[t * k + j]] = topk_w[t * k + j] * (s_dw[j] - S);
    }
  }
}

struct DgParams {
  int32_t E, M, N, I;            // stack [E, M rows, N columns]; I: the gate_up half width (mode 0)
  const uint8_t* codes;          // [E, M, N/2] packed
  const void* scales;            // NF4 fp32 [E*M*N/64]; MXFP4 e8m0 [E*M*N/32]
  const uint16_t* act;           // [R, M] bf16: dY (mode 0) or dG (mode 1)
  const int32_t* expert_offsets;
  // mode 0 (down stack -> dG): saved G [R, 2I] fp32 in, dG [R, 2I] bf16 out
  const float* G;
  uint16_t* dG;
  Epilogue ep;
  // mode 1 (gate_up stack -> dX): dX [R, N] fp32 out (+ dxa [R, 16] A_e^T with LoRA)
  float* dX;
  const float* dxa;
  const uint16_t* lora_A;        // [E, N, r]
  int32_t lora_rank;
  float lut[16];                 // NF4 levels
};

// Tile (expert, first routed row, rows) of chunk index `chunk`: experts in
// order, ceil(count / kDgTok) chunks each.  One warp scans the offsets.
__device__ __forceinline__ bool dgrad_tile(const int32_t* __restrict__ offs, int E, int chunk, int& e_out, int& r0,
                                           int& rows, int* s_tile) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int base = 0, found = -1;
    for (int e0 = 0; e0 < E && found < 0; e0 += 32) {
      const int e = e0 + lane;
      const int cnt = e < E ? offs[e + 1] - offs[e] : 0;
      const int nch = (cnt + kDgTok - 1) / kDgTok;
      int inc = nch;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, inc, o);
        if (lane >= o) inc += v;
      }
      const int excl = base + inc - nch;
      const bool mine = e < E && chunk >= excl && chunk < excl + nch;
      const uint32_t b = __ballot_sync(kFull, mine);
      if (b) {
        const int src = __ffs(b) - 1;
        const int ee = __shfl_sync(kFull, e, src), ex = __shfl_sync(kFull, excl, src);
        found = ee;
        if (lane == 0) {
          const int start = offs[ee] + (chunk - ex) * kDgTok;
          s_tile[0] = ee;
          s_tile[1] = start;
          s_tile[2] = min(kDgTok, offs[ee + 1] - start);
        }
      }
      base += __shfl_sync(kFull, inc, 31);
    }
    if (lane == 0 && found < 0) s_tile[0] = -1;
  }
  __syncthreads();
  e_out = s_tile[0];
  r0 = s_tile[1];
  rows = s_tile[2];
  return e_out >= 0;
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
               "{%0, %1, %2, %3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float e2m1_f32(uint32_t nib) {
  return __uint_as_float(((nib & 8u) << 28) | ((nib & 7u) << 22)) * 0x1p126f;
}

__device__ __forceinline__ float e8m0_f32(uint32_t s) {
  return __uint_as_float(s == 0u ? 0x00400000u : (s == 255u ? 0x7FC00000u : (s << 23)));
}


// out[r, n] = sum_m act[r, m] * W[e][m, n] for one (64 routed rows) x (128
// columns) tile, then the mode's epilogue.  256 threads: warp (wt, wn) owns
// rows 16wt..16wt+15 and columns 64wn..64wn+63.  The stored rows go by in
// slabs of 64; the next slab's codes, scales and activation rows are loaded
// into registers while the current one is multiplied, and the decoded tiles
// are double-buffered in shared memory (one barrier per slab).
template <int FMT, int MODE>
__global__ void __launch_bounds__(256, 3) dgrad_kernel(const DgParams p) {
  extern __shared__ __align__(16) uint8_t dg_smem[];
  uint16_t (*sW)[kDgK][kPadW] = reinterpret_cast<uint16_t (*)[kDgK][kPadW]>(dg_smem);                 // [2][m][n]
  uint16_t (*sA)[kDgTok][kPad] = reinterpret_cast<uint16_t (*)[kDgTok][kPad]>(dg_smem + 2 * kDgK * kPadW * 2);
  __shared__ float s_lut[16];
  __shared__ int s_tile[3];
  if (FMT == E4B_NF4 && threadIdx.x < 16) s_lut[threadIdx.x] = p.lut[threadIdx.x];
  pdl_wait();
  pdl_launch_dependents();
  int e, r0, rows;
  if (!dgrad_tile(p.expert_offsets, p.E, blockIdx.y, e, r0, rows, s_tile)) return;
  const int n0 = blockIdx.x * kDgCols;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wt = warp & 3, wn = warp >> 2;
  const int g = lane >> 2, c = lane & 3;
  // loader: stored row lm = tid / 4, 32 columns (16 code bytes) at 32 * ls; those columns
  // lie in one quantisation block and are either all inside the stack or all past its end
  const int lm = tid >> 2, ls = tid & 3;
  const bool col_ok = n0 + 32 * ls < p.N;
  const int64_t row_bytes = p.N / 2;
  const uint8_t* cbase = p.codes + (static_cast<int64_t>(e) * p.M + lm) * row_bytes + n0 / 2 + 16 * ls;
  const int64_t ebase = (static_cast<int64_t>(e) * p.M + lm) * p.N + n0 + 32 * ls;    // element index at m0 = 0
  // activation rows: routed row lr = tid / 4 (clamped into the tile), 16 stored rows at 16 * ls
  const int lr = min(tid >> 2, rows - 1);
  const uint16_t* abase = p.act + static_cast<int64_t>(r0 + lr) * p.M + 16 * ls;
  uint4 qn = make_uint4(0u, 0u, 0u, 0u), an0, an1;
  float sn = 0.0f;
  auto load = [&](int m0) {
    if (col_ok) {
      qn = __ldg(reinterpret_cast<const uint4*>(cbase + static_cast<int64_t>(m0) * row_bytes));
      const int64_t el = ebase + static_cast<int64_t>(m0) * p.N;
      sn = FMT == E4B_NF4 ? __ldg(static_cast<const float*>(p.scales) + el / 64)
                          : e8m0_f32(__ldg(static_cast<const uint8_t*>(p.scales) + el / 32));
    }
    an0 = __ldg(reinterpret_cast<const uint4*>(abase + m0));
    an1 = __ldg(reinterpret_cast<const uint4*>(abase + m0) + 1);
  };
  auto store = [&](int buf) {          // decode the registers' slab into buffer buf
    const uint32_t wd[4] = {qn.x, qn.y, qn.z, qn.w};
    uint32_t w[16];
#pragma unroll
    for (int b = 0; b < 16; ++b) {
      const uint32_t by = (wd[b >> 2] >> (8 * (b & 3))) & 0xFFu;
      if (FMT == E4B_NF4)        // element 2b in the high nibble; one rounding of level * absmax
        w[b] = pack_bf16x2(s_lut[by >> 4] * sn, s_lut[by & 15u] * sn);
      else                       // element 2b in the low nibble; exact
        w[b] = pack_bf16x2(e2m1_f32(by & 15u) * sn, e2m1_f32(by >> 4) * sn);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint4*>(&sW[buf][lm][32 * ls + 8 * i]) = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2],
                                                                             w[4 * i + 3]);
    *reinterpret_cast<uint4*>(&sA[buf][tid >> 2][16 * ls]) = an0;
    *reinterpret_cast<uint4*>(&sA[buf][tid >> 2][16 * ls + 8]) = an1;
  };
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;
  const int nslab = p.M / kDgK;
  load(0);
  store(0);
  __syncthreads();
  for (int s = 0; s < nslab; ++s) {
    const int buf = s & 1;
    if (s + 1 < nslab) load((s + 1) * kDgK);
#pragma unroll
    for (int kk = 0; kk < kDgK / 16; ++kk) {
      uint32_t af[4];
      ldsm_x4(af, &sA[buf][16 * wt + (lane & 15)][16 * kk + 8 * (lane >> 4)]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t b[4];
        ldsm_x4_t(b, &sW[buf][16 * kk + (lane & 15)][64 * wn + 16 * q + 8 * (lane >> 4)]);
        mma16816(acc[2 * q], af, b[0], b[1]);
        mma16816(acc[2 * q + 1], af, b[2], b[3]);
      }
    }
    if (s + 1 < nslab) store(buf ^ 1);
    __syncthreads();
  }

  // epilogue: acc[nt][h * 2 + i] is row 16wt + g + 8h, column 64wn + 8nt + 2c + i of the tile;
  // a thread's columns come in adjacent pairs (i = 0, 1; N is even), moved as one word
  if constexpr (MODE == 0) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int tr = 16 * wt + g + 8 * h;
        const int n = n0 + 64 * wn + 8 * nt + 2 * c;
        if (tr >= rows || n >= p.N) continue;
        const int64_t gi = (r0 + tr) * 2 * p.I + n;
        const float2 gg = *reinterpret_cast<const float2*>(p.G + gi);
        const float2 gu = *reinterpret_cast<const float2*>(p.G + gi + p.I);
        float dg0, du0, dg1, du1;
        act_grads(p.ep, gg.x, gu.x, dg0, du0);
        act_grads(p.ep, gg.y, gu.y, dg1, du1);
        const float v0 = acc[nt][2 * h], v1 = acc[nt][2 * h + 1];
        *reinterpret_cast<uint32_t*>(p.dG + gi) = pack_bf16x2(v0 * dg0, v1 * dg1);
        *reinterpret_cast<uint32_t*>(p.dG + gi + p.I) = pack_bf16x2(v0 * du0, v1 * du1);
      }
    }
  } else {
    // the LoRA term dxa_r A_e^T: the tile's dxa rows (fp32 [64][16]) and A_e rows of
    // its columns (bf16 [128][16]) are staged in the now idle tile buffers
    const int rk = p.lora_rank;
    float* s_dxa = reinterpret_cast<float*>(dg_smem);
    uint16_t* s_A = reinterpret_cast<uint16_t*>(dg_smem + kDgTok * 16 * 4);
    if (rk > 0) {
      for (int i = tid; i < kDgTok * 16; i += 256) {
        const int rr = i >> 4, j = i & 15;
        s_dxa[i] = (rr < rows && j < rk) ? p.dxa[static_cast<int64_t>(r0 + rr) * 16 + j] : 0.0f;
      }
      for (int i = tid; i < kDgCols * 16; i += 256) {
        const int cc = i >> 4, j = i & 15;
        const int n = n0 + cc;
        s_A[i] = (n < p.N && j < rk) ? p.lora_A[(static_cast<int64_t>(e) * p.N + n) * rk + j] : uint16_t(0);
      }
      __syncthreads();
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int tr = 16 * wt + g + 8 * h;
      if (tr >= rows) continue;
      float dr[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) dr[j] = rk > 0 ? s_dxa[tr * 16 + j] : 0.0f;
      const int64_t r = r0 + tr;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int cc = 64 * wn + 8 * nt + 2 * c + i;
          const int n = n0 + cc;
          if (n >= p.N) continue;
          float o = acc[nt][2 * h + i];
          if (rk > 0) {
            const uint4 a0 = *reinterpret_cast<const uint4*>(s_A + cc * 16);
            const uint4 a1 = *reinterpret_cast<const uint4*>(s_A + cc * 16 + 8);
            const uint32_t aw[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (j >= rk) break;
              o = fmaf(dr[j], bf16_to_f32((aw[j >> 1] >> (16 * (j & 1))) & 0xFFFFu), o);
            }
          }
          p.dX[r * p.N + n] = o;
        }
      }
    }
  }
}

// dxa[r, j] = s * sum_n dG[r, n] B_e[j, n], one warp per routed row (j < rank;
// fp32 [R, 16]).  The block's 8 rows are consecutive in expert order: B_e of its
// first row is staged in shared memory (rows of another expert read global memory).
__global__ void __launch_bounds__(256) lora_dxa_kernel(const uint16_t* __restrict__ dG, const uint16_t* __restrict__ B,
                                                       const int32_t* __restrict__ sorted_slot,
                                                       const int32_t* __restrict__ topk_ids, int R, int I2, int rank,
                                                       float scale, float* __restrict__ dxa, int stage_b) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint16_t s_B[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 8;
  int e_cached = -1;
  if (stage_b) {
    e_cached = topk_ids[sorted_slot[r0 < R ? r0 : R - 1]];
    const uint4* gb = reinterpret_cast<const uint4*>(B + static_cast<int64_t>(e_cached) * rank * I2);
    uint4* sb = reinterpret_cast<uint4*>(s_B);
    for (int i = threadIdx.x; i < rank * I2 / 8; i += blockDim.x) sb[i] = __ldg(gb + i);
    __syncthreads();
  }
  const int64_t r = r0 + warp;
  if (r >= R) return;
  const int e = topk_ids[sorted_slot[r]];
  const uint16_t* Be = e == e_cached ? s_B : B + static_cast<int64_t>(e) * rank * I2;
  const uint4* gr = reinterpret_cast<const uint4*>(dG + r * I2);
  float acc[kMaxLoraRank];
#pragma unroll
  for (int j = 0; j < kMaxLoraRank; ++j) acc[j] = 0.0f;
  for (int v = lane; v < I2 / 8; v += 32) {           // eight columns per lane and step
    const uint4 d = __ldg(gr + v);
    const uint32_t dw[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
    for (int j = 0; j < kMaxLoraRank; ++j) {
      if (j < rank) {
        const uint4 b = *reinterpret_cast<const uint4*>(Be + static_cast<int64_t>(j) * I2 + 8 * v);
        const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
          acc[j] = fmaf(bf16_to_f32(dw[q] & 0xFFFFu), bf16_to_f32(bw[q] & 0xFFFFu),
                        fmaf(bf16_to_f32(dw[q] >> 16), bf16_to_f32(bw[q] >> 16), acc[j]));
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kMaxLoraRank; ++j) {
    float v = acc[j];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kFull, v, off);
    if (lane == j) dxa[r * 16 + j] = j < rank ? scale * v : 0.0f;
  }
}

// dB[e, j, n] = sum over e's rows of xa[r, j] dG[r, n] (blockIdx.z = 0) and
// dA[e, h, j] = sum over e's rows of x_sorted[r, h] dxa[r, j] (blockIdx.z = 1);
// one thread per output column, rows walked in order (deterministic).
__global__ void __launch_bounds__(256) lora_grads_kernel(const uint16_t* __restrict__ xa, const uint16_t* __restrict__ dG,
                                                         const uint16_t* __restrict__ x_sorted,
                                                         const float* __restrict__ dxa,
                                                         const int32_t* __restrict__ expert_offsets, int H, int I2,
                                                         int rank, float* __restrict__ dA, float* __restrict__ dB) {
  pdl_wait();
  pdl_launch_dependents();
  const int e = blockIdx.y;
  const bool db = blockIdx.z == 0;
  const int ncols = db ? I2 : H;
  const int col = blockIdx.x * blockDim.x + threadIdx.x;
  const int lo = expert_offsets[e], hi = expert_offsets[e + 1];
  __shared__ float s_f[32][kMaxLoraRank];                // per-row factors of 32 rows at a time
  float acc[kMaxLoraRank];
#pragma unroll
  for (int j = 0; j < kMaxLoraRank; ++j) acc[j] = 0.0f;
  for (int r0 = lo; r0 < hi; r0 += 32) {
    const int nr = min(32, hi - r0);
    __syncthreads();
    for (int i = threadIdx.x; i < 32 * kMaxLoraRank; i += blockDim.x) {
      const int rr = i / kMaxLoraRank, j = i % kMaxLoraRank;
      float v = 0.0f;
      if (rr < nr && j < rank)
        v = db ? bf16_to_f32(xa[static_cast<int64_t>(r0 + rr) * 64 + j]) : dxa[static_cast<int64_t>(r0 + rr) * 16 + j];
      s_f[rr][j] = v;
    }
    __syncthreads();
    if (col < ncols) {
      for (int rr = 0; rr < nr; ++rr) {
        const int64_t r = r0 + rr;
        const float v = db ? bf16_to_f32(dG[r * I2 + col]) : bf16_to_f32(x_sorted[r * H + col]);
#pragma unroll
        for (int j = 0; j < kMaxLoraRank; ++j) acc[j] = fmaf(s_f[rr][j], v, acc[j]);
      }
    }
  }
  if (col >= ncols) return;
#pragma unroll
  for (int j = 0; j < kMaxLoraRank; ++j) {
    if (j >= rank) break;
    if (db) dB[(static_cast<int64_t>(e) * rank + j) * I2 + col] = acc[j];
    else dA[(static_cast<int64_t>(e) * H + col) * rank + j] = acc[j];
  }
}

// dx[t, h] = sum_j dX[slot_pos(t, j), h], j ascending (fp32).
__global__ void __launch_bounds__(256) dx_combine_kernel(const float* __restrict__ dX,
                                                         const int32_t* __restrict__ slot_pos, int k, int H,
                                                         float* __restrict__ dx) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t t = blockIdx.x;
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  if (c >= H / 4) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const float4 v = reinterpret_cast<const float4*>(dX + static_cast<int64_t>(slot_pos[t * k + j]) * H)[c];
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  reinterpret_cast<float4*>(dx + t * H)[c] = acc;
}

template <int FMT, int MODE>
cudaError_t launch_dgrad_typed(const DgParams& prm, dim3 grid, cudaStream_t s) {
  static cudaError_t attr = cudaFuncSetAttribute(dgrad_kernel<FMT, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kDgSmem);
  if (attr != cudaSuccess) return attr;
  return launch_pdl(dgrad_kernel<FMT, MODE>, grid, dim3(256), kDgSmem, s, prm);
}

template <int MODE>
cudaError_t launch_dgrad_mode(int32_t fmt, const DgParams& prm, int R, cudaStream_t s) {
  const dim3 grid((prm.N + kDgCols - 1) / kDgCols, (R + kDgTok - 1) / kDgTok + prm.E);
  return fmt == E4B_NF4 ? launch_dgrad_typed<E4B_NF4, MODE>(prm, grid, s)
                        : launch_dgrad_typed<E4B_MXFP4, MODE>(prm, grid, s);
}

}  // namespace

e4b_status launch_moe_backward(const BackwardLaunch& b, cudaStream_t s) {
  const int R = b.T * b.k;
  const int I2 = 2 * b.I;
  if (b.T == 0) {
    if (b.lora_rank > 0) {   // no routed rows: the factor gradients are zero
      if (cudaMemsetAsync(b.dA, 0, sizeof(float) * b.E * b.H * b.lora_rank, s) != cudaSuccess ||
          cudaMemsetAsync(b.dB, 0, sizeof(float) * b.E * b.lora_rank * I2, s) != cudaSuccess)
        return E4B_ERR_CUDA;
    }
    return E4B_OK;
  }
  if (launch_pdl(bwd_gate_kernel, dim3(b.T), dim3(256), 0, s, b.dout, static_cast<const float*>(b.y), b.topk_w,
                 b.topk_ids, b.slot_pos, b.logits, b.E, b.k, b.H, b.gating, b.dY, b.dlogits) != cudaSuccess)
    return E4B_ERR_CUDA;
  DgParams p = {};
  p.E = b.E;
  p.I = b.I;
  p.expert_offsets = b.expert_offsets;
  p.ep = b.ep;
  const Nf4Table& tab = nf4_table();
  for (int i = 0; i < 16; ++i) p.lut[i] = tab.level[i];
  // dh = dY W_dn[e] over the down stack's H stored rows, then dG in the epilogue
  p.M = b.H;
  p.N = b.I;
  p.codes = b.dn_codes;
  p.scales = b.dn_scales;
  p.act = b.dY;
  p.G = b.G;
  p.dG = b.dG;
  if (launch_dgrad_mode<0>(b.fmt, p, R, s) != cudaSuccess) return E4B_ERR_CUDA;
  if (b.lora_rank > 0) {
    constexpr size_t kStageMax = 200 * 1024;          // B_e in shared memory up to this size
    size_t smem = static_cast<size_t>(b.lora_rank) * I2 * 2;
    if (smem > kStageMax) smem = 0;
    if (smem > 48 * 1024) {
      static cudaError_t attr = cudaFuncSetAttribute(lora_dxa_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     static_cast<int>(kStageMax));
      if (attr != cudaSuccess) return E4B_ERR_CUDA;
    }
    if (launch_pdl(lora_dxa_kernel, dim3((R + 7) / 8), dim3(256), smem, s, static_cast<const uint16_t*>(b.dG),
                   b.lora_B, b.sorted_slot, b.topk_ids, R, I2, b.lora_rank, b.lora_scale, b.dxa,
                   smem > 0 ? 1 : 0) != cudaSuccess)
      return E4B_ERR_CUDA;
  }
  // dX = dG W_gu[e] (+ dxa A_e^T) over the gate_up stack's 2I stored rows
  p.M = I2;
  p.N = b.H;
  p.codes = b.gu_codes;
  p.scales = b.gu_scales;
  p.act = b.dG;
  p.dX = b.dX;
  p.dxa = b.dxa;
  p.lora_A = b.lora_A;
  p.lora_rank = b.lora_rank;
  if (launch_dgrad_mode<1>(b.fmt, p, R, s) != cudaSuccess) return E4B_ERR_CUDA;
  if (launch_pdl(dx_combine_kernel, dim3(b.T, (b.H / 4 + 255) / 256), dim3(256), 0, s,
                 static_cast<const float*>(b.dX), b.slot_pos, b.k, b.H, b.dx) != cudaSuccess)
    return E4B_ERR_CUDA;
  if (b.lora_rank > 0) {
    const int maxc = I2 > b.H ? I2 : b.H;
    if (launch_pdl(lora_grads_kernel, dim3((maxc + 255) / 256, b.E, 2), dim3(256), 0, s, b.xa,
                   static_cast<const uint16_t*>(b.dG), b.x_sorted, static_cast<const float*>(b.dxa),
                   b.expert_offsets, b.H, I2, b.lora_rank, b.dA, b.dB) != cudaSuccess)
      return E4B_ERR_CUDA;
  }
  return E4B_OK;
}

}  // namespace e4b
