// Standalone format kernels: MXFP4 -> bf16 decode and the NF4 quantiser.
//
// Both are pure HBM streams.  Each warp owns a contiguous span of the flat
// tensor, every lane moves 16 bytes per store (128-bit, fully coalesced), and
// the grid is a multiple of the SM count with a grid-stride loop.
//
// MXFP4 decode ("How do I train and serve MoE models released in MXFP4 ...?",
// "Why it happens" and "Two fidelity paths"): an E2M1 nibble
// s.e1.e0.m is turned into an fp32 value exactly by placing its three
// magnitude bits at fp32 bits 24..22 (which reads as e2m1 * 2^-126, subnormal
// encoding included) and multiplying by 2^126; the E8M0 scale is the fp32
// 2^(s-127) (s = 0 is the fp32 subnormal 2^-127, s = 255 NaN).  The product is
// exact in fp32 and in bf16 unless it overflows, so one round-to-nearest
// conversion reproduces the definition bit for bit.
#include <cmath>
#include <cstring>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "e4b_device.cuh"
#include "e4b_internal.h"

namespace e4b {
namespace {

__device__ __forceinline__ float e2m1_to_f32(uint32_t nib) {
  const uint32_t bits = ((nib & 8u) << 28) | ((nib & 7u) << 22);
  return __uint_as_float(bits) * 0x1p126f;
}

__device__ __forceinline__ float e8m0_to_f32(uint32_t s) {
  const uint32_t bits = (s == 0u) ? 0x00400000u : ((s == 255u) ? 0x7FC00000u : (s << 23));
  return __uint_as_float(bits);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // .x = lo (low half), .y = hi
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint4 decode_unit8(uint32_t w, uint32_t s) {
  if (s == 255u) return make_uint4(0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u);
  const float sc = e8m0_to_f32(s);
  uint32_t r[4];
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const uint32_t byte = (w >> (8 * b)) & 0xFFu;
    r[b] = pack_bf16x2(e2m1_to_f32(byte & 0xFu) * sc, e2m1_to_f32(byte >> 4) * sc);
  }
  return make_uint4(r[0], r[1], r[2], r[3]);
}

// 8 elements = 4 code bytes -> 16 output bytes.  Unit u covers elements [8u, 8u+8);
// each thread takes two units per trip (u and u + stride) so two loads are in flight.
__global__ void __launch_bounds__(256) dequant_mxfp4_kernel(const uint32_t* __restrict__ codes,
                                                              const uint8_t* __restrict__ scales, int64_t units,
                                                              uint4* __restrict__ out) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < units; u += 2 * stride) {
    const int64_t u2 = u + stride;
    const bool two = u2 < units;
    const uint32_t w = __ldcs(codes + u);
    const uint32_t s = __ldg(scales + (u >> 2));
    const uint32_t w2 = two ? __ldcs(codes + u2) : 0u;
    const uint32_t s2 = two ? __ldg(scales + (u2 >> 2)) : 0u;
    __stcs(out + u, decode_unit8(w, s));
    if (two) __stcs(out + u2, decode_unit8(w2, s2));
  }
}

// Exact decision table for the NF4 code of a quotient y in [-1, 1]: the code
// is #{i : y > m_i} over the 15 midpoints.  |y| in [2^-5, 1] falls in one of 161
// buckets given by its exponent and the top five mantissa bits (exact float
// boundaries [lo, hi)); each bucket holds at most one midpoint (buckets are at
// most 1/64 wide, midpoints at least 0.08 apart), so per bucket and sign
// code = base + (y > mid): positive y counts the midpoints below lo and tests
// the one in [lo, hi); negative y counts those at or below -hi and tests the
// one in (-hi, -lo].  |y| < 2^-5 lies between the two midpoints next to zero,
// code 7, which is also what bucket 0 gives for either sign (no midpoint in it,
// seven below it), so small quotients are clamped into bucket 0.  Entry 2j + s
// holds bucket j for sign s.  The host builds and checks the table
// (nf4_bucket_table).
constexpr int kNf4Buckets = 161;
constexpr int kNf4BucketBias = 122 << 5;              // exponent of 2^-5, five mantissa bits
struct Nf4Buckets {
  uint2 e[2 * kNf4Buckets];                           // {midpoint bits (or +inf), base}
};

// One half-warp per 64-block: each lane holds 4 consecutive fp32 (16 bytes),
// the half-warp reduces |x| to absmax, each lane emits 4 codes (2 bytes).
// Branch-free: every element takes the same instruction sequence.
__device__ __forceinline__ void quantize_quad(float4 v, int64_t q, uint32_t half_mask,
                                              const uint2* __restrict__ s_tab, uint16_t* __restrict__ codes,
                                              float* __restrict__ absmax) {
  float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(half_mask, a, off));
  if ((threadIdx.x & 15) == 0) absmax[q >> 4] = a;
  // y = fl32(x / a) by Markstein's FMA correction (P. Markstein, "Computation of
  // elementary functions on the IBM RISC System/6000 processor", IBM J. Res. Dev.
  // 34(1), 1990): with r = RN(1/a), q = RN(x*r), the residual x - a*q is exact in
  // one FMA and RN(q + residual*r) is the correctly rounded quotient unless it
  // underflows (an underflowing quotient lies far below the smallest decision
  // midpoint, so the code is the same either way).  A block with a tiny absmax
  // is first scaled by 2^96 (exact, and it changes no quotient) so that 1/a and
  // the residuals stay normal; an all-zero block takes r = 0, so all its
  // quotients are 0 and its codes 7.
  float xv[4] = {v.x, v.y, v.z, v.w};
  if (a < 0x1p-60f) {                      // uniform across the half-warp
    a *= 0x1p96f;
#pragma unroll
    for (int i = 0; i < 4; ++i) xv[i] *= 0x1p96f;
  }
  const float r = a == 0.0f ? 0.0f : __frcp_rn(a);
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float qq = xv[i] * r;
    const float y = fmaf(fmaf(-a, qq, xv[i]), r, qq);
    const uint32_t bits = __float_as_uint(y);
    // bucket of |y|; the upper clamp only keeps non-finite input inside the table
    const int j = min(max(static_cast<int>((bits << 1) >> 19) - kNf4BucketBias, 0), kNf4Buckets - 1);
    const uint2 t = s_tab[__funnelshift_l(bits, static_cast<uint32_t>(j), 1)];   // 2j + sign
    c[i] = t.y + (y > __uint_as_float(t.x) ? 1u : 0u);
  }
  codes[q] = static_cast<uint16_t>(((c[2] * 16u + c[3]) << 8) | (c[0] * 16u + c[1]));
}

// Each thread takes two quads per trip (q and q + stride): two loads in flight.
__global__ void __launch_bounds__(256) quantize_nf4_kernel(const float4* __restrict__ x, int64_t quads,
                                                             uint16_t* __restrict__ codes,
                                                             float* __restrict__ absmax, const Nf4Buckets tab) {
  __shared__ uint2 s_tab[2 * kNf4Buckets];
  for (int i = threadIdx.x; i < 2 * kNf4Buckets; i += blockDim.x) s_tab[i] = tab.e[i];
  __syncthreads();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const uint32_t half_mask = 0xFFFFu << (threadIdx.x & 16u);   // this half-warp only
  // quads and the stride are multiples of 16, so every half-warp stays inside one
  // block and the trip count and the second-quad test are uniform across it.
  for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < quads; q += 2 * stride) {
    const int64_t q2 = q + stride;
    const float4 v = __ldcs(x + q);
    const float4 v2 = q2 < quads ? __ldcs(x + q2) : make_float4(0.f, 0.f, 0.f, 0.f);
    quantize_quad(v, q, half_mask, s_tab, codes, absmax);
    if (q2 < quads) quantize_quad(v2, q2, half_mask, s_tab, codes, absmax);
  }
}

int grid_for(int64_t work_items, int threads, int per_sm) {
  const int64_t need = (work_items + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * per_sm;
  return static_cast<int>(need < cap ? (need > 0 ? need : 1) : cap);
}

}  // namespace

// gpt-oss gate_up de-interleave ("How do I train and serve MoE models released
// in MXFP4 ...?", "Why it happens": interleaved gate/up rows; "Which project
// solves it": the gpt-oss module de-interleaves them): row n of expert e in
// the output is input row 2n (gate, n < I) or 2(n - I) + 1 (up).  A plain row
// gather, moved in the widest word the row size and the pointers allow.
template <typename W>
__global__ void __launch_bounds__(256) deinterleave_rows_kernel(const W* __restrict__ in, W* __restrict__ out,
                                                                int64_t rows, int32_t I, int64_t words_per_row) {
  const int64_t total = rows * words_per_row;
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = u / words_per_row, w = u - row * words_per_row;
    const int64_t e = row / (2 * I), n = row - e * 2 * I;
    const int64_t src = e * 2 * I + (n < I ? 2 * n : 2 * (n - I) + 1);
    out[u] = __ldg(in + src * words_per_row + w);
  }
}

cudaError_t launch_deinterleave_rows(const void* in, void* out, int32_t E, int32_t I, int64_t row_bytes,
                                     cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(E) * 2 * I;
  const uintptr_t a = reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(out);
  if (rows == 0 || row_bytes == 0) return cudaSuccess;
  if (row_bytes % 16 == 0 && a % 16 == 0) {
    const int64_t wpr = row_bytes / 16;
    deinterleave_rows_kernel<uint4><<<grid_for(rows * wpr, 256, 8), 256, 0, s>>>(
        static_cast<const uint4*>(in), static_cast<uint4*>(out), rows, I, wpr);
  } else if (row_bytes % 4 == 0 && a % 4 == 0) {
    const int64_t wpr = row_bytes / 4;
    deinterleave_rows_kernel<uint32_t><<<grid_for(rows * wpr, 256, 8), 256, 0, s>>>(
        static_cast<const uint32_t*>(in), static_cast<uint32_t*>(out), rows, I, wpr);
  } else {
    deinterleave_rows_kernel<uint8_t><<<grid_for(rows * row_bytes, 256, 8), 256, 0, s>>>(
        static_cast<const uint8_t*>(in), static_cast<uint8_t*>(out), rows, I, row_bytes);
  }
  return cudaGetLastError();
}

// Double-quantised NF4 absmax ("experts4bit-qlora" limits list: bitsandbytes'
// nested form -- offset, 8-bit codes, one fp32 per 256 values -- expanded to
// fp32 just in time for one layer):
//   absmax[b] = fl32(fl32(table[code[b]] * absmax2[b / 256]) + offset),
// two explicit roundings (__fmul_rn / __fadd_rn, never contracted to an FMA).
// With expert_offsets, blocks of experts that no routed row touches are
// skipped: the GEMMs read only touched experts' absmax.  Four codes per thread
// (one 32-bit load, one 16-byte store) when the sizes and pointers allow.
__global__ void __launch_bounds__(256) expand_absmax_dq_kernel(const uint8_t* __restrict__ codes,
                                                               const float* __restrict__ absmax2,
                                                               const float* __restrict__ offset,
                                                               const float* __restrict__ table, int64_t n,
                                                               int64_t per_expert,
                                                               const int32_t* __restrict__ expert_offsets,
                                                               float* __restrict__ out, int vec4) {
  __shared__ float s_table[256];
  s_table[threadIdx.x] = __ldg(table + threadIdx.x);
  const float off = __ldg(offset);
  __syncthreads();
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t first = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (vec4) {
    for (int64_t q = first; q < n / 4; q += step) {
      const int64_t b = 4 * q;
      if (expert_offsets) {
        const int64_t e = b / per_expert;
        if (__ldg(expert_offsets + e + 1) == __ldg(expert_offsets + e)) continue;
      }
      const uint32_t c4 = __ldg(reinterpret_cast<const uint32_t*>(codes) + q);
      const float s2 = __ldg(absmax2 + b / 256);          // the four share a second-level block
      float4 v;
      v.x = __fadd_rn(__fmul_rn(s_table[c4 & 0xFFu], s2), off);
      v.y = __fadd_rn(__fmul_rn(s_table[(c4 >> 8) & 0xFFu], s2), off);
      v.z = __fadd_rn(__fmul_rn(s_table[(c4 >> 16) & 0xFFu], s2), off);
      v.w = __fadd_rn(__fmul_rn(s_table[c4 >> 24], s2), off);
      reinterpret_cast<float4*>(out)[q] = v;
    }
  } else {
    for (int64_t b = first; b < n; b += step) {
      if (expert_offsets) {
        const int64_t e = b / per_expert;
        if (__ldg(expert_offsets + e + 1) == __ldg(expert_offsets + e)) continue;
      }
      out[b] = __fadd_rn(__fmul_rn(s_table[__ldg(codes + b)], __ldg(absmax2 + b / 256)), off);
    }
  }
}

cudaError_t launch_expand_absmax_dq(const uint8_t* codes, const float* absmax2, const float* offset,
                                    const float* table, int64_t n, int64_t per_expert,
                                    const int32_t* expert_offsets, float* out, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  const bool vec4 = n % 4 == 0 && per_expert % 4 == 0 && reinterpret_cast<uintptr_t>(codes) % 4 == 0 &&
                    reinterpret_cast<uintptr_t>(out) % 16 == 0;
  const int64_t items = vec4 ? n / 4 : n;
  expand_absmax_dq_kernel<<<grid_for(items, 256, 8), 256, 0, s>>>(codes, absmax2, offset, table, n, per_expert,
                                                                  expert_offsets, out, vec4 ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_dequant_mxfp4(const uint8_t* codes, const uint8_t* scales, int64_t n, uint16_t* out,
                                 cudaStream_t s) {
  const int64_t units = n / 8;
  if (units == 0) return cudaSuccess;
  dequant_mxfp4_kernel<<<grid_for(units, 256, 8), 256, 0, s>>>(reinterpret_cast<const uint32_t*>(codes), scales,
                                                              units, reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

namespace {

// The bucket table of quantize_quad, from the fp32 midpoints; null if a premise fails
// (a bucket with two midpoints, a midpoint within 2^-5 of zero, or a bucket 0
// whose code is not 7 for either sign).
const Nf4Buckets* nf4_bucket_table() {
  static Nf4Buckets tab;
  static bool ok = [] {
    const float* m = nf4_table().mid;
    if (!(m[6] < -0x1p-5f && m[7] > 0x1p-5f)) return false;
    for (int j = 0; j < kNf4Buckets; ++j) {
      const float lo = std::ldexp(1.0f + static_cast<float>(j % 32) / 32.0f, j / 32 - 5);
      const float hi = lo + std::ldexp(1.0f / 32.0f, j / 32 - 5);
      uint32_t base_p = 0, base_n = 0, inpos = 0, inneg = 0;
      float mid_p = INFINITY, mid_n = INFINITY;
      for (int i = 0; i < 15; ++i) {
        if (m[i] < lo) ++base_p;
        if (m[i] >= lo && m[i] < hi) { mid_p = m[i]; ++inpos; }
        if (m[i] <= -hi) ++base_n;
        if (m[i] > -hi && m[i] <= -lo) { mid_n = m[i]; ++inneg; }
      }
      if (inpos > 1 || inneg > 1) return false;
      if (j == 0 && (base_p != 7 || base_n != 7 || inpos || inneg)) return false;
      uint32_t bp, bn;
      std::memcpy(&bp, &mid_p, 4);
      std::memcpy(&bn, &mid_n, 4);
      tab.e[2 * j] = make_uint2(bp, base_p);
      tab.e[2 * j + 1] = make_uint2(bn, base_n);
    }
    return true;
  }();
  return ok ? &tab : nullptr;
}

}  // namespace

cudaError_t launch_quantize_nf4(const float* x, int64_t n, uint8_t* codes, float* absmax, cudaStream_t s) {
  const int64_t quads = n / 4;
  if (quads == 0) return cudaSuccess;
  const Nf4Buckets* tab = nf4_bucket_table();
  if (!tab) return cudaErrorInvalidValue;
  quantize_nf4_kernel<<<grid_for(quads, 256, 8), 256, 0, s>>>(reinterpret_cast<const float4*>(x), quads,
                                                              reinterpret_cast<uint16_t*>(codes), absmax, *tab);
  return cudaGetLastError();
}

}  // namespace e4b
