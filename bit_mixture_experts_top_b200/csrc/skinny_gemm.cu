// Grouped 4-bit GEMMs for decode-sized batches: few routed rows per expert.
//
// Same contraction as grouped_gemm.cu ("MoE Training & Inference Guides",
// grouped-nf4-gemm table: packed 4-bit expert stacks, codes decoded on chip,
// fp32 accumulation, one launch over all experts; "experts4bit-qlora" limits
// list: the stock epilogue act(gate)*up; "experts4bit-qlora" index table:
// ExpertsLoRA's per-expert low-rank delta before the activation), organised
// for the case where each expert sees only a handful of tokens and streaming
// the packed weights from HBM is the whole cost.
//
// Why a second kernel: with <= 8 tokens per expert a 128-row tcgen05 tile
// spends one UMMA (a fixed issue cost, whatever N is) per 1 KB of packed codes
// and hands every dequantised stage from the converting warps to the single
// MMA thread through a barrier.  Here the decoded weights never leave
// registers: consumer warps read the packed codes from shared memory, decode
// them through a byte table straight into the A fragments of warp-level bf16
// MMAs (m16n8k16, the 8 tokens of a chunk as N) and accumulate in registers.
//
// Work unit: (chunk of <= 8 tokens of one expert, 128 weight rows), full K.
// chunk_off[E+1] is the router's prefix of ceil(count_e / 8).
//  * mode 0 (gate_up): rows are gate columns 64nb..64nb+63 and the matching up
//    columns I+64nb..; MMA tile t pairs gate rows 8t..8t+7 with up rows
//    64+8t..64+8t+7, so one thread holds gate and up of the same (token,
//    column) and applies the biases and the activation (SwiGLU, or the
//    gpt-oss clamped GLU) in registers;
//  * mode 1 (down): output rows 128nb..128nb+127; tile t = rows 16t..16t+15.
//
// Warp roles (one CTA per SM, persistent):
//  * warp 8, lane 0, the producer: takes units from a global counter (dynamic,
//    so every CTA finishes within one unit of the others), copies each unit's
//    scale rows to a shared buffer one unit ahead (2 buffers; a TMA box with the hardware
//    swizzle when a scale row is 32, 64 or 128 bytes, else one bulk copy per
//    contiguous run) and issues the 256-K stages: 128 rows x 128 code bytes
//    (128-byte swizzle) and the chunk's 8 activation rows x 256 K;
//  * warps 0-7, consumers: warp (wr, wk) owns MMA tiles 4wr..4wr+3 (64 rows)
//    and the 64-K block wk of every stage, so the activation fragments it
//    loads serve 64 rows (shared-memory bandwidth is the scarce resource:
//    per 16 KB stage the byte table takes 512 wavefronts, codes 128, TMA
//    writes 160, activations 64, scales 64).  At the end of a unit the four
//    K-partials of each tile are summed through shared memory and warp
//    (wr, wk) finishes tile 4wr+wk (LoRA step, SwiGLU or the fp32 store).
//
// Fragment/byte mapping.  Lane (g = lane / 4, c = lane % 4) takes, per 64-K
// block, code bytes [8c, 8c+8) of fragment rows g and g+8 of a tile (fragment
// row g is tile row rho(g) = 2(g mod 4) + g/4, a bank-spreading permutation).  MMA i (0..3) of
// the block uses byte 2i (elements 16c+4i, +1) as the low K pair and byte
// 2i+1 (elements 16c+4i+2, +3) as the high K pair of the A fragment; the B
// fragment takes the activations with the same K permutation, so the dot
// product is unchanged.
//
// Scales.  NF4: the byte table holds the bf16-rounded codebook levels and the
// fp32 absmax multiplies each block's fp32 partial sum, so the weights are
// never rounded after scaling.  MXFP4: exact bf16 e2m1 pairs times the bf16
// power-of-two scale (exact).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "e4b_device.cuh"
#include "e4b_internal.h"

namespace e4b {
namespace {

constexpr int SK_CONSUMERS = 8;
constexpr int SK_PRODUCER = 8;                   // warp index
constexpr int SK_THREADS = 9 * 32;
constexpr int SK_TPW = 4;                        // MMA tiles per consumer warp
constexpr int SK_SBUF = 2;                       // per-unit scale buffers
constexpr int SK_ROWS = 128;                     // weight rows per unit
constexpr int SK_KST = 256;                      // K per stage
constexpr int SK_CODE_BYTES = SK_ROWS * SK_KST / 2;          // 16 KB
// a chunk is TG token groups of 8 (MMA N = 8): its activation rows take
// 4 KB per group and stage; every decoded A fragment feeds TG MMAs
__host__ __device__ constexpr int sk_stage_bytes(int tg) { return SK_CODE_BYTES + tg * 8 * SK_KST * 2; }
constexpr int SK_MAX_STAGES = 8;
// byte table: entry b holds one copy per lane at 256*b + 4*lane (the upper
// 128 bytes of each entry are unused), so a single byte permute of the code
// word and the lane offset forms the address
constexpr int SK_LUT_BYTES = 256 * 256;
constexpr int SK_RED_BYTES = SK_CONSUMERS * SK_TPW * 4 * 32 * 4;  // K-partials of a unit
constexpr int SK_TAB_BYTES = 2 * (kMaxExperts + 1) * 4;
constexpr int SK_SMEM_LIMIT = 232448;

struct SkParams {
  int32_t E, N, K, I;
  int32_t n_blocks;       // units per chunk
  int32_t lora_rank;
  int32_t stages;         // ring depth
  int32_t srow;           // scale bytes per weight row (K/64 fp32 or K/32 e8m0)
  int32_t scale_bytes;    // bytes of one scale buffer (128 rows, 1024-aligned)
  int32_t scale_tma;      // 1: scale rows by TMA box (swizzled), 0: bulk copies of the raw runs
  uint32_t scale_swz;     // XOR mask of the scale buffer's swizzle (0 = none)
  const uint8_t* codes;   // [E, N, K/2]
  const void* scales;     // NF4 fp32 [E, N, K/64]; MXFP4 u8 [E, N, K/32]
  const uint16_t* xa;     // [R, 64] bf16 (mode 0 with LoRA)
  const uint16_t* lora_B; // [E, r, 2I]
  const int32_t* expert_offsets;
  const int32_t* chunk_off;
  void* out;              // mode 0: bf16 h [R, I]; mode 1: fp32 y [R, N]
  int32_t* status;
  uint32_t* counters;     // [2]: next unit, CTAs done (zero between launches)
  uint64_t wait_limit_ns;
  Epilogue ep;            // biases and activation
  float* g_out;           // mode 0: pre-activation outputs G [R, 2I] fp32, or null
  uint32_t level2[8];     // NF4: bf16 levels, two per word (level 2w low half)
};

struct SkLayout {
  int lut, ring, scale, red, tab, bar, total;
};

__host__ __device__ inline SkLayout sk_layout(int stages, int scale_bytes, int tg) {
  SkLayout L;
  L.lut = 0;
  L.ring = SK_LUT_BYTES;                                     // 1024-aligned (swizzle atoms)
  L.scale = L.ring + stages * sk_stage_bytes(tg);
  L.red = L.scale + SK_SBUF * scale_bytes;
  L.tab = L.red + SK_RED_BYTES;
  L.bar = L.tab + SK_TAB_BYTES;
  L.total = L.bar + 256 + 1024;   // barriers, unit ids, NF4 levels; base-alignment slack
  return L;
}

// d = A * B (accumulator starts at zero)
__device__ __forceinline__ void mma_bf16_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %10, %10, %10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Contiguous global -> shared copy (16-byte aligned, size a multiple of 16),
// completion counted in bytes on `bar`.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Table value of code byte `byte` of `word`: __byte_perm places that byte at
// bits 8..15 and this lane's offset (lane_off = 4 * lane) at bits 0..7.
__device__ __forceinline__ uint32_t lut_at(const uint8_t* lut, uint32_t lane_off, uint32_t word, int byte) {
  return *reinterpret_cast<const uint32_t*>(lut + __byte_perm(word, lane_off, 0x7704u | (byte << 4)));
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

// Warp-uniform bounded wait: every lane polls the barrier (so every lane
// acquires what the completed phase publishes) and the warp leaves together,
// either when all lanes saw the phase or when lane 0 found the abort flag or
// the time limit.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w, int32_t where) {
  const uint32_t a = smem_u32(bar);
  if (__all_sync(0xFFFFFFFFu, mbar_try_wait(a, parity))) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (__all_sync(0xFFFFFFFFu, mbar_try_wait(a, parity))) return true;
    if ((it & 15) == 0) {
      int bad = 0;
      if ((threadIdx.x & 31) == 0) {
        if (*w.abort_flag) {
          bad = 1;
        } else if (globaltimer_ns() - t0 > w.limit_ns) {
          *w.abort_flag = 1;
          record_error(w.status, E4B_ERR_TIMEOUT, where);
          bad = 1;
        }
      }
      if (__shfl_sync(0xFFFFFFFFu, bad, 0)) return false;
    }
  }
}

struct Unit {
  int e, t0, m, nb;
};

// Unit u -> (expert, first token, tokens, weight block), from the CTA's copies
// of chunk_off[E+1] and expert_offsets[E+1].
template <int TOK>
__device__ __forceinline__ Unit decode_unit(int u, int n_blocks, int E, const int32_t* s_chunk,
                                            const int32_t* s_off) {
  const int chunk = u / n_blocks;
  Unit r;
  r.nb = u - chunk * n_blocks;
  int lo = 0, hi = E;                   // last e with chunk_off[e] <= chunk
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_chunk[mid] <= chunk) lo = mid; else hi = mid;
  }
  r.e = lo;
  r.t0 = s_off[lo] + TOK * (chunk - s_chunk[lo]);
  const int rem = s_off[lo + 1] - r.t0;
  r.m = rem < TOK ? rem : TOK;
  return r;
}

// Stack rows of the two 64-row halves of a unit.
template <int MODE>
__device__ __forceinline__ void unit_rows(const SkParams& p, const Unit& u, int& row_a, int& row_b) {
  row_a = MODE == 0 ? 64 * u.nb : SK_ROWS * u.nb;
  row_b = MODE == 0 ? p.I + 64 * u.nb : row_a + 64;
}

__device__ __forceinline__ uint32_t lora_pair(const uint16_t* col, int64_t rstride, int j0, int rank) {
  const uint32_t lo = j0 < rank ? __ldg(col + j0 * rstride) : 0u;
  const uint32_t hi = j0 + 1 < rank ? __ldg(col + (j0 + 1) * rstride) : 0u;
  return lo | (hi << 16);
}

template <int FMT, int MODE, int TG>
__global__ void __launch_bounds__(SK_THREADS, 1)
    skinny_gemm_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
                       const __grid_constant__ CUtensorMap tm_scales, const __grid_constant__ SkParams p) {
  extern __shared__ uint8_t sk_dyn[];
  // 1024-aligned base (swizzle atoms), kept as an offset from the shared array so
  // that every access below compiles to a shared-memory load
  uint8_t* smem = sk_dyn + ((1024u - (smem_u32(sk_dyn) & 1023u)) & 1023u);
  constexpr int TOK = 8 * TG;                         // tokens per chunk
  constexpr int STAGE_BYTES = sk_stage_bytes(TG);
  const SkLayout L = sk_layout(p.stages, p.scale_bytes, TG);
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + L.lut);
  const uint8_t* lut_b = smem + L.lut;
  uint8_t* ring = smem + L.ring;
  uint8_t* sbuf = smem + L.scale;
  float* red = reinterpret_cast<float*>(smem + L.red);
  int32_t* s_chunk = reinterpret_cast<int32_t*>(smem + L.tab);
  int32_t* s_off = s_chunk + (kMaxExperts + 1);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar);
  uint64_t* empty = full + SK_MAX_STAGES;
  uint64_t* sfull = empty + SK_MAX_STAGES;      // [SK_SBUF]
  uint64_t* sempty = sfull + SK_SBUF;           // [SK_SBUF]
  uint64_t* rfull = sempty + SK_SBUF;
  uint64_t* rempty = rfull + 1;
  int32_t* s_unit = reinterpret_cast<int32_t*>(rempty + 1);   // [SK_SBUF]
  int32_t* s_abort = s_unit + SK_SBUF;
  uint16_t* s_level = reinterpret_cast<uint16_t*>(smem + L.bar + 224);   // [16], after barriers and unit ids

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], SK_CONSUMERS);
    }
    for (int b = 0; b < SK_SBUF; ++b) {
      mbar_init(&sfull[b], 1);
      mbar_init(&sempty[b], SK_CONSUMERS);
    }
    mbar_init(rfull, SK_CONSUMERS);
    mbar_init(rempty, (SK_CONSUMERS / 4) * SK_TPW);   // the warps that finish tiles
    *s_abort = 0;
    fence_mbar_init();
  }
  if (FMT == E4B_NF4 && threadIdx.x < 16)
    s_level[threadIdx.x] = static_cast<uint16_t>(p.level2[threadIdx.x >> 1] >> (16 * (threadIdx.x & 1)));
  if (warp == SK_PRODUCER && lane == 0) {
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_x);
    if (p.scale_tma) tma_prefetch_desc(&tm_scales);
  }
  __syncthreads();
  // Byte -> bf16 pair table, one copy per lane so every lane reads its own bank.
  for (int i = threadIdx.x; i < 256 * 32; i += SK_THREADS) {
    const uint32_t b = static_cast<uint32_t>(i) >> 5;
    const uint32_t at = b * 64 + (static_cast<uint32_t>(i) & 31u);
    uint32_t v;
    if (FMT == E4B_NF4) {   // element 2j in the high nibble -> low half
      v = static_cast<uint32_t>(s_level[b >> 4]) | (static_cast<uint32_t>(s_level[b & 15u]) << 16);
    } else {                // element 2j in the low nibble -> low half
      __nv_bfloat162 t = __floats2bfloat162_rn(e2m1_value(b & 15u), e2m1_value(b >> 4));
      v = *reinterpret_cast<uint32_t*>(&t);
    }
    lut[at] = v;
  }
  // everything above depends on nothing an earlier kernel writes; the unit
  // tables, activations and counters below do
  pdl_wait();
  pdl_launch_dependents();
  for (int i = threadIdx.x; i <= p.E; i += SK_THREADS) {
    s_chunk[i] = __ldg(p.chunk_off + i);
    s_off[i] = __ldg(p.expert_offsets + i);
  }
  __syncthreads();

  const WaitCtx wctx{s_abort, p.status, p.wait_limit_ns};
  const int total = s_chunk[p.E] * p.n_blocks;
  const int KB = p.K >> 6;
  const int nst = (p.K + SK_KST - 1) / SK_KST;

  if (warp == SK_PRODUCER) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // Unit blockIdx.x first (no atomic ahead of the first copy), then units
      // gridDim.x + 0, 1, ... in the order CTAs ask for them.  A fetched index is
      // compared with `total` only where it is used, so the atomic's round trip
      // overlaps the copies issued before that point; an index >= total ends the CTA.
      auto fetch = [&]() { return static_cast<int>(gridDim.x + atomicAdd(&p.counters[0], 1u)); };
      uint32_t armed = 0, par = 0, sarmed = 0, spar = 0;
      bool ok = true;
      // unit k's scale rows go to buffer k % SK_SBUF, one unit ahead of its stages
      auto issue_scales = [&](int k, int u) -> bool {
        const int sb = k % SK_SBUF;
        const uint32_t sph = static_cast<uint32_t>(k / SK_SBUF) & 1u;
        if (!mbar_wait(&sempty[sb], sph ^ 1u, wctx, 711)) return false;
        if (u >= total) {
          s_unit[sb] = -1;
          mbar_arrive(&sfull[sb]);
          return true;
        }
        const Unit un = decode_unit<TOK>(u, p.n_blocks, p.E, s_chunk, s_off);
        int row_a, row_b;
        unit_rows<MODE>(p, un, row_a, row_b);
        const int ya = un.e * p.N + row_a, yb = un.e * p.N + row_b;
        s_unit[sb] = u;
        uint8_t* sdst = sbuf + sb * p.scale_bytes;
        if (p.scale_tma) {
          mbar_arrive_expect_tx(&sfull[sb], 2 * 64 * p.srow);
          tma_load_2d(sdst, &tm_scales, &sfull[sb], 0, ya);
          tma_load_2d(sdst + 64 * p.srow, &tm_scales, &sfull[sb], 0, yb);
        } else {
          const int na = max(0, min(64, p.N - row_a)), nb = max(0, min(64, p.N - row_b));
          mbar_arrive_expect_tx(&sfull[sb], (na + nb) * p.srow);
          const uint8_t* sc = static_cast<const uint8_t*>(p.scales);
          if (na) bulk_copy_g2s(sdst, sc + static_cast<int64_t>(ya) * p.srow, na * p.srow, &sfull[sb]);
          if (nb) bulk_copy_g2s(sdst + 64 * p.srow, sc + static_cast<int64_t>(yb) * p.srow, nb * p.srow, &sfull[sb]);
        }
        sarmed |= 1u << sb;
        spar = (spar & ~(1u << sb)) | (sph << sb);
        return true;
      };
      const int q0 = static_cast<int>(blockIdx.x);
      int q1 = q0 < total ? fetch() : total, q2 = total;
      int slot = 0;
      uint32_t ph = 0;
      int u = q0;
      ok = issue_scales(0, u);
      for (int k = 0; ok && u < total; ++k) {
        const Unit un = decode_unit<TOK>(u, p.n_blocks, p.E, s_chunk, s_off);
        int row_a, row_b;
        unit_rows<MODE>(p, un, row_a, row_b);
        const int ya = un.e * p.N + row_a;
        for (int st = 0; st < nst; ++st) {
          if (!mbar_wait(&empty[slot], ph ^ 1u, wctx, 712)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[slot], STAGE_BYTES);
          uint8_t* dst = ring + slot * STAGE_BYTES;
          // Two copies per stage (the copy engine's throughput per SM, about 23 bytes per
          // clock plus a fixed cost per copy instruction, bounds the stream): the codes of
          // both 64-row halves of the unit (gate and up rows through the view
          // [expert x half][row][K], or 128 consecutive rows), and the chunk's activation
          // rows of the stage's four 64-K blocks (view [block][row][64 K]).
          if (MODE == 0)
            tma_load_3d(dst, &tm_codes, &full[slot], SK_KST / 2 * st, 64 * un.nb, 2 * un.e);
          else
            tma_load_2d(dst, &tm_codes, &full[slot], SK_KST / 2 * st, ya);
          tma_load_3d(dst + SK_CODE_BYTES, &tm_x, &full[slot], 0, un.t0, 4 * st);
          armed |= 1u << slot;
          par = (par & ~(1u << slot)) | (ph << slot);
          if (++slot == p.stages) { slot = 0; ph ^= 1u; }
        }
        if (!ok) break;
        if (k == 0) q2 = fetch();     // the second request goes out once the first unit's copies are issued
        u = q1;
        q1 = q2;
        q2 = u < total ? fetch() : total;
        ok = issue_scales(k + 1, u);
      }
      // the last CTA through resets the counters for the next launch
      __threadfence();
      if (atomicAdd(&p.counters[1], 1u) == gridDim.x - 1) {
        atomicExch(&p.counters[0], 0u);
        atomicExch(&p.counters[1], 0u);
      }
      if (!ok) {   // let every issued copy land before the CTA's shared memory is released
        for (int s = 0; s < p.stages; ++s)
          if (armed & (1u << s)) mbar_drain(&full[s], (par >> s) & 1u, p.wait_limit_ns);
        for (int b = 0; b < SK_SBUF; ++b)
          if (sarmed & (1u << b)) mbar_drain(&sfull[b], (spar >> b) & 1u, p.wait_limit_ns);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int wr = warp >> 2, wk = warp & 3;   // tiles SK_TPW*wr.., 64-K block wk of each stage
    const int g = lane >> 2, c = lane & 3;
    // fragment row g reads stage row 8t + rho (rho even for g < 4, odd for g >= 4),
    // so the eight 16-byte chunks a half-warp loads sit in different banks
    const int rho = 2 * (g & 3) + (g >> 2);
    const uint32_t lane_off = 4u * lane;
    constexpr int esz = FMT == E4B_NF4 ? 4 : 2;
    // per-warp constant offsets: code bytes [8c, 8c+8) of block wk in rows r0, r1
    // of each tile (128-byte swizzle), this lane's activation chunks, scale rows
    int co[SK_TPW][2], so[SK_TPW][2];
#pragma unroll
    for (int j = 0; j < SK_TPW; ++j) {
      const int t = SK_TPW * wr + j;
      const int r[2] = {MODE == 0 ? 8 * t + rho : 16 * t + rho, MODE == 0 ? 64 + 8 * t + rho : 16 * t + 8 + rho};
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        co[j][rr] = 128 * r[rr] + 16 * ((2 * wk + (c >> 1)) ^ rho) + 8 * (c & 1);
        so[j][rr] = r[rr] * p.srow;
      }
    }
    // activation box wk holds the chunk's TOK rows x 64 K; row 8tg+g of it feeds token group tg
    const int xo0 = SK_CODE_BYTES + 1024 * TG * wk + 128 * g + 16 * ((2 * c) ^ g);
    const int xo1 = SK_CODE_BYTES + 1024 * TG * wk + 128 * g + 16 * ((2 * c + 1) ^ g);
    // the scale buffer's swizzle flips bits 4..6 by bits 7..9 of the row offset,
    // which are the same for every row this lane reads
    const uint32_t xg = (static_cast<uint32_t>(so[0][0]) >> 3) & p.scale_swz;
    int sb = 0, slot = 0;
    uint32_t sph = 0, ph = 0, rph = 0;
    bool ok = true;
    for (;;) {
      if (!warp_wait(&sfull[sb], sph, wctx, 721)) break;
      const int u = s_unit[sb];
      if (u < 0) break;
      const Unit un = decode_unit<TOK>(u, p.n_blocks, p.E, s_chunk, s_off);
      const uint8_t* scb = sbuf + sb * p.scale_bytes;
      float acc[SK_TPW][TG][4];
#pragma unroll
      for (int j = 0; j < SK_TPW; ++j)
#pragma unroll
        for (int q = 0; q < TG; ++q) acc[j][q][0] = acc[j][q][1] = acc[j][q][2] = acc[j][q][3] = 0.f;
      for (int st = 0; st < nst; ++st) {
        if (!warp_wait(&full[slot], ph, wctx, 722)) { ok = false; break; }
        const int blk = 4 * st + wk;
        if (blk < KB) {
          const uint8_t* cs = ring + slot * STAGE_BYTES;
          const uint8_t* sc = scb + ((static_cast<uint32_t>(blk * esz)) ^ xg);
          uint32_t xw[TG][8];
#pragma unroll
          for (int q = 0; q < TG; ++q) {
            const uint4 xa = *reinterpret_cast<const uint4*>(cs + xo0 + 1024 * q);
            const uint4 xb = *reinterpret_cast<const uint4*>(cs + xo1 + 1024 * q);
            xw[q][0] = xa.x; xw[q][1] = xa.y; xw[q][2] = xa.z; xw[q][3] = xa.w;
            xw[q][4] = xb.x; xw[q][5] = xb.y; xw[q][6] = xb.z; xw[q][7] = xb.w;
          }
#pragma unroll
          for (int j = 0; j < SK_TPW; ++j) {
            const uint2 q0 = *reinterpret_cast<const uint2*>(cs + co[j][0]);
            const uint2 q1 = *reinterpret_cast<const uint2*>(cs + co[j][1]);
            const uint32_t s0 = FMT == E4B_NF4 ? *reinterpret_cast<const uint32_t*>(sc + so[j][0])
                                               : *reinterpret_cast<const uint16_t*>(sc + so[j][0]);
            const uint32_t s1 = FMT == E4B_NF4 ? *reinterpret_cast<const uint32_t*>(sc + so[j][1])
                                               : *reinterpret_cast<const uint16_t*>(sc + so[j][1]);
            if (FMT == E4B_NF4) {
              float bs[TG][4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const uint32_t w0 = i < 2 ? q0.x : q0.y, w1 = i < 2 ? q1.x : q1.y;
                const int by = 2 * (i & 1);
                const uint32_t a[4] = {lut_at(lut_b, lane_off, w0, by), lut_at(lut_b, lane_off, w1, by),
                                       lut_at(lut_b, lane_off, w0, by + 1), lut_at(lut_b, lane_off, w1, by + 1)};
#pragma unroll
                for (int q = 0; q < TG; ++q) {
                  if (i == 0) mma_bf16_z(bs[q], a, xw[q][0], xw[q][1]);
                  else mma_bf16(bs[q], a, xw[q][2 * i], xw[q][2 * i + 1]);
                }
              }
              const float f0 = __uint_as_float(s0), f1 = __uint_as_float(s1);
#pragma unroll
              for (int q = 0; q < TG; ++q) {
                acc[j][q][0] = fmaf(f0, bs[q][0], acc[j][q][0]);
                acc[j][q][1] = fmaf(f0, bs[q][1], acc[j][q][1]);
                acc[j][q][2] = fmaf(f1, bs[q][2], acc[j][q][2]);
                acc[j][q][3] = fmaf(f1, bs[q][3], acc[j][q][3]);
              }
            } else {
              const uint32_t e0 = e8m0_bf16x2((s0 >> (8 * (c >> 1))) & 0xFFu);
              const uint32_t e1 = e8m0_bf16x2((s1 >> (8 * (c >> 1))) & 0xFFu);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const uint32_t w0 = i < 2 ? q0.x : q0.y, w1 = i < 2 ? q1.x : q1.y;
                const int by = 2 * (i & 1);
                const uint32_t a[4] = {bf16x2_mul(lut_at(lut_b, lane_off, w0, by), e0),
                                       bf16x2_mul(lut_at(lut_b, lane_off, w1, by), e1),
                                       bf16x2_mul(lut_at(lut_b, lane_off, w0, by + 1), e0),
                                       bf16x2_mul(lut_at(lut_b, lane_off, w1, by + 1), e1)};
#pragma unroll
                for (int q = 0; q < TG; ++q) mma_bf16(acc[j][q], a, xw[q][2 * i], xw[q][2 * i + 1]);
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        if (++slot == p.stages) { slot = 0; ph ^= 1u; }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sempty[sb]);
      // sum the four K-partials of each tile, one token group per round; warp
      // (wr, wk < SK_TPW) finishes tile SK_TPW*wr+wk
      const int t = SK_TPW * wr + wk;
      const bool fin = wk < SK_TPW;
      uint32_t la[4] = {0u, 0u, 0u, 0u};             // LoRA step A fragment of the finished tile
      if (MODE == 0 && fin && p.lora_rank > 0) {
        const int col = 64 * un.nb + 8 * t + rho;
        const int64_t rs = 2 * static_cast<int64_t>(p.I);
        const uint16_t* Be = p.lora_B + static_cast<int64_t>(un.e) * p.lora_rank * rs;
        la[0] = lora_pair(Be + col, rs, 2 * c, p.lora_rank);
        la[1] = lora_pair(Be + p.I + col, rs, 2 * c, p.lora_rank);
        la[2] = lora_pair(Be + col, rs, 2 * c + 8, p.lora_rank);
        la[3] = lora_pair(Be + p.I + col, rs, 2 * c + 8, p.lora_rank);
      }
      // biases of the two output rows this lane finishes (gate/up pair, or rows n, n + 8)
      float b_lo = 0.f, b_hi = 0.f;
      if (fin && p.ep.bias) {
        if (MODE == 0) {
          const float* be = p.ep.bias + static_cast<int64_t>(un.e) * 2 * p.I + 64 * un.nb + 8 * t + rho;
          b_lo = __ldg(be);
          b_hi = __ldg(be + p.I);
        } else {
          const int n = SK_ROWS * un.nb + 16 * t + rho;
          const float* be = p.ep.bias + static_cast<int64_t>(un.e) * p.N + n;
          if (n < p.N) b_lo = __ldg(be);
          if (n + 8 < p.N) b_hi = __ldg(be + 8);
        }
      }
#pragma unroll
      for (int q = 0; q < TG; ++q) {
        if (!warp_wait(rempty, rph ^ 1u, wctx, 723)) { ok = false; break; }
#pragma unroll
        for (int j = 0; j < SK_TPW; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i) red[((warp * SK_TPW + j) * 4 + i) * 32 + lane] = acc[j][q][i];
        __syncwarp();
        if (lane == 0) mbar_arrive(rfull);
        if (fin) {
          if (!warp_wait(rfull, rph, wctx, 724)) { ok = false; break; }
          float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int i = 0; i < 4; ++i) v[i] += red[(((4 * wr + k) * SK_TPW + wk) * 4 + i) * 32 + lane];
          __syncwarp();
          if (lane == 0) mbar_arrive(rempty);
          const int tok0 = 8 * q;                    // first token of this group in the chunk
          if (MODE == 0) {
            const int col = 64 * un.nb + 8 * t + rho;
            if (p.lora_rank > 0) {
              // LoRA step: A = B_e^T (rows n, K = rank padded to 16), B = xa (scale folded in)
              uint32_t b0 = 0u, b1 = 0u;
              if (tok0 + g < un.m) {
                const uint32_t* xr =
                    reinterpret_cast<const uint32_t*>(p.xa + static_cast<int64_t>(un.t0 + tok0 + g) * 64);
                b0 = __ldg(xr + c);
                b1 = __ldg(xr + 4 + c);
              }
              mma_bf16(v, la, b0, b1);
            }
            __nv_bfloat16* h = static_cast<__nv_bfloat16*>(p.out);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              if (tok0 + 2 * c + r < un.m) {
                const int64_t row = un.t0 + tok0 + 2 * c + r;
                const float gate = v[r] + b_lo, up = v[2 + r] + b_hi;
                h[row * p.I + col] = __float2bfloat16_rn(expert_act(p.ep, gate, up));
                if (p.g_out) {   // kept for the backward
                  p.g_out[row * 2 * p.I + col] = gate;
                  p.g_out[row * 2 * p.I + p.I + col] = up;
                }
              }
            }
          } else {
            const int n = SK_ROWS * un.nb + 16 * t + rho;
            float* y = static_cast<float*>(p.out);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              if (tok0 + 2 * c + r < un.m) {
                float* yr = y + static_cast<int64_t>(un.t0 + tok0 + 2 * c + r) * p.N + n;
                if (n < p.N) yr[0] = v[r] + b_lo;
                if (n + 8 < p.N) yr[8] = v[2 + r] + b_hi;
              }
            }
          }
        }
        rph ^= 1u;
      }
      if (!ok) break;
      if (++sb == SK_SBUF) { sb = 0; sph ^= 1u; }
    }
  }
}

template <int FMT, int MODE, int TG>
e4b_status launch_typed(const CUtensorMap& tc, const CUtensorMap& tx, const CUtensorMap& ts, const SkParams& prm,
                        int smem, cudaStream_t s) {
  auto kern = skinny_gemm_kernel<FMT, MODE, TG>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SK_SMEM_LIMIT);
  });
  if (attr_err != cudaSuccess) return E4B_ERR_CUDA;
  return launch_pdl(kern, dim3(device_sm_count()), dim3(SK_THREADS), smem, s, tc, tx, ts, prm) == cudaSuccess
             ? E4B_OK
             : E4B_ERR_CUDA;
}

int scale_row_bytes(int32_t K, int32_t fmt) { return fmt == E4B_NF4 ? K / 16 : K / 32; }
int scale_buffer_bytes(int32_t K, int32_t fmt) { return (SK_ROWS * scale_row_bytes(K, fmt) + 1023) & ~1023; }

}  // namespace

bool skinny_gemm_supported(int32_t K, int32_t fmt) {
  return sk_layout(3, scale_buffer_bytes(K, fmt), 4).total <= SK_SMEM_LIMIT;
}

template <int TG>
e4b_status launch_tg(int32_t fmt, int32_t mode, const CUtensorMap& tc, const CUtensorMap& tx, const CUtensorMap& ts,
                     const SkParams& prm, int smem, cudaStream_t s) {
  if (fmt == E4B_NF4)
    return mode == 0 ? launch_typed<E4B_NF4, 0, TG>(tc, tx, ts, prm, smem, s)
                     : launch_typed<E4B_NF4, 1, TG>(tc, tx, ts, prm, smem, s);
  return mode == 0 ? launch_typed<E4B_MXFP4, 0, TG>(tc, tx, ts, prm, smem, s)
                   : launch_typed<E4B_MXFP4, 1, TG>(tc, tx, ts, prm, smem, s);
}

e4b_status launch_skinny_gemm(const GroupedGemmLaunch& g, cudaStream_t s) {
  if (g.R == 0) return E4B_OK;
  const int tok = g.tokens_per_tile;                  // 8, 16 or 32 tokens per chunk
  if (g.K % 64 != 0 || (g.mode == 0 && g.I % 64 != 0) || !skinny_gemm_supported(g.K, g.fmt) ||
      (tok != 8 && tok != 16 && tok != 32))
    return E4B_ERR_UNSUPPORTED;
  const int tg = tok / 8;
  SkParams prm;
  prm.E = g.E;
  prm.N = g.N;
  prm.K = g.K;
  prm.I = g.I;
  prm.n_blocks = g.mode == 0 ? g.I / 64 : (g.N + SK_ROWS - 1) / SK_ROWS;
  prm.lora_rank = g.mode == 0 ? g.lora_rank : 0;
  prm.srow = scale_row_bytes(g.K, g.fmt);
  prm.scale_bytes = scale_buffer_bytes(g.K, g.fmt);
  // scale rows of 32, 64 or 128 bytes go through a swizzled TMA box, so the
  // eight rows a fragment reads fall in different banks
  prm.scale_tma = (prm.srow == 32 || prm.srow == 64 || prm.srow == 128) ? 1 : 0;
  prm.scale_swz = prm.scale_tma ? static_cast<uint32_t>(((prm.srow >> 4) - 1) << 4) : 0u;
  int stages = SK_MAX_STAGES;
  while (stages > 3 && sk_layout(stages, prm.scale_bytes, tg).total > SK_SMEM_LIMIT) --stages;
  prm.stages = stages;
  prm.codes = g.codes;
  prm.scales = g.scales;
  prm.xa = g.xa;
  prm.lora_B = g.lora_B;
  prm.expert_offsets = g.expert_offsets;
  prm.chunk_off = g.chunk_off;
  prm.out = g.out;
  prm.status = g.status;
  prm.ep = Epilogue{g.bias, g.mode == 0 ? g.glu : E4B_ACT_SWIGLU, g.glu_alpha, g.glu_limit, g.glu_beta};
  prm.g_out = g.mode == 0 ? g.g_out : nullptr;
  prm.counters = reinterpret_cast<uint32_t*>(g.status) + 8 + 2 * g.mode;
  prm.wait_limit_ns = g.wait_limit_ns;
  const Nf4Table& t = nf4_table();
  for (int w = 0; w < 8; ++w) {
    const __nv_bfloat16 lo = __float2bfloat16_rn(t.level[2 * w]);
    const __nv_bfloat16 hi = __float2bfloat16_rn(t.level[2 * w + 1]);
    prm.level2[w] = static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&lo)) |
                    (static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&hi)) << 16);
  }
  CUtensorMap tc, tx, ts;
  const uint64_t code_rows = static_cast<uint64_t>(g.E) * g.N;
  const bool coded = g.mode == 0
                         // gate_up: [E x {gate, up}] x I rows x K/2 bytes; one box holds both 64-row halves
                         ? encode_tma_3d(&tc, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.codes, g.K / 2, g.I,
                                         2 * static_cast<uint64_t>(g.E), g.K / 2,
                                         static_cast<uint64_t>(g.I) * (g.K / 2), SK_KST / 2, 64, 2,
                                         CU_TENSOR_MAP_SWIZZLE_128B)
                         : encode_tma_2d(&tc, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.codes, g.K / 2, code_rows, g.K / 2,
                                         SK_KST / 2, SK_ROWS, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!coded) return E4B_ERR_CUDA;
  // activations [R, K] viewed as [K / 64 blocks][R rows][64 K]: one box = the stage's four blocks
  if (!encode_tma_3d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.act, 64, g.R, g.K / 64, static_cast<uint64_t>(g.K) * 2,
                     128, 64, tok, 4, CU_TENSOR_MAP_SWIZZLE_128B))
    return E4B_ERR_CUDA;
  if (prm.scale_tma) {
    const CUtensorMapSwizzle sw = prm.srow == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : prm.srow == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                   : CU_TENSOR_MAP_SWIZZLE_32B;
    if (!encode_tma_2d(&ts, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.scales, prm.srow, code_rows, prm.srow, prm.srow, 64, sw))
      return E4B_ERR_CUDA;
  } else {
    ts = tc;
  }
  const int smem = sk_layout(stages, prm.scale_bytes, tg).total;
  if (tg == 1) return launch_tg<1>(g.fmt, g.mode, tc, tx, ts, prm, smem, s);
  if (tg == 2) return launch_tg<2>(g.fmt, g.mode, tc, tx, ts, prm, smem, s);
  return launch_tg<4>(g.fmt, g.mode, tc, tx, ts, prm, smem, s);
}

}  // namespace e4b
