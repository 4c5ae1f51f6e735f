// Grouped 4-bit expert GEMMs on sm_100a tensor cores (tcgen05 / TMEM).
//
// What it computes (solutions index, grouped-nf4-gemm table: the routed MoE
// expert GEMM straight on NF4 packed weights or on E2M1 blocks with E8M0
// scales, one launch over all experts, fp32 accumulation, no bf16 expert
// tensor; "experts4bit-qlora" limits list: the stock epilogue act(gate)*up;
// experts4bit-qlora table of the index: ExpertsLoRA's per-expert low-rank
// delta before the activation):
//
//   mode 0 (gate_up): G = X_e W_gu[e]^T (+ xa_e B_e) (+ b_gu[e]), h = act(G_gate, G_up) -> bf16 [R, I]
//   mode 1 (down)   : Y = h_e W_dn[e]^T (+ b_dn[e])                           -> fp32 [R, H]
//
// act is silu(gate) * up, or the gpt-oss clamped GLU with per-expert biases
// ("How do I train and serve MoE models released in MXFP4 (gpt-oss,
// DeepSeek-V4)?", "Why it happens"); see Epilogue in e4b_device.cuh.
//
// B200 design.  The weights are the UMMA M operand (128 rows per tile; in
// tensor memory for decode-sized tiles, in shared memory for prefill tiles)
// and the routed rows of one expert the N operand (tokens_per_tile = BN
// columns, in shared memory), so a decode batch with a handful of rows per
// expert still issues full-height MMAs, and one dequantised weight tile serves
// up to 256 rows in prefill.
// One persistent CTA per SM walks a tile list (expert, weight block, row
// chunk); consecutive tiles share a weight block so its bytes are read from
// HBM once and from L2 after.  Warp roles:
//   warp 0      TMA producer of packed codes (64-byte swizzled boxes) into a
//               raw ring; warms L2 with whole tiles (contiguous runs) ahead;
//   warp 1      TMA producer of activation tiles (128-byte swizzled) into the
//               B ring;
//   warp 2      TMEM owner and single-thread UMMA issuer (kind::f16, M=128,
//               N=BN, K=16, fp32 accumulators in TMEM, two buffers);
//   warps 3-10  dequant: 4-bit codes + per-block scale -> bf16 rows written
//               into tensor memory (tcgen05.st) or 128-byte-swizzled shared
//               memory, the UMMA A operand;
//   warps 11-14 epilogue: tcgen05.ld, activation and bf16 store (gate_up) or
//               bias and fp32 store (down).
// Every wait is bounded: on timeout the kernel records E4B_ERR_TIMEOUT, lets
// copies and MMAs in flight land, frees its TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "e4b_device.cuh"
#include "e4b_internal.h"

namespace e4b {
namespace {

constexpr int BM = 128;                      // weight rows per tile (UMMA M)
constexpr int ATOM_K = 64;                   // K per 128-byte swizzle row of bf16
constexpr int RAW_K = 128;                   // K per packed-code stage
constexpr int RAW_ROW_BYTES = RAW_K / 2;     // 64 bytes of codes per weight row
constexpr int RAW_STAGE_BYTES = BM * RAW_ROW_BYTES;
constexpr int LUT_BYTES = 32768;             // byte -> element-pair table, one copy per bank
constexpr int NUM_DQ_WARPS = 8;             // dequant warps that produce one A stage (4 lane quarters x 2)
constexpr int NUM_EPI_WARPS = 4;
constexpr int WARP_RAW = 0;                  // TMA producer of packed codes
constexpr int WARP_ACT = 1;                  // TMA producer of activation tiles
constexpr int WARP_MMA = 2;
constexpr int WARP_DQ0 = 3;
constexpr uint64_t kDrainNs = 50000000ull;   // error path: wait at most 50 ms per in-flight stage

// Two placements of the dequantised weight tile (the UMMA A operand):
//  * BN <= 192: A lives in tensor memory.  Columns [0, 2*BN) hold the two
//    fp32 accumulators, the rest a ring of A stages (BKS/2 columns each);
//    shared memory only carries the packed codes, the activation tiles and
//    the byte LUT.  Decode-sized tiles (BN <= 64) stage 128 K so each dequant
//    thread converts 64 elements per barrier round.
//  * BN = 256: A lives in shared memory (128-byte swizzled, K-major, 64 K per
//    stage), so the two 256-column accumulators can fill tensor memory.
template <int BN>
struct Cfg {
  static constexpr bool TMEM_A = BN != 256;
  static constexpr int BKS = BN <= 64 ? 128 : 64;
  static constexpr int ATOMS = BKS / ATOM_K;
  static constexpr int A_COLS = BKS / 2;                    // TMEM columns per A stage
  static constexpr int A_COL0 = 2 * BN > 256 ? 2 * BN : 256;   // first TMEM column of the A ring
  static constexpr int STAGES = TMEM_A ? (512 - A_COL0) / A_COLS : 3;
  static constexpr int A_STAGE_BYTES = TMEM_A ? 0 : BM * 128;   // shared-memory A (one atom)
  static constexpr int B_ATOM_BYTES = BN * 128;
  static constexpr int B_STAGE_BYTES = ATOMS * B_ATOM_BYTES;
  static constexpr int RAW_STAGES = BN <= 64 ? 12 : (TMEM_A ? 6 : 4);
  // 64-K stages (prefill tiles): two groups of 8 dequant warps take alternate
  // 128-K code stages, so each warp converts and synchronises half as often
  static constexpr int DQ_GROUPS = BKS == 64 ? 2 : 1;
  static constexpr int WARP_EPI0 = WARP_DQ0 + NUM_DQ_WARPS * DQ_GROUPS;
  static constexpr int THREADS = 32 * (WARP_EPI0 + NUM_EPI_WARPS);
  static constexpr int TMEM_COLS = 512;
  static constexpr int OFF_LUT = 0;
  static constexpr int OFF_A = OFF_LUT + LUT_BYTES;
  static constexpr int OFF_B = OFF_A + STAGES * A_STAGE_BYTES;
  static constexpr int OFF_RAW = OFF_B + STAGES * B_STAGE_BYTES;
  static constexpr int OFF_BAR = OFF_RAW + RAW_STAGES * RAW_STAGE_BYTES;
  static constexpr int NUM_BARS = 3 * STAGES + 2 * RAW_STAGES + 4;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_TAB = OFF_MISC + 16;              // chunk_off and expert_offsets, [E+1] each
  static constexpr int SMEM_BYTES = OFF_TAB + 2 * (kMaxExperts + 1) * 4 + 1024;   // + slack to align the base
  static_assert(TMEM_A ? 2 * BN <= A_COL0 : 2 * BN <= 512, "accumulators must fit in tensor memory");
  static_assert(B_ATOM_BYTES % 1024 == 0, "B atoms must keep 1024-byte alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct Params {
  int32_t E, N, K, I;
  int32_t n_blocks;       // weight blocks per expert (mode 0: I/64 gate+up pairs; mode 1: ceil(N/128))
  int32_t lora_rank;      // 0 = none (mode 0 only)
  const uint8_t* codes;   // packed stack [E, N, K/2] (for L2 warming)
  const void* scales;
  const uint16_t* lora_B; // [E, r, 2I]
  const int32_t* expert_offsets;
  const int32_t* chunk_off;
  void* out;
  int32_t* status;
  uint64_t wait_limit_ns;
  Epilogue ep;            // biases and activation
  float* g_out;           // mode 0: pre-activation outputs G [R, 2I] fp32, or null
  float lut[16];          // NF4 levels
};

struct Tile {
  int e, nb, row0, rows;
};

// Tile lookup from the CTA's shared copies of chunk_off[E+1] and
// expert_offsets[E+1] (tile order: expert, weight block, row chunk).
template <int BN>
__device__ __forceinline__ bool get_tile(const Params& p, const int32_t* s_chunk, const int32_t* s_off, int tile,
                                         int total, Tile& t) {
  if (tile >= total) return false;
  int lo = 0, hi = p.E;                 // last e with chunk_off[e] * n_blocks <= tile
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_chunk[mid] * p.n_blocks <= tile) lo = mid; else hi = mid;
  }
  const int c0 = s_chunk[lo];
  const int nch = s_chunk[lo + 1] - c0;
  const int local = tile - c0 * p.n_blocks;
  t.e = lo;
  t.nb = local / nch;
  const int chunk = local - t.nb * nch;
  t.row0 = s_off[lo] + chunk * BN;
  t.rows = min(BN, s_off[lo + 1] - t.row0);
  return true;
}

// Row of the weight stack behind A-tile row `prow` and its row in the raw code
// tile.  Mode 0 pairs gate and up rows: within each 32-row group (one epilogue
// warp's TMEM lanes), rows 0..15 are gate features and 16..31 the matching up
// features, and within each half row r < 8 is feature 2r and row r + 8 feature
// 2r + 1, so a 16x256b TMEM load hands every thread two adjacent features.
template <int MODE>
__device__ __forceinline__ void tile_row(const Params& p, int nb, int prow, int& wrow, int& raw_row) {
  if (MODE == 0) {
    const int g = prow >> 5, wi = prow & 31;
    const int fi = 2 * (wi & 7) + ((wi >> 3) & 1);
    const int f = 64 * nb + 16 * g + fi;
    raw_row = (wi < 16 ? 0 : 64) + 16 * g + fi;
    wrow = (wi < 16) ? f : p.I + f;
  } else {
    raw_row = prow;
    wrow = BM * nb + prow;
  }
}

__device__ __forceinline__ float e2m1_to_f32(uint32_t nib) {
  return __uint_as_float(((nib & 8u) << 28) | ((nib & 7u) << 22)) * 0x1p126f;
}

// bf16x2 of the E8M0 scale 2^(s-127) in both halves (s = 0: bf16 subnormal, 255: NaN).
__device__ __forceinline__ uint32_t e8m0_to_bf16x2(uint32_t s) {
  const uint32_t b = s == 0u ? 0x0040u : (s == 255u ? 0x7FC0u : (s << 7));
  return b | (b << 16);
}

// NF4: one code byte -> two bf16 (element 2j from the high nibble in the low
// half).  The LUT holds fp32 level pairs; the fp32 products round once.
__device__ __forceinline__ uint32_t nf4_pair(uint32_t addr, uint64_t a2) {
  uint32_t r;
  asm("{\n\t.reg .b64 t;\n\t.reg .f32 lo, hi;\n\t"
      "ld.shared.b64 t, [%1];\n\t"
      "mul.rn.f32x2 t, t, %2;\n\t"
      "mov.b64 {lo, hi}, t;\n\t"
      "cvt.rn.bf16x2.f32 %0, hi, lo;\n\t}"
      : "=r"(r)
      : "r"(addr), "l"(a2));
  return r;
}

// MXFP4: one code byte -> two bf16 (element 2j from the low nibble in the low
// half).  The LUT holds exact bf16 pairs; the power-of-two scale keeps them exact.
__device__ __forceinline__ uint32_t mx_pair(uint32_t addr, uint32_t s2) {
  uint32_t r;
  asm("{\n\t.reg .b32 t;\n\t"
      "ld.shared.b32 t, [%1];\n\t"
      "mul.rn.bf16x2 %0, t, %2;\n\t}"
      : "=r"(r)
      : "r"(addr), "r"(s2));
  return r;
}

// 16 code bytes (32 elements sharing one scale) -> 4 x 16 bytes of bf16.
// lut_l already includes this lane's table copy; scale is the fp32 absmax
// (NF4) or the bf16x2 E8M0 scale (MXFP4).
template <int FMT>
__device__ __forceinline__ void dequant32(const uint4 q, uint32_t lut_l, uint64_t a2, uint32_t s2, uint4 (&o)[4]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t r[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t addr = lut_l + (((w[i] >> (8 * b)) & 0xFFu) << 7);
      r[b] = FMT == E4B_NF4 ? nf4_pair(addr, a2) : mx_pair(addr, s2);
    }
    o[i] = make_uint4(r[0], r[1], r[2], r[3]);
  }
}

__device__ __forceinline__ uint64_t dup_f32(float a) {
  const uint64_t u = __float_as_uint(a);
  return u | (u << 32);
}

template <int BN, int FMT, int MODE>
__global__ void __launch_bounds__(Cfg<BN>::THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_act,
                        const __grid_constant__ CUtensorMap tm_xa, const Params p) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~uintptr_t(1023));
  uint8_t* sLut = smem + C::OFF_LUT;
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sB = smem + C::OFF_B;
  uint8_t* sRaw = smem + C::OFF_RAW;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* a_full = bars;
  uint64_t* b_full = a_full + C::STAGES;
  uint64_t* empty = b_full + C::STAGES;
  uint64_t* raw_full = empty + C::STAGES;
  uint64_t* raw_empty = raw_full + C::RAW_STAGES;
  uint64_t* acc_full = raw_empty + C::RAW_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int32_t* s_abort = reinterpret_cast<int32_t*>(smem + C::OFF_MISC + 8);
  int32_t* s_chunk = reinterpret_cast<int32_t*>(smem + C::OFF_TAB);
  int32_t* s_off = s_chunk + (kMaxExperts + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&a_full[s], NUM_DQ_WARPS);
      mbar_init(&b_full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < C::RAW_STAGES; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], NUM_DQ_WARPS);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], NUM_EPI_WARPS);
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  // Byte -> element-pair tables, replicated so that every lane of a warp reads
  // its own bank: NF4 fp32 pairs (16 copies of 8 bytes per byte value), MXFP4
  // bf16 pairs (32 copies of 4 bytes).
  if (FMT == E4B_NF4) {
    float2* lut = reinterpret_cast<float2*>(sLut);
    for (int i = threadIdx.x; i < 256 * 16; i += C::THREADS) {
      const int b = i >> 4;
      lut[i] = make_float2(p.lut[b >> 4], p.lut[b & 15]);
    }
  } else {
    uint32_t* lut = reinterpret_cast<uint32_t*>(sLut);
    for (int i = threadIdx.x; i < 256 * 32; i += C::THREADS) {
      const int b = i >> 5;
      __nv_bfloat162 v = __floats2bfloat162_rn(e2m1_to_f32(b & 15), e2m1_to_f32(b >> 4));
      lut[i] = *reinterpret_cast<uint32_t*>(&v);
    }
  }
  if (warp == WARP_RAW && lane == 0) {
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_act);
    if (MODE == 0 && p.lora_rank > 0) tma_prefetch_desc(&tm_xa);
  }
  // the set-up above depends on nothing an earlier kernel writes; the tile tables,
  // activations and tensor memory (held by an earlier grid until it ends) below do
  pdl_wait();
  pdl_launch_dependents();
  for (int i = threadIdx.x; i <= p.E; i += C::THREADS) {
    s_chunk[i] = __ldg(p.chunk_off + i);
    s_off[i] = __ldg(p.expert_offsets + i);
  }
  if (warp == WARP_MMA) {
    tmem_alloc(s_tmem, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;

  const WaitCtx wctx{s_abort, p.status, p.wait_limit_ns};
  const int total = s_chunk[p.E] * p.n_blocks;
  const bool lora = (MODE == 0) && p.lora_rank > 0;
  const int raw_steps = (p.K + RAW_K - 1) / RAW_K;
  const int mma_steps = (p.K + C::BKS - 1) / C::BKS;   // K stages per tile (before the LoRA step)
  const int nsteps = mma_steps + (lora ? 1 : 0);

  if (warp == WARP_RAW) {
    // ------------------------------------------------------------ packed-code producer
    if (lane == 0) {
      int rstage = 0;
      uint32_t rphase = 0, armed_r = 0, par_r = 0;   // per-stage "armed" bit and parity
      bool ok = true;
      // Each tile's packed codes are one (down) or two (gate_up) contiguous runs
      // of the stack, and so are its scale rows: warm L2 with whole runs, one
      // tile ahead, so HBM streams them sequentially and the per-stage boxes hit L2.
      auto warm_tile = [&](int tile_id) {
        Tile wt;
        if (!get_tile<BN>(p, s_chunk, s_off, tile_id, total, wt)) return;
        const int nrun = MODE == 0 ? 2 : 1;
        for (int run = 0; run < nrun; ++run) {
          const int row0 = MODE == 0 ? (run == 0 ? 64 * wt.nb : p.I + 64 * wt.nb) : BM * wt.nb;
          const int nrows = MODE == 0 ? 64 : min(BM, p.N - row0);
          const int64_t grow = static_cast<int64_t>(wt.e) * p.N + row0;
          bulk_prefetch_l2(p.codes + grow * (p.K / 2), static_cast<uint32_t>(nrows) * (p.K / 2));
          const int sbytes = FMT == E4B_NF4 ? p.K / 16 : p.K / 32;     // scale bytes per row
          const uint32_t sz = (static_cast<uint32_t>(nrows) * sbytes) & ~15u;
          const uint8_t* sp = reinterpret_cast<const uint8_t*>(p.scales) + grow * sbytes;
          const uint8_t* spa = reinterpret_cast<const uint8_t*>(reinterpret_cast<uintptr_t>(sp) & ~uintptr_t(15));
          if (sz) bulk_prefetch_l2(spa, sz);
        }
      };
      warm_tile(blockIdx.x);
      warm_tile(blockIdx.x + gridDim.x);
      Tile t;
      for (int tile = blockIdx.x; ok && get_tile<BN>(p, s_chunk, s_off, tile, total, t); tile += gridDim.x) {
        warm_tile(tile + 2 * gridDim.x);
        for (int r = 0; r < raw_steps; ++r) {
          if (!mbar_wait(&raw_empty[rstage], rphase ^ 1u, wctx, 101)) { ok = false; break; }
          mbar_arrive_expect_tx(&raw_full[rstage], RAW_STAGE_BYTES);
          uint8_t* dst = sRaw + rstage * RAW_STAGE_BYTES;
          const int x = r * RAW_ROW_BYTES;
          if (MODE == 0) {
            tma_load_2d(dst, &tm_codes, &raw_full[rstage], x, t.e * p.N + 64 * t.nb);
            tma_load_2d(dst + 64 * RAW_ROW_BYTES, &tm_codes, &raw_full[rstage], x, t.e * p.N + p.I + 64 * t.nb);
          } else {
            tma_load_2d(dst, &tm_codes, &raw_full[rstage], x, t.e * p.N + BM * t.nb);
          }
          armed_r |= 1u << rstage;
          par_r = (par_r & ~(1u << rstage)) | (rphase << rstage);
          if (++rstage == C::RAW_STAGES) { rstage = 0; rphase ^= 1u; }
        }
      }
      if (!ok) {   // let every issued copy land before the CTA's shared memory is released
        for (int s = 0; s < C::RAW_STAGES; ++s)
          if (armed_r & (1u << s)) mbar_drain(&raw_full[s], (par_r >> s) & 1u, kDrainNs);
      }
    }
  } else if (warp == WARP_ACT) {
    // ------------------------------------------------------------ activation producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, armed_b = 0, par_b = 0;
      bool ok = true;
      Tile t;
      for (int tile = blockIdx.x; ok && get_tile<BN>(p, s_chunk, s_off, tile, total, t); tile += gridDim.x) {
        for (int ks = 0; ks < nsteps; ++ks) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, wctx, 102)) { ok = false; break; }
          if (ks < mma_steps) {
            const int k0 = ks * C::BKS;
            const int natoms = min(C::ATOMS, (p.K - k0) / ATOM_K);
            mbar_arrive_expect_tx(&b_full[stage], natoms * C::B_ATOM_BYTES);
            for (int a = 0; a < natoms; ++a)
              tma_load_2d(sB + stage * C::B_STAGE_BYTES + a * C::B_ATOM_BYTES, &tm_act, &b_full[stage],
                          k0 + a * ATOM_K, t.row0);
          } else {                                   // LoRA step: the xa tile
            mbar_arrive_expect_tx(&b_full[stage], C::B_ATOM_BYTES);
            tma_load_2d(sB + stage * C::B_STAGE_BYTES, &tm_xa, &b_full[stage], 0, t.row0);
          }
          armed_b |= 1u << stage;
          par_b = (par_b & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        for (int s = 0; s < C::STAGES; ++s)
          if (armed_b & (1u << s)) mbar_drain(&b_full[s], (par_b >> s) & 1u, kDrainNs);
      }
    }
  } else if (warp == WARP_MMA) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
      int stage = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      uint64_t* last_bar = nullptr;
      uint32_t last_par = 0;
      Tile t;
      for (int tile = blockIdx.x; ok && get_tile<BN>(p, s_chunk, s_off, tile, total, t); tile += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t aphase = (it >> 1) & 1;
        if (!mbar_wait(&acc_empty[buf], aphase ^ 1u, wctx, 201)) { ok = false; break; }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
        for (int ks = 0; ks < nsteps; ++ks) {
          if (!mbar_wait(&a_full[stage], phase, wctx, 202)) { ok = false; break; }
          if (!mbar_wait(&b_full[stage], phase, wctx, 203)) { ok = false; break; }
          tc_fence_after_sync();
          const uint32_t a0 = C::TMEM_A ? tmem_base + static_cast<uint32_t>(C::A_COL0 + stage * C::A_COLS)
                                        : smem_u32(sA + stage * C::A_STAGE_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * C::B_STAGE_BYTES);
          // K16 steps: 4 per valid atom; the LoRA step is a single K=16 MMA
          const int nk = ks < mma_steps ? 4 * min(C::ATOMS, (p.K - ks * C::BKS) / ATOM_K) : 1;
          for (int kk = 0; kk < nk; ++kk) {
            const uint32_t bo = (kk >> 2) * C::B_ATOM_BYTES + (kk & 3) * 32;
            if constexpr (C::TMEM_A)
              umma_bf16_ts(d_tmem, a0 + kk * 8, smem_desc_sw128(b0 + bo), idesc, (ks > 0 || kk > 0) ? 1u : 0u);
            else
              umma_bf16_ss(d_tmem, smem_desc_sw128(a0 + (kk & 3) * 32), smem_desc_sw128(b0 + bo), idesc,
                           (ks > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          issued = true;
          last_bar = &empty[stage];
          last_par = phase;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&acc_full[buf]);
        last_bar = &acc_full[buf];
        last_par = aphase;
      }
      if (!ok && issued) mbar_drain(last_bar, last_par, kDrainNs);   // MMAs in flight finish first
    }
  } else if (warp < C::WARP_EPI0) {
    // ------------------------------------------------------------ dequant
    // With A in tensor memory, A row = TMEM lane and a warp may only touch its
    // own quarter of the lanes; with A in shared memory any mapping works.
    const int quarter = warp & 3;
    const int prow = 32 * quarter + lane;          // A-tile row written by this thread
    const int half = ((warp - WARP_DQ0) >> 2) & 1; // BKS 128: atom; BKS 64: 32-element half of the atom
    const int group = (warp - WARP_DQ0) >> 3;      // BKS 64: takes the 128-K code stages of its parity
    int64_t gs = 0, gr = 0;                        // BKS 64: MMA / code stages of the tiles before this one
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(32 * quarter) << 16);
    const uint32_t lut_l =
        smem_u32(sLut) + (FMT == E4B_NF4 ? static_cast<uint32_t>(lane & 15) * 8u : static_cast<uint32_t>(lane) * 4u);
    const int kb64 = p.K / 64, kb32 = p.K / 32;
    int stage = 0, rstage = 0;
    uint32_t phase = 0, rphase = 0;
    bool ok = true;
    Tile t;
    for (int tile = blockIdx.x; ok && get_tile<BN>(p, s_chunk, s_off, tile, total, t); tile += gridDim.x) {
      int wrow, raw_row;
      tile_row<MODE>(p, t.nb, prow, wrow, raw_row);
      const int64_t grow = static_cast<int64_t>(t.e) * p.N + min(wrow, p.N - 1);
      const float* sc_nf4 = reinterpret_cast<const float*>(p.scales) + grow * kb64;
      const uint8_t* sc_mx = reinterpret_cast<const uint8_t*>(p.scales) + grow * kb32;
      if constexpr (C::BKS == 128) {
        // each thread: 64 elements of its row per stage (atom `half`)
        // scales of this thread's 64 elements: NF4 one absmax, MXFP4 two E8M0 (one per 32)
        auto load_scale = [&](int r, uint64_t& a2, uint32_t& s2a, uint32_t& s2b) {
          const int blk = 2 * r + half;                     // 64-element block along K
          if (blk >= kb64) return;                          // ragged tail: nothing to decode
          if (FMT == E4B_NF4) {
            a2 = dup_f32(__ldg(sc_nf4 + blk));
          } else {
            const uint32_t v = __ldg(reinterpret_cast<const uint16_t*>(sc_mx + 2 * blk));
            s2a = e8m0_to_bf16x2(v & 0xFFu);
            s2b = e8m0_to_bf16x2(v >> 8);
          }
        };
        uint64_t a2n = 0;
        uint32_t san = 0, sbn = 0;
        load_scale(0, a2n, san, sbn);
        for (int r = 0; r < raw_steps; ++r) {
          const uint64_t a2 = a2n;
          const uint32_t sa = san, sb = sbn;
          if (r + 1 < raw_steps) load_scale(r + 1, a2n, san, sbn);
          if (!mbar_wait(&raw_full[rstage], rphase, wctx, 301)) { ok = false; break; }
          if (!mbar_wait(&empty[stage], phase ^ 1u, wctx, 302)) { ok = false; break; }
          if (r * RAW_K + half * ATOM_K < p.K) {       // warp-uniform (half is per warp)
            const uint8_t* raw = sRaw + rstage * RAW_STAGE_BYTES;
            const uint32_t acol = static_cast<uint32_t>(C::A_COL0 + stage * C::A_COLS + half * 32);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const uint4 q =
                  *reinterpret_cast<const uint4*>(raw + swizzled_offset(raw_row, half * 2 + c, RAW_ROW_BYTES));
              uint4 o[4];
              dequant32<FMT>(q, lut_l, a2, c == 0 ? sa : sb, o);
              const uint32_t v[16] = {o[0].x, o[0].y, o[0].z, o[0].w, o[1].x, o[1].y, o[1].z, o[1].w,
                                      o[2].x, o[2].y, o[2].z, o[2].w, o[3].x, o[3].y, o[3].z, o[3].w};
              tmem_st_32x32b_x16(t_lane + acol + c * 16, v);
            }
            tmem_st_wait();
          }
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&a_full[stage]);
            mbar_arrive(&raw_empty[rstage]);
          }
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
          if (++rstage == C::RAW_STAGES) { rstage = 0; rphase ^= 1u; }
        }
      } else {
        // each thread: 32 elements (half of one 64-wide atom row) per MMA stage; the
        // group takes code stage j of the tile when gr + j has its parity
        const int ksteps = p.K / ATOM_K;
        const int nraw = (ksteps + 1) / 2;
        // scales of code stage j (two MMA stages), loaded one owned stage ahead
        auto load_scales = [&](int j, uint64_t (&a2)[2], uint32_t (&s2)[2]) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int ks = 2 * j + h;
            if (j < nraw && ks < ksteps) {
              if (FMT == E4B_NF4) a2[h] = dup_f32(__ldg(sc_nf4 + ks));
              else s2[h] = e8m0_to_bf16x2(__ldg(sc_mx + 2 * ks + half));
            }
          }
        };
        const int j0 = static_cast<int>((group - gr) & 1);
        uint64_t a2n[2] = {0, 0};
        uint32_t s2n[2] = {0, 0};
        load_scales(j0, a2n, s2n);
        for (int j = j0; j < nraw; j += 2) {
          const int64_t rg = gr + j;
          const int rs = static_cast<int>(rg % C::RAW_STAGES);
          const uint32_t rph = static_cast<uint32_t>(rg / C::RAW_STAGES) & 1u;
          const uint64_t a2[2] = {a2n[0], a2n[1]};
          const uint32_t s2[2] = {s2n[0], s2n[1]};
          load_scales(j + 2, a2n, s2n);
          if (!mbar_wait(&raw_full[rs], rph, wctx, 301)) { ok = false; break; }
          const uint8_t* raw = sRaw + rs * RAW_STAGE_BYTES;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int ks = 2 * j + h;
            if (ks >= ksteps) break;
            const int64_t sg = gs + ks;
            const int st = static_cast<int>(sg % C::STAGES);
            const uint32_t sph = static_cast<uint32_t>(sg / C::STAGES) & 1u;
            if (!mbar_wait(&empty[st], sph ^ 1u, wctx, 302)) { ok = false; break; }
            const uint4 q = *reinterpret_cast<const uint4*>(raw + swizzled_offset(raw_row, h * 2 + half, RAW_ROW_BYTES));
            uint4 o[4];
            dequant32<FMT>(q, lut_l, a2[h], s2[h], o);
            if constexpr (C::TMEM_A) {
              const uint32_t v[16] = {o[0].x, o[0].y, o[0].z, o[0].w, o[1].x, o[1].y, o[1].z, o[1].w,
                                      o[2].x, o[2].y, o[2].z, o[2].w, o[3].x, o[3].y, o[3].z, o[3].w};
              tmem_st_32x32b_x16(t_lane + static_cast<uint32_t>(C::A_COL0 + st * C::A_COLS + half * 16), v);
              tmem_st_wait();
              tc_fence_before_sync();
            } else {
              uint8_t* a = sA + st * C::A_STAGE_BYTES;
#pragma unroll
              for (int i = 0; i < 4; ++i)
                *reinterpret_cast<uint4*>(a + swizzled_offset(prow, half * 4 + i, 128)) = o[i];
              fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[st]);
          }
          if (!ok) break;
          __syncwarp();
          if (lane == 0) mbar_arrive(&raw_empty[rs]);
        }
        if (!ok) break;
        if (lora && group == 0) {                  // the LoRA step: group 0 fills the stage after K
          const int64_t sg = gs + ksteps;
          const int st = static_cast<int>(sg % C::STAGES);
          if (!mbar_wait(&empty[st], (static_cast<uint32_t>(sg / C::STAGES) & 1u) ^ 1u, wctx, 303)) {
            ok = false;
            break;
          }
          if (half == 0) {                           // warp-uniform
            const uint16_t* bcol = p.lora_B + static_cast<int64_t>(t.e) * p.lora_rank * (2 * p.I) + wrow;
            uint32_t v[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              const uint32_t lo = (2 * jj < p.lora_rank) ? __ldg(bcol + static_cast<int64_t>(2 * jj) * 2 * p.I) : 0u;
              const uint32_t hi =
                  (2 * jj + 1 < p.lora_rank) ? __ldg(bcol + static_cast<int64_t>(2 * jj + 1) * 2 * p.I) : 0u;
              v[jj] = lo | (hi << 16);
            }
            if constexpr (C::TMEM_A) {
              tmem_st_32x32b_x8(t_lane + static_cast<uint32_t>(C::A_COL0 + st * C::A_COLS), v);
              tmem_st_wait();
            } else {
              uint8_t* a = sA + st * C::A_STAGE_BYTES;
              *reinterpret_cast<uint4*>(a + swizzled_offset(prow, 0, 128)) = make_uint4(v[0], v[1], v[2], v[3]);
              *reinterpret_cast<uint4*>(a + swizzled_offset(prow, 1, 128)) = make_uint4(v[4], v[5], v[6], v[7]);
            }
          }
          if constexpr (C::TMEM_A) tc_fence_before_sync();
          else fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_full[st]);
        }
        gs += ksteps + (lora ? 1 : 0);
        gr += nraw;
        continue;                                  // the LoRA step is done above for these tiles
      }
      if (!ok) break;
      if (lora) {                                   // A rows of the LoRA step: B_e[:, wrow]^T, rank padded to 16
        if (!mbar_wait(&empty[stage], phase ^ 1u, wctx, 303)) { ok = false; break; }
        if (half == 0) {                              // warp-uniform
          const uint16_t* bcol = p.lora_B + static_cast<int64_t>(t.e) * p.lora_rank * (2 * p.I) + wrow;
          uint32_t v[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t lo = (2 * j < p.lora_rank) ? __ldg(bcol + static_cast<int64_t>(2 * j) * 2 * p.I) : 0u;
            const uint32_t hi = (2 * j + 1 < p.lora_rank) ? __ldg(bcol + static_cast<int64_t>(2 * j + 1) * 2 * p.I) : 0u;
            v[j] = lo | (hi << 16);
          }
          if constexpr (C::TMEM_A) {
            tmem_st_32x32b_x8(t_lane + static_cast<uint32_t>(C::A_COL0 + stage * C::A_COLS), v);
            tmem_st_wait();
          } else {
            uint8_t* a = sA + stage * C::A_STAGE_BYTES;
            *reinterpret_cast<uint4*>(a + swizzled_offset(prow, 0, 128)) = make_uint4(v[0], v[1], v[2], v[3]);
            *reinterpret_cast<uint4*>(a + swizzled_offset(prow, 1, 128)) = make_uint4(v[4], v[5], v[6], v[7]);
          }
        }
        if constexpr (C::TMEM_A) tc_fence_before_sync();
        else fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[stage]);
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                        // TMEM lanes 32q..32q+31
    int it = 0;
    Tile t;
    for (int tile = blockIdx.x; get_tile<BN>(p, s_chunk, s_off, tile, total, t); tile += gridDim.x, ++it) {
      const int buf = it & 1;
      const uint32_t aphase = (it >> 1) & 1;
      if (!mbar_wait_sleep(&acc_full[buf], aphase, wctx, 401, 256)) break;
      tc_fence_after_sync();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * BN);
      if constexpr (MODE == 0) {
        // Thread t holds the adjacent features f, f + 1 (rows t/4 and t/4 + 8 of
        // the gate slab, lanes 32q..32q+15, and of the up slab, 32q+16..32q+31)
        // for the tokens 8i + 2(t%4) + {0, 1} of each 32-column chunk: the
        // activation of every (feature, token) is formed in the thread that holds
        // its gate and up values, and two features go out in one 4-byte store.
        const int f = 64 * t.nb + 16 * q + 2 * (lane >> 2);
        const int tc = 2 * (lane & 3);
        __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(p.out);
        float bg0 = 0.f, bg1 = 0.f, bu0 = 0.f, bu1 = 0.f;
        if (p.ep.bias) {
          const float* b = p.ep.bias + static_cast<int64_t>(t.e) * 2 * p.I + f;
          bg0 = __ldg(b);
          bg1 = __ldg(b + 1);
          bu0 = __ldg(b + p.I);
          bu1 = __ldg(b + p.I + 1);
        }
        for (int c0 = 0; c0 < BN && c0 < t.rows; c0 += 32) {
          uint32_t g[16], u[16];
          tmem_ld_16x256b_x4(taddr + c0, g);
          tmem_ld_16x256b_x4(taddr + (16u << 16) + c0, u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int tok = c0 + 8 * i + tc + hh;
              if (tok < t.rows) {
                const float g0 = __uint_as_float(g[4 * i + hh]) + bg0;
                const float g1 = __uint_as_float(g[4 * i + 2 + hh]) + bg1;
                const float u0 = __uint_as_float(u[4 * i + hh]) + bu0;
                const float u1 = __uint_as_float(u[4 * i + 2 + hh]) + bu1;
                const int64_t row = t.row0 + tok;
                *reinterpret_cast<__nv_bfloat162*>(h + row * p.I + f) =
                    __floats2bfloat162_rn(expert_act(p.ep, g0, u0), expert_act(p.ep, g1, u1));
                if (p.g_out) {              // kept for the backward: pre-activation gate and up
                  float* go = p.g_out + row * 2 * p.I + f;
                  *reinterpret_cast<float2*>(go) = make_float2(g0, g1);
                  *reinterpret_cast<float2*>(go + p.I) = make_float2(u0, u1);
                }
              }
            }
          }
        }
      } else {
        // lane = output feature n, one 128-byte row segment per store
        const int n = BM * t.nb + 32 * q + lane;
        float* y = reinterpret_cast<float*>(p.out);
        const float bv = (p.ep.bias && n < p.N) ? __ldg(p.ep.bias + static_cast<int64_t>(t.e) * p.N + n) : 0.f;
        for (int c0 = 0; c0 < BN && c0 < t.rows; c0 += 16) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(taddr + c0, r);
          tmem_ld_wait();
          if (n < p.N) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (c0 + j < t.rows) y[static_cast<int64_t>(t.row0 + c0 + j) * p.N + n] = __uint_as_float(r[j]) + bv;
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------- host side

template <int BN, int FMT, int MODE>
e4b_status launch_typed(const GroupedGemmLaunch& g, const CUtensorMap& tc, const CUtensorMap& ta,
                        const CUtensorMap& tx, const Params& prm, cudaStream_t s) {
  using C = Cfg<BN>;
  auto kern = grouped_gemm_kernel<BN, FMT, MODE>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return E4B_ERR_CUDA;
  const int64_t active = g.R < g.E ? g.R : g.E;
  const int64_t max_tiles = (active + (g.R + BN - 1) / BN) * prm.n_blocks;
  const int64_t sms = device_sm_count();
  const int grid = static_cast<int>(max_tiles < sms ? (max_tiles > 0 ? max_tiles : 1) : sms);
  return launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, s, tc, ta, tx, prm) == cudaSuccess
             ? E4B_OK
             : E4B_ERR_CUDA;
}

template <int BN>
e4b_status dispatch_fmt_mode(const GroupedGemmLaunch& g, const CUtensorMap& tc, const CUtensorMap& ta,
                             const CUtensorMap& tx, const Params& prm, cudaStream_t s) {
  if (g.fmt == E4B_NF4)
    return g.mode == 0 ? launch_typed<BN, E4B_NF4, 0>(g, tc, ta, tx, prm, s)
                       : launch_typed<BN, E4B_NF4, 1>(g, tc, ta, tx, prm, s);
  return g.mode == 0 ? launch_typed<BN, E4B_MXFP4, 0>(g, tc, ta, tx, prm, s)
                     : launch_typed<BN, E4B_MXFP4, 1>(g, tc, ta, tx, prm, s);
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool encode_tma_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tma_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t d0, uint64_t d1,
                   uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2,
                   CUtensorMapSwizzle swz) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

e4b_status launch_grouped_gemm(const GroupedGemmLaunch& g, cudaStream_t s) {
  if (g.R == 0) return E4B_OK;
  const int BN = g.tokens_per_tile;
  CUtensorMap tc, ta, tx;
  const uint64_t code_rows = static_cast<uint64_t>(g.E) * g.N;
  if (!encode_tma_2d(&tc, CU_TENSOR_MAP_DATA_TYPE_UINT8, g.codes, g.K / 2, code_rows, g.K / 2, RAW_ROW_BYTES,
                 g.mode == 0 ? 64 : BM, CU_TENSOR_MAP_SWIZZLE_64B))
    return E4B_ERR_CUDA;
  if (!encode_tma_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.act, g.K, g.R, static_cast<uint64_t>(g.K) * 2, ATOM_K, BN,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return E4B_ERR_CUDA;
  const bool lora = g.mode == 0 && g.lora_rank > 0;
  if (lora) {
    if (!encode_tma_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.xa, 64, g.R, 128, ATOM_K, BN, CU_TENSOR_MAP_SWIZZLE_128B))
      return E4B_ERR_CUDA;
  } else {
    tx = ta;
  }
  Params prm;
  prm.E = g.E;
  prm.N = g.N;
  prm.K = g.K;
  prm.I = g.I;
  prm.n_blocks = g.mode == 0 ? g.I / 64 : (g.N + BM - 1) / BM;
  prm.lora_rank = lora ? g.lora_rank : 0;
  prm.codes = g.codes;
  prm.scales = g.scales;
  prm.lora_B = g.lora_B;
  prm.expert_offsets = g.expert_offsets;
  prm.chunk_off = g.chunk_off;
  prm.out = g.out;
  prm.status = g.status;
  prm.wait_limit_ns = g.wait_limit_ns;
  prm.ep = Epilogue{g.bias, g.mode == 0 ? g.glu : E4B_ACT_SWIGLU, g.glu_alpha, g.glu_limit, g.glu_beta};
  prm.g_out = g.mode == 0 ? g.g_out : nullptr;
  for (int i = 0; i < 16; ++i) prm.lut[i] = nf4_table().level[i];
  switch (BN) {
    case 32: return dispatch_fmt_mode<32>(g, tc, ta, tx, prm, s);
    case 64: return dispatch_fmt_mode<64>(g, tc, ta, tx, prm, s);
    case 128: return dispatch_fmt_mode<128>(g, tc, ta, tx, prm, s);
    case 192: return dispatch_fmt_mode<192>(g, tc, ta, tx, prm, s);
    case 256: return dispatch_fmt_mode<256>(g, tc, ta, tx, prm, s);
    default: return E4B_ERR_UNSUPPORTED;
  }
}

}  // namespace e4b
