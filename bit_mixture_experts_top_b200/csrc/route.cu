// Top-k routing, expert histogram, stable expert permute, row gather (with the
// LoRA left factor) and the weighted combine.
//
// Routing (solutions index, grouped-nf4-gemm table: the routed expert GEMM runs
// over all experts in one launch, so routed rows are grouped by expert first;
// "experts4bit-qlora", "Current measured position": routing is decided on the
// router logits):
//   * one warp per token; lane l holds the logits of experts l, l+32, ...
//     packed into 32-bit keys (order-preserving bf16 bits << 16 | 0xFFFF - id),
//     so one unsigned max picks the largest logit and, on ties, the lowest id;
//     each lane sorts its keys once, then k rounds of __reduce_max_sync over the
//     lanes' largest remaining keys select the k experts (keys are unique, so
//     exactly one lane owns each pick and steps to its next key);
//   * gate weights are the fp32 softmax of the k selected logits, or (gating
//     E4B_GATE_SOFTMAX_ALL) the softmax over all E logits read at the k picks,
//     not renormalised: the denominator is summed from the keys before the
//     first pick is removed;
//   * the block histogram feeds per-block counts; the last block to finish
//     turns them into expert offsets, per-block bases and tile-chunk offsets;
//   * the rank kernel orders each block's slots by (expert, slot) with
//     warp-level __match_any_sync ranks, which makes the permute stable and
//     deterministic.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "e4b_device.cuh"
#include "e4b_internal.h"

namespace e4b {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTopkThreads = 1024;         // top-k: 4 tokens per warp at 128 tokens per block
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTokPerWarp = kRouteTokensPerBlock / kTopkWarps;
constexpr uint32_t kFull = 0xFFFFFFFFu;

__device__ __forceinline__ uint32_t route_key(uint16_t bits, int e) {
  if (bits == 0x8000u) bits = 0;                                    // -0 == +0
  const uint32_t ord = (bits & 0x8000u) ? (~bits & 0xFFFFu) : (bits | 0x8000u);
  return (ord << 16) | (0xFFFFu - static_cast<uint32_t>(e));
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

// The logit a key holds (inverse of route_key's order-preserving map).
__device__ __forceinline__ float key_logit(uint32_t key) {
  const uint32_t ord = key >> 16;
  return bf16_bits_to_f32(static_cast<uint16_t>((ord & 0x8000u) ? (ord & 0x7FFFu) : (~ord & 0xFFFFu)));
}

// sum over the row of exp(logit - m), from this warp's keys (0 = no expert)
template <int J>
__device__ __forceinline__ float row_exp_sum(const uint32_t (&key)[J], float m) {
  float s = 0.0f;
#pragma unroll
  for (int j = 0; j < J; ++j)
    if (key[j]) s += expf(key_logit(key[j]) - m);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(kFull, s, off);
  return s;
}

__device__ __forceinline__ void cas_desc(uint32_t& a, uint32_t& b) {
  const uint32_t hi = max(a, b), lo = min(a, b);
  a = hi;
  b = lo;
}

// Sorts J <= 8 keys in descending order (Batcher's odd-even merge networks).
template <int J>
__device__ __forceinline__ void sort_desc(uint32_t (&x)[J]) {
  if constexpr (J == 2) {
    cas_desc(x[0], x[1]);
  } else if constexpr (J == 4) {
    cas_desc(x[0], x[1]); cas_desc(x[2], x[3]);
    cas_desc(x[0], x[2]); cas_desc(x[1], x[3]);
    cas_desc(x[1], x[2]);
  } else if constexpr (J == 8) {
    cas_desc(x[0], x[1]); cas_desc(x[2], x[3]); cas_desc(x[4], x[5]); cas_desc(x[6], x[7]);
    cas_desc(x[0], x[2]); cas_desc(x[1], x[3]); cas_desc(x[4], x[6]); cas_desc(x[5], x[7]);
    cas_desc(x[1], x[2]); cas_desc(x[5], x[6]);
    cas_desc(x[0], x[4]); cas_desc(x[1], x[5]); cas_desc(x[2], x[6]); cas_desc(x[3], x[7]);
    cas_desc(x[2], x[4]); cas_desc(x[3], x[5]);
    cas_desc(x[1], x[2]); cas_desc(x[3], x[4]); cas_desc(x[5], x[6]);
  }
}

// One token's top k (one warp, keys already loaded, 0 = no expert): lane r < k
// returns the r-th largest key, and all_sum the full-softmax denominator when
// `gating` asks for it (summed before any key is taken).
template <int J>
__device__ __forceinline__ uint32_t warp_topk(uint32_t (&key)[J], int k, int gating, int lane, float& all_sum) {
  sort_desc<J>(key);
  uint32_t mine = 0;
  for (int r = 0; r < k; ++r) {
    const uint32_t best = __reduce_max_sync(kFull, key[0]);
    if (r == 0 && gating == E4B_GATE_SOFTMAX_ALL) all_sum = row_exp_sum(key, key_logit(best));
    if (key[0] == best) {                  // the owner steps to its next key
#pragma unroll
      for (int j = 0; j + 1 < J; ++j) key[j] = key[j + 1];
      key[J - 1] = 0u;
    }
    if (lane == r) mine = best;
  }
  return mine;
}

// Stable rank: block b's slots [s0, s1) take positions base[b][e] + (# earlier
// slots of the block with the same expert).  Each warp owns a contiguous
// segment; per-warp histograms are scanned across warps first.
template <int NW>
__device__ __forceinline__ void rank_block(int b, const int32_t* __restrict__ topk_ids, int T, int E, int k,
                                           const int32_t* block_base, int32_t* __restrict__ sorted_slot,
                                           int32_t* __restrict__ slot_pos, int32_t (*s_wc)[kMaxExperts]) {
  constexpr int kWarps = NW, kThreads = NW * 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t s0 = static_cast<int64_t>(b) * kRouteTokensPerBlock * k;
  const int64_t s1 = min(static_cast<int64_t>(T), static_cast<int64_t>(b + 1) * kRouteTokensPerBlock) * k;
  const int64_t n = s1 - s0;
  const int64_t seg = ((n + kWarps - 1) / kWarps + 31) / 32 * 32;
  const int64_t w0 = s0 + warp * seg, w1 = min(s1, w0 + seg);
  for (int i = tid; i < kWarps * kMaxExperts; i += kThreads) (&s_wc[0][0])[i] = 0;
  __syncthreads();
  for (int64_t s = w0 + lane; s < w1; s += 32) atomicAdd(&s_wc[warp][topk_ids[s]], 1);
  __syncthreads();
  for (int e = tid; e < E; e += kThreads) {
    int32_t run = __ldcg(block_base + static_cast<int64_t>(b) * E + e);
    for (int w = 0; w < kWarps; ++w) {
      const int32_t c = s_wc[w][e];
      s_wc[w][e] = run;
      run += c;
    }
  }
  __syncthreads();
  const uint32_t lt = (1u << lane) - 1u;
  for (int64_t c0 = w0; c0 < w1; c0 += 32) {
    const int64_t s = c0 + lane;
    const bool valid = s < w1;
    const int id = valid ? topk_ids[s] : (kMaxExperts + lane);   // invalid lanes never match
    const uint32_t peers = __match_any_sync(kFull, id);
    const int rank = __popc(peers & lt);
    int32_t pos = 0;
    if (valid) pos = s_wc[warp][id] + rank;
    __syncwarp();
    if (valid && rank == __popc(peers) - 1) s_wc[warp][id] += __popc(peers);
    __syncwarp();
    if (valid) {
      sorted_slot[pos] = static_cast<int32_t>(s);
      slot_pos[s] = pos;
    }
  }
}

__global__ void __launch_bounds__(kThreads) route_rank_kernel(const int32_t* __restrict__ topk_ids, int T, int E,
                                                              int k, const int32_t* __restrict__ block_base,
                                                              int32_t* __restrict__ sorted_slot,
                                                              int32_t* __restrict__ slot_pos) {
  __shared__ int32_t s_wc[kWarps][kMaxExperts];
  pdl_wait();
  pdl_launch_dependents();
  rank_block<kWarps>(blockIdx.x, topk_ids, T, E, k, block_base, sorted_slot, slot_pos, s_wc);
}

template <int J>
__global__ void __launch_bounds__(kTopkThreads, 1) route_topk_kernel(const uint16_t* __restrict__ logits, int T, int E,
                                                                  int k, int gating, int tokens_per_tile, int nblk,
                                                                  int32_t* __restrict__ topk_ids,
                                                                  float* __restrict__ topk_w, int32_t* block_counts,
                                                                  uint32_t* done_counter, int32_t* expert_offsets,
                                                                  int32_t* chunk_off, int32_t* __restrict__ sorted_slot,
                                                                  int32_t* __restrict__ slot_pos) {
  __shared__ int32_t s_wc[kTopkWarps][kMaxExperts];
  __shared__ int32_t s_cnt[kMaxExperts];
  __shared__ int32_t s_tot[kMaxExperts + 1];
  __shared__ bool s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();
  pdl_launch_dependents();
  for (int e = tid; e < E; e += kTopkThreads) s_cnt[e] = 0;
  __syncthreads();

  // warp w takes tokens t_begin + w + kTopkWarps * q; all their logits are loaded first
  const int t_begin = blockIdx.x * kRouteTokensPerBlock;
  uint32_t key[kTokPerWarp][J];            // J = ceil(E / 32) keys per lane
#pragma unroll
  for (int q = 0; q < kTokPerWarp; ++q) {
    const int t = t_begin + warp + kTopkWarps * q;
    const uint16_t* row = logits + static_cast<int64_t>(t) * E;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int e = lane + 32 * j;
      key[q][j] = (t < T && e < E) ? route_key(__ldg(row + e), e) : 0u;   // real keys are never 0
    }
  }
#pragma unroll
  for (int q = 0; q < kTokPerWarp; ++q) {
    const int t = t_begin + warp + kTopkWarps * q;
    if (t >= T) break;
    float all_sum = 0.0f;                  // full-softmax denominator (E4B_GATE_SOFTMAX_ALL)
    const uint32_t mine = warp_topk(key[q], k, gating, lane, all_sum);   // lane j keeps the j-th pick
    int id = 0;
    float v = 0.0f;
    if (lane < k) {
      id = 0xFFFF - static_cast<int>(mine & 0xFFFFu);
      v = key_logit(mine);
    }
    const float m = __shfl_sync(kFull, v, 0);          // the first pick holds the maximum
    float ex = (lane < k) ? expf(v - m) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(kFull, sum, off);
    if (lane < k) {
      topk_ids[static_cast<int64_t>(t) * k + lane] = id;
      topk_w[static_cast<int64_t>(t) * k + lane] = ex / (gating == E4B_GATE_SOFTMAX_ALL ? all_sum : sum);
      atomicAdd(&s_cnt[id], 1);
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += kTopkThreads) block_counts[static_cast<int64_t>(blockIdx.x) * E + e] = s_cnt[e];
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(done_counter, 1u) == static_cast<uint32_t>(nblk - 1));
  __syncthreads();
  if (!s_last) return;

  // Last block: totals, exclusive offsets, per-block bases, tile-chunk offsets.
  __threadfence();
  for (int e = tid; e < E; e += kTopkThreads) {
    int32_t tot = 0;
    for (int b = 0; b < nblk; ++b) tot += __ldcg(block_counts + static_cast<int64_t>(b) * E + e);
    s_tot[e] = tot;
  }
  __syncthreads();
  if (warp == 0) {
    // warp-wide exclusive scans of the counts and of the chunk counts; lane l owns
    // experts [8l, 8l+8)
    int32_t c[kMaxExperts / 32], ch[kMaxExperts / 32];
    int32_t run = 0, crun = 0;
#pragma unroll
    for (int j = 0; j < kMaxExperts / 32; ++j) {
      const int e = lane * (kMaxExperts / 32) + j;
      c[j] = e < E ? s_tot[e] : 0;
      ch[j] = tokens_per_tile > 0 ? (c[j] + tokens_per_tile - 1) / tokens_per_tile : 0;
      run += c[j];
      crun += ch[j];
    }
    int32_t inc = run, cinc = crun;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t a = __shfl_up_sync(kFull, inc, off), ca = __shfl_up_sync(kFull, cinc, off);
      if (lane >= off) { inc += a; cinc += ca; }
    }
    run = inc - run;
    crun = cinc - crun;
#pragma unroll
    for (int j = 0; j < kMaxExperts / 32; ++j) {
      const int e = lane * (kMaxExperts / 32) + j;
      if (e < E) {
        expert_offsets[e] = run;
        if (chunk_off) chunk_off[e] = crun;
        s_tot[e] = run;
      }
      run += c[j];
      crun += ch[j];
    }
    if (lane == 31) {
      expert_offsets[E] = run;
      if (chunk_off) chunk_off[E] = crun;
      *done_counter = 0u;                             // ready for the next call
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += kTopkThreads) {
    int32_t run = s_tot[e];
    for (int b = 0; b < nblk; ++b) {
      int32_t* p = block_counts + static_cast<int64_t>(b) * E + e;
      const int32_t c = __ldcg(p);
      *p = run;                                       // becomes block b's base for expert e
      run += c;
    }
  }
  if (nblk == 1) {          // a single routing block also ranks its slots: one launch for small batches
    __threadfence_block();
    __syncthreads();
    rank_block<kTopkWarps>(0, topk_ids, T, E, k, block_counts, sorted_slot, slot_pos, s_wc);
  }
}

// T <= 4 * NW (one routing block of NW warps, 4 tokens per warp): top-k,
// histogram, scans and the stable rank in one block with every intermediate in
// shared memory, no cross-block protocol.  The block also zeroes the status
// words of the workspace first (the caller skips its memset), so a small
// forward starts with a single launch.  Decode batches (T <= 32) take an
// 8-warp block, whose barriers and shared-memory clears cost a quarter of the
// 32-warp block's.
template <int NW, int J>
__global__ void __launch_bounds__(NW * 32, 1) route_small_kernel(const uint16_t* __restrict__ logits, int T, int E,
                                                                  int k, int gating, int tokens_per_tile,
                                                                  int32_t* status_words,
                                                                  int32_t* __restrict__ topk_ids,
                                                                  float* __restrict__ topk_w,
                                                                  int32_t* __restrict__ expert_offsets,
                                                                  int32_t* __restrict__ chunk_off,
                                                                  int32_t* __restrict__ sorted_slot,
                                                                  int32_t* __restrict__ slot_pos) {
  __shared__ int16_t s_ids[kRouteTokensPerBlock * kMaxTopK];
  constexpr int kW = NW, kT = NW * 32;
  __shared__ __align__(16) int16_t s_wc[kW][kMaxExperts];   // per-warp counts, then running positions
  __shared__ int32_t s_cnt[kMaxExperts];
  __shared__ int32_t s_off[kMaxExperts];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();
  pdl_launch_dependents();
  if (status_words && tid < kStatusBytes / 4) status_words[tid] = 0;
  for (int e = tid; e < kMaxExperts; e += kT) s_cnt[e] = 0;
  for (int i = tid; i < kW * kMaxExperts; i += kT) (&s_wc[0][0])[i] = 0;
  __syncthreads();

  uint32_t key[kTokPerWarp][J];            // J = ceil(E / 32) keys per lane
#pragma unroll
  for (int q = 0; q < kTokPerWarp; ++q) {
    const int t = warp + kW * q;
    const uint16_t* row = logits + static_cast<int64_t>(t) * E;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int e = lane + 32 * j;
      key[q][j] = (t < T && e < E) ? route_key(__ldg(row + e), e) : 0u;
    }
  }
#pragma unroll
  for (int q = 0; q < kTokPerWarp; ++q) {
    const int t = warp + kW * q;
    if (t >= T) break;
    float all_sum = 0.0f;
    const uint32_t mine = warp_topk(key[q], k, gating, lane, all_sum);
    int id = 0;
    float v = 0.0f;
    if (lane < k) {
      id = 0xFFFF - static_cast<int>(mine & 0xFFFFu);
      v = key_logit(mine);
    }
    const float m = __shfl_sync(kFull, v, 0);
    float ex = (lane < k) ? expf(v - m) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(kFull, sum, off);
    if (lane < k) {
      topk_ids[static_cast<int64_t>(t) * k + lane] = id;
      topk_w[static_cast<int64_t>(t) * k + lane] = ex / (gating == E4B_GATE_SOFTMAX_ALL ? all_sum : sum);
      s_ids[t * k + lane] = static_cast<int16_t>(id);
      atomicAdd(&s_cnt[id], 1);
    }
  }
  __syncthreads();
  if (warp == 0) {          // exclusive scans of the counts and chunk counts; lane l owns experts [8l, 8l+8)
    int32_t c[kMaxExperts / 32], ch[kMaxExperts / 32];
    int32_t run = 0, crun = 0;
#pragma unroll
    for (int j = 0; j < kMaxExperts / 32; ++j) {
      const int e = lane * (kMaxExperts / 32) + j;
      c[j] = e < E ? s_cnt[e] : 0;
      ch[j] = tokens_per_tile > 0 ? (c[j] + tokens_per_tile - 1) / tokens_per_tile : 0;
      run += c[j];
      crun += ch[j];
    }
    int32_t inc = run, cinc = crun;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t a = __shfl_up_sync(kFull, inc, off), ca = __shfl_up_sync(kFull, cinc, off);
      if (lane >= off) { inc += a; cinc += ca; }
    }
    run = inc - run;
    crun = cinc - crun;
#pragma unroll
    for (int j = 0; j < kMaxExperts / 32; ++j) {
      const int e = lane * (kMaxExperts / 32) + j;
      if (e < E) {
        expert_offsets[e] = run;
        if (chunk_off) chunk_off[e] = crun;
        s_off[e] = run;
      }
      run += c[j];
      crun += ch[j];
    }
    if (lane == 31) {
      expert_offsets[E] = run;
      if (chunk_off) chunk_off[E] = crun;
    }
  }
  // stable rank: warp w owns the contiguous slot segment [w0, w1)
  const int n = T * k;
  const int seg = ((n + kW - 1) / kW + 31) / 32 * 32;
  const int w0 = warp * seg, w1 = min(n, w0 + seg);
  for (int s = w0 + lane; s < w1; s += 32) {
    const int id = s_ids[s];
    // 16-bit counters: add through the containing word
    atomicAdd(reinterpret_cast<int*>(&s_wc[warp][id & ~1]), 1 << (16 * (id & 1)));
  }
  __syncthreads();
  for (int e = tid; e < E; e += kT) {
    int32_t run = s_off[e];
    for (int w = 0; w < kW; ++w) {
      const int32_t c = s_wc[w][e];
      s_wc[w][e] = static_cast<int16_t>(run);
      run += c;
    }
  }
  __syncthreads();
  const uint32_t lt = (1u << lane) - 1u;
  for (int c0 = w0; c0 < w1; c0 += 32) {
    const int s = c0 + lane;
    const bool valid = s < w1;
    const int id = valid ? s_ids[s] : (kMaxExperts + lane);
    const uint32_t peers = __match_any_sync(kFull, id);
    const int rank = __popc(peers & lt);
    int32_t pos = 0;
    if (valid) pos = static_cast<uint16_t>(s_wc[warp][id]) + rank;
    __syncwarp();
    if (valid && rank == __popc(peers) - 1) s_wc[warp][id] = static_cast<int16_t>(pos + 1);
    __syncwarp();
    if (valid) {
      sorted_slot[pos] = s;
      slot_pos[s] = pos;
    }
  }
}

// One warp per routed row: copy the token's activations into expert order and,
// with LoRA, form xa = scale * x . A_e (bf16, rank padded with zeros to 64).
__global__ void __launch_bounds__(kThreads) gather_kernel(const uint16_t* __restrict__ x, int H, int k, int R,
                                                          const int32_t* __restrict__ sorted_slot,
                                                          const int32_t* __restrict__ topk_ids,
                                                          uint16_t* __restrict__ x_sorted,
                                                          const uint16_t* __restrict__ lora_A, int rank,
                                                          float scale, uint16_t* __restrict__ xa) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  pdl_launch_dependents();
  const int64_t r = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  if (r >= R) return;
  const int32_t slot = sorted_slot[r];
  const int64_t t = slot / k;
  const uint4* src = reinterpret_cast<const uint4*>(x + t * H);
  uint4* dst = reinterpret_cast<uint4*>(x_sorted + r * H);
  const int nvec = H / 8;
  float acc[kMaxLoraRank];
#pragma unroll
  for (int j = 0; j < kMaxLoraRank; ++j) acc[j] = 0.0f;
  if (!lora_A) {            // plain copy: eight 16-byte loads in flight per lane
    for (int v0 = lane; v0 < nvec; v0 += 32 * 8) {
      uint4 q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (v0 + 32 * i < nvec) q[i] = __ldg(src + v0 + 32 * i);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (v0 + 32 * i < nvec) dst[v0 + 32 * i] = q[i];
    }
    return;
  }
  const uint16_t* Ae = lora_A ? lora_A + static_cast<int64_t>(topk_ids[slot]) * H * rank : nullptr;
  const bool vec8 = Ae && (rank == 8 || rank == 16) &&            // A rows are whole 16-byte vectors
                    (reinterpret_cast<uintptr_t>(lora_A) & 15u) == 0;
  for (int v = lane; v < nvec; v += 32) {
    const uint4 q = __ldg(src + v);
    dst[v] = q;
    if (Ae) {
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float xv = bf16_bits_to_f32(static_cast<uint16_t>(w[i >> 1] >> (16 * (i & 1))));
        const uint16_t* arow = Ae + static_cast<int64_t>(v * 8 + i) * rank;
        if (vec8) {
#pragma unroll
          for (int h = 0; h < kMaxLoraRank / 8; ++h) {
            if (h * 8 < rank) {
              const uint4 a = __ldg(reinterpret_cast<const uint4*>(arow) + h);
              const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
              for (int j = 0; j < 8; ++j)
                acc[h * 8 + j] = fmaf(xv, bf16_bits_to_f32(static_cast<uint16_t>(aw[j >> 1] >> (16 * (j & 1)))),
                                      acc[h * 8 + j]);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < kMaxLoraRank; ++j)
            if (j < rank) acc[j] = fmaf(xv, bf16_bits_to_f32(__ldg(arow + j)), acc[j]);
        }
      }
    }
  }
  if (!Ae) return;
#pragma unroll
  for (int j = 0; j < kMaxLoraRank; ++j) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[j] += __shfl_xor_sync(kFull, acc[j], off);
  }
  // lane l writes columns 2l, 2l+1 of the 64-wide row
  float lo = 0.0f, hi = 0.0f;
#pragma unroll
  for (int j = 0; j < kMaxLoraRank; ++j) {
    if (j < rank && j == 2 * lane) lo = acc[j] * scale;
    if (j < rank && j == 2 * lane + 1) hi = acc[j] * scale;
  }
  __nv_bfloat162 pr = __floats2bfloat162_rn(lo, hi);
  reinterpret_cast<uint32_t*>(xa + r * 64)[lane] = *reinterpret_cast<uint32_t*>(&pr);
}

// out[t] = sum_j w[t, j] * y[slot_pos[t*k + j]], j ascending.  Block (t, cb)
// covers columns [4 * kThreads * cb, ...) of token t, one float4 per thread;
// the k rows are loaded eight at a time before they are summed in order.
__global__ void __launch_bounds__(kThreads) combine_kernel(const float* __restrict__ y,
                                                           const float* __restrict__ topk_w,
                                                           const int32_t* __restrict__ slot_pos, int k, int H,
                                                           uint16_t* __restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t t = blockIdx.x;
  const int c = blockIdx.y * kThreads + threadIdx.x;
  if (c >= H / 4) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j0 = 0; j0 < k; j0 += 8) {
    float4 v[8];
    float w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (j0 + i < k) {
        w[i] = __ldg(topk_w + t * k + j0 + i);
        v[i] = __ldcs(reinterpret_cast<const float4*>(y + static_cast<int64_t>(__ldg(slot_pos + t * k + j0 + i)) * H) + c);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (j0 + i < k) {
        acc.x = fmaf(w[i], v[i].x, acc.x);
        acc.y = fmaf(w[i], v[i].y, acc.y);
        acc.z = fmaf(w[i], v[i].z, acc.z);
        acc.w = fmaf(w[i], v[i].w, acc.w);
      }
    }
  }
  __nv_bfloat162 a = __floats2bfloat162_rn(acc.x, acc.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(acc.z, acc.w);
  uint2 o = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
  reinterpret_cast<uint2*>(out + t * H)[c] = o;
}

}  // namespace

namespace {

// The routing launches for J = ceil(E / 32) keys per lane (J in {1, 2, 4, 8}).
template <int J>
cudaError_t launch_route_keys(const uint16_t* logits, int32_t T, int32_t E, int32_t k, int32_t gating,
                              int32_t tokens_per_tile, const RouteBuffers& b, int32_t* status_words,
                              cudaStream_t s) {
  const int nblk = route_blocks(T);
  if (nblk == 1) {
    if (T <= 4 * 8)
      return launch_pdl(route_small_kernel<8, J>, dim3(1), dim3(8 * 32), 0, s, logits, T, E, k, gating,
                        tokens_per_tile, status_words, b.topk_ids, b.topk_w, b.expert_offsets, b.chunk_off,
                        b.sorted_slot, b.slot_pos);
    return launch_pdl(route_small_kernel<kTopkWarps, J>, dim3(1), dim3(kTopkThreads), 0, s, logits, T, E, k,
                      gating, tokens_per_tile, status_words, b.topk_ids, b.topk_w, b.expert_offsets, b.chunk_off,
                      b.sorted_slot, b.slot_pos);
  }
  if (status_words && cudaMemsetAsync(status_words, 0, kStatusBytes, s) != cudaSuccess) return cudaGetLastError();
  cudaError_t err = launch_pdl(route_topk_kernel<J>, dim3(nblk), dim3(kTopkThreads), 0, s, logits, T, E, k, gating,
                               tokens_per_tile, nblk, b.topk_ids, b.topk_w, b.block_counts, b.done_counter,
                               b.expert_offsets, b.chunk_off, b.sorted_slot, b.slot_pos);
  if (err != cudaSuccess) return err;
  return launch_pdl(route_rank_kernel, dim3(nblk), dim3(kThreads), 0, s, b.topk_ids, T, E, k,
                    static_cast<const int32_t*>(b.block_counts), b.sorted_slot, b.slot_pos);
}

}  // namespace

cudaError_t launch_route(const uint16_t* logits, int32_t T, int32_t E, int32_t k, int32_t gating,
                         int32_t tokens_per_tile,
                         const RouteBuffers& b, int32_t* status_words, cudaStream_t s) {
  if (T == 0) {
    cudaError_t err = status_words ? cudaMemsetAsync(status_words, 0, kStatusBytes, s) : cudaSuccess;
    if (err == cudaSuccess) err = cudaMemsetAsync(b.expert_offsets, 0, sizeof(int32_t) * (E + 1), s);
    if (err == cudaSuccess && b.chunk_off) err = cudaMemsetAsync(b.chunk_off, 0, sizeof(int32_t) * (E + 1), s);
    return err;
  }
  if (E <= 32) return launch_route_keys<1>(logits, T, E, k, gating, tokens_per_tile, b, status_words, s);
  if (E <= 64) return launch_route_keys<2>(logits, T, E, k, gating, tokens_per_tile, b, status_words, s);
  if (E <= 128) return launch_route_keys<4>(logits, T, E, k, gating, tokens_per_tile, b, status_words, s);
  return launch_route_keys<8>(logits, T, E, k, gating, tokens_per_tile, b, status_words, s);
}

cudaError_t launch_gather(const uint16_t* x, int32_t H, int32_t k, int32_t R, const int32_t* sorted_slot,
                          const int32_t* topk_ids, int32_t E, uint16_t* x_sorted, const uint16_t* lora_A,
                          int32_t lora_rank, float lora_scale, uint16_t* xa, cudaStream_t s) {
  (void)E;
  if (R == 0) return cudaSuccess;
  const int grid = (R + kWarps - 1) / kWarps;
  return launch_pdl(gather_kernel, dim3(grid), dim3(kThreads), 0, s, x, H, k, R, sorted_slot, topk_ids, x_sorted,
                    lora_A, lora_rank, lora_scale, xa);
}

cudaError_t launch_combine(const float* y, const float* topk_w, const int32_t* slot_pos, int32_t T, int32_t k,
                           int32_t H, uint16_t* out, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const dim3 grid(T, (H / 4 + kThreads - 1) / kThreads);
  return launch_pdl(combine_kernel, grid, dim3(kThreads), 0, s, y, topk_w, slot_pos, k, H, out);
}

}  // namespace e4b

// ---------------------------------------------------------------------------
// Routing for callers that cannot allocate device memory.
//
// Some callers have no way to hand the library a workspace: a host runtime
// that owns every byte of device memory through its own pool and forbids
// cudaMalloc once it has started, or a latency-critical serving loop where an
// allocation could synchronise the device.  e4b_route_noalloc runs the same
// routing kernels as e4b_route but keeps their scratch (status word, per-block
// histograms, slot positions) in one file-scope device array of fixed size
// that every GPU loading the library holds until the process exits.
// ---------------------------------------------------------------------------
#include <mutex>

namespace e4b {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;     // 1 MiB per device
static __device__ __align__(256) uint8_t g_route_scratch[kNoAllocScratchBytes];

// Device addresses of g_route_scratch, looked up once per device.  In host
// code the array's name is only a host-side handle: the address the kernels
// need comes from cudaGetSymbolAddress with that device current.  The cached
// address belongs to the device's current context: a cudaDeviceReset between
// calls would leave it stale, so callers must not reset the device while
// they use this entry point.
uint8_t* g_route_scratch_addr[64] = {};
std::mutex g_route_scratch_mu;

e4b_status route_scratch_address(uint8_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return E4B_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_route_scratch_mu);
  if (!g_route_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return E4B_ERR_CUDA;
    g_route_scratch_addr[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_route_scratch_addr[dev];
  return E4B_OK;
}

}  // namespace
}  // namespace e4b

extern "C" e4b_status e4b_route_noalloc(const uint16_t* logits, int32_t T, int32_t E, int32_t k, int32_t gating,
                                        int32_t* topk_ids, float* topk_w, int32_t* expert_offsets,
                                        int32_t* sorted_slot, e4b_stream stream) {
  using namespace e4b;
  if (T < 0 || E < 1 || k < 1 || k > E) return E4B_ERR_INVALID_ARG;
  if (gating != E4B_GATE_SOFTMAX_TOPK && gating != E4B_GATE_SOFTMAX_ALL) return E4B_ERR_INVALID_ARG;
  if (E > kMaxExperts || k > kMaxTopK) return E4B_ERR_UNSUPPORTED;
  if (!expert_offsets) return E4B_ERR_INVALID_ARG;
  if (T > 0 && (!logits || !topk_ids || !topk_w || !sorted_slot)) return E4B_ERR_INVALID_ARG;
  // scratch layout: status word + done counter, per-block histograms, slot positions
  const size_t nblk = static_cast<size_t>(route_blocks(T) > 0 ? route_blocks(T) : 1);
  const size_t off_counts = align_up(kStatusBytes);
  const size_t off_pos = off_counts + align_up(nblk * static_cast<size_t>(E) * 4);
  const size_t need = off_pos + align_up(static_cast<size_t>(T) * k * 4);
  if (need > kNoAllocScratchBytes) return E4B_ERR_UNSUPPORTED;   // beyond the fixed scratch size
  uint8_t* scratch = nullptr;
  const e4b_status st = route_scratch_address(&scratch);
  if (st != E4B_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents.  The status word and the
  // last-block counter must start at zero; launch_route clears them itself
  // (inside the single routing block for T <= 128, else by a memset ahead of
  // the multi-block kernels), and every other region is written before it is
  // read, so nothing else needs clearing.
  RouteBuffers b;
  b.status = reinterpret_cast<int32_t*>(scratch);
  b.done_counter = reinterpret_cast<uint32_t*>(b.status + 2);
  b.topk_ids = topk_ids;
  b.topk_w = topk_w;
  b.expert_offsets = expert_offsets;
  b.chunk_off = nullptr;
  b.block_counts = reinterpret_cast<int32_t*>(scratch + off_counts);
  b.sorted_slot = sorted_slot;
  b.slot_pos = reinterpret_cast<int32_t*>(scratch + off_pos);
  return launch_route(logits, T, E, k, gating, 0, b, b.status, s) == cudaSuccess ? E4B_OK : E4B_ERR_CUDA;
}
