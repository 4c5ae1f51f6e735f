// C ABI of the library: argument validation, workspace layout and the launch
// sequence of the layer forward (route -> gather -> gate_up -> down -> combine).
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>

#include "e4b.h"
#include "e4b_device.cuh"
#include "e4b_internal.h"

namespace e4b {

int device_sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev < 64) cache[dev] = n;
  return n;
}

namespace {

__global__ void wait_timeout_probe_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtx w{&abort_flag, status, limit_ns};
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, w, 9001);   // nothing ever arrives
  __syncthreads();
}

struct ForwardLayout {
  size_t status, topk_ids, topk_w, offsets, chunk_off, block_counts, sorted_slot, slot_pos, x_sorted, xa, h, y;
  size_t gu_absmax, dn_absmax;   // expanded double-quantised absmax (E4B_NF4_DQ only)
  size_t total;
};

// Absmax values of one stack [E, N, K] (one per 64 weights).
size_t absmax_count(const e4b_moe_desc& d, bool gate_up) {
  return static_cast<size_t>(d.E) * (gate_up ? 2 * static_cast<size_t>(d.I) : d.H) *
         (gate_up ? d.H : d.I) / 64;
}

// The format the GEMM kernels see: a double-quantised stack runs as NF4 on its expanded absmax.
int32_t gemm_format(int32_t format) { return format == E4B_NF4_DQ ? E4B_NF4 : format; }

// A nested-form absmax description: every array present, the fp32 ones 4-byte aligned.
bool valid_dq(const e4b_nf4_dq* q) {
  return q && q->codes && q->absmax2 && q->offset && q->table && aligned(q->absmax2, 4) && aligned(q->offset, 4) &&
         aligned(q->table, 4);
}

ForwardLayout forward_layout(const e4b_moe_desc& d, int32_t T) {
  const size_t R = static_cast<size_t>(T) * d.k;
  const size_t nblk = static_cast<size_t>(route_blocks(T) > 0 ? route_blocks(T) : 1);
  ForwardLayout L;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += align_up(bytes);
    return at;
  };
  L.status = take(kStatusBytes);
  L.topk_ids = take(R * 4);
  L.topk_w = take(R * 4);
  L.offsets = take((d.E + 1) * 4);
  L.chunk_off = take((d.E + 1) * 4);
  L.block_counts = take(nblk * d.E * 4);
  L.sorted_slot = take(R * 4);
  L.slot_pos = take(R * 4);
  L.x_sorted = take(R * d.H * 2);
  L.xa = take(d.lora_rank > 0 ? R * 128 : 0);
  L.h = take(R * d.I * 2);
  L.y = take(R * d.H * 4);
  const bool dq = d.format == E4B_NF4_DQ;
  L.gu_absmax = take(dq ? absmax_count(d, true) * 4 : 0);
  L.dn_absmax = take(dq ? absmax_count(d, false) * 4 : 0);
  L.total = o;
  return L;
}

// The training workspace: the forward's layout, then what the backward needs
// besides it (the saved pre-activation G) and its own scratch.
struct TrainLayout {
  ForwardLayout fwd;
  size_t g, dY, dG, dxa, dX, total;
};

TrainLayout train_layout(const e4b_moe_desc& d, int32_t T) {
  TrainLayout L;
  L.fwd = forward_layout(d, T);
  const size_t R = static_cast<size_t>(T) * d.k;
  size_t o = L.fwd.total;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += align_up(bytes);
    return at;
  };
  L.g = take(R * 2 * d.I * 4);
  L.dY = take(R * d.H * 2);
  L.dG = take(R * 2 * d.I * 2);
  L.dxa = take(d.lora_rank > 0 ? R * 16 * 4 : 0);
  L.dX = take(R * d.H * 4);
  L.total = o;
  return L;
}

struct RouteLayout {
  size_t status, block_counts, slot_pos, total;
};

RouteLayout route_layout(int32_t T, int32_t E, int32_t k) {
  const size_t nblk = static_cast<size_t>(route_blocks(T) > 0 ? route_blocks(T) : 1);
  RouteLayout L;
  size_t o = 0;
  L.status = o;
  o += align_up(kStatusBytes);
  L.block_counts = o;
  o += align_up(nblk * E * 4);
  L.slot_pos = o;
  o += align_up(static_cast<size_t>(T) * k * 4);
  L.total = o;
  return L;
}

e4b_status validate_desc(const e4b_moe_desc* d, int32_t T) {
  if (!d || T < 0) return E4B_ERR_INVALID_ARG;
  if (d->E < 1 || d->E > kMaxExperts || d->k < 1 || d->k > d->E || d->k > kMaxTopK) return E4B_ERR_UNSUPPORTED;
  if (d->H < 64 || d->H % 64 != 0 || d->I < 64 || d->I % 64 != 0) return E4B_ERR_UNSUPPORTED;
  if (d->format != E4B_NF4 && d->format != E4B_MXFP4 && d->format != E4B_NF4_DQ) return E4B_ERR_UNSUPPORTED;
  if (d->act != E4B_ACT_SWIGLU && d->act != E4B_ACT_CLAMPED_GLU) return E4B_ERR_UNSUPPORTED;
  if (d->act == E4B_ACT_CLAMPED_GLU &&
      (!std::isfinite(d->glu_alpha) || !std::isfinite(d->glu_beta) || !(d->glu_limit > 0.0f)))
    return E4B_ERR_INVALID_ARG;
  if (d->lora_rank < 0 || d->lora_rank > kMaxLoraRank) return E4B_ERR_UNSUPPORTED;
  if (d->gating != E4B_GATE_SOFTMAX_TOPK && d->gating != E4B_GATE_SOFTMAX_ALL) return E4B_ERR_INVALID_ARG;
  const int tpt = d->tokens_per_tile;
  const int32_t gf = gemm_format(d->format);
  if (tpt == 8 && !(skinny_gemm_supported(d->H, gf) && skinny_gemm_supported(d->I, gf)))
    return E4B_ERR_UNSUPPORTED;
  if (tpt != 0 && tpt != 8 && tpt != 32 && tpt != 64 && tpt != 128 && tpt != 192 && tpt != 256) return E4B_ERR_UNSUPPORTED;
  const int64_t R = static_cast<int64_t>(T) * d->k;
  if (R > (int64_t(1) << 30)) return E4B_ERR_UNSUPPORTED;
  // TMA row coordinates are 32-bit: E * 2I rows of codes must fit.
  if (static_cast<int64_t>(d->E) * 2 * d->I >= (int64_t(1) << 31)) return E4B_ERR_UNSUPPORTED;
  return E4B_OK;
}

struct KernelChoice {
  bool decode;        // skinny_gemm (decode kernel) or grouped_gemm (tcgen05 tiles)
  int32_t tokens;     // decode: tokens per chunk; tcgen05: tile width
};

// Mean routed rows per active expert decides: a handful per expert -> the decode
// kernel (weight-stream bound), with chunks of 8, 16 or 32 tokens so that one
// decoded weight fragment serves up to 32 tokens; more -> the smallest tcgen05
// tile that holds most experts' rows in one chunk, 256 for prefill (each
// dequantised weight stage then feeds the most tokens).
KernelChoice pick_kernel(const e4b_moe_desc& d, int32_t T) {
  const int64_t R = static_cast<int64_t>(T) * d.k;
  const int64_t active = R < d.E ? R : d.E;
  const int64_t avg = active > 0 ? (R + active - 1) / active : 1;
  const int32_t gf = gemm_format(d.format);
  const bool decode_ok = skinny_gemm_supported(d.H, gf) && skinny_gemm_supported(d.I, gf);
  const int32_t chunk = avg <= 8 ? 8 : (avg <= 16 ? 16 : 32);
  if (d.tokens_per_tile == 8) return {true, chunk};
  if (d.tokens_per_tile) return {false, d.tokens_per_tile};
  if (avg <= kDecodeMaxRows && decode_ok) return {true, chunk};
  if (avg <= 16) return {false, 32};
  if (avg <= 48) return {false, 64};
  if (avg <= 96) return {false, 128};
  return {false, 256};
}

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}

}  // namespace
}  // namespace e4b

using namespace e4b;

extern "C" {

int32_t e4b_abi_version(void) { return E4B_ABI_VERSION; }

const char* e4b_status_string(int32_t status) {
  switch (status) {
    case E4B_OK: return "E4B_OK";
    case E4B_ERR_INVALID_ARG: return "E4B_ERR_INVALID_ARG: bad pointer, size, alignment or workspace";
    case E4B_ERR_UNSUPPORTED: return "E4B_ERR_UNSUPPORTED: shape or option outside what the kernels implement";
    case E4B_ERR_CUDA: return "E4B_ERR_CUDA: a CUDA call or kernel launch failed";
    case E4B_ERR_TIMEOUT: return "E4B_ERR_TIMEOUT: a bounded device-side wait ran out";
    default: return "E4B_ERR_UNKNOWN";
  }
}

void e4b_nf4_codebook(float* out) {
  if (!out) return;
  std::memcpy(out, nf4_table().level, sizeof(float) * 16);
}

e4b_status e4b_dequant_mxfp4(const uint8_t* codes, const uint8_t* scales, int64_t n, uint16_t* out,
                             e4b_stream stream) {
  if (n < 0 || n % 32 != 0) return E4B_ERR_INVALID_ARG;
  if (n == 0) return E4B_OK;
  if (!codes || !scales || !out || !aligned(codes, 16) || !aligned(out, 16)) return E4B_ERR_INVALID_ARG;
  return launch_dequant_mxfp4(codes, scales, n, out, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? E4B_OK
             : E4B_ERR_CUDA;
}

e4b_status e4b_expand_absmax_dq(const e4b_nf4_dq* dq, int64_t n, float* out, e4b_stream stream) {
  if (n < 0) return E4B_ERR_INVALID_ARG;
  if (n == 0) return E4B_OK;
  if (!valid_dq(dq) || !out || !aligned(out, 4)) return E4B_ERR_INVALID_ARG;
  return launch_expand_absmax_dq(dq->codes, dq->absmax2, dq->offset, dq->table, n, n, nullptr, out,
                                 reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? E4B_OK
             : E4B_ERR_CUDA;
}

e4b_status e4b_deinterleave_rows(const void* in, void* out, int32_t E, int32_t I, int64_t row_bytes,
                                 e4b_stream stream) {
  if (E < 0 || I < 0 || row_bytes < 0) return E4B_ERR_INVALID_ARG;
  const int64_t bytes = static_cast<int64_t>(E) * 2 * I * row_bytes;
  if (bytes == 0) return E4B_OK;
  if (!in || !out) return E4B_ERR_INVALID_ARG;
  const uintptr_t a = reinterpret_cast<uintptr_t>(in), b = reinterpret_cast<uintptr_t>(out);
  if (a < b + static_cast<uintptr_t>(bytes) && b < a + static_cast<uintptr_t>(bytes)) return E4B_ERR_INVALID_ARG;
  return launch_deinterleave_rows(in, out, E, I, row_bytes, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? E4B_OK
             : E4B_ERR_CUDA;
}

e4b_status e4b_quantize_nf4(const float* x, int64_t n, uint8_t* codes, float* absmax, e4b_stream stream) {
  if (n < 0 || n % 64 != 0) return E4B_ERR_INVALID_ARG;
  if (n == 0) return E4B_OK;
  if (!x || !codes || !absmax || !aligned(x, 16) || !aligned(codes, 4) || !aligned(absmax, 4))
    return E4B_ERR_INVALID_ARG;
  return launch_quantize_nf4(x, n, codes, absmax, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? E4B_OK
             : E4B_ERR_CUDA;
}

size_t e4b_route_workspace_bytes(int32_t T, int32_t E, int32_t k) {
  if (T < 0 || E < 1 || E > kMaxExperts || k < 1 || k > E || k > kMaxTopK) return 0;
  return route_layout(T, E, k).total;
}

e4b_status e4b_route(const uint16_t* logits, int32_t T, int32_t E, int32_t k, int32_t gating, int32_t* topk_ids,
                     float* topk_w,
                     int32_t* expert_offsets, int32_t* sorted_slot, void* ws, size_t ws_bytes,
                     e4b_stream stream) {
  if (T < 0 || E < 1 || k < 1 || k > E) return E4B_ERR_INVALID_ARG;
  if (gating != E4B_GATE_SOFTMAX_TOPK && gating != E4B_GATE_SOFTMAX_ALL) return E4B_ERR_INVALID_ARG;
  if (E > kMaxExperts || k > kMaxTopK) return E4B_ERR_UNSUPPORTED;
  if (!expert_offsets || !ws || !aligned(ws, kAlign)) return E4B_ERR_INVALID_ARG;
  if (T > 0 && (!logits || !topk_ids || !topk_w || !sorted_slot)) return E4B_ERR_INVALID_ARG;
  if (static_cast<int64_t>(T) * k > (int64_t(1) << 30)) return E4B_ERR_UNSUPPORTED;
  const RouteLayout L = route_layout(T, E, k);
  if (ws_bytes < L.total) return E4B_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  RouteBuffers b;
  b.status = at<int32_t>(ws, L.status);
  b.done_counter = reinterpret_cast<uint32_t*>(b.status + 2);
  b.topk_ids = topk_ids;
  b.topk_w = topk_w;
  b.expert_offsets = expert_offsets;
  b.chunk_off = nullptr;
  b.block_counts = at<int32_t>(ws, L.block_counts);
  b.sorted_slot = sorted_slot;
  b.slot_pos = at<int32_t>(ws, L.slot_pos);
  // the status words are zeroed by the launch sequence (in-kernel for one routing block)
  return launch_route(logits, T, E, k, gating, 0, b, b.status, s) == cudaSuccess ? E4B_OK : E4B_ERR_CUDA;
}

size_t e4b_moe_workspace_bytes(const e4b_moe_desc* d, int32_t T) {
  if (validate_desc(d, T) != E4B_OK) return 0;
  return forward_layout(*d, T).total;
}

e4b_status e4b_moe_workspace_region(const e4b_moe_desc* d, int32_t T, int32_t region, size_t* offset,
                                    size_t* bytes) {
  const e4b_status v = validate_desc(d, T);
  if (v != E4B_OK) return v;
  if (!offset || !bytes) return E4B_ERR_INVALID_ARG;
  const ForwardLayout L = forward_layout(*d, T);
  const size_t R = static_cast<size_t>(T) * d->k;
  switch (region) {
    case E4B_WS_TOPK_IDS: *offset = L.topk_ids; *bytes = R * 4; break;
    case E4B_WS_TOPK_W: *offset = L.topk_w; *bytes = R * 4; break;
    case E4B_WS_EXPERT_OFFSETS: *offset = L.offsets; *bytes = (d->E + 1) * 4; break;
    case E4B_WS_SORTED_SLOT: *offset = L.sorted_slot; *bytes = R * 4; break;
    case E4B_WS_X_SORTED: *offset = L.x_sorted; *bytes = R * d->H * 2; break;
    case E4B_WS_H: *offset = L.h; *bytes = R * d->I * 2; break;
    case E4B_WS_Y: *offset = L.y; *bytes = R * d->H * 4; break;
    case E4B_WS_GU_ABSMAX:
      *offset = L.gu_absmax;
      *bytes = d->format == E4B_NF4_DQ ? absmax_count(*d, true) * 4 : 0;
      break;
    case E4B_WS_DN_ABSMAX:
      *offset = L.dn_absmax;
      *bytes = d->format == E4B_NF4_DQ ? absmax_count(*d, false) * 4 : 0;
      break;
    default: return E4B_ERR_INVALID_ARG;
  }
  return E4B_OK;
}

static e4b_status run_stages(int32_t first, int32_t last, const e4b_moe_desc* d, int32_t T, const uint16_t* x,
                             const uint16_t* logits, const uint8_t* gu_codes, const void* gu_scales,
                             const uint8_t* dn_codes, const void* dn_scales, const uint16_t* lora_A,
                             const uint16_t* lora_B, const float* gu_bias, const float* dn_bias, uint16_t* out,
                             void* ws, size_t ws_bytes, e4b_stream stream, bool train = false) {
  const e4b_status v = validate_desc(d, T);
  if (v != E4B_OK) return v;
  if (first < E4B_STAGE_ROUTE || last > E4B_STAGE_COMBINE || first > last) return E4B_ERR_INVALID_ARG;
  const bool lora = d->lora_rank > 0;
  if ((lora_A != nullptr) != lora || (lora_B != nullptr) != lora) return E4B_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, kAlign)) return E4B_ERR_INVALID_ARG;
  const ForwardLayout L = forward_layout(*d, T);
  if (ws_bytes < (train ? train_layout(*d, T).total : L.total)) return E4B_ERR_INVALID_ARG;
  const bool dq = d->format == E4B_NF4_DQ;
  if (T > 0) {
    if (!x || !logits || !gu_codes || !gu_scales || !dn_codes || !dn_scales || !out) return E4B_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out, 16) || !aligned(gu_codes, 16) || !aligned(dn_codes, 16))
      return E4B_ERR_INVALID_ARG;
    if (dq ? !(valid_dq(static_cast<const e4b_nf4_dq*>(gu_scales)) && valid_dq(static_cast<const e4b_nf4_dq*>(dn_scales)))
           : !(aligned(gu_scales, 16) && aligned(dn_scales, 16)))
      return E4B_ERR_INVALID_ARG;
    if (lora && (!aligned(lora_A, 2) || !aligned(lora_B, 2))) return E4B_ERR_INVALID_ARG;
    if ((gu_bias && !aligned(gu_bias, 4)) || (dn_bias && !aligned(dn_bias, 4))) return E4B_ERR_INVALID_ARG;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const KernelChoice kc = pick_kernel(*d, T);
  const int32_t tpt = kc.tokens;
  const int32_t R = T * d->k;

  RouteBuffers b;
  b.status = at<int32_t>(ws, L.status);
  b.done_counter = reinterpret_cast<uint32_t*>(b.status + 2);
  b.topk_ids = at<int32_t>(ws, L.topk_ids);
  b.topk_w = at<float>(ws, L.topk_w);
  b.expert_offsets = at<int32_t>(ws, L.offsets);
  b.chunk_off = at<int32_t>(ws, L.chunk_off);
  b.block_counts = at<int32_t>(ws, L.block_counts);
  b.sorted_slot = at<int32_t>(ws, L.sorted_slot);
  b.slot_pos = at<int32_t>(ws, L.slot_pos);
  uint16_t* x_sorted = at<uint16_t>(ws, L.x_sorted);
  uint16_t* xa = lora ? at<uint16_t>(ws, L.xa) : nullptr;
  uint16_t* h = at<uint16_t>(ws, L.h);
  float* y = at<float>(ws, L.y);
  float* gu_absmax = at<float>(ws, L.gu_absmax);
  float* dn_absmax = at<float>(ws, L.dn_absmax);

  GroupedGemmLaunch g;
  g.fmt = gemm_format(d->format);
  g.E = d->E;
  g.I = d->I;
  g.R = R;
  g.tokens_per_tile = tpt;
  g.decode = kc.decode ? 1 : 0;
  g.expert_offsets = b.expert_offsets;
  g.chunk_off = b.chunk_off;
  g.status = b.status;
  g.wait_limit_ns = kWaitLimitNs;
  g.glu = d->act;
  g.glu_alpha = d->glu_alpha;
  g.glu_limit = d->glu_limit;
  g.glu_beta = d->glu_beta;
  g.g_out = nullptr;
  float* g_keep = train ? at<float>(ws, train_layout(*d, T).g) : nullptr;

  for (int32_t stage = first; stage <= last; ++stage) {
    switch (stage) {
      case E4B_STAGE_ROUTE:
        // zeroes the status words first (in the routing kernel when one block routes)
        if (launch_route(logits, T, d->E, d->k, d->gating, tpt, b, b.status, s) != cudaSuccess) return E4B_ERR_CUDA;
        break;
      case E4B_STAGE_GATHER:
        if (launch_gather(x, d->H, d->k, R, b.sorted_slot, b.topk_ids, d->E, x_sorted, lora_A, d->lora_rank,
                          d->lora_scale, xa, s) != cudaSuccess)
          return E4B_ERR_CUDA;
        if (dq && T > 0) {   // the touched experts' absmax, expanded to fp32 for this forward
          const e4b_nf4_dq* gq = static_cast<const e4b_nf4_dq*>(gu_scales);
          const e4b_nf4_dq* dqs = static_cast<const e4b_nf4_dq*>(dn_scales);
          const size_t ng = absmax_count(*d, true), nd = absmax_count(*d, false);
          if (launch_expand_absmax_dq(gq->codes, gq->absmax2, gq->offset, gq->table, ng, ng / d->E,
                                      b.expert_offsets, gu_absmax, s) != cudaSuccess ||
              launch_expand_absmax_dq(dqs->codes, dqs->absmax2, dqs->offset, dqs->table, nd, nd / d->E,
                                      b.expert_offsets, dn_absmax, s) != cudaSuccess)
            return E4B_ERR_CUDA;
        }
        break;
      case E4B_STAGE_GATE_UP: {
        g.mode = 0;
        g.N = 2 * d->I;
        g.K = d->H;
        g.codes = gu_codes;
        g.scales = dq ? static_cast<const void*>(gu_absmax) : gu_scales;
        g.act = x_sorted;
        g.xa = xa;
        g.lora_B = lora_B;
        g.lora_rank = d->lora_rank;
        g.bias = gu_bias;
        g.out = h;
        g.g_out = g_keep;
        const e4b_status st = kc.decode ? launch_skinny_gemm(g, s) : launch_grouped_gemm(g, s);
        if (st != E4B_OK) return st;
        break;
      }
      case E4B_STAGE_DOWN: {
        g.mode = 1;
        g.N = d->H;
        g.K = d->I;
        g.codes = dn_codes;
        g.scales = dq ? static_cast<const void*>(dn_absmax) : dn_scales;
        g.act = h;
        g.xa = nullptr;
        g.lora_B = nullptr;
        g.lora_rank = 0;
        g.bias = dn_bias;
        g.out = y;
        g.g_out = nullptr;
        const e4b_status st = kc.decode ? launch_skinny_gemm(g, s) : launch_grouped_gemm(g, s);
        if (st != E4B_OK) return st;
        break;
      }
      case E4B_STAGE_COMBINE:
        if (launch_combine(y, b.topk_w, b.slot_pos, T, d->k, d->H, out, s) != cudaSuccess) return E4B_ERR_CUDA;
        break;
    }
  }
  return E4B_OK;
}

e4b_status e4b_moe_forward(const e4b_moe_desc* d, int32_t T, const uint16_t* x, const uint16_t* logits,
                           const uint8_t* gu_codes, const void* gu_scales, const uint8_t* dn_codes,
                           const void* dn_scales, const uint16_t* lora_A, const uint16_t* lora_B,
                           const float* gu_bias, const float* dn_bias, uint16_t* out, void* ws, size_t ws_bytes,
                           e4b_stream stream) {
  return run_stages(E4B_STAGE_ROUTE, E4B_STAGE_COMBINE, d, T, x, logits, gu_codes, gu_scales, dn_codes, dn_scales,
                    lora_A, lora_B, gu_bias, dn_bias, out, ws, ws_bytes, stream);
}

e4b_status e4b_moe_forward_stage(int32_t stage, const e4b_moe_desc* d, int32_t T, const uint16_t* x,
                                 const uint16_t* logits, const uint8_t* gu_codes, const void* gu_scales,
                                 const uint8_t* dn_codes, const void* dn_scales, const uint16_t* lora_A,
                                 const uint16_t* lora_B, const float* gu_bias, const float* dn_bias, uint16_t* out,
                                 void* ws, size_t ws_bytes, e4b_stream stream) {
  return run_stages(stage, stage, d, T, x, logits, gu_codes, gu_scales, dn_codes, dn_scales, lora_A, lora_B, gu_bias,
                    dn_bias, out, ws, ws_bytes, stream);
}

size_t e4b_moe_train_workspace_bytes(const e4b_moe_desc* d, int32_t T) {
  if (validate_desc(d, T) != E4B_OK) return 0;
  return train_layout(*d, T).total;
}

e4b_status e4b_moe_forward_train(const e4b_moe_desc* d, int32_t T, const uint16_t* x, const uint16_t* logits,
                                 const uint8_t* gu_codes, const void* gu_scales, const uint8_t* dn_codes,
                                 const void* dn_scales, const uint16_t* lora_A, const uint16_t* lora_B,
                                 const float* gu_bias, const float* dn_bias, uint16_t* out, void* ws,
                                 size_t ws_bytes, e4b_stream stream) {
  return run_stages(E4B_STAGE_ROUTE, E4B_STAGE_COMBINE, d, T, x, logits, gu_codes, gu_scales, dn_codes, dn_scales,
                    lora_A, lora_B, gu_bias, dn_bias, out, ws, ws_bytes, stream, true);
}

e4b_status e4b_moe_backward(const e4b_moe_desc* d, int32_t T, const uint16_t* logits, const uint16_t* dout,
                            const uint8_t* gu_codes, const void* gu_scales, const uint8_t* dn_codes,
                            const void* dn_scales, const uint16_t* lora_A, const uint16_t* lora_B, float* dx,
                            float* dlogits, float* dA, float* dB, void* ws, size_t ws_bytes, e4b_stream stream) {
  const e4b_status v = validate_desc(d, T);
  if (v != E4B_OK) return v;
  const bool lora = d->lora_rank > 0;
  if ((lora_A != nullptr) != lora || (lora_B != nullptr) != lora || (dA != nullptr) != lora ||
      (dB != nullptr) != lora)
    return E4B_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, kAlign)) return E4B_ERR_INVALID_ARG;
  const TrainLayout L = train_layout(*d, T);
  if (ws_bytes < L.total) return E4B_ERR_INVALID_ARG;
  const bool dq = d->format == E4B_NF4_DQ;
  if (T > 0) {
    if (!logits || !dout || !gu_codes || !gu_scales || !dn_codes || !dn_scales || !dx || !dlogits)
      return E4B_ERR_INVALID_ARG;
    if (!aligned(dout, 8) || !aligned(dx, 16) || !aligned(dlogits, 4) || !aligned(gu_codes, 16) ||
        !aligned(dn_codes, 16))
      return E4B_ERR_INVALID_ARG;
    if (dq ? !(valid_dq(static_cast<const e4b_nf4_dq*>(gu_scales)) && valid_dq(static_cast<const e4b_nf4_dq*>(dn_scales)))
           : !(aligned(gu_scales, 16) && aligned(dn_scales, 16)))
      return E4B_ERR_INVALID_ARG;
    if (lora && (!aligned(lora_A, 2) || !aligned(lora_B, 16) || !aligned(dA, 4) || !aligned(dB, 4)))
      return E4B_ERR_INVALID_ARG;
  }
  BackwardLaunch b;
  b.T = T;
  b.k = d->k;
  b.E = d->E;
  b.H = d->H;
  b.I = d->I;
  b.fmt = gemm_format(d->format);
  b.gating = d->gating;
  b.lora_rank = d->lora_rank;
  b.lora_scale = d->lora_scale;
  b.ep = Epilogue{nullptr, d->act, d->glu_alpha, d->glu_limit, d->glu_beta};
  b.logits = logits;
  b.dout = dout;
  b.y = at<float>(ws, L.fwd.y);
  b.topk_w = at<float>(ws, L.fwd.topk_w);
  b.topk_ids = at<int32_t>(ws, L.fwd.topk_ids);
  b.slot_pos = at<int32_t>(ws, L.fwd.slot_pos);
  b.sorted_slot = at<int32_t>(ws, L.fwd.sorted_slot);
  b.expert_offsets = at<int32_t>(ws, L.fwd.offsets);
  b.x_sorted = at<uint16_t>(ws, L.fwd.x_sorted);
  b.xa = lora ? at<uint16_t>(ws, L.fwd.xa) : nullptr;
  b.G = at<float>(ws, L.g);
  b.dY = at<uint16_t>(ws, L.dY);
  b.dG = at<uint16_t>(ws, L.dG);
  b.dxa = lora ? at<float>(ws, L.dxa) : nullptr;
  b.dX = at<float>(ws, L.dX);
  b.dx = dx;
  b.dlogits = dlogits;
  b.dA = dA;
  b.dB = dB;
  b.gu_codes = gu_codes;
  b.dn_codes = dn_codes;
  // the nested-form absmax was expanded into the workspace by the training forward
  b.gu_scales = dq ? static_cast<const void*>(at<float>(ws, L.fwd.gu_absmax)) : gu_scales;
  b.dn_scales = dq ? static_cast<const void*>(at<float>(ws, L.fwd.dn_absmax)) : dn_scales;
  b.lora_A = lora_A;
  b.lora_B = lora_B;
  return launch_moe_backward(b, reinterpret_cast<cudaStream_t>(stream));
}

e4b_status e4b_device_status(void* ws, e4b_stream stream) {
  if (!ws || !aligned(ws, kAlign)) return E4B_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return E4B_ERR_CUDA;
  int32_t h[2] = {0, 0};
  if (cudaMemcpy(h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return E4B_ERR_CUDA;
  if (h[0] != 0 && cudaMemset(ws, 0, sizeof(h)) != cudaSuccess) return E4B_ERR_CUDA;
  return static_cast<e4b_status>(h[0]);
}

e4b_status e4b_debug_wait_timeout(uint32_t limit_ns, void* ws, size_t ws_bytes, e4b_stream stream) {
  if (!ws || !aligned(ws, kAlign) || ws_bytes < kStatusBytes || limit_ns > 1000000000u) return E4B_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, kStatusBytes, s) != cudaSuccess) return E4B_ERR_CUDA;
  wait_timeout_probe_kernel<<<1, 32, 0, s>>>(static_cast<int32_t*>(ws), limit_ns);
  return cudaGetLastError() == cudaSuccess ? E4B_OK : E4B_ERR_CUDA;
}

}  // extern "C"
