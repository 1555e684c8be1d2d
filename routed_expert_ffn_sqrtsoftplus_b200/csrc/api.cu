// Host runtime behind include/moe.h: argument validation, the handle (repacked
// weights + workspace), TMA descriptors, and the launch sequence of one layer
// invocation. Every step of the layer runs in this library's kernels.
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <utility>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/moe.h"
#include "common.cuh"
#include "kernels.h"

using namespace moe;

namespace {

// Token counts above this use the tensor-core router GEMM for the logits.
constexpr int kTcRouterMinTokens = 256;
// Token counts up to this use the sliced CUDA-core router and the per-token top-k.
constexpr int kSmallRouterMaxTokens = 32;
// Router logits of at most kSmallRouterMaxTokens tokens on the tensor cores (the
// dense grouped-GEMM mode, K split in slices of 128) (1), or on the CUDA cores,
// hidden-sliced (0). Measured at decode: the logits take half the time on the
// tensor cores, but the top-k then sums 40 slices instead of 5, and the step is
// the same.
#ifndef MOE_ROUTER_TC_SMALL
#define MOE_ROUTER_TC_SMALL 0
#endif
constexpr bool kRouterTcSmall = MOE_ROUTER_TC_SMALL != 0;
// Top-k with one CTA per token up to this many tokens (the candidates of a token
// are re-scored by 8 warps in parallel); one warp per token above (measured on
// B200: the CTA form halves the time at T=256 and is slower from T=2048 on).
constexpr int kTopkCtaMaxTokens = 1024;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// BF16 [rows, cols] row-major, 128-byte swizzled boxes of 64 columns x box_rows.
bool make_tmap_bf16(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

const char* kKernelNames[kKNumKinds] = {"router_logits", "router_gemm",  "topk_refine", "perm_count",
                                        "perm_scan",     "perm_scatter", "gather_rows", "gemm_gateup",
                                        "gemm_down",     "combine",      "quant_x",     "gemm_gateup_mx",
                                        "gemm_down_mx",  "swiglu_reduce", "hash_route",  "gemm_fused"};

// 2-D tensor map, box of box_cols x box_rows elements, 128-byte swizzle unless stated.
bool make_tmap(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, uint64_t rows, uint64_t cols,
               uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows,
               CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

struct moe_handle {
  moe_config cfg{};
  int device = 0;
  int num_sms = 148;
  int G = 0;       // routed + shared groups
  int64_t R = 0;   // max rows of h / O
  int nchunks_max = 0;
  int m_tiles_gu = 0, m_tiles_dn = 0;
  int64_t max_tiles_gu = 0, max_tiles_dn = 0;

  void* wg = nullptr;
  float* bias = nullptr;
  void* w13 = nullptr;
  void* w2 = nullptr;

  float* z = nullptr;
  float* zpart = nullptr;       // logit slices for T <= kSmallRouterMaxTokens
  int32_t* idx = nullptr;
  float* wts = nullptr;
  int32_t* chunk_cnt = nullptr;
  int32_t* cnt = nullptr;
  int32_t* off = nullptr;
  int32_t* perm = nullptr;
  int32_t* inv = nullptr;
  int4* tiles_gu = nullptr;
  int4* tiles_dn = nullptr;
  int* ntiles = nullptr;
  void* xp = nullptr;
  void* h = nullptr;
  float* o = nullptr;
  int* status = nullptr;
  void* x_stage = nullptr;
  void* y_stage = nullptr;
  // pipelined host path (moe_forward_host_async), set up on first use: slot 0 stages
  // through x_stage / y_stage, slot 1 through buffers of its own
  bool pipe_ready = false;
  cudaStream_t pipe_in = nullptr, pipe_out = nullptr;  // host-to-device and device-to-host copies
  cudaEvent_t pipe_copied_in[2] = {nullptr, nullptr};  // x of the slot on the device
  cudaEvent_t pipe_done[2] = {nullptr, nullptr};       // the layer finished with the slot's x and y
  cudaEvent_t pipe_copied_out[2] = {nullptr, nullptr}; // y of the slot on the host
  void* pipe_x[2] = {nullptr, nullptr};
  void* pipe_y[2] = {nullptr, nullptr};
  int pipe_slot = 0;
  uint64_t pipe_bytes = 0;

  CUtensorMap tm_w13, tm_w2, tm_xp, tm_h, tm_wg;
  CUtensorMap tm_w2w;           // W2 with 256-row boxes (wide down tiles)
  bool wide_ok = false;         // H % 256 == 0

  // MXFP4 routed experts (expert_dtype == MOE_DT_MXFP4)
  bool mx = false;              // routed experts block-scaled (MXFP4 or MXFP8)
  bool a8 = false;              // ... and MXFP8 (E4M3 weights, one byte per value)
  int e_begin = 0, e_local = 0; // routed experts held: [e_begin, e_begin + e_local) of cfg.n_routed
  uint8_t* w13q = nullptr;      // packed E2M1, gate/up tile order
  uint8_t* w2q = nullptr;       // packed E2M1
  uint8_t* sfa13 = nullptr;     // scale atoms of W1|W3
  uint8_t* sfa2 = nullptr;      // scale atoms of W2
  void* w13sh = nullptr;        // shared experts, BF16
  void* w2sh = nullptr;
  uint8_t* xq = nullptr;        // MXFP8 routed token rows
  uint8_t* hq = nullptr;        // MXFP8 routed h rows
  uint8_t* sfb_gu = nullptr;    // activation scale atoms, gate/up token tiles
  uint8_t* sfb_dn = nullptr;    // h scale atoms, down token tiles
  int32_t* ntile_base_gu = nullptr;
  int* bn_choice = nullptr;     // token-tile width the permutation chose (many-token BF16 path)
  int* sched = nullptr;         // tile counters of the dual-width GEMMs (gate/up wide, thin; down wide, thin)
  int32_t* ntile_base_dn = nullptr;
  int* bad = nullptr;
  int* bad_flag = nullptr;      // device flag of the hash-table check
  int* done = nullptr;          // per-group gate/up completion counters of the fused GEMM
  int64_t max_ntiles_r = 0;
  CUtensorMap tm_w13q, tm_w2q, tm_w2qw, tm_xq, tm_hq, tm_w13sh, tm_w2sh, tm_w2shw;
  // shared experts alone (MXFP4 layers, few tokens): split-K partial sums
  float* sh_parts_gu = nullptr;  // [S][ks_gu][T][2I]
  float* sh_parts_dn = nullptr;  // [S][ks_dn][T][H]
  int ks_gu = 1, ks_dn = 1;

  // hash-routed layers: the vocabulary table [hash_vocab, k] (library copy), or none
  int32_t* hash_table = nullptr;
  int32_t hash_vocab = 0;

  uint64_t timeout_ns = 2000000000ull;
  std::vector<void*> allocs;
  std::vector<std::pair<void*, size_t>> ws_allocs;  // per-forward scratch (moe_fill_workspace)
  int fail_after = -1;          // test hook: allocations allowed before one is made to fail (-1: off)
  int nvtx_open = 0;            // NVTX kernel ranges pushed and not yet popped
  uint64_t weight_bytes = 0, workspace_bytes = 0;
  int last_T = 0;

  // profiling
  bool prof_on = false;
  std::vector<cudaEvent_t> ev;  // pairs
  std::vector<int> ev_kind;
  size_t ev_used = 0;

  template <class T>
  bool alloc(T** p, size_t bytes, uint64_t* counter) {
    void* q = nullptr;
    if (bytes == 0) bytes = 16;
    if (fail_after == 0) return false;
    if (fail_after > 0) --fail_after;
    if (cudaMalloc(&q, bytes) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    allocs.push_back(q);
    *p = static_cast<T*>(q);
    *counter += bytes;
    if (counter == &workspace_bytes) ws_allocs.emplace_back(q, bytes);
    return true;
  }

  void release() {
    for (void* p : allocs) cudaFree(p);
    allocs.clear();
    for (int i = 0; i < 2; ++i) {
      if (pipe_copied_in[i]) cudaEventDestroy(pipe_copied_in[i]);
      if (pipe_done[i]) cudaEventDestroy(pipe_done[i]);
      if (pipe_copied_out[i]) cudaEventDestroy(pipe_copied_out[i]);
      pipe_copied_in[i] = pipe_done[i] = pipe_copied_out[i] = nullptr;
    }
    if (pipe_in) cudaStreamDestroy(pipe_in);
    if (pipe_out) cudaStreamDestroy(pipe_out);
    pipe_in = pipe_out = nullptr;
    pipe_ready = false;
    if (hash_table != nullptr) cudaFree(hash_table);
    hash_table = nullptr;
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
    ev.clear();
  }

  void prof_mark(int kind, cudaStream_t s) {
    nvtxRangePushA(kKernelNames[kind]);
    ++nvtx_open;
    if (!prof_on || ev_used + 2 > ev.size()) return;
    cudaEventRecord(ev[ev_used], s);
    ev_kind[ev_used / 2] = kind;
  }
  void prof_done(cudaStream_t s) {
    if (nvtx_open > 0) {
      nvtxRangePop();
      --nvtx_open;
    }
    if (!prof_on || ev_used + 2 > ev.size()) return;
    cudaEventRecord(ev[ev_used + 1], s);
    ev_used += 2;
  }
};

namespace {

// Largest divisor of n that is <= cap.
int divisor_at_most(int n, int cap) {
  for (int d = cap; d > 1; --d)
    if (n % d == 0) return d;
  return 1;
}

moe_status validate_config(const moe_config* c) {
  if (!(c->route_scale > 0.f) || !std::isfinite(c->route_scale)) return MOE_ERR_INVALID_ARG;
  if (std::isnan(c->swiglu_limit) || c->swiglu_limit < 0.f) return MOE_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->inter <= 0 || c->n_routed <= 0 || c->top_k <= 0 || c->max_tokens <= 0 ||
      c->n_shared < 0)
    return MOE_ERR_INVALID_ARG;
  if (c->top_k > c->n_routed) return MOE_ERR_INVALID_ARG;
  if (c->hidden % 128 != 0 || c->inter % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (c->n_routed > 512 || c->top_k > 32 || c->n_shared > 4 || c->max_tokens > 65536) return MOE_ERR_UNSUPPORTED;
  if (c->hidden > 16384 || c->inter > 16384) return MOE_ERR_UNSUPPORTED;
  if (c->expert_dtype != MOE_DT_BF16 && c->expert_dtype != MOE_DT_MXFP4 && c->expert_dtype != MOE_DT_MXFP8)
    return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

#define MOE_TRY_CUDA(expr)                 \
  do {                                     \
    if ((expr) != cudaSuccess) {           \
      cudaGetLastError();                  \
      return MOE_ERR_CUDA;                 \
    }                                      \
  } while (0)

}  // namespace

extern "C" {

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_OOM: return "MOE_ERR_OOM";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
  }
  return "MOE_ERR_UNKNOWN";
}

int32_t moe_num_kernel_kinds(void) { return kKNumKinds; }

const char* moe_kernel_name(int32_t kind) {
  if (kind < 0 || kind >= kKNumKinds) return nullptr;
  return kKernelNames[kind];
}

}  // extern "C"

namespace {

// A layer instance holding the routed experts [e_begin, e_begin + e_count) of the
// router's n_routed (all of them for moe_create; a window for moe_create_ep).
moe_status create_impl(const moe_config* cfg, const moe_weights* w, int32_t e_begin, int32_t e_count,
                       moe_stream_t stream, moe_handle** out) {
  if (out == nullptr) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (cfg == nullptr || w == nullptr) return MOE_ERR_INVALID_ARG;
  moe_status st = validate_config(cfg);
  if (st != MOE_OK) return st;
  if (e_begin < 0 || e_count < 1 || e_begin > cfg->n_routed - e_count) return MOE_ERR_INVALID_ARG;
  const bool mx = cfg->expert_dtype == MOE_DT_MXFP4 || cfg->expert_dtype == MOE_DT_MXFP8;
  const bool a8 = cfg->expert_dtype == MOE_DT_MXFP8;
  const void* req[] = {w->router_w, w->w1, w->w3, w->w2};
  for (const void* p : req)
    if (p == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  if (mx && (w->s1 == nullptr || w->s3 == nullptr || w->s2 == nullptr)) return MOE_ERR_INVALID_ARG;
  if (cfg->n_shared > 0) {
    const void* sh[] = {w->sh_w1, w->sh_w3, w->sh_w2};
    for (const void* p : sh)
      if (p == nullptr || !aligned16(p)) return MOE_ERR_INVALID_ARG;
  }
  if (w->router_bias != nullptr && !aligned16(w->router_bias)) return MOE_ERR_INVALID_ARG;
  {
    // the repacking kernels read the weights on the current device
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return MOE_ERR_CUDA;
    const void* all[] = {w->router_w, w->router_bias, w->w1, w->w3, w->w2, w->s1, w->s3, w->s2,
                         w->sh_w1, w->sh_w3, w->sh_w2};
    for (const void* p : all)
      if (p != nullptr && !device_pointer_on(p, cur)) return MOE_ERR_INVALID_ARG;
  }
  if (get_encode_fn() == nullptr) return MOE_ERR_CUDA;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  moe_handle* h = new (std::nothrow) moe_handle();
  if (h == nullptr) return MOE_ERR_OOM;
  h->cfg = *cfg;
  if (const char* f = std::getenv("MOE_TEST_FAIL_ALLOC_AFTER")) h->fail_after = std::atoi(f);
  h->mx = mx;
  h->a8 = a8;
  h->e_begin = e_begin;
  h->e_local = e_count;
  if (cudaGetDevice(&h->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess ||
      gemm_set_attributes() != cudaSuccess || gemm_mx_set_attributes() != cudaSuccess ||
      router_set_attributes() != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return MOE_ERR_CUDA;
  }
  // E: the router's experts; El: the routed experts this instance holds
  const int64_t H = cfg->hidden, I = cfg->inter, E = cfg->n_routed, El = e_count, S = cfg->n_shared,
                k = cfg->top_k, Tm = cfg->max_tokens;
  h->G = static_cast<int>(El + S);
  h->R = Tm * k + S * Tm;
  h->nchunks_max = static_cast<int>((Tm * k + kPermChunk - 1) / kPermChunk);
  h->m_tiles_gu = static_cast<int>(I / 128);
  h->m_tiles_dn = static_cast<int>(H / 128);
  h->max_tiles_gu = h->m_tiles_gu * (h->G + (h->R + 31) / 32);
  h->max_tiles_dn = h->m_tiles_dn * (h->G + (h->R + 31) / 32);
  h->max_ntiles_r = El + (Tm * k + 31) / 32;

  bool ok = true;
  uint64_t* wb = &h->weight_bytes;
  uint64_t* ws = &h->workspace_bytes;
  ok = ok && h->alloc(&h->wg, E * H * 2, wb);
  if (w->router_bias) ok = ok && h->alloc(&h->bias, E * 4, wb);
  if (!mx) {
    ok = ok && h->alloc(&h->w13, (El + S) * 2 * I * H * 2, wb);
    ok = ok && h->alloc(&h->w2, (El + S) * H * I * 2, wb);
    if (!kGatherX) ok = ok && h->alloc(&h->xp, Tm * k * H * 2, ws);
  } else {
    ok = ok && h->alloc(&h->w13q, El * 2 * I * (a8 ? H : H / 2), wb);
    ok = ok && h->alloc(&h->w2q, El * H * (a8 ? I : I / 2), wb);
    ok = ok && h->alloc(&h->sfa13, El * (I / 128) * (H / 128) * 1024, wb);
    ok = ok && h->alloc(&h->sfa2, El * (H / 128) * (I / 128) * 512, wb);
    if (S > 0) {
      ok = ok && h->alloc(&h->w13sh, S * 2 * I * H * 2, wb);
      ok = ok && h->alloc(&h->w2sh, S * H * I * 2, wb);
    }
    ok = ok && h->alloc(&h->xq, Tm * k * H, ws);
    ok = ok && h->alloc(&h->hq, Tm * k * I, ws);
    ok = ok && h->alloc(&h->sfb_gu, h->max_ntiles_r * (H / 128) * 512, ws);
    ok = ok && h->alloc(&h->sfb_dn, h->max_ntiles_r * (I / 128) * 512, ws);
    ok = ok && h->alloc(&h->ntile_base_gu, (El + 1) * 4, ws);
    ok = ok && h->alloc(&h->ntile_base_dn, (El + 1) * 4, ws);
    ok = ok && h->alloc(&h->bad, 16, ws);
    if (S > 0) {
      const int64_t tsmall = Tm < kSmallRouterMaxTokens ? Tm : kSmallRouterMaxTokens;
      h->ks_gu = divisor_at_most(static_cast<int>(H / 64), 8);
      h->ks_dn = divisor_at_most(static_cast<int>(I / 64), 4);
      ok = ok && h->alloc(&h->sh_parts_gu, S * h->ks_gu * tsmall * 2 * I * 4, ws);
      ok = ok && h->alloc(&h->sh_parts_dn, S * h->ks_dn * tsmall * H * 4, ws);
    }
  }
  ok = ok && h->alloc(&h->z, Tm * E * 4, ws);
  ok = ok && h->alloc(&h->zpart, (H / 128) * (Tm < kSmallRouterMaxTokens ? Tm : kSmallRouterMaxTokens) * E * 4, ws);
  ok = ok && h->alloc(&h->idx, Tm * k * 4, ws);
  ok = ok && h->alloc(&h->wts, Tm * k * 4, ws);
  ok = ok && h->alloc(&h->chunk_cnt, static_cast<size_t>(h->nchunks_max) * El * 4, ws);
  ok = ok && h->alloc(&h->cnt, (El + S) * 4, ws);
  ok = ok && h->alloc(&h->off, (El + S + 1) * 4, ws);
  ok = ok && h->alloc(&h->perm, Tm * k * 4, ws);
  ok = ok && h->alloc(&h->inv, Tm * k * 4, ws);
  ok = ok && h->alloc(&h->bn_choice, 16, ws);
  ok = ok && h->alloc(&h->sched, 16, ws);
  ok = ok && h->alloc(&h->tiles_gu, h->max_tiles_gu * 16, ws);
  ok = ok && h->alloc(&h->tiles_dn, h->max_tiles_dn * 16, ws);
  ok = ok && h->alloc(&h->ntiles, 32, ws);   // 4 tile counts, the routed row count, 2 thin-tile starts
  ok = ok && h->alloc(&h->h, h->R * I * 2, ws);
  ok = ok && h->alloc(&h->o, h->R * H * 4, ws);
  ok = ok && h->alloc(&h->status, 16, ws);
  ok = ok && h->alloc(&h->bad_flag, 16, ws);
  ok = ok && h->alloc(&h->done, (El + S) * 4, ws);
  ok = ok && h->alloc(&h->x_stage, Tm * H * 2, ws);
  ok = ok && h->alloc(&h->y_stage, Tm * H * 2, ws);
  if (!ok) {
    h->release();
    delete h;
    return MOE_ERR_OOM;
  }

  bool err = false;
  err |= cudaMemsetAsync(h->status, 0, 16, s) != cudaSuccess;
  err |= cudaMemsetAsync(h->ntiles, 0, 32, s) != cudaSuccess;
  err |= cudaMemcpyAsync(h->wg, w->router_w, E * H * 2, cudaMemcpyDeviceToDevice, s) != cudaSuccess;
  if (w->router_bias) err |= cudaMemcpyAsync(h->bias, w->router_bias, E * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess;
  if (!mx) {
    err |= launch_repack_w13(w->w1, w->w3, w->sh_w1, w->sh_w3, static_cast<int>(El), static_cast<int>(S),
                             static_cast<int>(I), static_cast<int>(H), h->w13, s) != cudaSuccess;
    err |= cudaMemcpyAsync(h->w2, w->w2, El * H * I * 2, cudaMemcpyDeviceToDevice, s) != cudaSuccess;
    if (S > 0)
      err |= cudaMemcpyAsync(static_cast<uint8_t*>(h->w2) + El * H * I * 2, w->sh_w2, S * H * I * 2,
                             cudaMemcpyDeviceToDevice, s) != cudaSuccess;
    err |= !make_tmap_bf16(&h->tm_w13, h->w13, (El + S) * 2 * I, H, 256);
    err |= !make_tmap_bf16(&h->tm_w2, h->w2, (El + S) * H, I, 128);
    h->wide_ok = H % 256 == 0;
    if (h->wide_ok) err |= !make_tmap_bf16(&h->tm_w2w, h->w2, (El + S) * H, I, 256);
    if (!kGatherX) err |= !make_tmap_bf16(&h->tm_xp, h->xp, Tm * k, H, 32);
  } else {
    err |= cudaMemsetAsync(h->bad, 0, 16, s) != cudaSuccess;
    err |= launch_repack_w13_bytes(w->w1, w->w3, nullptr, nullptr, static_cast<int>(El), 0, static_cast<int>(I),
                                   static_cast<int>(a8 ? H : H / 2), h->w13q, s) != cudaSuccess;
    err |= cudaMemcpyAsync(h->w2q, w->w2, El * H * (a8 ? I : I / 2), cudaMemcpyDeviceToDevice, s) != cudaSuccess;
    err |= launch_sf_atoms(w->s1, w->s3, static_cast<int>(El), static_cast<int>(I), static_cast<int>(H), h->sfa13,
                           h->bad, s) != cudaSuccess;
    err |= launch_sf_atoms(w->s2, nullptr, static_cast<int>(El), static_cast<int>(H), static_cast<int>(I), h->sfa2,
                           h->bad, s) != cudaSuccess;
    if (S > 0) {
      err |= launch_repack_w13(nullptr, nullptr, w->sh_w1, w->sh_w3, 0, static_cast<int>(S), static_cast<int>(I),
                               static_cast<int>(H), h->w13sh, s) != cudaSuccess;
      err |= cudaMemcpyAsync(h->w2sh, w->sh_w2, S * H * I * 2, cudaMemcpyDeviceToDevice, s) != cudaSuccess;
      err |= !make_tmap_bf16(&h->tm_w13sh, h->w13sh, S * 2 * I, H, 256);
      err |= !make_tmap_bf16(&h->tm_w2sh, h->w2sh, S * H, I, 128);
      // 256-row W2 boxes: the shared groups share the down tile list with the
      // routed ones, whose tiles are 256 rows of W2 when H % 256 == 0
      if (H % 256 == 0) err |= !make_tmap_bf16(&h->tm_w2shw, h->w2sh, S * H, I, 256);
    }
    // MXFP4: packed E2M1 pairs, unpacked by the TMA to one value per byte in shared
    // memory; MXFP8: E4M3 bytes as stored. Either way 128 values = 128 smem bytes per row.
    // (With packed staging the MXFP4 weights are plain bytes: 64 per row per K step,
    // unswizzled, and the kernel's expander warps lay them out for the MMA.)
    if (!a8 && kMxPacked) {
      const CUtensorMapDataType u8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
      const CUtensorMapSwizzle none = CU_TENSOR_MAP_SWIZZLE_NONE;
      err |= !make_tmap(&h->tm_w13q, h->w13q, u8, El * 2 * I, H / 2, H / 2, 64, 256, none);
      err |= !make_tmap(&h->tm_w2q, h->w2q, u8, El * H, I / 2, I / 2, 64, 128, none);
      h->wide_ok = H % 256 == 0;
      if (h->wide_ok) err |= !make_tmap(&h->tm_w2qw, h->w2q, u8, El * H, I / 2, I / 2, 64, 256, none);
    } else {
      const CUtensorMapDataType wdt = a8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B;
      err |= !make_tmap(&h->tm_w13q, h->w13q, wdt, El * 2 * I, H, a8 ? H : H / 2, 128, 256);
      err |= !make_tmap(&h->tm_w2q, h->w2q, wdt, El * H, I, a8 ? I : I / 2, 128, 128);
      h->wide_ok = H % 256 == 0;
      if (h->wide_ok) err |= !make_tmap(&h->tm_w2qw, h->w2q, wdt, El * H, I, a8 ? I : I / 2, 128, 256);
    }
    err |= !make_tmap(&h->tm_xq, h->xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, Tm * k, H, H, 128, 32);
    err |= !make_tmap(&h->tm_hq, h->hq, CU_TENSOR_MAP_DATA_TYPE_UINT8, Tm * k, I, I, 128, 32);
  }
  err |= !make_tmap_bf16(&h->tm_h, h->h, h->R, I, 32);
  err |= !make_tmap_bf16(&h->tm_wg, h->wg, E, H, 128);
  if (!err && mx) {
    // NaN scale codes (0xFF) are rejected: check what the atom packer saw.
    int bad = 0;
    err |= cudaMemcpyAsync(&bad, h->bad, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess;
    err |= cudaStreamSynchronize(s) != cudaSuccess;
    if (!err && bad) {
      h->release();
      delete h;
      return MOE_ERR_INVALID_ARG;
    }
  }
  if (err) {
    cudaGetLastError();
    cudaStreamSynchronize(s);
    h->release();
    delete h;
    return MOE_ERR_CUDA;
  }
  *out = h;
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_create(const moe_config* cfg, const moe_weights* w, moe_stream_t stream, moe_handle** out) {
  return create_impl(cfg, w, 0, cfg != nullptr ? cfg->n_routed : 0, stream, out);
}

moe_status moe_create_ep(const moe_config* cfg, const moe_weights* w, int32_t expert_begin, int32_t expert_count,
                         moe_stream_t stream, moe_handle** out) {
  return create_impl(cfg, w, expert_begin, expert_count, stream, out);
}

}  // extern "C"

namespace {

// One layer invocation; token_ids != nullptr selects the hash routing of the
// handle's table instead of the learned router and top-k.
// y_f32: y is fp32 [T, H] and receives this instance's partial output (its expert
// window's slots, plus the shared experts it holds), else BF16 [T, H].
moe_status forward_impl(moe_handle* h, const void* x, const int32_t* token_ids, int32_t T, void* y, bool y_f32,
                        int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
  if (h == nullptr) return MOE_ERR_INVALID_ARG;
  if (T < 0 || T > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (T == 0) {
    h->last_T = 0;
    return MOE_OK;
  }
  if (x == nullptr || y == nullptr || !aligned16(x) || !aligned16(y) || x == y) return MOE_ERR_INVALID_ARG;
  {
    // kernels launch on the current device and read x / write y directly
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess || cur != h->device) return MOE_ERR_INVALID_ARG;
    if (!device_pointer_on(x, h->device) || !device_pointer_on(y, h->device)) return MOE_ERR_INVALID_ARG;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // NVTX: one range per forward and one per kernel launch (the kernel ranges of a
  // launch that failed are closed here too)
  struct ForwardRange {
    moe_handle* h;
    explicit ForwardRange(moe_handle* hh, bool hashed) : h(hh) {
      nvtxRangePushA(hashed ? "moe_forward_hashed" : "moe_forward");
    }
    ~ForwardRange() {
      for (; h->nvtx_open > 0; --h->nvtx_open) nvtxRangePop();
      nvtxRangePop();
    }
  } range(h, token_ids != nullptr);
  const moe_config& c = h->cfg;
  // E: the router's experts; El: the routed expert groups this instance holds,
  // experts [eb, eb + El)
  const int H = c.hidden, I = c.inter, E = c.n_routed, S = c.n_shared, k = c.top_k;
  const int El = h->e_local, eb = h->e_begin;
  const int nslots = T * k;
  const int nchunks = (nslots + kPermChunk - 1) / kPermChunk;
  // Token tiles. Few tokens: 32-row tiles and deep smem rings (weight streaming).
  // Many tokens per expert: kBnLarge-row tiles so each weight tile is read once
  // (one TMEM accumulator for gate/up).
  const bool small = T <= 32;
  const bool large = !small && static_cast<int64_t>(T) * k >= 24LL * E;
  const int bn_gu = small ? 32 : (large ? kBnLarge : 128);   // BF16 token tiles
  const int bn_dn = small ? 32 : kBnLarge;
  const bool wide = large && h->wide_ok && !h->mx;      // 256-row W2 tiles
  const bool wide_small = small && h->wide_ok && !h->mx;  // 256-row W2 tiles, 32-token tiles
  // many tokens per expert, BF16: the permutation picks kBnAlt-row tiles (a deeper
  // ring, one tile per expert) when no routed expert has more rows than that, else
  // kBnLarge; one dual-width launch per GEMM runs the chosen body
  const bool alt = kBnAlt > 0 && wide;
  const int bn_mx = small ? 32 : (large ? kBnMxLarge : 64);  // MXFP4 token tiles (gate/up and down)

  CUtensorMap tm_x;
  if (!make_tmap_bf16(&tm_x, x, static_cast<uint64_t>(T), static_cast<uint64_t>(H), 32)) return MOE_ERR_CUDA;

  // 1-2. router logits (+ bias), scores, top-k, weights
  if (token_ids != nullptr) {
    h->prof_mark(kKHashRoute, s);
    MOE_TRY_CUDA(launch_hash_route(x, h->wg, h->bias, h->hash_table, token_ids, T, H, E, k, h->hash_vocab,
                                   c.route_scale, h->idx, h->wts, h->status, s));
    h->prof_done(s);
  } else if (T <= kSmallRouterMaxTokens) {
    int nparts = 0;
    if (kRouterTcSmall) {
      // the logits on the tensor cores: 128-expert x 32-token tiles, K cut into
      // H / 128 slices of two K blocks, each slice's fp32 partial sums a slice of zpart
      GemmArgs a{};
      a.dense_m_tiles = (E + 127) / 128;
      a.dense_rows = T;
      a.num_kb = H / 64;
      a.dense_k_splits = H / 128;
      a.split_stride = static_cast<size_t>(T) * E;
      a.out = h->zpart;
      a.out_ld = E;
      a.out_rows = T;
      a.m_limit = E;
      a.status = h->status;
      a.timeout_ns = h->timeout_ns;
      const int nt = a.dense_m_tiles * a.dense_k_splits;
      h->prof_mark(kKRouterGemm, s);
      MOE_TRY_CUDA(launch_gemm_down(h->tm_wg, tm_x, a, 32, nt < h->num_sms ? nt : h->num_sms, s));
      h->prof_done(s);
      nparts = a.dense_k_splits;
    } else {
      h->prof_mark(kKRouterLogits, s);
      MOE_TRY_CUDA(launch_router_small(x, h->wg, h->zpart, T, H, E, s));
      h->prof_done(s);
      nparts = H / router_small_slice(H);
    }
    h->prof_mark(kKTopk, s);
    MOE_TRY_CUDA(launch_topk_small(h->zpart, nparts, x, h->wg, h->bias, T, H, E, k, c.route_scale, kRefineDelta,
                                   h->idx, h->wts, h->z, h->status, s, h->bias));
    h->prof_done(s);
  } else if (T < kTcRouterMinTokens) {
    h->prof_mark(kKRouterLogits, s);
    MOE_TRY_CUDA(launch_router_logits(x, h->wg, h->bias, h->z, T, H, E, s));
    h->prof_done(s);
  } else {
    GemmArgs a{};
    a.dense_m_tiles = (E + 127) / 128;
    a.dense_rows = T;
    a.num_kb = H / 64;
    a.out = h->z;
    a.out_ld = E;
    a.out_rows = T;
    a.m_limit = E;
    a.col_bias = h->bias;
    a.status = h->status;
    a.timeout_ns = h->timeout_ns;
    const int nt = a.dense_m_tiles * ((T + kBnLarge - 1) / kBnLarge);
    h->prof_mark(kKRouterGemm, s);
    MOE_TRY_CUDA(launch_gemm_down(h->tm_wg, tm_x, a, kBnLarge, nt < h->num_sms ? nt : h->num_sms, s));
    h->prof_done(s);
  }
  if (token_ids == nullptr && T > kSmallRouterMaxTokens) {
    // scores, top-k with exact refinement of the near-tie candidates, weights
    h->prof_mark(kKTopk, s);
    if (T <= kTopkCtaMaxTokens) {
      // one CTA per token: the logits (bias included) are a single slice; the
      // exact re-scoring adds the bias itself
      MOE_TRY_CUDA(launch_topk_small(h->z, 1, x, h->wg, nullptr, T, H, E, k, c.route_scale, kRefineDelta, h->idx,
                                     h->wts, nullptr, h->status, s, h->bias));
    } else {
      // one warp per token: with thousands of tokens the warps keep every SM busy
      MOE_TRY_CUDA(launch_topk_refine(h->z, x, h->wg, h->bias, T, H, E, k, c.route_scale, kRefineDelta, h->idx,
                                      h->wts, h->status, s));
    }
    h->prof_done(s);
  }
  // 3. permutation and tile lists
  if (nchunks > 1) {
    h->prof_mark(kKPermCount, s);
    MOE_TRY_CUDA(launch_perm_count(h->idx, nslots, El, eb, E, h->chunk_cnt, h->status, s));
    h->prof_done(s);
  }
  ScanArgs sa{};
  sa.chunk_cnt = h->chunk_cnt;
  sa.nchunks = nchunks;
  sa.E = El;
  sa.e_begin = eb;
  sa.e_global = E;
  sa.S = S;
  sa.T = T;
  sa.k = k;
  sa.cnt = h->cnt;
  sa.off = h->off;
  sa.tiles_gu = h->tiles_gu;
  sa.tiles_dn = h->tiles_dn;
  sa.ntiles = h->ntiles;
  sa.m_tiles_gu = h->m_tiles_gu;
  const bool wide_mx = h->mx && h->wide_ok;             // 256-row MXFP4 W2 tiles
  sa.m_tiles_dn = (wide || wide_small || wide_mx) ? H / 256 : h->m_tiles_dn;
  sa.bn_gu_r = h->mx ? bn_mx : bn_gu;
  sa.bn_dn_r = h->mx ? bn_mx : bn_dn;
  sa.bn_gu_s = bn_gu;
  sa.bn_dn_s = bn_dn;
  sa.mx = h->mx ? 1 : 0;
  sa.ntile_base_gu = h->ntile_base_gu;
  sa.ntile_base_dn = h->ntile_base_dn;
  // with few tokens every tile streams the same weight bytes and its rows cost
  // next to nothing: the order of the partial tiles does not matter
  sa.sort_partial = small ? 0 : 1;
  // few tokens, BF16: gate/up and down in one persistent launch
  const bool fused = kFusedDecode && !kGatherX && !h->mx && wide_small;
  sa.done = fused ? h->done : nullptr;
  sa.nrows_routed = h->ntiles + 4;
  sa.bn_alt = alt ? kBnAlt : 0;
  sa.bn_choice = alt ? h->bn_choice : nullptr;
  sa.sched_zero = alt ? h->sched : nullptr;
  if (nchunks == 1) {
    h->prof_mark(kKPermScan, s);
    MOE_TRY_CUDA(launch_perm_fused(sa, h->idx, nslots, h->perm, h->inv, h->status, s));
    h->prof_done(s);
  } else {
    h->prof_mark(kKPermScan, s);
    MOE_TRY_CUDA(launch_perm_scan(sa, s));
    h->prof_done(s);
    h->prof_mark(kKPermScatter, s);
    MOE_TRY_CUDA(launch_perm_scatter(h->idx, nslots, El, eb, h->chunk_cnt, h->perm, h->inv, s));
    h->prof_done(s);
  }

  if (!h->mx) {
    // 4. gate/up grouped GEMM with the clamped SwiGLU epilogue (routed and shared
    // groups). The routed token rows come straight from x through the permutation
    // (tile::gather4 on a one-row-box map of x), or from a gathered copy.
    CUtensorMap tm_xg;
    if (kGatherX) {
      if (!make_tmap_bf16(&tm_xg, x, static_cast<uint64_t>(T), static_cast<uint64_t>(H), 1)) return MOE_ERR_CUDA;
    } else {
      h->prof_mark(kKGather, s);
      MOE_TRY_CUDA(launch_gather_rows(x, h->perm, nslots, h->ntiles + 4, k, H, h->xp, s));
      h->prof_done(s);
    }
    const CUtensorMap& tm_b = kGatherX ? tm_xg : h->tm_xp;
    GemmArgs a{};
    if (kGatherX) {
      a.gather_perm = h->perm;
      a.gather_k = k;
    }
    a.tiles = h->tiles_gu;
    a.ntiles = h->ntiles;
    a.num_kb = H / 64;
    a.a_rows_per_group = 2 * I;
    a.n_routed = El;
    a.out = h->h;
    a.out_ld = I;
    a.out_rows = static_cast<int>(h->R);
    a.m_limit = I;
    a.limit = c.swiglu_limit;
    a.status = h->status;
    a.timeout_ns = h->timeout_ns;
    if (!fused) {
      h->prof_mark(kKGateUp, s);
      if (alt) {
        a.bn_select = h->bn_choice;
        a.thin_begin = h->ntiles + 5;
        a.sched = h->sched;
        MOE_TRY_CUDA(launch_gemm_gateup_dual(h->tm_w13, tm_b, tm_x, a, h->num_sms, s));
      } else {
        MOE_TRY_CUDA(launch_gemm_gateup(h->tm_w13, tm_b, tm_x, a, bn_gu, h->num_sms, s));
      }
      h->prof_done(s);
    }
    // 5. down grouped GEMM
    GemmArgs d{};
    d.tiles = h->tiles_dn;
    d.ntiles = h->ntiles + 1;
    d.num_kb = I / 64;
    d.a_rows_per_group = H;
    d.n_routed = El;
    d.out = h->o;
    d.out_ld = H;
    d.out_rows = static_cast<int>(h->R);
    d.m_limit = H;
    d.status = h->status;
    d.timeout_ns = h->timeout_ns;
    if (fused) {
      // 4-5 together: the down tiles of a group start once its gate/up tiles are done
      FusedArgs f{};
      f.gu = a;
      f.dn = d;
      f.done = h->done;
      f.cnt = h->cnt;
      f.m_tiles_gu = h->m_tiles_gu;
      h->prof_mark(kKGemmFused, s);
      MOE_TRY_CUDA(launch_gemm_fused_small(h->tm_w13, tm_b, tm_x, h->tm_w2w, h->tm_h, f, h->num_sms, s));
    } else if (alt) {
      h->prof_mark(kKDown, s);
      d.bn_select = h->bn_choice;
      d.thin_begin = h->ntiles + 6;
      d.sched = h->sched + 2;
      MOE_TRY_CUDA(launch_gemm_down_wide_dual(h->tm_w2w, h->tm_h, d, h->num_sms, s));
    } else {
      h->prof_mark(kKDown, s);
      MOE_TRY_CUDA(launch_gemm_down(wide || wide_small ? h->tm_w2w : h->tm_w2, h->tm_h, d, bn_dn, h->num_sms, s,
                                    wide || wide_small));
    }
    h->prof_done(s);
  } else {
    // MXFP8 token rows of the routed slots
    h->prof_mark(kKQuantX, s);
    MOE_TRY_CUDA(launch_quant_gather_mx(x, h->perm, h->idx, h->off, h->ntile_base_gu, nslots, h->ntiles + 4, k, H,
                                        bn_mx, eb, El, h->xq, h->sfb_gu, s));
    h->prof_done(s);
    // 4a. routed gate/up on block-scaled MMAs (tiles after the shared ones)
    MxGemmArgs g{};
    g.tiles = h->tiles_gu;
    g.ntiles = h->ntiles;
    g.tile_begin = h->ntiles + 2;
    g.num_kb = H / 128;
    g.a_rows_per_group = 2 * I;
    g.m_tiles = I / 128;
    g.sfa = h->sfa13;
    g.sfb = h->sfb_gu;
    g.out = h->hq;
    g.out_ld = I;
    g.out_rows = T * k;
    g.m_limit = I;
    g.limit = c.swiglu_limit;
    g.sf_out = h->sfb_dn;
    g.sf_out_kb4 = I / 128;
    g.bn_dn = bn_mx;
    g.group_off = h->off;
    g.dn_ntile_base = h->ntile_base_dn;
    g.status = h->status;
    g.timeout_ns = h->timeout_ns;
    g.a_base = h->w13q;
    g.a_row_bytes = h->a8 ? H : H / 2;
    h->prof_mark(kKGateUpMx, s);
    MOE_TRY_CUDA(launch_gemm_mx_gateup(h->tm_w13q, h->tm_xq, g, bn_mx, h->num_sms, s, h->a8));
    h->prof_done(s);
    // 4b. shared experts' gate/up in BF16. With few tokens the shared expert has
    // only I/128 weight tiles: split K so every SM streams part of it, then sum
    // the slices and apply the SwiGLU.
    const bool sh_split = S > 0 && T <= kSmallRouterMaxTokens;
    if (sh_split) {
      for (int j = 0; j < S; ++j) {
        GemmArgs a{};
        a.dense_m_tiles = I / 128;
        a.dense_rows = T;
        a.dense_k_splits = h->ks_gu;
        a.num_kb = H / 64;
        a.a_rows_per_group = 2 * I;
        a.group_base = -j;
        a.out = h->sh_parts_gu + static_cast<size_t>(j) * h->ks_gu * T * 2 * I;
        a.out_ld = 2 * I;
        a.out_rows = T;
        a.m_limit = I;
        a.raw_gateup = 1;
        a.split_stride = static_cast<size_t>(T) * 2 * I;
        a.limit = c.swiglu_limit;
        a.status = h->status;
        a.timeout_ns = h->timeout_ns;
        const int nt = a.dense_m_tiles * a.dense_k_splits;
        h->prof_mark(kKGateUp, s);
        MOE_TRY_CUDA(launch_gemm_gateup(h->tm_w13sh, tm_x, tm_x, a, 32, nt < h->num_sms ? nt : h->num_sms, s));
        h->prof_done(s);
        h->prof_mark(kKSwigluReduce, s);
        MOE_TRY_CUDA(launch_swiglu_reduce(a.out ? static_cast<float*>(a.out) : nullptr, h->ks_gu, T, I,
                                          c.swiglu_limit,
                                          static_cast<__nv_bfloat16*>(h->h) + (static_cast<size_t>(T) * k +
                                                                               static_cast<size_t>(j) * T) * I,
                                          s));
        h->prof_done(s);
      }
    } else if (S > 0) {
      GemmArgs a{};
      a.tiles = h->tiles_gu;
      a.ntiles = h->ntiles + 2;
      a.group_base = El;
      a.num_kb = H / 64;
      a.a_rows_per_group = 2 * I;
      a.n_routed = El;
      a.out = h->h;
      a.out_ld = I;
      a.out_rows = static_cast<int>(h->R);
      a.m_limit = I;
      a.limit = c.swiglu_limit;
      a.status = h->status;
      a.timeout_ns = h->timeout_ns;
      h->prof_mark(kKGateUp, s);
      MOE_TRY_CUDA(launch_gemm_gateup(h->tm_w13sh, tm_x, tm_x, a, bn_gu, h->num_sms, s));
      h->prof_done(s);
    }
    // 5a. routed down on block-scaled MMAs
    MxGemmArgs d{};
    d.tiles = h->tiles_dn;
    d.ntiles = h->ntiles + 1;
    d.tile_begin = h->ntiles + 3;
    d.num_kb = I / 128;
    d.a_rows_per_group = H;
    d.m_tiles = H / 128;
    d.sfa = h->sfa2;
    d.sfb = h->sfb_dn;
    d.out = h->o;
    d.out_ld = H;
    d.out_rows = static_cast<int>(h->R);
    d.m_limit = H;
    d.status = h->status;
    d.timeout_ns = h->timeout_ns;
    d.a_base = h->w2q;
    d.a_row_bytes = h->a8 ? I : I / 2;
    h->prof_mark(kKDownMx, s);
    MOE_TRY_CUDA(
        launch_gemm_mx_down(wide_mx ? h->tm_w2qw : h->tm_w2q, h->tm_hq, d, bn_mx, h->num_sms, s, wide_mx, h->a8));
    h->prof_done(s);
    // 5b. shared experts' down in BF16 (split K for few tokens; the combine sums the slices)
    if (sh_split) {
      for (int j = 0; j < S; ++j) {
        GemmArgs a{};
        a.dense_m_tiles = H / 128;
        a.dense_rows = T;
        a.dense_b_row0 = T * k + j * T;
        a.dense_k_splits = h->ks_dn;
        a.num_kb = I / 64;
        a.a_rows_per_group = H;
        a.group_base = -j;
        a.out = h->sh_parts_dn + static_cast<size_t>(j) * h->ks_dn * T * H;
        a.out_ld = H;
        a.out_rows = T;
        a.m_limit = H;
        a.split_stride = static_cast<size_t>(T) * H;
        a.status = h->status;
        a.timeout_ns = h->timeout_ns;
        const int nt = a.dense_m_tiles * a.dense_k_splits;
        h->prof_mark(kKDown, s);
        MOE_TRY_CUDA(launch_gemm_down(h->tm_w2sh, h->tm_h, a, 32, nt < h->num_sms ? nt : h->num_sms, s));
        h->prof_done(s);
      }
    } else if (S > 0) {
      GemmArgs a{};
      a.tiles = h->tiles_dn;
      a.ntiles = h->ntiles + 3;
      a.group_base = El;
      a.num_kb = I / 64;
      a.a_rows_per_group = H;
      a.n_routed = El;
      a.out = h->o;
      a.out_ld = H;
      a.out_rows = static_cast<int>(h->R);
      a.m_limit = H;
      a.status = h->status;
      a.timeout_ns = h->timeout_ns;
      h->prof_mark(kKDown, s);
      MOE_TRY_CUDA(launch_gemm_down(wide_mx ? h->tm_w2shw : h->tm_w2sh, h->tm_h, a, bn_dn, h->num_sms, s, wide_mx));
      h->prof_done(s);
    }
  }
  // 6. weighted combine with the shared experts
  h->prof_mark(kKCombine, s);
  const bool parts = h->mx && S > 0 && T <= kSmallRouterMaxTokens;
  MOE_TRY_CUDA(launch_combine(h->o, h->inv, h->idx, eb, El, h->wts, T, H, k, S, y, y_f32,
                              parts ? h->sh_parts_dn : nullptr, parts ? h->ks_dn : 0, s));
  h->prof_done(s);
  if (topk_idx) MOE_TRY_CUDA(cudaMemcpyAsync(topk_idx, h->idx, static_cast<size_t>(nslots) * 4, cudaMemcpyDefault, s));
  if (topk_w) MOE_TRY_CUDA(cudaMemcpyAsync(topk_w, h->wts, static_cast<size_t>(nslots) * 4, cudaMemcpyDefault, s));
  h->last_T = T;
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_forward(moe_handle* h, const void* x, int32_t T, void* y, int32_t* topk_idx, float* topk_w,
                       moe_stream_t stream) {
  if (h != nullptr && h->e_local != h->cfg.n_routed) return MOE_ERR_INVALID_ARG;  // an expert window: partial only
  return forward_impl(h, x, nullptr, T, y, false, topk_idx, topk_w, stream);
}

moe_status moe_forward_partial(moe_handle* h, const void* x, int32_t T, float* y_partial, int32_t* topk_idx,
                               float* topk_w, moe_stream_t stream) {
  return forward_impl(h, x, nullptr, T, y_partial, true, topk_idx, topk_w, stream);
}

moe_status moe_set_hash_table(moe_handle* h, const int32_t* table, int32_t vocab, moe_stream_t stream) {
  if (h == nullptr || table == nullptr || vocab <= 0) return MOE_ERR_INVALID_ARG;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess || cur != h->device) return MOE_ERR_INVALID_ARG;
  if (!device_pointer_on(table, h->device)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(vocab) * h->cfg.top_k * 4;
  int32_t* copy = nullptr;
  if (cudaMalloc(&copy, bytes) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_OOM;
  }
  int bad = 0;
  bool err = cudaMemcpyAsync(copy, table, bytes, cudaMemcpyDeviceToDevice, s) != cudaSuccess;
  err |= cudaMemsetAsync(h->bad_flag, 0, sizeof(int), s) != cudaSuccess;
  err |= launch_hash_table_check(copy, vocab, h->cfg.top_k, h->cfg.n_routed, h->bad_flag, s) != cudaSuccess;
  err |= cudaMemcpyAsync(&bad, h->bad_flag, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess;
  err |= cudaStreamSynchronize(s) != cudaSuccess;
  if (err || bad) {
    cudaGetLastError();
    cudaFree(copy);
    return err ? MOE_ERR_CUDA : MOE_ERR_INVALID_ARG;
  }
  if (h->hash_table != nullptr) cudaFree(h->hash_table);
  h->hash_table = copy;
  h->hash_vocab = vocab;
  return MOE_OK;
}

moe_status moe_forward_hashed(moe_handle* h, const void* x, const int32_t* token_ids, int32_t T, void* y,
                              int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
  if (h == nullptr || h->hash_table == nullptr) return MOE_ERR_INVALID_ARG;
  if (T > 0) {
    if (token_ids == nullptr) return MOE_ERR_INVALID_ARG;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess || cur != h->device) return MOE_ERR_INVALID_ARG;
    if (!device_pointer_on(token_ids, h->device)) return MOE_ERR_INVALID_ARG;
  }
  if (h->e_local != h->cfg.n_routed) return MOE_ERR_INVALID_ARG;
  return forward_impl(h, x, token_ids, T, y, false, topk_idx, topk_w, stream);
}

moe_status moe_forward_host(moe_handle* h, const void* x_host, int32_t T, void* y_host, int32_t* topk_idx_host,
                            float* topk_w_host, moe_stream_t stream) {
  if (h == nullptr) return MOE_ERR_INVALID_ARG;
  if (T < 0 || T > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (x_host == nullptr || y_host == nullptr) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(T) * h->cfg.hidden * 2;
  MOE_TRY_CUDA(cudaMemcpyAsync(h->x_stage, x_host, bytes, cudaMemcpyHostToDevice, s));
  moe_status st = moe_forward(h, h->x_stage, T, h->y_stage, nullptr, nullptr, stream);
  if (st != MOE_OK) return st;
  MOE_TRY_CUDA(cudaMemcpyAsync(y_host, h->y_stage, bytes, cudaMemcpyDeviceToHost, s));
  const size_t kb = static_cast<size_t>(T) * h->cfg.top_k * 4;
  if (topk_idx_host) MOE_TRY_CUDA(cudaMemcpyAsync(topk_idx_host, h->idx, kb, cudaMemcpyDeviceToHost, s));
  if (topk_w_host) MOE_TRY_CUDA(cudaMemcpyAsync(topk_w_host, h->wts, kb, cudaMemcpyDeviceToHost, s));
  return MOE_OK;
}

moe_status moe_forward_host_async(moe_handle* h, const void* x_host, int32_t T, void* y_host, moe_stream_t stream) {
  if (h == nullptr) return MOE_ERR_INVALID_ARG;
  if (T < 0 || T > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (x_host == nullptr || y_host == nullptr) return MOE_ERR_INVALID_ARG;
  if (!h->pipe_ready) {
    // two copy streams, the slots' events, and the second slot's staging buffers
    // (each made once; a failed set-up is resumed by the next call)
    const size_t stage = static_cast<size_t>(h->cfg.max_tokens) * h->cfg.hidden * 2;
    auto stream_once = [](cudaStream_t* p) {
      return *p != nullptr || cudaStreamCreateWithFlags(p, cudaStreamNonBlocking) == cudaSuccess;
    };
    auto event_once = [](cudaEvent_t* p) {
      return *p != nullptr || cudaEventCreateWithFlags(p, cudaEventDisableTiming) == cudaSuccess;
    };
    bool ok = stream_once(&h->pipe_in) && stream_once(&h->pipe_out);
    for (int i = 0; ok && i < 2; ++i)
      ok = event_once(&h->pipe_copied_in[i]) && event_once(&h->pipe_done[i]) && event_once(&h->pipe_copied_out[i]);
    if (!ok) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    if ((h->pipe_x[1] == nullptr && !h->alloc(&h->pipe_x[1], stage, &h->pipe_bytes)) ||
        (h->pipe_y[1] == nullptr && !h->alloc(&h->pipe_y[1], stage, &h->pipe_bytes)))
      return MOE_ERR_OOM;
    h->pipe_x[0] = h->x_stage;
    h->pipe_y[0] = h->y_stage;
    h->pipe_ready = true;
  }
  const int k = h->pipe_slot;
  h->pipe_slot ^= 1;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(T) * h->cfg.hidden * 2;
  // x into slot k once the layer two calls back has finished reading it
  MOE_TRY_CUDA(cudaStreamWaitEvent(h->pipe_in, h->pipe_done[k], 0));
  MOE_TRY_CUDA(cudaMemcpyAsync(h->pipe_x[k], x_host, bytes, cudaMemcpyHostToDevice, h->pipe_in));
  MOE_TRY_CUDA(cudaEventRecord(h->pipe_copied_in[k], h->pipe_in));
  // the layer on `stream`, after that copy and after slot k's previous y has left
  MOE_TRY_CUDA(cudaStreamWaitEvent(s, h->pipe_copied_in[k], 0));
  MOE_TRY_CUDA(cudaStreamWaitEvent(s, h->pipe_copied_out[k], 0));
  const moe_status st = moe_forward(h, h->pipe_x[k], T, h->pipe_y[k], nullptr, nullptr, stream);
  if (st != MOE_OK) return st;
  MOE_TRY_CUDA(cudaEventRecord(h->pipe_done[k], s));
  // y out on the copy-out stream
  MOE_TRY_CUDA(cudaStreamWaitEvent(h->pipe_out, h->pipe_done[k], 0));
  MOE_TRY_CUDA(cudaMemcpyAsync(y_host, h->pipe_y[k], bytes, cudaMemcpyDeviceToHost, h->pipe_out));
  MOE_TRY_CUDA(cudaEventRecord(h->pipe_copied_out[k], h->pipe_out));
  return MOE_OK;
}

moe_status moe_forward_host_wait(moe_handle* h, moe_stream_t stream) {
  if (h == nullptr) return MOE_ERR_INVALID_ARG;
  if (!h->pipe_ready) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MOE_TRY_CUDA(cudaStreamWaitEvent(s, h->pipe_copied_out[0], 0));
  MOE_TRY_CUDA(cudaStreamWaitEvent(s, h->pipe_copied_out[1], 0));
  return MOE_OK;
}

moe_status moe_get_status(moe_handle* h) {
  if (h == nullptr) return MOE_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  int v = 0;
  if (cudaMemcpy(&v, h->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemset(h->status, 0, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (v & kStatusTimeout) return MOE_ERR_TIMEOUT;
  if (v & kStatusDevice) return MOE_ERR_DEVICE;
  return MOE_OK;
}

void moe_destroy(moe_handle* h) {
  if (h == nullptr) return;
  cudaDeviceSynchronize();
  cudaGetLastError();
  h->release();
  delete h;
}

moe_status moe_quantize_mxfp4(const void* src_bf16, int64_t rows, int32_t cols, uint8_t* dst_packed,
                              uint8_t* dst_scales, moe_stream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (src_bf16 == nullptr || dst_packed == nullptr || dst_scales == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(src_bf16) || !aligned16(dst_packed)) return MOE_ERR_INVALID_ARG;
  MOE_TRY_CUDA(launch_quantize_mxfp4(src_bf16, rows, cols, dst_packed, dst_scales,
                                     reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_quantize_mxfp8(const void* src_bf16, int64_t rows, int32_t cols, uint8_t* dst_codes,
                              uint8_t* dst_scales, moe_stream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (src_bf16 == nullptr || dst_codes == nullptr || dst_scales == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(src_bf16) || !aligned16(dst_codes)) return MOE_ERR_INVALID_ARG;
  MOE_TRY_CUDA(launch_quantize_mxfp8(src_bf16, rows, cols, dst_codes, dst_scales,
                                     reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_inspect(moe_handle* h, int32_t what, void* dst, size_t bytes, moe_stream_t stream) {
  if (h == nullptr || dst == nullptr) return MOE_ERR_INVALID_ARG;
  const int64_t Tm = h->cfg.max_tokens, k = h->cfg.top_k, E = h->cfg.n_routed, I = h->cfg.inter;
  const void* src = nullptr;
  size_t cap = 0;
  switch (what) {
    case MOE_BUF_LOGITS: src = h->z; cap = Tm * E * 4; break;
    case MOE_BUF_TOPK_IDX: src = h->idx; cap = Tm * k * 4; break;
    case MOE_BUF_TOPK_W: src = h->wts; cap = Tm * k * 4; break;
    case MOE_BUF_COUNTS: src = h->cnt; cap = h->G * 4; break;
    case MOE_BUF_OFFSETS: src = h->off; cap = (h->G + 1) * 4; break;
    case MOE_BUF_PERM: src = h->perm; cap = Tm * k * 4; break;
    case MOE_BUF_INV: src = h->inv; cap = Tm * k * 4; break;
    case MOE_BUF_H: src = h->h; cap = h->R * I * 2; break;
    case MOE_BUF_XQ:
      if (!h->mx) return MOE_ERR_INVALID_ARG;
      src = h->xq;
      cap = Tm * k * h->cfg.hidden;
      break;
    case MOE_BUF_XQ_SCALES:
      if (!h->mx) return MOE_ERR_INVALID_ARG;
      src = h->sfb_gu;
      cap = h->max_ntiles_r * (h->cfg.hidden / 128) * 512;
      break;
    case MOE_BUF_HQ:
      if (!h->mx) return MOE_ERR_INVALID_ARG;
      src = h->hq;
      cap = Tm * k * I;
      break;
    case MOE_BUF_HQ_SCALES:
      if (!h->mx) return MOE_ERR_INVALID_ARG;
      src = h->sfb_dn;
      cap = h->max_ntiles_r * (I / 128) * 512;
      break;
    case MOE_BUF_NTILES: src = h->ntiles; cap = 28; break;
    case MOE_BUF_TILES_GU: src = h->tiles_gu; cap = h->max_tiles_gu * 16; break;
    case MOE_BUF_TILES_DN: src = h->tiles_dn; cap = h->max_tiles_dn * 16; break;
    default: return MOE_ERR_INVALID_ARG;
  }
  if (bytes > cap) return MOE_ERR_INVALID_ARG;
  if (bytes == 0) return MOE_OK;
  MOE_TRY_CUDA(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDefault, reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_fill_workspace(moe_handle* h, int32_t byte_value, moe_stream_t stream) {
  if (h == nullptr || byte_value < 0 || byte_value > 255) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (const auto& a : h->ws_allocs) {
    // the status word and the check flags keep their meaning
    if (a.first == h->status || a.first == h->bad || a.first == h->bad_flag) continue;
    MOE_TRY_CUDA(cudaMemsetAsync(a.first, byte_value, a.second, s));
  }
  return MOE_OK;
}

moe_status moe_read_bandwidth(const void* buf, size_t bytes, int32_t reps, moe_stream_t stream, double* gbs) {
  if (buf == nullptr || gbs == nullptr || reps < 1 || bytes < (size_t(1) << 20) || !aligned16(buf))
    return MOE_ERR_INVALID_ARG;
  int dev = -1, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || !device_pointer_on(buf, dev)) return MOE_ERR_INVALID_ARG;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t used = bytes / (32 * 1024) * (32 * 1024);
  int* status = nullptr;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  moe_status st = MOE_OK;
  if (cudaMalloc(&status, sizeof(int)) != cudaSuccess || cudaEventCreate(&e0) != cudaSuccess ||
      cudaEventCreate(&e1) != cudaSuccess || cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess ||
      launch_stream_read(buf, used, sms, status, 2000000000ull, s) != cudaSuccess ||  // warm-up
      cudaEventRecord(e0, s) != cudaSuccess) {
    st = MOE_ERR_CUDA;
  }
  for (int i = 0; st == MOE_OK && i < reps; ++i)
    if (launch_stream_read(buf, used, sms, status, 2000000000ull, s) != cudaSuccess) st = MOE_ERR_CUDA;
  float ms = 0.f;
  int v = 0;
  if (st == MOE_OK && (cudaEventRecord(e1, s) != cudaSuccess || cudaEventSynchronize(e1) != cudaSuccess ||
                       cudaEventElapsedTime(&ms, e0, e1) != cudaSuccess ||
                       cudaMemcpy(&v, status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess))
    st = MOE_ERR_CUDA;
  if (st == MOE_OK && v != 0) st = MOE_ERR_TIMEOUT;
  if (st == MOE_OK) *gbs = static_cast<double>(used) * reps / (ms * 1e-3) / 1e9;
  cudaGetLastError();
  if (e0) cudaEventDestroy(e0);
  if (e1) cudaEventDestroy(e1);
  if (status) cudaFree(status);
  return st;
}

moe_status moe_set_wait_timeout(moe_handle* h, uint64_t timeout_ns) {
  if (h == nullptr || timeout_ns == 0) return MOE_ERR_INVALID_ARG;
  h->timeout_ns = timeout_ns;
  return MOE_OK;
}

moe_status moe_selftest_wait_timeout(moe_handle* h, uint64_t timeout_ns, moe_stream_t stream) {
  if (h == nullptr || timeout_ns == 0 || timeout_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;
  MOE_TRY_CUDA(launch_wait_timeout_probe(h->status, timeout_ns, reinterpret_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_get_info(moe_handle* h, moe_info* out) {
  if (h == nullptr || out == nullptr) return MOE_ERR_INVALID_ARG;
  out->weight_bytes = h->weight_bytes;
  out->workspace_bytes = h->workspace_bytes;
  out->num_sms = h->num_sms;
  out->last_tokens = h->last_T;
  return MOE_OK;
}

moe_status moe_profile_begin(moe_handle* h, int32_t max_calls) {
  if (h == nullptr || max_calls <= 0 || max_calls > 100000) return MOE_ERR_INVALID_ARG;
  const size_t need = static_cast<size_t>(max_calls) * 2 * 16;
  while (h->ev.size() < need) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    h->ev.push_back(e);
  }
  h->ev_kind.assign(h->ev.size() / 2, -1);
  h->ev_used = 0;
  h->prof_on = true;
  return MOE_OK;
}

moe_status moe_profile_end(moe_handle* h, double* ms, int64_t* launches, int32_t n) {
  if (h == nullptr || ms == nullptr || launches == nullptr || n < 0) return MOE_ERR_INVALID_ARG;
  h->prof_on = false;
  for (int i = 0; i < n; ++i) {
    ms[i] = 0.0;
    launches[i] = 0;
  }
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  for (size_t p = 0; p + 1 < h->ev_used; p += 2) {
    float t = 0.f;
    const int kind = h->ev_kind[p / 2];
    if (kind < 0 || kind >= n) continue;
    if (cudaEventElapsedTime(&t, h->ev[p], h->ev[p + 1]) == cudaSuccess) {
      ms[kind] += t;
      launches[kind] += 1;
    } else {
      cudaGetLastError();
    }
  }
  h->ev_used = 0;
  return MOE_OK;
}

}  // extern "C"
