// Launchers of the MoE layer's device kernels (host-callable, internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// True when p is device (or managed) memory the kernels of device `dev` may read
// and write: a host pointer or another GPU's memory handed to a kernel would
// fault the device, so the entry points reject them before launching anything.
inline bool device_pointer_on(const void* p, int dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (a.type == cudaMemoryTypeManaged) return true;
  return a.type == cudaMemoryTypeDevice && a.device == dev;
}

// One GEMM tile: x = group | (m_tile << 16), y = first B row, z = first output row,
// w = number of valid rows (tokens) in the tile.
using TileEntry = int4;

struct GemmArgs {
  const int4* tiles;            // grouped mode: tile list; nullptr = dense mode
  const int* ntiles;            // grouped mode: device index one past the last tile to run
  const int* tile_begin;        // grouped mode: device index of the first tile to run (nullptr = 0)
  int group_base;               // A rows of group g start at (g - group_base) * a_rows_per_group
  int dense_m_tiles;            // dense mode: 128-row tiles of A
  int dense_rows;               // dense mode: rows of B (tokens)
  int dense_b_row0;             // dense mode: first B row
  int num_kb;                   // K / 64
  int a_rows_per_group;         // rows of A per group
  int n_routed;                 // gate/up: groups >= n_routed read B through the shared-token map
  void* out;                    // gate/up: BF16 h rows; down / dense: fp32 rows
  int out_ld;                   // elements per output row
  int out_rows;                 // rows of the output buffer (device bounds check)
  int m_limit;                  // output columns >= m_limit are not stored
  float limit;                  // swiglu limit (gate/up)
  const float* col_bias;        // down / dense: added to output column m (nullptr = none)
  int dense_k_splits;           // dense mode: K split into this many slices (partial sums)
  size_t split_stride;          // dense mode with k splits: elements between the slices' outputs
  int raw_gateup;               // gate/up: store fp32 G | U (ld = out_ld, U at + I) instead of h
  int* status;                  // device status word
  unsigned long long timeout_ns;
  const int* bn_select;         // dual-width launch: the token-tile width the permutation chose
  const int* thin_begin;        // dual-width launch: device index from which every tile has at most
                                //   kThinRows rows (nullptr: one tile list, taken by stride)
  int* sched;                   // dual-width launch with thin_begin: two tile counters (wide, thin),
                                //   zero before the launch
  const int32_t* gather_perm;   // gate/up: routed B rows are x rows perm[row] / gather_k, fetched by
  int gather_k;                 //   tile::gather4 through tmB (a one-row box map of x); nullptr = B rows as stored
};
// The BF16 gate/up GEMM fetches the routed token rows straight from x through the
// permutation (tile::gather4) instead of a gathered copy (1), or reads the copy (0).
// Measured on B200: the gathers (a TMA instruction per four 128-byte rows, up to 64
// per ring stage) made gate/up 1.7x slower at prefill than the copy kernel plus
// 32-row boxes, so the copy is the default.
#ifndef MOE_GATHER_X
#define MOE_GATHER_X 0
#endif
constexpr bool kGatherX = MOE_GATHER_X != 0;

// Kernel kinds for profiling (order = moe_kernel_name()).
enum KernelKind {
  kKRouterLogits = 0,
  kKRouterGemm,
  kKTopk,
  kKPermCount,
  kKPermScan,
  kKPermScatter,
  kKGather,
  kKGateUp,
  kKDown,
  kKCombine,
  kKQuantX,
  kKGateUpMx,
  kKDownMx,
  kKSwigluReduce,
  kKHashRoute,
  kKGemmFused,
  kKNumKinds
};

// ---- router
// Logit error of the approximate router is far below this (fp32 sums of exact
// BF16 products, or tensor-core fp32 accumulation); every expert whose
// approximate score lies within kRefineDelta of the k-th is re-scored exactly.
// moe_forward and moe_route_noalloc use the same band.
constexpr float kRefineDelta = 2e-3f;
cudaError_t launch_router_logits(const void* x, const void* wg, const float* bias, float* z, int T, int H, int E,
                                 cudaStream_t s);
// Few tokens (T <= 32): fp32 logit slices [H / router_small_slice(H)][T][E] over
// CTAs of 8 experts x one hidden slice, then one CTA per token sums the slices,
// picks the candidates and re-scores them exactly in parallel.
int router_small_slice(int H);
cudaError_t router_set_attributes();
cudaError_t launch_router_small(const void* x, const void* wg, float* part, int T, int H, int E, cudaStream_t s);
cudaError_t launch_topk_small(const float* part, int nparts, const void* x, const void* wg, const float* bias, int T,
                              int H, int E, int k, float route_scale, float delta, int32_t* idx, float* w, float* z,
                              int* status, cudaStream_t s, const float* exact_bias);
cudaError_t launch_topk_refine(const float* z, const void* x, const void* wg, const float* bias, int T, int H,
                               int E, int k, float route_scale, float delta, int32_t* idx, float* w, int* status,
                               cudaStream_t s);

// Hash-routed layers: selection from table[ids[t]] [vocab, k], exact sqrtsoftplus weights.
cudaError_t launch_hash_route(const void* x, const void* wg, const float* bias, const int32_t* table,
                              const int32_t* ids, int T, int H, int E, int k, int vocab, float route_scale,
                              int32_t* idx, float* w, int* status, cudaStream_t s);
// Sets *bad when an entry lies outside [0, E) or a row repeats an expert.
cudaError_t launch_hash_table_check(const int32_t* table, int vocab, int k, int E, int* bad, cudaStream_t s);

// ---- permutation
constexpr int kPermChunk = 1024;
// Expert window: this instance holds routed experts [e_begin, e_begin + E) of e_global
// (the whole layer: e_begin 0, E = e_global); slots of other experts are skipped.
cudaError_t launch_perm_count(const int32_t* idx, int nslots, int E, int e_begin, int e_global, int32_t* chunk_cnt,
                              int* status, cudaStream_t s);
struct ScanArgs {
  int32_t* chunk_cnt;
  int nchunks, E, S, T, k;     // E: routed groups of this instance (its expert window)
  int e_begin, e_global;        // the window's first expert and the router's expert count
  int32_t* cnt;
  int32_t* off;
  int4* tiles_gu;
  int4* tiles_dn;
  int* ntiles;                  // [gu_end, dn_end, gu_shared_end, dn_shared_end, (routed rows),
                                //  gu_thin_begin, dn_thin_begin]
  int* sched_zero;              // when not null: 4 tile counters of the dual-width GEMMs, zeroed here
  int m_tiles_gu, m_tiles_dn;
  int bn_gu_r, bn_dn_r;         // token tile of routed groups (gate/up, down)
  int bn_gu_s, bn_dn_s;         // token tile of shared groups
  int mx;                       // routed tiles carry their token-tile id in .y
  int32_t* ntile_base_gu;       // [E + 1] first token tile of each routed group (gate/up)
  int32_t* ntile_base_dn;       // [E + 1] same for the down GEMM
  int bn_alt;                   // > 0: use this width for every tile when no routed group has more rows
  int* bn_choice;               // out: the width the tile lists were built with (bn_alt, or bn_gu_r)
  int sort_partial;             // order the partial token tiles longest first (tile costs differ)
  int* done;                    // when not null: per-group counters of the fused GEMM, zeroed here
  int32_t* nrows_routed;        // out: rows of the routed groups (T*k, or fewer in an expert window)
};
cudaError_t launch_perm_scan(const ScanArgs& a, cudaStream_t s);
// count + scan + scatter in one launch when all slots fit one chunk
cudaError_t launch_perm_fused(const ScanArgs& a, const int32_t* idx, int nslots, int32_t* perm, int32_t* inv,
                              int* status, cudaStream_t s);
cudaError_t launch_perm_scatter(const int32_t* idx, int nslots, int E, int e_begin, const int32_t* chunk_base,
                                int32_t* perm, int32_t* inv, cudaStream_t s);
// rows >= min(nrows, *nrows_dev) are not routed to this instance and are skipped
cudaError_t launch_gather_rows(const void* x, const int32_t* perm, int nrows, const int32_t* nrows_dev, int k, int H,
                               void* xp, cudaStream_t s);

// ---- grouped GEMMs (tcgen05)
// Token-tile width of the many-tokens-per-expert GEMMs (gate/up, down and the
// router GEMM): a multiple of 32 in [32, 256].
#ifndef MOE_BN_LARGE
#define MOE_BN_LARGE 256
#endif
constexpr int kBnLarge = MOE_BN_LARGE;
static_assert(kBnLarge % 32 == 0 && kBnLarge >= 32 && kBnLarge <= 256, "large token tile");
// Narrower many-token width the permutation picks on the device when no routed
// expert has more rows (one tile per expert with a deeper ring); 0 = never.
#ifndef MOE_BN_ALT
#define MOE_BN_ALT 192
#endif
constexpr int kBnAlt = MOE_BN_ALT;
static_assert(kBnAlt == 0 || (kBnAlt % 32 == 0 && kBnAlt >= 32 && kBnAlt < kBnLarge && kBnAlt != 128 &&
                              kBnAlt != 32), "alternative token tile");
// Thin tiles: in a longest-first list of many-token tiles the partial token tiles
// of at most kThinRows rows come last (a skewed batch's cold experts). They only
// stream weights, which a ring of kThinRows-token stages does with about twice the
// bytes in flight of the wide-tile ring. With kThinSplit the dual-width launch
// takes tiles from two counters, one per list: some CTAs start on the thin list
// (on that ring) while the others run the wide tiles, so the weight streaming
// overlaps the compute-bound tiles, and each CTA moves to the other list when its
// own runs dry.
constexpr int kThinRows = 32;
#ifndef MOE_THIN_SPLIT
#define MOE_THIN_SPLIT 1
#endif
constexpr bool kThinSplit = MOE_THIN_SPLIT != 0;
// bn: 32 (few tokens per group), 128 or kBnLarge (gate/up) and 32 or kBnLarge
// (down).
cudaError_t launch_gemm_gateup(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmBsh,
                               const GemmArgs& a, int bn, int grid, cudaStream_t s);
// wide: each tile covers 256 rows of W2 (two 128-row MMAs sharing the token tile);
// the tile list's m tiles are then H / 256.
cudaError_t launch_gemm_down(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a, int bn, int grid,
                             cudaStream_t s, bool wide = false);
// Gate/up and down of the few-token path (32-token tiles, 256 W2 rows per down
// tile) in one persistent launch: the CTAs walk the gate/up tiles and then the down
// tiles; a down tile of group g starts once every gate/up tile of g has stored its
// h rows (done[g] counts the epilogue warps that finished one). Cooperative launch.
struct FusedArgs {
  GemmArgs gu, dn;
  int* done;                    // per group, zeroed by the permutation kernel
  const int32_t* cnt;           // rows per group
  int m_tiles_gu;               // weight tiles per group of the gate/up GEMM
};
#ifndef MOE_FUSED_DECODE
#define MOE_FUSED_DECODE 1
#endif
constexpr bool kFusedDecode = MOE_FUSED_DECODE != 0;
cudaError_t launch_gemm_fused_small(const CUtensorMap& tmA_gu, const CUtensorMap& tmB_gu, const CUtensorMap& tmBsh,
                                   const CUtensorMap& tmA_dn, const CUtensorMap& tmB_dn, const FusedArgs& f,
                                   int grid, cudaStream_t s);
// One launch for both many-token widths (kBnLarge and kBnAlt): a.bn_select holds
// the permutation kernel's choice; wide W2 tiles for the down GEMM.
cudaError_t launch_gemm_gateup_dual(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmBsh,
                                    const GemmArgs& a, int grid, cudaStream_t s);
cudaError_t launch_gemm_down_wide_dual(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a, int grid,
                                       cudaStream_t s);
cudaError_t gemm_set_attributes();

// ---- MX (MXFP4 routed experts)
// Token-tile width of the MX GEMMs when many tokens meet each expert (32 and 64
// are always built): a multiple of 32 in [32, 128].
#ifndef MOE_BN_MX_LARGE
#define MOE_BN_MX_LARGE 96
#endif
constexpr int kBnMxLarge = MOE_BN_MX_LARGE;
// MXFP4 weights staged packed in the ring and expanded by warps (1), or unpacked
// by the 16U4_ALIGN16B TMA type (0); expanded buffers of the packed form.
#ifndef MOE_MX_PACKED
#define MOE_MX_PACKED 0
#endif
#ifndef MOE_MX_PACKED_BUFS
#define MOE_MX_PACKED_BUFS 2
#endif
constexpr bool kMxPacked = MOE_MX_PACKED != 0;
static_assert(kBnMxLarge % 32 == 0 && kBnMxLarge >= 32 && kBnMxLarge <= 128, "large MX token tile");
struct MxGemmArgs {
  const int4* tiles;            // {group | m_tile << 16, token tile id, first row, rows}
  const int* ntiles;            // device index one past the last tile
  const int* tile_begin;        // device index of the first tile (nullptr = 0)
  int num_kb;                   // K / 128
  int a_rows_per_group;
  int m_tiles;                  // weight tiles per group
  const uint8_t* sfa;           // weight scale atoms [groups][m_tiles][num_kb][atoms of this GEMM]
  const uint8_t* sfb;           // activation scale atoms [token tiles][num_kb][512]
  void* out;                    // gate/up: E4M3 h rows; down: fp32 rows
  int out_ld;
  int out_rows;
  int m_limit;
  float limit;
  uint8_t* sf_out;              // gate/up: scale atoms of h for the down GEMM
  int sf_out_kb4;               // I / 128
  int bn_dn;                    // token tile of the down GEMM
  const int32_t* group_off;     // first row of each group
  const int32_t* dn_ntile_base; // first down token tile of each group
  int* status;
  unsigned long long timeout_ns;
  const uint8_t* a_base;        // the weights as stored: a tile's rows are contiguous, a_row_bytes each
  int a_row_bytes;
};
cudaError_t gemm_mx_set_attributes();
// a_fp8: the weights are MXFP8 (E4M3, one byte per value) instead of MXFP4
cudaError_t launch_gemm_mx_gateup(const CUtensorMap& tmA, const CUtensorMap& tmB, const MxGemmArgs& a, int bn,
                                  int grid, cudaStream_t s, bool a_fp8);
// wide: tiles of 256 W2 rows (two 128-row MMAs per K step); the tile list's m tiles are H / 256
cudaError_t launch_gemm_mx_down(const CUtensorMap& tmA, const CUtensorMap& tmB, const MxGemmArgs& a, int bn,
                                int grid, cudaStream_t s, bool wide, bool a_fp8);
// x rows of the routed slots -> MXFP8: xq[row] = E4M3 codes of x[perm[row] / k], scale
// atoms by gate/up token tile.
cudaError_t launch_quant_gather_mx(const void* x, const int32_t* perm, const int32_t* idx, const int32_t* off,
                                   const int32_t* ntile_base_gu, int nrows, const int32_t* nrows_dev, int k, int H,
                                   int bn_gu, int e_begin, int e_count, uint8_t* xq, uint8_t* sfb, cudaStream_t s);
// Weight scales [groups, rows, K/32] -> atoms [groups][rows/128][K/128][parts * 512]; for
// gate/up the two parts are W1 and W3 of the same 128 rows. Codes 0xFF raise *bad.
cudaError_t launch_sf_atoms(const uint8_t* s_a, const uint8_t* s_b, int groups, int rows, int K, uint8_t* dst,
                            int* bad, cudaStream_t s);
// Row permutation of the W1/W3 rows into 256-row gate/up tiles for any row width
// (bytes per row a multiple of 16); groups >= E come from the shared pointers.
cudaError_t launch_repack_w13_bytes(const void* w1, const void* w3, const void* sh1, const void* sh3, int E, int S,
                                    int I, int row_bytes, void* w13, cudaStream_t s);

// ---- combine
// sh_parts: when not null, the shared experts' outputs are the sum of n_parts fp32
// slices [n_parts][S][T][H] (split-K partial sums) instead of O's shared rows.
// Only the slots whose expert (idx) lies in [e_begin, e_begin + e_count) are summed;
// y is BF16, or fp32 when y_f32 (an expert-parallel partial output).
cudaError_t launch_combine(const float* O, const int32_t* inv, const int32_t* idx, int e_begin, int e_count,
                           const float* w, int T, int H, int k, int S, void* y, bool y_f32, const float* sh_parts,
                           int n_parts, cudaStream_t s);
// h[row0 + t] = clamped SwiGLU of the sum over n_parts slices of fp32 G | U rows [n_parts][T][2I].
cudaError_t launch_swiglu_reduce(const float* parts, int n_parts, int T, int I, float limit, void* h,
                                 cudaStream_t s);

// ---- MX utilities
cudaError_t launch_quantize_mxfp4(const void* src, int64_t rows, int cols, uint8_t* packed, uint8_t* scales,
                                  cudaStream_t s);
cudaError_t launch_quantize_mxfp8(const void* src, int64_t rows, int cols, uint8_t* codes, uint8_t* scales,
                                  cudaStream_t s);

// ---- repack
cudaError_t launch_repack_w13(const void* w1, const void* w3, const void* sh1, const void* sh3, int E, int S,
                              int I, int H, void* w13, cudaStream_t s);

// ---- read-only streaming (roofline denominator): reads bytes / 32 KiB chunks of buf
cudaError_t launch_stream_read(const void* buf, size_t bytes, int grid, int* status, unsigned long long timeout_ns,
                               cudaStream_t s);

// ---- self test
cudaError_t launch_wait_timeout_probe(int* status, unsigned long long timeout_ns, cudaStream_t s);

}  // namespace moe
