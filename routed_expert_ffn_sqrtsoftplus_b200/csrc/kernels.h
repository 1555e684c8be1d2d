// Launchers of the MoE layer's device kernels (host-callable, internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// One GEMM tile: x = group | (m_tile << 16), y = first B row, z = first output row,
// w = number of valid rows (tokens) in the tile.
using TileEntry = int4;

struct GemmArgs {
  const int4* tiles;            // grouped mode: tile list; nullptr = dense mode
  const int* ntiles;            // grouped mode: device tile count
  int dense_m_tiles;            // dense mode: 128-row tiles of A
  int dense_rows;               // dense mode: rows of B (tokens)
  int num_kb;                   // K / 64
  int a_rows_per_group;         // rows of A per group
  int n_routed;                 // gate/up: groups >= n_routed read B through the shared-token map
  void* out;                    // gate/up: BF16 h rows; down / dense: fp32 rows
  int out_ld;                   // elements per output row
  int out_rows;                 // rows of the output buffer (device bounds check)
  int m_limit;                  // output columns >= m_limit are not stored
  float limit;                  // swiglu limit (gate/up)
  const float* col_bias;        // down / dense: added to output column m (nullptr = none)
  int* status;                  // device status word
  unsigned long long timeout_ns;
};

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
  kKNumKinds
};

// ---- router
cudaError_t launch_router_logits(const void* x, const void* wg, const float* bias, float* z, int T, int H, int E,
                                 cudaStream_t s);
cudaError_t launch_topk_refine(const float* z, const void* x, const void* wg, const float* bias, int T, int H,
                               int E, int k, float route_scale, float delta, int32_t* idx, float* w, int* status,
                               cudaStream_t s);

// ---- permutation
constexpr int kPermChunk = 1024;
cudaError_t launch_perm_count(const int32_t* idx, int nslots, int E, int32_t* chunk_cnt, int* status,
                              cudaStream_t s);
struct ScanArgs {
  int32_t* chunk_cnt;
  int nchunks, E, S, T, k;
  int32_t* cnt;
  int32_t* off;
  int4* tiles_gu;
  int4* tiles_dn;
  int* ntiles;
  int m_tiles_gu, bn_gu, m_tiles_dn, bn_dn;
};
cudaError_t launch_perm_scan(const ScanArgs& a, cudaStream_t s);
cudaError_t launch_perm_scatter(const int32_t* idx, int nslots, int E, const int32_t* chunk_base, int32_t* perm,
                                int32_t* inv, cudaStream_t s);
cudaError_t launch_gather_rows(const void* x, const int32_t* perm, int nrows, int k, int H, void* xp,
                               cudaStream_t s);

// ---- grouped GEMMs (tcgen05)
// bn: 32 (few tokens per group) or the large-tile variant (gate/up 128, down 256).
cudaError_t launch_gemm_gateup(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmBsh,
                               const GemmArgs& a, int bn, int grid, cudaStream_t s);
cudaError_t launch_gemm_down(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a, int bn, int grid,
                             cudaStream_t s);
cudaError_t gemm_set_attributes();

// ---- combine
cudaError_t launch_combine(const float* O, const int32_t* inv, const float* w, int T, int H, int k, int S,
                           void* y, cudaStream_t s);

// ---- MX utilities
cudaError_t launch_quantize_mxfp4(const void* src, int64_t rows, int cols, uint8_t* packed, uint8_t* scales,
                                  cudaStream_t s);

// ---- repack
cudaError_t launch_repack_w13(const void* w1, const void* w3, const void* sh1, const void* sh3, int E, int S,
                              int I, int H, void* w13, cudaStream_t s);

// ---- self test
cudaError_t launch_wait_timeout_probe(int* status, unsigned long long timeout_ns, cudaStream_t s);

}  // namespace moe
