// Token permutation: group the (token, slot) pairs by expert so each expert's
// rows are contiguous for the grouped GEMMs (the dispatch of routed experts the
// MAX DeepseekV41Config ep_config describes across devices, here inside one GPU).
//
// Deterministic counting sort of the flat slots s = t*k + j by expert:
//   perm_count   per chunk of kPermChunk slots, a histogram over experts
//   perm_scan    per-expert counts and offsets (routed experts first, then the
//                shared experts with T rows each), per-chunk base positions,
//                and the gate/up and down tile lists
//   perm_scatter positions in ascending slot order inside each expert: perm
//                (row -> slot) and inv (slot -> row)
//   gather_rows  Xp[row] = x[perm[row] / k], the B operand of the gate/up GEMM
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kMaxGroups = 1024;      // routed experts of the histogram and scatter kernels
constexpr int kMaxScanGroups = 544;   // routed (<= 512) + shared (<= 4) groups of the scan kernel
constexpr int kMaxSegs = 2 * kMaxScanGroups;  // tile-list segments (shared, full, partial)
// Partial token tiles by row count, descending (1), or in group order (0).
#ifndef MOE_TILE_ORDER_LPT
#define MOE_TILE_ORDER_LPT 1
#endif
constexpr bool kTileOrderLongestFirst = MOE_TILE_ORDER_LPT != 0;
// In a longest-first list, the partial last token tile of a group that also has
// full tiles follows that group's full tiles of the same weight tile (1), so that
// the CTAs taking consecutive tiles read the weight box together, through L2; only
// the groups without a full tile make up the longest-first tail. Or every partial
// tile in that tail (0), where a hot expert's partial tiles read their weights from
// HBM again.
#ifndef MOE_TILE_ORDER_HOT_PARTIAL
#define MOE_TILE_ORDER_HOT_PARTIAL 1
#endif
constexpr bool kTileOrderHotPartial = MOE_TILE_ORDER_HOT_PARTIAL != 0;

// Token tiles of routed group g (n rows) in its full-tile segment: the full ones,
// and with `hp` (a group that has full tiles) its partial last one as well.
__device__ __forceinline__ int full_seg_tiles(int n, int bn, bool hp) {
  if (!hp) return n / bn;
  return n >= bn ? (n + bn - 1) / bn : 0;
}

// Expert windows (expert parallelism): this layer instance holds routed experts
// [e_begin, e_begin + E) of e_global; a slot whose expert lies outside the window
// belongs to another instance and is skipped, one outside [0, e_global) is an error.
__global__ void __launch_bounds__(256)
    perm_count_kernel(const int32_t* __restrict__ idx, int nslots, int E, int e_begin, int e_global,
                      int32_t* __restrict__ chunk_cnt, int* status) {
  __shared__ int hist[kMaxGroups];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int base = blockIdx.x * kPermChunk;
  const int end = min(nslots, base + kPermChunk);
  for (int s = base + threadIdx.x; s < end; s += blockDim.x) {
    const int g = idx[s];
    const int e = g - e_begin;
    if (g < 0 || g >= e_global)
      report_status(status, kStatusDevice);
    else if (e >= 0 && e < E)
      atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_cnt[static_cast<size_t>(blockIdx.x) * E + e] = hist[e];
}

// Exclusive scan of one int per thread over a 1024-thread block; returns the
// thread's exclusive prefix, *total gets the block sum. Uses warp shuffles and
// one shared array of 32 warp totals.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = lane < static_cast<int>(blockDim.x / 32) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    warp_tot[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int before = warp > 0 ? warp_tot[warp - 1] : 0;
  *total = warp_tot[blockDim.x / 32 - 1];
  __syncthreads();
  return before + inc - v;
}

// Counts, offsets, token-tile bases and both tile lists, one thread per group.
// With `fused` (all slots in one chunk) the kernel also builds the histogram
// and scatters the slots itself, so one launch replaces three.
__global__ void __launch_bounds__(1024) perm_scan_kernel(ScanArgs a, int fused, const int32_t* idx, int nslots,
                                                        int32_t* perm, int32_t* inv, int* status) {
  __shared__ int cnt_s[kMaxScanGroups];
  __shared__ int off_s[kMaxScanGroups + 1];
  __shared__ int ngu_s[kMaxScanGroups + 1];      // first token tile of each routed group
  __shared__ int ndn_s[kMaxScanGroups + 1];
  __shared__ int seg_pre[2][kMaxSegs + 1];       // first tile of each list segment (gate/up, down)
  __shared__ int part_g[2][kMaxScanGroups];      // routed group of each partial-tile segment
  __shared__ int rem_s[kMaxScanGroups];          // rows of each routed group's partial token tile
  __shared__ int nseg_s[2];
  __shared__ bool hp_list[2];
  __shared__ int nbig_s[2];
  __shared__ int slot_e[kPermChunk];             // fused: each slot's group (-1: not this instance's)
  __shared__ int warp_tot[32];
  __shared__ int tot;
  __shared__ int maxc_s;
  const int G = a.E + a.S;
  const int tid = threadIdx.x;
  // 1. per-group row counts
  if (fused) {
    for (int g = tid; g < a.E; g += blockDim.x) cnt_s[g] = 0;
    __syncthreads();
    for (int s = tid; s < nslots; s += blockDim.x) {
      const int g = idx[s];
      const int e = g - a.e_begin;
      const bool mine = g >= 0 && g < a.e_global && e >= 0 && e < a.E;
      if (g < 0 || g >= a.e_global) report_status(status, kStatusDevice);
      if (mine) atomicAdd(&cnt_s[e], 1);
      slot_e[s] = mine ? e : -1;  // kept for the scatter below (no second pass over global memory)
    }
    __syncthreads();
    for (int g = a.E + tid; g < G; g += blockDim.x) cnt_s[g] = a.T;
  } else {
    for (int g = tid; g < G; g += blockDim.x) {
      if (g < a.E) {
        int run = 0;
        for (int c = 0; c < a.nchunks; ++c) {
          const size_t i = static_cast<size_t>(c) * a.E + g;
          const int v = a.chunk_cnt[i];
          a.chunk_cnt[i] = run;
          run += v;
        }
        cnt_s[g] = run;
      } else {
        cnt_s[g] = a.T;
      }
    }
  }
  // token-tile widths: the narrower alternative when no routed group exceeds it
  if (tid == 0) maxc_s = 0;
  __syncthreads();
  for (int g = tid; g < a.E; g += blockDim.x) atomicMax(&maxc_s, cnt_s[g]);
  __syncthreads();
  const bool alt = a.bn_alt > 0 && maxc_s <= a.bn_alt;
  const int bn_gu_r = alt ? a.bn_alt : a.bn_gu_r, bn_dn_r = alt ? a.bn_alt : a.bn_dn_r;
  const int bn_gu_s = alt ? a.bn_alt : a.bn_gu_s, bn_dn_s = alt ? a.bn_alt : a.bn_dn_s;
  if (tid == 0 && a.bn_choice != nullptr) *a.bn_choice = alt ? a.bn_alt : a.bn_gu_r;
  // 2. scans (G <= 1024: one group per thread)
  {
    // rows: the routed groups packed from 0 in group order; shared group j always
    // at T*k + j*T (where the combine and the split shared GEMMs read it), also
    // when an expert window holds fewer than T*k routed rows
    const int g = tid;
    const int n = g < a.E ? cnt_s[g] : 0;
    int o = block_exclusive_scan(n, warp_tot, &tot);
    if (g < a.E) off_s[g] = o;
    else if (g <= G) off_s[g] = a.T * a.k + (g - a.E) * a.T;
    if (tid == 0 && a.nrows_routed != nullptr) *a.nrows_routed = tot;
    // token-tile bases of the routed groups, in group order (MX scale atoms)
    const bool routed = g < a.E;
    int ng = block_exclusive_scan(routed ? (n + bn_gu_r - 1) / bn_gu_r : 0, warp_tot, &tot);
    if (routed) ngu_s[g] = ng;
    if (tid == 0) ngu_s[a.E] = tot;
    int nd = block_exclusive_scan(routed ? (n + bn_dn_r - 1) / bn_dn_r : 0, warp_tot, &tot);
    if (routed) ndn_s[g] = nd;
    if (tid == 0) ndn_s[a.E] = tot;
  }
  // Tile-list order, for persistent CTAs that take every gridDim-th tile: the
  // costliest tiles first, so the last round holds the cheapest ones.
  //   segments 0 .. S-1          every tile of shared group j (T rows)
  //   segments S .. S+E-1        the full token tiles of routed group g, all m tiles
  //                              (with hp: and its partial last tile, after the
  //                              full ones of the same m tile)
  //   segments S+E .. S+E+P-1    the partial last token tile of each routed group
  //                              that has one (with hp: of each group without a
  //                              full tile), by its row count descending
  //                              (ties: lower group first), all m tiles
  // Thread i owns segments 2i and 2i + 1 of the scan (S + 2E <= 2 * blockDim).
  for (int list = 0; list < 2; ++list) {
    const int bnr = list == 0 ? bn_gu_r : bn_dn_r, bns = list == 0 ? bn_gu_s : bn_dn_s;
    const int mtl = list == 0 ? a.m_tiles_gu : a.m_tiles_dn;
    const bool hp = kTileOrderHotPartial && kTileOrderLongestFirst && a.sort_partial;
    for (int g = tid; g < a.E; g += blockDim.x) rem_s[g] = (hp && cnt_s[g] >= bnr) ? 0 : cnt_s[g] % bnr;
    __syncthreads();
    if (kTileOrderLongestFirst && a.sort_partial) {
      // rank of each partial tile: longer ones first, ties by group (O(E) per thread)
      for (int g = tid; g < a.E; g += blockDim.x) {
        const int rg = rem_s[g];
        if (rg > 0) {
          int rank = 0;
          for (int h = 0; h < a.E; ++h) {
            const int rh = rem_s[h];
            rank += (rh > rg) || (rh == rg && h < g);
          }
          part_g[list][rank] = g;
        }
      }
    } else {
      // group order: a prefix count over the groups (E <= blockDim, one per thread)
      const bool has = tid < a.E && rem_s[tid] > 0;
      const int rank = block_exclusive_scan(has ? 1 : 0, warp_tot, &tot);
      if (has) part_g[list][rank] = tid;
    }
    const int npart = __syncthreads_count(tid < a.E && rem_s[tid] > 0);
    const int nbig = __syncthreads_count(tid < a.E && rem_s[tid] > kThinRows);  // partial tiles before the thin ones
    const int ns = a.S + a.E + npart;
    const int sh_tiles = mtl * ((a.T + bns - 1) / bns);
    int c[2];
    for (int q = 0; q < 2; ++q) {
      const int sgi = 2 * tid + q;
      c[q] = sgi >= ns ? 0 : sgi < a.S ? sh_tiles : sgi < a.S + a.E ? mtl * full_seg_tiles(cnt_s[sgi - a.S], bnr, hp) : mtl;
    }
    const int ex = block_exclusive_scan(c[0] + c[1], warp_tot, &tot);
    if (2 * tid <= ns) seg_pre[list][2 * tid] = ex;
    if (2 * tid + 1 <= ns) seg_pre[list][2 * tid + 1] = ex + c[0];
    if (tid == 0) {
      nseg_s[list] = ns;
      nbig_s[list] = nbig;
      hp_list[list] = hp;
      a.ntiles[list] = tot;
    }
    __syncthreads();
  }
  if (tid == 0) {
    a.ntiles[2] = seg_pre[0][a.S];   // shared tiles end (= 0 without shared experts)
    a.ntiles[3] = seg_pre[1][a.S];
    // where the thin tiles (at most kThinRows rows) begin: they end a list ordered
    // longest first; the list's end otherwise
    const bool sorted = kTileOrderLongestFirst && a.sort_partial;
    for (int list = 0; list < 2; ++list)
      a.ntiles[5 + list] = sorted ? seg_pre[list][a.S + a.E + nbig_s[list]] : seg_pre[list][nseg_s[list]];
  }
  if (a.sched_zero != nullptr && tid < 4) a.sched_zero[tid] = 0;
  // 3. outputs
  for (int g = tid; g <= G; g += blockDim.x) {
    a.off[g] = off_s[g];
    if (g < G) a.cnt[g] = cnt_s[g];
    if (g < G && a.done != nullptr) a.done[g] = 0;
  }
  if (a.ntile_base_gu != nullptr)
    for (int g = tid; g <= a.E; g += blockDim.x) {
      a.ntile_base_gu[g] = ngu_s[g];
      a.ntile_base_dn[g] = ndn_s[g];
    }
  if (!fused)
    for (int g = tid; g < a.E; g += blockDim.x)
      for (int c = 0; c < a.nchunks; ++c) a.chunk_cnt[static_cast<size_t>(c) * a.E + g] += off_s[g];
  // tile lists, spread over all threads: tile -> segment by binary search over the
  // segment prefix (the last segment starting at or before it is never empty),
  // then (group, m tile, token tile) inside the segment
  for (int list = 0; list < 2; ++list) {
    const int* pre = seg_pre[list];
    const int ns = nseg_s[list];
    const int bnr = list == 0 ? bn_gu_r : bn_dn_r, bns = list == 0 ? bn_gu_s : bn_dn_s;
    int4* out = list == 0 ? a.tiles_gu : a.tiles_dn;
    const int total = pre[ns];
    for (int t = tid; t < total; t += blockDim.x) {
      int lo = 0, hi = ns - 1;
      while (lo < hi) {  // last segment with pre <= t
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= t) lo = mid; else hi = mid - 1;
      }
      const int local = t - pre[lo];
      int g, mt, nt;
      if (lo < a.S) {
        g = a.E + lo;
        const int ntn = (a.T + bns - 1) / bns;
        mt = local / ntn;
        nt = local % ntn;
      } else if (lo < a.S + a.E) {
        g = lo - a.S;
        const int nf = full_seg_tiles(cnt_s[g], bnr, hp_list[list]);
        mt = local / nf;
        nt = local % nf;
      } else {
        g = part_g[list][lo - a.S - a.E];
        mt = local;
        nt = cnt_s[g] / bnr;
      }
      const bool shared = g >= a.E;
      const bool mx = a.mx && !shared;
      const int bn = shared ? bns : bnr;
      const int n = cnt_s[g];
      const int r0 = nt * bn;
      int y;
      if (list == 0)
        y = mx ? ngu_s[g] + nt : (shared ? r0 : off_s[g] + r0);
      else
        y = mx ? ndn_s[g] + nt : off_s[g] + r0;
      out[t] = make_int4(g | (mt << 16), y, off_s[g] + r0, min(bn, n - r0));
    }
  }
  // 4. fused small case: scatter the slots (one warp, 32 slots at a time, in order)
  __syncthreads();
  if (fused && tid < 32) {
    const int lane = tid;
    for (int e = lane; e < a.E; e += 32) cnt_s[e] = off_s[e];  // reuse as running position
    __syncwarp();
    for (int b = 0; b < nslots; b += 32) {
      const int s = b + lane;
      const int e = s < nslots ? slot_e[s] : -1;
      const bool valid = e >= 0;
      const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      if (valid) {
        const int pos = cnt_s[e] + rank;
        perm[pos] = s;
        inv[s] = pos;
      }
      __syncwarp();
      if (valid && rank == 0) cnt_s[e] += __popc(peers);
      __syncwarp();
    }
  }
}

// One warp per chunk walks its slots in order, 32 at a time; peers with the
// same expert get consecutive positions in lane order.
__global__ void __launch_bounds__(32)
    perm_scatter_kernel(const int32_t* __restrict__ idx, int nslots, int E, int e_begin,
                        const int32_t* __restrict__ chunk_base, int32_t* __restrict__ perm,
                        int32_t* __restrict__ inv) {
  __shared__ int ctr[kMaxGroups];
  const int lane = threadIdx.x;
  for (int e = lane; e < E; e += 32) ctr[e] = chunk_base[static_cast<size_t>(blockIdx.x) * E + e];
  __syncwarp();
  const int base = blockIdx.x * kPermChunk;
  const int end = min(nslots, base + kPermChunk);
  for (int b = base; b < end; b += 32) {
    const int s = b + lane;
    const int e = s < end ? idx[s] - e_begin : -1;
    const bool valid = e >= 0 && e < E;
    const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    int pos = 0;
    if (valid) {
      pos = ctr[e] + rank;
      perm[pos] = s;
      inv[s] = pos;
    }
    __syncwarp();
    if (valid && rank == 0) ctr[e] += __popc(peers);
    __syncwarp();
  }
}

// Xp[row] = x[perm[row] / k]: one warp per row, 16-byte vectors.
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm, int nrows,
                       const int32_t* __restrict__ nrows_dev, int k, int hv, uint4* __restrict__ xp) {
  const int row = blockIdx.x * 8 + threadIdx.x / 32;
  if (row >= nrows || row >= *nrows_dev) return;
  const int t = perm[row] / k;
  const uint4* src = x + static_cast<size_t>(t) * hv;
  uint4* dst = xp + static_cast<size_t>(row) * hv;
  int c = threadIdx.x % 32;
  for (; c + 96 < hv; c += 128) {  // four 16-byte loads in flight per lane
    const uint4 a = __ldg(src + c), b = __ldg(src + c + 32), d = __ldg(src + c + 64), e = __ldg(src + c + 96);
    dst[c] = a;
    dst[c + 32] = b;
    dst[c + 64] = d;
    dst[c + 96] = e;
  }
  for (; c < hv; c += 32) dst[c] = __ldg(src + c);
}

// MXFP8 quantisation of the routed token rows (OCP MX v1.0 rule, E4M3 with
// round-to-nearest-even and saturation): one warp per row, one 32-value block
// per lane per step. The E8M0 codes go straight into the scale-factor atoms of
// the gate/up token tile that holds the row.
__global__ void __launch_bounds__(256)
    quant_gather_mx_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm,
                           const int32_t* __restrict__ idx, const int32_t* __restrict__ off,
                           const int32_t* __restrict__ ntile_base, int nrows, const int32_t* __restrict__ nrows_dev,
                           int k, int H, int bn, int e_begin, int e_count, uint4* __restrict__ xq,
                           uint8_t* __restrict__ sfb) {
  const int row = blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= nrows || row >= *nrows_dev) return;
  const int slot = perm[row];
  const int t = slot / k;
  const int g = idx[slot] - e_begin;
  if (g < 0 || g >= e_count) return;  // never for a routed row of this instance
  const int j = row - off[g];
  const int ntile = ntile_base[g] + j / bn;
  const int n = j % bn;
  const int nblk = H / 32;
  const uint4* src = x + static_cast<size_t>(t) * (H / 8);
  uint4* dst = xq + static_cast<size_t>(row) * (H / 16);
  for (int b = lane; b < nblk; b += 32) {
    float v[32];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 u = __ldg(src + b * 4 + q);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(p[i]);
        v[q * 8 + 2 * i] = f.x;
        v[q * 8 + 2 * i + 1] = f.y;
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    int code;
    float inv;
    mx_scale(amax, 8, code, inv);
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __nv_fp8x2_storage_t lo =
          __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i] * inv, v[4 * i + 1] * inv), __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi =
          __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i + 2] * inv, v[4 * i + 3] * inv), __NV_SATFINITE, __NV_E4M3);
      w[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    }
    dst[b * 2] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[b * 2 + 1] = make_uint4(w[4], w[5], w[6], w[7]);
    sfb[(static_cast<size_t>(ntile) * (H / 128) + b / 4) * 512 + (n % 32) * 16 + (n / 32) * 4 + (b % 4)] =
        static_cast<uint8_t>(code);
  }
}

}  // namespace

cudaError_t launch_quant_gather_mx(const void* x, const int32_t* perm, const int32_t* idx, const int32_t* off,
                                   const int32_t* ntile_base_gu, int nrows, const int32_t* nrows_dev, int k, int H,
                                   int bn_gu, int e_begin, int e_count, uint8_t* xq, uint8_t* sfb, cudaStream_t s) {
  if (nrows == 0) return cudaSuccess;
  quant_gather_mx_kernel<<<(nrows + 7) / 8, 256, 0, s>>>(static_cast<const uint4*>(x), perm, idx, off,
                                                          ntile_base_gu, nrows, nrows_dev, k, H, bn_gu, e_begin,
                                                          e_count, reinterpret_cast<uint4*>(xq), sfb);
  return cudaGetLastError();
}

cudaError_t launch_perm_count(const int32_t* idx, int nslots, int E, int e_begin, int e_global, int32_t* chunk_cnt,
                              int* status, cudaStream_t s) {
  if (E > kMaxGroups) return cudaErrorInvalidValue;
  const int nchunks = (nslots + kPermChunk - 1) / kPermChunk;
  perm_count_kernel<<<nchunks, 256, 0, s>>>(idx, nslots, E, e_begin, e_global, chunk_cnt, status);
  return cudaGetLastError();
}

cudaError_t launch_perm_scan(const ScanArgs& a, cudaStream_t s) {
  if (a.E + a.S > kMaxScanGroups) return cudaErrorInvalidValue;
  perm_scan_kernel<<<1, 1024, 0, s>>>(a, 0, nullptr, 0, nullptr, nullptr, nullptr);
  return cudaGetLastError();
}

cudaError_t launch_perm_fused(const ScanArgs& a, const int32_t* idx, int nslots, int32_t* perm, int32_t* inv,
                              int* status, cudaStream_t s) {
  if (a.E + a.S > kMaxScanGroups || nslots > kPermChunk) return cudaErrorInvalidValue;
  perm_scan_kernel<<<1, 1024, 0, s>>>(a, 1, idx, nslots, perm, inv, status);
  return cudaGetLastError();
}

cudaError_t launch_perm_scatter(const int32_t* idx, int nslots, int E, int e_begin, const int32_t* chunk_base,
                                int32_t* perm, int32_t* inv, cudaStream_t s) {
  const int nchunks = (nslots + kPermChunk - 1) / kPermChunk;
  perm_scatter_kernel<<<nchunks, 32, 0, s>>>(idx, nslots, E, e_begin, chunk_base, perm, inv);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* x, const int32_t* perm, int nrows, const int32_t* nrows_dev, int k, int H,
                               void* xp, cudaStream_t s) {
  if (nrows == 0) return cudaSuccess;
  gather_rows_kernel<<<(nrows + 7) / 8, 256, 0, s>>>(static_cast<const uint4*>(x), perm, nrows, nrows_dev, k, H / 8,
                                                     static_cast<uint4*>(xp));
  return cudaGetLastError();
}

}  // namespace moe
